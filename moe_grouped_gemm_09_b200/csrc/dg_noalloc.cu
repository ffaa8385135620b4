// dg_fp8_gemm_nt_noalloc: the dense GEMM for callers that cannot allocate
// device memory.  Its scratch -- the device error word the kernel's bounded
// waits report into -- lives in one file-scope __device__ array of fixed size
// instead of memory the library would otherwise cudaMalloc on first use.
// (Split-K reduces through distributed shared memory and needs no global
// scratch.)  The declaration and the contract are in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>
#include <utility>

#include "../../include/dg.h"
#include "dg_config.h"
#include "sm100_fp8_gemm.cuh"

namespace dg {
namespace {

// Layout of the static scratch: [error word | pad to 256 bytes]
constexpr size_t kNaScratchBytes = 256;

// Every GPU that loads the library holds this array until the process exits.
// In host code `g_noalloc_scratch` is only a host-side stand-in for the
// symbol; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNaScratchBytes];

constexpr int kNaMaxDevices = 64;

struct NaDevice {
  bool ready = false;
  int num_sms = 0;
  unsigned char* scratch = nullptr;  // device address of g_noalloc_scratch
  bool smem_attr_set[kNumVariants] = {};
  ClusterLimits limits = {};         // co-resident split-K clusters (0: not known)
};

std::mutex g_na_mutex;
NaDevice g_na_dev[kNaMaxDevices];

using NaEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
NaEncodeFn g_na_encode = nullptr;

template <int V>
using NaShape = KernelShape<kVariants[V].block_n, kVariants[V].stages, kVariants[V].num_acc,
                            kVariants[V].kps, kVariants[V].a_rows, kVariants[V].small>;
// (instantiated only for the variants this entry point launches: not the pair ones)

template <int V>
auto na_kernel() {
  constexpr Variant var = kVariants[V];
  static_assert(!var.pair, "pair variants are not launched by this entry point");
  return fp8_gemm_kernel<kDense, var.block_n, var.stages, var.num_acc, var.kps, var.a_rows,
                         var.small>;
}

template <int V>
dg_status na_smem_attr(NaDevice& st) {
  if constexpr (kVariants[V].pair) {
    return DG_ERR_UNSUPPORTED;  // the picker offers this entry point no pair variant
  } else {
  if (!st.smem_attr_set[V]) {
    if (cudaFuncSetAttribute(na_kernel<V>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                             NaShape<V>::kSmemBytes) != cudaSuccess)
      return DG_ERR_CUDA;
    st.smem_attr_set[V] = true;
  }
  return DG_OK;
  }
}

// Split-K clusters of each size the device co-schedules for decode variant V.
template <int V>
dg_status na_cluster_limits(NaDevice& st) {
  if constexpr (kVariants[V].decode) {
    dg_status s = na_smem_attr<V>(st);
    if (s != DG_OK) return s;
    for (int c = 1; c <= kMaxSplitK; ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = NaShape<V>::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, na_kernel<V>(), &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
      }
      st.limits.max_clusters[V][c] = n;
    }
  }
  return DG_OK;
}

template <int... V>
dg_status na_all_cluster_limits(NaDevice& st, std::integer_sequence<int, V...>) {
  dg_status s = DG_OK;
  ((s = (s == DG_OK ? na_cluster_limits<V>(st) : s)), ...);
  return s;
}

// Once per device, with that device current: check the architecture, find the
// tensor-map encoder and the device address of the static scratch.  Nothing
// here allocates device memory.
dg_status na_setup(NaDevice** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
  if (dev < 0 || dev >= kNaMaxDevices) return DG_ERR_UNSUPPORTED;
  NaDevice& st = g_na_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DG_ERR_CUDA;
    if (major != 10 || minor != 0) return DG_ERR_ARCH;
    if (!g_na_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return DG_ERR_CUDA;
      g_na_encode = reinterpret_cast<NaEncodeFn>(fn);
    }
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || ptr == nullptr)
      return DG_ERR_CUDA;
    st.scratch = static_cast<unsigned char*>(ptr);
    st.num_sms = sms;
    dg_status s = na_all_cluster_limits(st, std::make_integer_sequence<int, kNumVariants>{});
    if (s != DG_OK) return s;
    st.ready = true;
  }
  *out = &st;
  return DG_OK;
}

// Same 4-D view of an E4M3 [rows][K] matrix as the regular entry points use.
dg_status na_map(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint32_t box_rows,
                 uint32_t kps) {
  cuuint64_t dims[4] = {128, rows, K / 128, 1};
  cuuint64_t strides[3] = {K, 128, K * rows};
  cuuint32_t box[4] = {128, box_rows, kps, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_na_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

dg_status na_d_map(CUtensorMap* map, void* base, uint64_t N, uint64_t rows) {
  cuuint64_t dims[2] = {N, rows};
  cuuint64_t strides[1] = {N * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_na_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

template <int V>
dg_status na_launch(NaDevice& st, const CUtensorMap& ta, const CUtensorMap& tb,
                    const CUtensorMap& td, const GemmArgs& args, int grid, cudaStream_t stream) {
  if constexpr (kVariants[V].pair) {
    return DG_ERR_UNSUPPORTED;
  } else {
  dg_status s = na_smem_attr<V>(st);
  if (s != DG_OK) return s;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = NaShape<V>::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (args.split_k > 1) {  // the CTAs of one output tile form a cluster
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = args.split_k;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  return cudaLaunchKernelEx(&cfg, na_kernel<V>(), ta, tb, td, args) == cudaSuccess ? DG_OK
                                                                                   : DG_ERR_CUDA;
  }
}

template <int... V>
dg_status na_dispatch(NaDevice& st, int variant, const CUtensorMap& ta, const CUtensorMap& tb,
                      const CUtensorMap& td, const GemmArgs& args, int grid, cudaStream_t stream,
                      std::integer_sequence<int, V...>) {
  dg_status s = DG_ERR_UNSUPPORTED;
  ((variant == V ? (s = na_launch<V>(st, ta, tb, td, args, grid, stream), 0) : 0), ...);
  return s;
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" dg_status dg_fp8_gemm_nt_noalloc(const void* a, const float* sfa, const void* b,
                                            const float* sfb, void* d, int M, int N, int K,
                                            dg_stream_t stream_) {
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (M < 0 || K <= 0 || K % 128 != 0 || N <= 0 || N % 16 != 0) return DG_ERR_INVALID_ARG;
  if (M == 0) return DG_OK;
  if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_ARG;
  auto al = [](const void* p, size_t n) { return reinterpret_cast<uintptr_t>(p) % n == 0; };
  if (!al(a, 16) || !al(b, 16) || !al(d, 16) || !al(sfa, 4) || !al(sfb, 4))
    return DG_ERR_INVALID_ARG;
  if (K > (1 << 24)) return DG_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_na_mutex);
  NaDevice* st = nullptr;
  dg_status s = na_setup(&st);
  if (s != DG_OK) return s;

  const PickedConfig pc = pick_config(kDense, M, N, K, 1, 0, st->num_sms, &st->limits,
                                      /*allow_pair=*/false);
  const Variant var = kVariants[pc.variant];
  GemmArgs args = {};
  args.rows = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.num_m_blocks = ceil_div(M, tile_rows(var));
  args.num_n_blocks = ceil_div(N, var.block_n);
  args.k_blocks = K / kBlockK;
  args.split_k = pc.split_k;
  args.kb_per_split = ceil_div(args.k_blocks, pc.split_k);
  args.nb128 = ceil_div(N, 128);
  args.sfa = sfa;
  args.sfb = sfb;
  args.d = static_cast<__nv_bfloat16*>(d);
  args.error_word = reinterpret_cast<int*>(st->scratch);
  args.timeout_ns = 1000ull * 1000 * 1000;
  args.a_box_rows = var.a_rows == 256 ? 256 : M >= kBlockM ? kBlockM : ((M + 15) / 16) * 16;
  args.prefetch = 1;
  if (args.a_box_rows > var.a_rows) return DG_ERR_UNSUPPORTED;
  if (var.small && pc.grid != args.num_m_blocks * args.num_n_blocks * pc.split_k)
    return DG_ERR_UNSUPPORTED;
  if (pc.split_k > 1 && (pc.grid != args.num_m_blocks * args.num_n_blocks * pc.split_k ||
                         M > kBlockM || !split_fits(var, M, pc.split_k)))
    return DG_ERR_UNSUPPORTED;

  CUtensorMap ta, tb;
  s = na_map(&ta, a, K, M, args.a_box_rows, var.kps);
  if (s != DG_OK) return s;
  s = na_map(&tb, b, K, N, var.block_n, var.kps);
  if (s != DG_OK) return s;
  CUtensorMap td;
  s = na_d_map(&td, d, N, M);
  if (s != DG_OK) return s;
  return na_dispatch(*st, pc.variant, ta, tb, td, args, pc.grid, stream,
                     std::make_integer_sequence<int, kNumVariants>{});
}
