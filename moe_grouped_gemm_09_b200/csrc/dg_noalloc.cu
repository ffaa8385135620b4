// dg_fp8_gemm_nt_noalloc: the dense GEMM for callers that cannot allocate
// device memory.  Its scratch (split-K partial sums, split-K arrival counters
// and the device error word) lives in one file-scope __device__ array of fixed
// size instead of memory the library would otherwise cudaMalloc on first use.
// The declaration and the contract are in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/dg.h"
#include "dg_config.h"
#include "sm100_fp8_gemm.cuh"

namespace dg {
namespace {

// Layout of the static scratch: [error word | pad][counters][split-K partials]
constexpr size_t kNaErrorBytes = 256;
constexpr int kNaCounters = 4096;
constexpr size_t kNaCounterBytes = kNaCounters * sizeof(int);
constexpr size_t kNaWorkspaceBytes = size_t(12) << 20;  // 12 MiB of FP32 partial sums
constexpr size_t kNaScratchBytes = kNaErrorBytes + kNaCounterBytes + kNaWorkspaceBytes;

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
};

std::mutex g_na_mutex;
NaDevice g_na_dev[kNaMaxDevices];

using NaEncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
NaEncodeFn g_na_encode = nullptr;

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
    st.ready = true;
  }
  *out = &st;
  return DG_OK;
}

dg_status na_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint32_t box1) {
  cuuint64_t dims[3] = {d0, d1, 1};
  cuuint64_t strides[2] = {d0, d0 * d1};
  cuuint32_t box[3] = {128, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_na_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

template <int V>
dg_status na_launch(NaDevice& st, const CUtensorMap& ta, const CUtensorMap& tb,
                    const GemmArgs& args, int grid, cudaStream_t stream) {
  constexpr Variant var = kVariants[V];
  using Shape = KernelShape<var.block_n, var.stages, var.num_acc>;
  auto kern = fp8_gemm_kernel<kDense, var.block_n, var.stages, var.num_acc>;
  if (!st.smem_attr_set[V]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Shape::kSmemBytes) != cudaSuccess)
      return DG_ERR_CUDA;
    st.smem_attr_set[V] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Shape::kSmemBytes;
  cfg.stream = stream;
  return cudaLaunchKernelEx(&cfg, kern, ta, tb, args) == cudaSuccess ? DG_OK : DG_ERR_CUDA;
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

  const PickedConfig pc = pick_config(kDense, M, N, K, 1, 0, st->num_sms);
  const Variant var = kVariants[pc.variant];
  GemmArgs args = {};
  args.rows = M;
  args.N = N;
  args.K = K;
  args.G = 1;
  args.num_m_blocks = ceil_div(M, kBlockM);
  args.num_n_blocks = ceil_div(N, var.block_n);
  args.k_blocks = K / kBlockK;
  args.split_k = pc.split_k;
  args.kb_per_split = ceil_div(args.k_blocks, pc.split_k);
  args.nb128 = ceil_div(N, 128);
  args.sfa = sfa;
  args.sfb = sfb;
  args.d = static_cast<__nv_bfloat16*>(d);
  args.error_word = reinterpret_cast<int*>(st->scratch);
  args.counters = reinterpret_cast<int*>(st->scratch + kNaErrorBytes);
  args.workspace = reinterpret_cast<float*>(st->scratch + kNaErrorBytes + kNaCounterBytes);
  args.timeout_ns = 1000ull * 1000 * 1000;
  if (pc.split_k > 1) {
    const size_t ws = static_cast<size_t>(pc.out_tiles) * pc.split_k * kBlockM * var.block_n *
                      sizeof(float);
    if (ws > kNaWorkspaceBytes || pc.out_tiles > kNaCounters) return DG_ERR_UNSUPPORTED;
    // the arrival counters must start at zero; the array keeps the last call's contents
    if (cudaMemsetAsync(args.counters, 0, pc.out_tiles * sizeof(int), stream) != cudaSuccess)
      return DG_ERR_CUDA;
  }

  CUtensorMap ta, tb;
  s = na_map(&ta, a, K, M, kBlockM);
  if (s != DG_OK) return s;
  s = na_map(&tb, b, K, N, var.block_n);
  if (s != DG_OK) return s;
  switch (pc.variant) {
    case 0: return na_launch<0>(*st, ta, tb, args, pc.grid, stream);
    case 1: return na_launch<1>(*st, ta, tb, args, pc.grid, stream);
    case 2: return na_launch<2>(*st, ta, tb, args, pc.grid, stream);
    case 3: return na_launch<3>(*st, ta, tb, args, pc.grid, stream);
    default: return DG_ERR_UNSUPPORTED;
  }
}
