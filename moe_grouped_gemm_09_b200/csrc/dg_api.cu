// C ABI of the FP8 block-scaled GEMM library: argument checks, per-device
// state, configuration choice, TMA descriptors and kernel launches.
// The operations are declared and documented in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "../../include/dg.h"
#include "dg_config.h"
#include "sm100_fp8_gemm.cuh"

namespace dg {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kCounterSlots = 1 << 16;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* error_word = nullptr;      // one int, device memory
  float* workspace = nullptr;     // split-K partials
  size_t workspace_bytes = 0;
  int* counters = nullptr;        // split-K arrival counters
  bool smem_attr_set[3][kNumVariants] = {};
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
int g_num_sms_cap = 0;            // 0: all SMs
unsigned long long g_timeout_ns = 1000ull * 1000 * 1000;
bool g_timeout_from_env = false;

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

dg_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DG_OK : DG_ERR_CUDA; }

bool print_configs() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("DG_PRINT_CONFIGS");
    v = (e && e[0] && e[0] != '0') ? 1 : 0;
  }
  return v == 1;
}

// Initialise (once) the state of the current device.  Caller holds g_mutex.
dg_status device_state(DeviceState** out, int* dev_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return DG_ERR_CUDA;
    if (prop.major != 10 || prop.minor != 0) return DG_ERR_ARCH;
    if (!g_encode) {
      cudaDriverEntryPointQueryResult q;
      void* fn = nullptr;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || fn == nullptr)
        return DG_ERR_CUDA;
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    if (!g_timeout_from_env) {
      g_timeout_from_env = true;
      const char* e = std::getenv("DG_WAIT_TIMEOUT_MS");
      if (e && std::atoi(e) > 0) g_timeout_ns = 1000000ull * std::atoi(e);
    }
    st.num_sms = prop.multiProcessorCount;
    if (cudaMalloc(&st.error_word, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaMemset(st.error_word, 0, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaMalloc(&st.counters, kCounterSlots * sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaMemset(st.counters, 0, kCounterSlots * sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
    st.ready = true;
  }
  *out = &st;
  if (dev_out) *dev_out = dev;
  return DG_OK;
}

// Grow the split-K workspace of a device to at least `bytes`.  The workspace
// is only ever grown (never freed) so that earlier launches stay valid.
dg_status ensure_workspace(DeviceState& st, size_t bytes) {
  if (bytes <= st.workspace_bytes) return DG_OK;
  size_t want = bytes < (size_t(16) << 20) ? (size_t(16) << 20) : bytes;
  if (st.workspace) {
    // A larger workspace replaces the old one once the device is idle.
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
    cudaFree(st.workspace);
    st.workspace = nullptr;
    st.workspace_bytes = 0;
  }
  if (cudaMalloc(&st.workspace, want) != cudaSuccess) return DG_ERR_CUDA;
  st.workspace_bytes = want;
  return DG_OK;
}

int effective_sms(const DeviceState& st) {
  int n = st.num_sms;
  if (g_num_sms_cap > 0 && g_num_sms_cap < n) n = g_num_sms_cap;
  return n;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 3-D tensor map over E4M3 bytes [d2][d1][d0] (d0 = K contiguous) with a
// box of box1 rows x 128 bytes and the 128-byte swizzle.
dg_status make_map(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                   uint32_t box1) {
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0, d0 * d1};  // bytes, for dims 1 and 2
  cuuint32_t box[3] = {128, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

template <int KIND, int V>
dg_status launch_variant(DeviceState& st, const CUtensorMap& ta, const CUtensorMap& tb,
                         const GemmArgs& args, int grid, cudaStream_t stream) {
  constexpr Variant var = kVariants[V];
  using Shape = KernelShape<var.block_n, var.stages, var.num_acc>;
  auto kern = fp8_gemm_kernel<KIND, var.block_n, var.stages, var.num_acc>;
  if (!st.smem_attr_set[KIND][V]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Shape::kSmemBytes) != cudaSuccess)
      return DG_ERR_CUDA;
    st.smem_attr_set[KIND][V] = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Shape::kSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ta, tb, args);
  return from_cuda(e);
}

template <int KIND>
dg_status launch(DeviceState& st, int variant, const CUtensorMap& ta, const CUtensorMap& tb,
                 const GemmArgs& args, int grid, cudaStream_t stream) {
  switch (variant) {
    case 0: return launch_variant<KIND, 0>(st, ta, tb, args, grid, stream);
    case 1: return launch_variant<KIND, 1>(st, ta, tb, args, grid, stream);
    case 2: return launch_variant<KIND, 2>(st, ta, tb, args, grid, stream);
    case 3: return launch_variant<KIND, 3>(st, ta, tb, args, grid, stream);
    default: return DG_ERR_UNSUPPORTED;
  }
}

// Shared path of the three GEMM forms.
dg_status run(int kind, const void* a, const float* sfa, const void* b, const float* sfb,
              void* d, const int* m_indices, const int* masked_m, int rows, int N, int K, int G,
              int expected_m, cudaStream_t stream) {
  // ---- argument checks (no device work) ----
  if (rows < 0 || G < 0) return DG_ERR_INVALID_ARG;
  if (K <= 0 || K % 128 != 0 || N <= 0 || N % 16 != 0) return DG_ERR_INVALID_ARG;
  if (rows == 0 || G == 0) return DG_OK;
  if (!a || !sfa || !b || !sfb || !d) return DG_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(sfa, 4) ||
      !aligned(sfb, 4))
    return DG_ERR_INVALID_ARG;
  if (kind == kContiguous && (!m_indices || !aligned(m_indices, 4) || rows % 128 != 0))
    return DG_ERR_INVALID_ARG;
  if (kind == kMasked && (!masked_m || !aligned(masked_m, 4))) return DG_ERR_INVALID_ARG;
  if (kind == kMasked && G > kMaxMaskedGroups) return DG_ERR_UNSUPPORTED;
  const long long a_rows = (kind == kMasked) ? static_cast<long long>(G) * rows : rows;
  if (a_rows > 0x7fffffffLL || static_cast<long long>(G) * N > 0x7fffffffLL)
    return DG_ERR_UNSUPPORTED;
  if (K > (1 << 24)) return DG_ERR_UNSUPPORTED;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  dg_status s = device_state(&st, nullptr);
  if (s != DG_OK) return s;
  const int sms = effective_sms(*st);
  const PickedConfig pc = pick_config(kind, rows, N, K, G, expected_m, sms);
  const Variant var = kVariants[pc.variant];

  GemmArgs args = {};
  args.rows = rows;
  args.N = N;
  args.K = K;
  args.G = (kind == kDense) ? 1 : G;
  args.num_m_blocks = ceil_div(rows, kBlockM);
  args.num_n_blocks = ceil_div(N, var.block_n);
  args.k_blocks = K / kBlockK;
  args.split_k = pc.split_k;
  args.kb_per_split = ceil_div(args.k_blocks, pc.split_k);
  args.nb128 = ceil_div(N, 128);
  args.sfa = sfa;
  args.sfb = sfb;
  args.d = static_cast<__nv_bfloat16*>(d);
  args.m_indices = m_indices;
  args.masked_m = masked_m;
  args.error_word = st->error_word;
  args.timeout_ns = g_timeout_ns;
  args.counters = st->counters;
  if (pc.split_k > 1) {
    if (pc.out_tiles > kCounterSlots) return DG_ERR_UNSUPPORTED;
    const size_t ws = static_cast<size_t>(pc.out_tiles) * pc.split_k * kBlockM * var.block_n *
                      sizeof(float);
    s = ensure_workspace(*st, ws);
    if (s != DG_OK) return s;
  }
  args.workspace = st->workspace;

  CUtensorMap ta, tb;
  const int b_groups = (kind == kDense) ? 1 : G;
  s = make_map(&ta, a, K, rows, kind == kMasked ? G : 1, kBlockM);
  if (s != DG_OK) return s;
  s = make_map(&tb, b, K, N, b_groups, var.block_n);
  if (s != DG_OK) return s;

  if (print_configs())
    std::fprintf(stderr,
                 "[dg] kind=%d rows=%d N=%d K=%d G=%d expected_m=%d -> BLOCK_N=%d stages=%d "
                 "acc=%d split_k=%d grid=%d\n",
                 kind, rows, N, K, G, expected_m, var.block_n, var.stages, var.num_acc,
                 pc.split_k, pc.grid);

  switch (kind) {
    case kDense: return launch<kDense>(*st, pc.variant, ta, tb, args, pc.grid, stream);
    case kContiguous: return launch<kContiguous>(*st, pc.variant, ta, tb, args, pc.grid, stream);
    default: return launch<kMasked>(*st, pc.variant, ta, tb, args, pc.grid, stream);
  }
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" {

dg_status dg_fp8_gemm_nt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return run(kDense, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, void* d, const int* m_indices,
                                              int M_sum, int N, int K, int G,
                                              dg_stream_t stream) {
  return run(kContiguous, a, sfa, b, sfb, d, m_indices, nullptr, M_sum, N, K, G, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const float* sfa, const void* b,
                                          const float* sfb, void* d, const int* masked_m, int G,
                                          int max_m, int N, int K, int expected_m,
                                          dg_stream_t stream) {
  return run(kMasked, a, sfa, b, sfb, d, nullptr, masked_m, max_m, N, K, G, expected_m,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_set_num_sms(int n) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_num_sms_cap = n > 0 ? n : 0;
  return DG_OK;
}

int dg_get_num_sms(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  if (device_state(&st, nullptr) != DG_OK) return -1;
  return effective_sms(*st);
}

dg_status dg_get_last_device_error(int* code) {
  if (!code) return DG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  dg_status s = device_state(&st, nullptr);
  if (s != DG_OK) return s;
  if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, st->error_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return DG_ERR_CUDA;
  *code = v;
  if (v != 0) {
    if (cudaMemset(st->error_word, 0, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaMemset(st->counters, 0, kCounterSlots * sizeof(int)) != cudaSuccess)
      return DG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
  }
  return DG_OK;
}

dg_status dg_set_wait_timeout_ms(int ms) {
  if (ms <= 0) return DG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  g_timeout_from_env = true;
  g_timeout_ns = 1000000ull * static_cast<unsigned long long>(ms);
  return DG_OK;
}

const char* dg_status_string(dg_status s) {
  switch (s) {
    case DG_OK: return "DG_OK";
    case DG_ERR_INVALID_ARG: return "DG_ERR_INVALID_ARG";
    case DG_ERR_UNSUPPORTED: return "DG_ERR_UNSUPPORTED";
    case DG_ERR_CUDA: return "DG_ERR_CUDA";
    case DG_ERR_ARCH: return "DG_ERR_ARCH";
    case DG_ERR_DEVICE: return "DG_ERR_DEVICE";
  }
  return "DG_ERR_UNKNOWN";
}

dg_status dg_query_config(int kind, int rows, int N, int K, int G, int expected_m, int num_sms,
                          dg_config* out) {
  if (!out || kind < 0 || kind > 2 || rows < 0 || N <= 0 || N % 16 != 0 || K <= 0 ||
      K % 128 != 0 || G < 1 || num_sms < 1)
    return DG_ERR_INVALID_ARG;
  const PickedConfig pc = pick_config(kind, rows, N, K, G, expected_m, num_sms);
  const Variant v = kVariants[pc.variant];
  out->block_m = kBlockM;
  out->block_n = v.block_n;
  out->stages = v.stages;
  out->num_acc = v.num_acc;
  out->split_k = pc.split_k;
  out->grid = pc.grid;
  switch (pc.variant) {
    case 0: out->smem_bytes = KernelShape<256, 4, 1>::kSmemBytes; out->tmem_cols = KernelShape<256, 4, 1>::kTmemCols; break;
    case 1: out->smem_bytes = KernelShape<128, 6, 2>::kSmemBytes; out->tmem_cols = KernelShape<128, 6, 2>::kTmemCols; break;
    case 2: out->smem_bytes = KernelShape<64, 8, 2>::kSmemBytes; out->tmem_cols = KernelShape<64, 8, 2>::kTmemCols; break;
    default: out->smem_bytes = KernelShape<32, 9, 2>::kSmemBytes; out->tmem_cols = KernelShape<32, 9, 2>::kTmemCols; break;
  }
  return DG_OK;
}

const char* dg_version(void) { return "0.1.0"; }

}  // extern "C"
