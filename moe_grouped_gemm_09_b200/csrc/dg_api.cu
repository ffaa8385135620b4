// C ABI of the FP8 block-scaled GEMM library: argument checks, per-device
// state, configuration choice, TMA descriptors and kernel launches.
// The operations are declared and documented in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <array>
#include <mutex>
#include <type_traits>
#include <utility>

#include "../../include/dg.h"
#include "dg_config.h"
#include "sm100_fp8_gemm.cuh"
#include "sm100_fp8_gemm_pair.cuh"

namespace dg {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kNumForms = 10;  // launch forms (enum Form below)

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* error_word = nullptr;      // one int, device memory
  bool smem_attr_set[kNumForms][kNumVariants] = {};  // per form and variant
  bool limits_known = false;
  ClusterLimits limits = {};      // co-resident split-K clusters per variant and size
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
    if (!st.error_word && cudaMalloc(&st.error_word, sizeof(int)) != cudaSuccess) {
      st.error_word = nullptr;
      return DG_ERR_CUDA;
    }
    // (a failure below keeps the word for the next attempt instead of leaking it)
    if (cudaMemset(st.error_word, 0, sizeof(int)) != cudaSuccess) return DG_ERR_CUDA;
    if (cudaDeviceSynchronize() != cudaSuccess) return DG_ERR_CUDA;
    st.ready = true;
  }
  *out = &st;
  if (dev_out) *dev_out = dev;
  return DG_OK;
}

// Rows per TMA box of A: a whole tile (128 rows, or 256 for a two-half
// variant), except that a dense A shorter than one 128-row block is fetched
// with a box of its own (16-row rounded) height, so the SM moves no padding.
int a_box_rows(int kind, int rows, const Variant& var) {
  if (var.a_rows == 256) return 256;
  if (var.pair) return kBlockM;
  if (kind != kDense || rows >= kBlockM) return kBlockM;
  return ((rows + 15) / 16) * 16;
}

// DG_FORCE_CONFIG="<block_n>:<split_k>[:<kps>:<a_rows>[:<small>]]" overrides
// the picker (tuning sweeps); without kps/a_rows a general (one K block per
// stage) variant.
// Ignored unless the variant exists and, for split_k > 1, the problem is a
// dense one with a single 128-row block.
void forced_config(int kind, int rows, int N, int K, int G, int sms, PickedConfig* pc) {
  const char* e = std::getenv("DG_FORCE_CONFIG");
  if (!e || !e[0]) return;
  int bn = 0, sk = 1;
  if (std::sscanf(e, "%d:%d", &bn, &sk) < 1) return;
  int kps = 0, ar = 0, sm = -1, pr = -1;
  std::sscanf(e, "%*d:%*d:%d:%d:%d:%d", &kps, &ar, &sm, &pr);
  int v = -1;
  for (int i = 0; i < kNumVariants; ++i) {
    const Variant& x = kVariants[i];
    if (x.block_n != bn) continue;
    if (kps ? (x.kps != kps || (ar && x.a_rows != ar)) : x.decode) continue;
    if (sm >= 0 && x.small != (sm != 0)) continue;
    if (x.pair != (pr > 0)) continue;
    if ((x.decode || x.a_rows == 256 || x.pair) && kind != kDense) continue;
    if ((x.a_rows == 256 || x.pair) && rows < 256) continue;
    if (a_box_rows(kind, rows, x) > x.a_rows) continue;
    v = i;
  }
  const int KB = K / kBlockK;
  if (v < 0 || sk < 1 || sk > kMaxSplitK || sk > KB) return;
  if (sk > 1 && (kind != kDense || rows > kBlockM)) return;
  if ((sk - 1) * ceil_div(KB, sk) >= KB) return;
  const long long groups = (kind == kMasked) ? G : 1;
  const long long tiles = groups * ceil_div(rows, tile_rows(kVariants[v])) * ceil_div(N, bn);
  pc->variant = v;
  pc->split_k = sk;
  pc->out_tiles = static_cast<int>(tiles);
  if (kVariants[v].pair) {
    const long long pairs = tiles < sms / 2 ? tiles : sms / 2;
    pc->grid = static_cast<int>(2 * (pairs > 0 ? pairs : 1));
    return;
  }
  pc->grid = sk > 1 ? static_cast<int>(tiles) * sk : static_cast<int>(tiles < sms ? tiles : sms);
}

// L2 prefetch of the first tile before the dependency wait; DG_NO_PREFETCH=1
// turns it off (for measurements).
int prefetch_enabled() {
  static int v = -1;
  if (v < 0) {
    const char* e = std::getenv("DG_NO_PREFETCH");
    v = (e && e[0] && e[0] != '0') ? 0 : 1;
  }
  return v;
}

int effective_sms(const DeviceState& st) {
  int n = st.num_sms;
  if (g_num_sms_cap > 0 && g_num_sms_cap < n) n = g_num_sms_cap;
  return n;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// 4-D tensor map over an operand [groups][rows][K] whose rows are kb = K *
// elem_bytes bytes (E4M3: 1, BF16: 2), viewed as {one 128-byte K block,
// rows, kb/128 blocks, groups} with byte strides {kb, 128, rows*kb}: a box of
// {128 bytes, box_rows, kps, 1} brings kps K blocks of box_rows rows, laid
// out in shared memory as kps consecutive [box_rows][128 B] tiles with the
// 128-byte swizzle.
dg_status make_map(CUtensorMap* map, const void* base, uint64_t K, uint64_t rows, uint64_t groups,
                   uint32_t box_rows, uint32_t kps, uint32_t elem_bytes = 1) {
  const uint64_t kb = K * elem_bytes;
  const cuuint32_t block = 128 / elem_bytes;  // elements of one 128-byte K block
  cuuint64_t dims[4] = {block, rows, kb / 128, groups};
  cuuint64_t strides[3] = {kb, 128, kb * rows};  // bytes, for dims 1..3
  cuuint32_t box[4] = {block, box_rows, kps, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = g_encode(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                             : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                        4, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 2-D tensor map over the BF16 output D [rows][N] with a box of 32 rows x
// 64 columns and the 128-byte swizzle (the epilogue's staging layout).
dg_status make_d_map(CUtensorMap* map, void* base, uint64_t N, uint64_t rows) {
  cuuint64_t dims[2] = {N, rows};
  cuuint64_t strides[1] = {N * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// Launch forms: the three GEMM forms, then the dense form with M-major A
// and/or N-major B, then the dense form with FP32 output (D = A B^T + C),
// then the three GEMM forms on BF16 operands; the forms differ in their
// kernel instantiation.
enum Form : int { kFormDense = 0, kFormContiguous = 1, kFormMasked = 2, kFormNN = 3, kFormTN = 4,
                  kFormTT = 5, kFormF32 = 6, kFormBf16Dense = 7, kFormBf16Contiguous = 8,
                  kFormBf16Masked = 9 };
static_assert(kFormBf16Masked + 1 == kNumForms, "one shared-memory attribute row per form");
constexpr bool is_bf16_form(int f) { return f >= kFormBf16Dense; }
constexpr int kind_of_form(int f) {
  return f < 3 ? f : is_bf16_form(f) ? f - kFormBf16Dense : kDense;
}
constexpr int layout_of_form(int f) {
  return f == kFormNN ? kLayoutNN : f == kFormTN ? kLayoutTN : f == kFormTT ? kLayoutTT : kLayoutNT;
}
// Variants that serve M-/N-major operands and the FP32 output form: general
// ones with 128-column B boxes.
constexpr bool mn_capable(const Variant& v) {
  return !v.decode && !v.small && !v.pair && v.kps == 1 && v.a_rows == 128 && v.block_n % 128 == 0;
}

// 2-D tensor map over an M-/N-major operand stored as [K, mn] bytes (mn
// contiguous), boxes of 128 mn bytes x 128 K rows with the 128-byte swizzle.
dg_status make_map_mn(CUtensorMap* map, const void* base, uint64_t mn, uint64_t K) {
  cuuint64_t dims[2] = {mn, K};
  cuuint64_t strides[1] = {mn};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

template <int V, bool SCALED = true>
using ShapeOf = std::conditional_t<
    kVariants[V].pair, PairShape<kVariants[V].block_n, kVariants[V].stages>,
    KernelShape<kVariants[V].block_n, kVariants[V].stages, kVariants[V].num_acc,
                kVariants[V].kps, kVariants[V].a_rows, kVariants[V].small, SCALED>>;
// The geometry a form's kernel is built with (BF16 operands: no scale factors).
template <int FORM, int V>
using FormShape = ShapeOf<V, !is_bf16_form(FORM)>;

// Kernels are instantiated only for the (form, variant) pairs that exist:
// the decode, 256-row and pair variants serve the dense form only.
// Per-variant shared-memory bytes (what = 0) or TMEM columns (what = 1).
template <int what, int... V>
constexpr std::array<int, sizeof...(V)> variant_table(std::integer_sequence<int, V...>) {
  return {(what == 0 ? ShapeOf<V>::kSmemBytes : ShapeOf<V>::kTmemCols)...};
}

template <int FORM, int V>
constexpr bool kBuilt =
    FORM == kFormDense ||
    ((FORM == kFormContiguous || FORM == kFormMasked || FORM == kFormBf16Contiguous ||
      FORM == kFormBf16Masked) &&
     !kVariants[V].decode && kVariants[V].a_rows != 256 && !kVariants[V].pair) ||
    (FORM == kFormBf16Dense && kVariants[V].a_rows != 256 && !kVariants[V].pair) ||
    (FORM >= kFormNN && FORM <= kFormF32 && mn_capable(kVariants[V]));

template <int FORM, int V>
auto kernel_of() {
  constexpr Variant var = kVariants[V];
  if constexpr (var.pair) {
    return fp8_gemm_pair_kernel<var.block_n, var.stages>;
  } else {
    return fp8_gemm_kernel<kind_of_form(FORM), var.block_n, var.stages, var.num_acc, var.kps,
                           var.a_rows, var.small, layout_of_form(FORM), FORM == kFormF32,
                           is_bf16_form(FORM)>;
  }
}

template <int KIND, int V>
dg_status set_smem_attr(DeviceState& st) {
  if constexpr (!kBuilt<KIND, V>) {
    return DG_ERR_UNSUPPORTED;
  } else {
    if (!st.smem_attr_set[KIND][V]) {
      if (cudaFuncSetAttribute(kernel_of<KIND, V>(), cudaFuncAttributeMaxDynamicSharedMemorySize,
                               FormShape<KIND, V>::kSmemBytes) != cudaSuccess)
        return DG_ERR_CUDA;
      st.smem_attr_set[KIND][V] = true;
    }
    return DG_OK;
  }
}

// How many clusters of each size the device co-schedules: split-K clusters of
// every decode variant, and SM pairs of every pair variant (a cluster must fit
// in one GPC, so fewer pairs than SMs / 2 may be resident at once).
template <int V>
dg_status query_cluster_limits(DeviceState& st) {
  if constexpr (kVariants[V].decode || kVariants[V].pair) {
    dg_status s = set_smem_attr<kDense, V>(st);
    if (s != DG_OK) return s;
    for (int c = kVariants[V].pair ? 2 : 1; c <= (kVariants[V].pair ? 2 : kMaxSplitK); ++c) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(c, 1, 1);
      cfg.blockDim = dim3(kThreads, 1, 1);
      cfg.dynamicSmemBytes = ShapeOf<V>::kSmemBytes;
      cudaLaunchAttribute attr[1];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = c;
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, kernel_of<kDense, V>(), &cfg) != cudaSuccess) {
        cudaGetLastError();  // clear; treat as "not known"
        n = 0;
      }
      st.limits.max_clusters[V][c] = n;
    }
  }
  return DG_OK;
}

template <int... V>
dg_status query_all_cluster_limits(DeviceState& st, std::integer_sequence<int, V...>) {
  dg_status s = DG_OK;
  ((s = (s == DG_OK ? query_cluster_limits<V>(st) : s)), ...);
  return s;
}

dg_status ensure_cluster_limits(DeviceState& st) {
  if (st.limits_known) return DG_OK;
  dg_status s = query_all_cluster_limits(st, std::make_integer_sequence<int, kNumVariants>{});
  if (s != DG_OK) return s;
  st.limits_known = true;
  return DG_OK;
}

template <int KIND, int V>
dg_status launch_variant(DeviceState& st, const CUtensorMap& ta, const CUtensorMap& tb,
                         const CUtensorMap& td, const GemmArgs& args, int grid,
                         cudaStream_t stream) {
  if constexpr (!kBuilt<KIND, V>) {
    return DG_ERR_UNSUPPORTED;
  } else {
    dg_status s = set_smem_attr<KIND, V>(st);
    if (s != DG_OK) return s;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid, 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = FormShape<KIND, V>::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    int n_attr = 1;
    if (args.split_k > 1 || kVariants[V].pair) {  // the CTAs of one output tile form a cluster
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = kVariants[V].pair ? 2 : args.split_k;
      attr[1].val.clusterDim.y = 1;
      attr[1].val.clusterDim.z = 1;
      n_attr = 2;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n_attr;
    return from_cuda(cudaLaunchKernelEx(&cfg, kernel_of<KIND, V>(), ta, tb, td, args));
  }
}

template <int KIND, int... V>
dg_status launch_dispatch(DeviceState& st, int variant, const CUtensorMap& ta,
                          const CUtensorMap& tb, const CUtensorMap& td, const GemmArgs& args,
                          int grid, cudaStream_t stream, std::integer_sequence<int, V...>) {
  dg_status s = DG_ERR_UNSUPPORTED;
  ((variant == V ? (s = launch_variant<KIND, V>(st, ta, tb, td, args, grid, stream), 0) : 0),
   ...);
  return s;
}

template <int KIND>
dg_status launch(DeviceState& st, int variant, const CUtensorMap& ta, const CUtensorMap& tb,
                 const CUtensorMap& td, const GemmArgs& args, int grid, cudaStream_t stream) {
  return launch_dispatch<KIND>(st, variant, ta, tb, td, args, grid, stream,
                               std::make_integer_sequence<int, kNumVariants>{});
}

// Shared path of the three GEMM forms.
dg_status run(int form, const void* a, const float* sfa, const void* b, const float* sfb,
              void* d, const int* m_indices, const int* masked_m, int rows, int N, int K, int G,
              int expected_m, cudaStream_t stream, const float* c = nullptr) {
  const int kind = kind_of_form(form);
  const int layout = layout_of_form(form);
  const bool a_mn = (layout & 1) != 0, b_mn = (layout & 2) != 0;
  const bool bf16 = is_bf16_form(form);
  // ---- argument checks (no device work) ----
  // A K block is 128 bytes of a row: 128 E4M3 or 64 BF16 elements.
  const int k_block = bf16 ? kBlockK / 2 : kBlockK;
  if (rows < 0 || G < 0) return DG_ERR_INVALID_ARG;
  if (K <= 0 || K % k_block != 0 || N <= 0 || N % 16 != 0) return DG_ERR_INVALID_ARG;
  if (rows == 0 || G == 0) return DG_OK;
  if (!a || !b || !d || (!bf16 && (!sfa || !sfb))) return DG_ERR_INVALID_ARG;
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) ||
      (!bf16 && (!aligned(sfa, 4) || !aligned(sfb, 4))))
    return DG_ERR_INVALID_ARG;
  if (kind == kContiguous && (!m_indices || !aligned(m_indices, 4) || rows % 128 != 0))
    return DG_ERR_INVALID_ARG;
  if (a_mn && rows % 16 != 0) return DG_ERR_INVALID_ARG;  // [K, M] rows of whole 16-byte units
  if (form == kFormF32 && c && !aligned(c, 16)) return DG_ERR_INVALID_ARG;
  if (kind == kMasked && (!masked_m || !aligned(masked_m, 4))) return DG_ERR_INVALID_ARG;
  if (kind == kMasked && G > kMaxMaskedGroups) return DG_ERR_UNSUPPORTED;
  const long long a_rows = (kind == kMasked) ? static_cast<long long>(G) * rows : rows;
  if (a_rows > 0x7fffffffLL || static_cast<long long>(G) * N > 0x7fffffffLL)
    return DG_ERR_UNSUPPORTED;
  if (K > (1 << 24)) return DG_ERR_UNSUPPORTED;
  // the picker and the kernel count K in 128-byte blocks of a row
  const int k_bytes = bf16 ? 2 * K : K;

  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  dg_status s = device_state(&st, nullptr);
  if (s != DG_OK) return s;
  const int sms = effective_sms(*st);
  if (kind == kDense) {
    s = ensure_cluster_limits(*st);
    if (s != DG_OK) return s;
  }
  PickedConfig pc = pick_config(kind, rows, N, k_bytes, G, expected_m, sms, &st->limits,
                                /*allow_pair=*/!bf16,
                                /*mn_operands=*/layout != kLayoutNT || form == kFormF32);
  forced_config(kind, rows, N, k_bytes, G, sms, &pc);
  const Variant var = kVariants[pc.variant];
  if ((layout != kLayoutNT || form == kFormF32) && (!mn_capable(var) || pc.split_k > 1))
    return DG_ERR_UNSUPPORTED;
  if (bf16 && (var.pair || var.a_rows == 256)) return DG_ERR_UNSUPPORTED;

  GemmArgs args = {};
  args.rows = rows;
  args.N = N;
  args.K = K;
  args.G = (kind == kDense) ? 1 : G;
  args.num_m_blocks = ceil_div(rows, tile_rows(var));
  args.num_n_blocks = ceil_div(N, var.block_n);
  args.k_blocks = k_bytes / kBlockK;
  args.split_k = pc.split_k;
  args.kb_per_split = ceil_div(args.k_blocks, pc.split_k);
  args.nb128 = ceil_div(N, 128);
  args.sfa = sfa;
  args.sfb = sfb;
  args.d = static_cast<__nv_bfloat16*>(d);
  args.d_f32 = form == kFormF32 ? static_cast<float*>(d) : nullptr;
  args.c_f32 = form == kFormF32 ? c : nullptr;
  args.m_indices = m_indices;
  args.masked_m = masked_m;
  args.error_word = st->error_word;
  args.timeout_ns = g_timeout_ns;
  args.a_box_rows = a_mn ? kBlockM : a_box_rows(kind, rows, var);
  if (args.a_box_rows > var.a_rows) return DG_ERR_UNSUPPORTED;
  if ((var.a_rows == 256 || var.pair) && (kind != kDense || pc.split_k > 1))
    return DG_ERR_UNSUPPORTED;
  if (var.pair) {
    // no more pairs than the device co-schedules: a pair launched beyond that
    // would only start once another has finished all its tiles
    const int resident = cluster_limit(&st->limits, pc.variant, 2, sms);
    if (pc.grid / 2 > resident) pc.grid = 2 * resident;
    if (pc.grid % 2 != 0 || pc.grid < 2) return DG_ERR_UNSUPPORTED;
  }
  args.prefetch = prefetch_enabled();
  // a small variant runs one tile per CTA (its epilogue reuses the ring)
  if (var.small && (kind != kDense || pc.grid != args.num_m_blocks * args.num_n_blocks * pc.split_k))
    return DG_ERR_UNSUPPORTED;
  // split-K runs one tile per CTA, one cluster per output tile
  if (pc.split_k > 1 &&
      (kind != kDense || pc.grid != args.num_m_blocks * args.num_n_blocks * pc.split_k ||
       rows > kBlockM || !split_fits(var, rows, pc.split_k)))
    return DG_ERR_UNSUPPORTED;

  CUtensorMap ta, tb;
  const int b_groups = (kind == kDense) ? 1 : G;
  const uint32_t elem = bf16 ? 2 : 1;
  s = a_mn ? make_map_mn(&ta, a, rows, K)
           : make_map(&ta, a, K, rows, kind == kMasked ? G : 1, args.a_box_rows, var.kps, elem);
  if (s != DG_OK) return s;
  s = b_mn ? make_map_mn(&tb, b, N, K)
           : make_map(&tb, b, K, N, b_groups, var.pair ? var.block_n / 2 : var.block_n, var.kps,
                      elem);
  if (s != DG_OK) return s;
  CUtensorMap td;
  s = make_d_map(&td, d, N, static_cast<uint64_t>(a_rows));
  if (s != DG_OK) return s;

  if (print_configs())
    std::fprintf(stderr,
                 "[dg] kind=%d rows=%d N=%d K=%d G=%d expected_m=%d -> BLOCK_N=%d stages=%d "
                 "acc=%d split_k=%d grid=%d\n",
                 kind, rows, N, K, G, expected_m, var.block_n, var.stages, var.num_acc,
                 pc.split_k, pc.grid);

  switch (form) {
    case kFormDense: return launch<kFormDense>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormContiguous:
      return launch<kFormContiguous>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormMasked:
      return launch<kFormMasked>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormNN: return launch<kFormNN>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormTN: return launch<kFormTN>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormTT: return launch<kFormTT>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormF32: return launch<kFormF32>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormBf16Dense:
      return launch<kFormBf16Dense>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    case kFormBf16Contiguous:
      return launch<kFormBf16Contiguous>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
    default:
      return launch<kFormBf16Masked>(*st, pc.variant, ta, tb, td, args, pc.grid, stream);
  }
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" {

dg_status dg_fp8_gemm_nt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return run(kFormDense, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_nn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return run(kFormNN, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_tn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return run(kFormTN, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_tt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return run(kFormTT, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_fp8_gemm_nt_f32(const void* a, const float* sfa, const void* b, const float* sfb,
                             const float* c, float* d, int M, int N, int K, dg_stream_t stream) {
  return run(kFormF32, a, sfa, b, sfb, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream), c);
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, void* d, const int* m_indices,
                                              int M_sum, int N, int K, int G,
                                              dg_stream_t stream) {
  return run(kFormContiguous, a, sfa, b, sfb, d, m_indices, nullptr, M_sum, N, K, G, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const float* sfa, const void* b,
                                          const float* sfb, void* d, const int* masked_m, int G,
                                          int max_m, int N, int K, int expected_m,
                                          dg_stream_t stream) {
  return run(kFormMasked, a, sfa, b, sfb, d, nullptr, masked_m, max_m, N, K, G, expected_m,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_bf16_gemm_nt(const void* a, const void* b, void* d, int M, int N, int K,
                          dg_stream_t stream) {
  return run(kFormBf16Dense, a, nullptr, b, nullptr, d, nullptr, nullptr, M, N, K, 1, 0,
             reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_bf16_gemm_nt_contiguous(const void* a, const void* b, void* d,
                                               const int* m_indices, int M_sum, int N, int K,
                                               int G, dg_stream_t stream) {
  return run(kFormBf16Contiguous, a, nullptr, b, nullptr, d, m_indices, nullptr, M_sum, N, K, G,
             0, reinterpret_cast<cudaStream_t>(stream));
}

dg_status dg_m_grouped_bf16_gemm_nt_masked(const void* a, const void* b, void* d,
                                           const int* masked_m, int G, int max_m, int N, int K,
                                           int expected_m, dg_stream_t stream) {
  return run(kFormBf16Masked, a, nullptr, b, nullptr, d, nullptr, masked_m, max_m, N, K, G,
             expected_m, reinterpret_cast<cudaStream_t>(stream));
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
  out->block_m = tile_rows(v);
  out->block_n = v.block_n;
  out->stages = v.stages;
  out->num_acc = v.num_acc;
  out->split_k = pc.split_k;
  out->grid = pc.grid;
  constexpr auto smem = variant_table<0>(std::make_integer_sequence<int, kNumVariants>{});
  constexpr auto tmem = variant_table<1>(std::make_integer_sequence<int, kNumVariants>{});
  out->smem_bytes = smem[pc.variant];
  out->tmem_cols = tmem[pc.variant];
  out->kps = v.kps;
  return DG_OK;
}

const char* dg_version(void) { return "0.1.0"; }

}  // extern "C"
