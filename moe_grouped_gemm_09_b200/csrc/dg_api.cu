// C ABI of the FP8 block-scaled GEMM library: argument checks, per-device
// state, configuration choice, TMA descriptors and kernel launches.
// The operations are declared and documented in include/dg.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <utility>

#include "../../include/dg.h"
#include "dg_internal.h"

namespace dg {
namespace {

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int num_sms = 0;
  int* error_word = nullptr;      // one int, device memory
  bool attr_set[kNumForms][kNumVariants] = {};  // shared-memory limit raised, per form and variant
  bool limits_known = false;
  ClusterLimits limits = {};      // co-resident split-K clusters per variant and size
};

std::mutex g_mutex;
DeviceState g_dev[kMaxDevices];
int g_num_sms_cap = 0;            // 0: all SMs

// Settings every entry point reads (guarded by their own mutex: the no-alloc
// entry point reads them without holding g_mutex).
std::mutex g_settings_mutex;
unsigned long long g_timeout_ns = 1000ull * 1000 * 1000;
bool g_timeout_from_env = false;
int g_check_scales = -1;          // -1: not decided yet (read DG_CHECK_SCALES)
int g_weight_preload = -1;        // -1: not decided yet (read DG_WEIGHT_PRELOAD)

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
std::once_flag g_encode_once;
EncodeTiledFn g_encode = nullptr;

EncodeTiledFn encoder() {
  std::call_once(g_encode_once, [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  });
  return g_encode;
}

bool env_flag(const char* name) {
  const char* e = std::getenv(name);
  return e && e[0] && e[0] != '0';
}

bool print_configs() {
  static const bool v = env_flag("DG_PRINT_CONFIGS");
  return v;
}

// Initialise (once) the state of the current device.  Caller holds g_mutex.
dg_status device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DG_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DG_ERR_UNSUPPORTED;
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return DG_ERR_CUDA;
    if (major != 10 || minor != 0) return DG_ERR_ARCH;
    if (!encoder()) return DG_ERR_CUDA;
    st.num_sms = sms;
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
  return DG_OK;
}

// Rows per TMA box of A: a whole 128-row tile, except that a dense A shorter
// than one 128-row block is fetched with a box of its own (16-row rounded)
// height, so the SM moves no padding.
int a_box_rows(int kind, int rows) {
  if (kind != kDense || rows >= kBlockM) return kBlockM;
  return ((rows + 15) / 16) * 16;
}

// DG_FORCE_CONFIG="<block_n>:<split_k>[:<kps>:<a_rows>[:<mode>]]" overrides
// the picker (tuning sweeps); without kps/a_rows a general (one K block per
// stage) variant; mode 0 general, 1 decode, 2 small decode.
// Ignored unless the variant exists and, for split_k > 1, the problem is a
// dense one with a single 128-row block.
void forced_config(int kind, int rows, int N, int K, int G, int sms, bool f32_out,
                   PickedConfig* pc) {
  const char* e = std::getenv("DG_FORCE_CONFIG");
  if (!e || !e[0]) return;
  int bn = 0, sk = 1;
  if (std::sscanf(e, "%d:%d", &bn, &sk) < 1) return;
  int kps = 0, ar = 0, mode = -1;
  std::sscanf(e, "%*d:%*d:%d:%d:%d", &kps, &ar, &mode);
  int v = -1;
  for (int i = 0; i < kNumVariants; ++i) {
    const Variant& x = kVariants[i];
    if (x.block_n != bn || x.f32 != f32_out) continue;
    if (kps ? (x.kps != kps || (ar && x.a_rows != ar)) : x.decode) continue;
    if (mode >= 0 && (x.small ? 2 : x.decode ? 1 : 0) != mode) continue;
    if (x.decode && kind != kDense) continue;
    if (a_box_rows(kind, rows) > x.a_rows) continue;
    v = i;
  }
  const int KB = K / kBlockK;
  if (v < 0 || sk < 1 || sk > kMaxSplitK || sk > KB) return;
  if (sk > 1 && (kind != kDense || rows > kBlockM)) return;
  if ((sk - 1) * ceil_div(KB, sk) >= KB) return;
  const long long groups = (kind == kMasked || kind == kKGrouped) ? G : 1;
  const long long tiles = groups * ceil_div(rows, tile_rows(kVariants[v])) * ceil_div(N, bn);
  pc->variant = v;
  pc->split_k = sk;
  pc->out_tiles = static_cast<int>(tiles);
  pc->grid = sk > 1 ? static_cast<int>(tiles) * sk : static_cast<int>(tiles < sms ? tiles : sms);
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
  CUresult r = encoder()(map, elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                              : CU_TENSOR_MAP_DATA_TYPE_UINT8,
                         4, const_cast<void*>(base), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 2-D tensor map over the BF16 output D [rows][N], rows ldd elements apart,
// with a box of 32 rows x 64 columns and the 128-byte swizzle (the
// epilogue's staging layout).
dg_status make_d_map(CUtensorMap* map, void* base, uint64_t N, uint64_t rows, uint64_t ldd) {
  cuuint64_t dims[2] = {N, rows};
  cuuint64_t strides[1] = {ldd * 2};
  cuuint32_t box[2] = {64, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encoder()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 3-D tensor map over an FP32 output D [groups][rows][N] (the FP32-output
// forms: groups = 1 for the dense one) with a box of 32 rows x 16 columns
// (64 bytes) and the 64-byte swizzle; rows past a group's end and columns
// past N are clipped by the TMA unit.
dg_status make_d_map_f32(CUtensorMap* map, void* base, uint64_t N, uint64_t rows, uint64_t groups) {
  cuuint64_t dims[3] = {N, rows, groups};
  cuuint64_t strides[2] = {N * 4, rows * N * 4};
  cuuint32_t box[3] = {16, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = encoder()(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                         CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

// 2-D tensor map over an M-/N-major operand stored as [K, mn] bytes (mn
// contiguous), boxes of 128 mn bytes x 128 K rows with the 128-byte swizzle.
dg_status make_map_mn(CUtensorMap* map, const void* base, uint64_t mn, uint64_t K) {
  cuuint64_t dims[2] = {mn, K};
  cuuint64_t strides[1] = {mn};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = encoder()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_CUDA;
}

int effective_sms(const DeviceState& st) {
  int n = st.num_sms;
  if (g_num_sms_cap > 0 && g_num_sms_cap < n) n = g_num_sms_cap;
  return n;
}

dg_status launch_plan(DeviceState& st, const LaunchPlan& pl, cudaStream_t stream) {
  bool* row = st.attr_set[pl.form];
  switch (pl.form) {
    case kFormDense: return launch_fp8_dense(row, pl, stream);
    case kFormContiguous:
    case kFormMasked: return launch_fp8_grouped(row, pl, stream);
    case kFormNN:
    case kFormTN:
    case kFormTT:
    case kFormF32:
    case kFormKGrouped: return launch_fp8_layouts(row, pl, stream);
    case kFormBf16Dense: return launch_bf16_dense(row, pl, stream);
    default: return launch_bf16_grouped(row, pl, stream);
  }
}

// Shared path of every GEMM entry point.
dg_status run(const GemmCall& call, cudaStream_t stream) {
  bool empty = false;
  dg_status s = check_gemm_call(call, &empty);  // before any device work
  if (s != DG_OK || empty) return s;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  s = device_state(&st);
  if (s != DG_OK) return s;
  if (kind_of_form(call.form) == kDense && !st->limits_known) {
    s = query_decode_cluster_limits(st->attr_set[kFormDense], &st->limits);
    if (s != DG_OK) return s;
    st->limits_known = true;
  }
  LaunchPlans plans;
  s = plan_gemm(call, DeviceFacts{effective_sms(*st), &st->limits}, st->error_word, &plans);
  if (s != DG_OK || plans.n == 0) return s;
  if (!is_bf16_form(call.form) && check_scales_enabled()) {
    s = launch_scale_check(call, st->error_word, stream);
    if (s != DG_OK) return s;
  }
  for (int i = 0; i < plans.n && s == DG_OK; ++i) s = launch_plan(*st, plans.plan[i], stream);
  return s;
}

// Checks n scales against the contract and records kDevBadScale if one breaks
// it.  Launched before a GEMM only when the check is turned on; the GEMM
// kernels themselves use the exponent byte without looking at the rest.
__global__ void check_scales_kernel(const float* __restrict__ s, long long n, int* error_word) {
  bool bad = false;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    bad |= !scale_ok(__ldg(s + i));
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicCAS(error_word, 0, kDevBadScale);
}

}  // namespace

int weight_preload_enabled() {
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  if (g_weight_preload < 0) g_weight_preload = env_flag("DG_WEIGHT_PRELOAD") ? 1 : 0;
  return g_weight_preload;
}

dg_status launch_scale_check(const GemmCall& call, int* error_word, cudaStream_t stream) {
  const int kind = kind_of_form(call.form);
  const long long kb = call.K / kBlockK;
  const long long a_rows = kind == kMasked ? static_cast<long long>(call.G) * call.rows : call.rows;
  // (K-grouped: one sfa [M, K/128] and one sfb for all groups)
  const long long b_groups = (kind == kDense || kind == kKGrouped) ? 1 : call.G;
  const long long n_sfa = a_rows * kb;
  const long long n_sfb = b_groups * ceil_div(call.N, 128) * kb;
  for (const auto& t : {std::make_pair(call.sfa, n_sfa), std::make_pair(call.sfb, n_sfb)}) {
    const int blocks = static_cast<int>(std::min<long long>((t.second + 255) / 256, 1024));
    check_scales_kernel<<<blocks, 256, 0, stream>>>(t.first, t.second, error_word);
    if (cudaGetLastError() != cudaSuccess) return DG_ERR_CUDA;
  }
  return DG_OK;
}

unsigned long long wait_timeout_ns() {
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  if (!g_timeout_from_env) {
    g_timeout_from_env = true;
    const char* e = std::getenv("DG_WAIT_TIMEOUT_MS");
    if (e && std::atoi(e) > 0) g_timeout_ns = 1000000ull * std::atoi(e);
  }
  return g_timeout_ns;
}

// L2 prefetch of the first tile before the dependency wait; DG_NO_PREFETCH=1
// turns it off (for measurements).
int prefetch_enabled() {
  static const int v = env_flag("DG_NO_PREFETCH") ? 0 : 1;
  return v;
}

// The kernels check every scale they read against the contract (a positive
// normal power of two) and report device error 0x301: off unless
// DG_CHECK_SCALES=1 or dg_set_check_scales(1).
int check_scales_enabled() {
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  if (g_check_scales < 0) g_check_scales = env_flag("DG_CHECK_SCALES") ? 1 : 0;
  return g_check_scales;
}

dg_status check_gemm_call(const GemmCall& call, bool* empty) {
  const int form = call.form;
  const int kind = kind_of_form(form);
  const int layout = layout_of_form(form);
  const bool a_mn = (layout & 1) != 0;
  const bool bf16 = is_bf16_form(form);
  const int rows = call.rows, N = call.N, K = call.K, G = call.G;
  *empty = false;
  // A K block is 128 bytes of a row: 128 E4M3 or 64 BF16 elements.
  const int k_block = bf16 ? kBlockK / 2 : kBlockK;
  if (rows < 0 || G < 0) return DG_ERR_INVALID_ARG;
  if (K <= 0 || K % k_block != 0 || N <= 0 || N % 16 != 0) return DG_ERR_INVALID_ARG;
  if (rows == 0 || G == 0) {
    *empty = true;
    return DG_OK;
  }
  if (!call.a || !call.b || !call.d || (!bf16 && (!call.sfa || !call.sfb)))
    return DG_ERR_INVALID_ARG;
  if (!aligned(call.a, 16) || !aligned(call.b, 16) || !aligned(call.d, 16) ||
      (!bf16 && (!aligned(call.sfa, 4) || !aligned(call.sfb, 4))))
    return DG_ERR_INVALID_ARG;
  if (kind == kContiguous &&
      (!call.m_indices || !aligned(call.m_indices, 4) || rows % 128 != 0))
    return DG_ERR_INVALID_ARG;
  if (a_mn && rows % 16 != 0) return DG_ERR_INVALID_ARG;  // [K, M] rows of whole 16-byte units
  if (is_f32_form(form) && call.c && !aligned(call.c, 16)) return DG_ERR_INVALID_ARG;
  if (kind == kMasked && (!call.masked_m || !aligned(call.masked_m, 4))) return DG_ERR_INVALID_ARG;
  if (kind == kKGrouped && (!call.ks || !aligned(call.ks, 4))) return DG_ERR_INVALID_ARG;
  if ((kind == kMasked || kind == kKGrouped) && G > kMaxMaskedGroups) return DG_ERR_UNSUPPORTED;
  // rows of D (and of A for the masked form)
  const long long a_rows =
      (kind == kMasked || kind == kKGrouped) ? static_cast<long long>(G) * rows : rows;
  if (a_rows > 0x7fffffffLL || static_cast<long long>(G) * N > 0x7fffffffLL)
    return DG_ERR_UNSUPPORTED;
  if (K > (1 << 24)) return DG_ERR_UNSUPPORTED;
  return DG_OK;
}

namespace {

// The last-wave split (see plan_tail) is on unless DG_NO_TAIL_SPLIT=1 (read
// at every call, like DG_FORCE_CONFIG, for measurements).
bool tail_split_enabled() { return !env_flag("DG_NO_TAIL_SPLIT"); }

// Fills one launch of `call` (the whole problem, or a rectangle of D with A,
// B and their scales offset to it): kernel arguments and tensor maps for the
// given variant, split and grid; `ldd` is the row stride of D in elements and
// `tile_limit` (> 0) stops the dense form after that many tiles.
dg_status fill_plan(const GemmCall& call, int variant, int split, int grid, int ldd,
                    int tile_limit, int* error_word, LaunchPlan* pl) {
  const int form = call.form;
  const int kind = kind_of_form(form);
  const int layout = layout_of_form(form);
  const bool a_mn = (layout & 1) != 0, b_mn = (layout & 2) != 0;
  const bool bf16 = is_bf16_form(form);
  const int rows = call.rows, N = call.N, K = call.K, G = call.G;
  const long long a_rows =
      (kind == kMasked || kind == kKGrouped) ? static_cast<long long>(G) * rows : rows;
  const int k_bytes = bf16 ? 2 * K : K;
  const Variant var = kVariants[variant];
  if ((layout != kLayoutNT || is_f32_form(form)) && (!mn_capable(var) || split > 1))
    return DG_ERR_UNSUPPORTED;

  GemmArgs& args = pl->args;
  args = GemmArgs{};
  args.rows = rows;
  args.N = N;
  args.K = K;
  args.G = (kind == kDense) ? 1 : G;  // K-grouped: groups of K, one D each
  args.num_m_blocks = ceil_div(rows, tile_rows(var));
  args.num_n_blocks = ceil_div(N, var.block_n);
  args.k_blocks = k_bytes / kBlockK;
  args.split_k = split;
  args.kb_per_split = ceil_div(args.k_blocks, split);
  args.nb128 = ceil_div(N, 128);
  args.sfa = call.sfa;
  args.sfb = call.sfb;
  args.d = static_cast<__nv_bfloat16*>(call.d);
  args.ldd = ldd;
  args.d_f32 = is_f32_form(form) ? static_cast<float*>(call.d) : nullptr;
  args.c_f32 = is_f32_form(form) ? call.c : nullptr;
  args.ks = call.ks;
  args.m_indices = call.m_indices;
  args.masked_m = call.masked_m;
  args.error_word = error_word;
  args.timeout_ns = wait_timeout_ns();
  args.a_box_rows = a_mn ? kBlockM : a_box_rows(kind, rows);
  args.prefetch = prefetch_enabled();
  args.preload_b = kind == kDense ? weight_preload_enabled() : 0;
  args.tile_limit = tile_limit;
  if (args.a_box_rows > var.a_rows) return DG_ERR_UNSUPPORTED;
  // a decode variant runs one tile per CTA (its epilogue reuses the ring)
  const long long tiles = static_cast<long long>(args.num_m_blocks) * args.num_n_blocks;
  if (var.decode && (kind != kDense || tile_limit != 0 || grid != tiles * split))
    return DG_ERR_UNSUPPORTED;
  // split-K runs one tile per CTA, one cluster per output tile
  if (split > 1 && (kind != kDense || tile_limit != 0 || grid != tiles * split ||
                    !split_fits(var, rows < kBlockM ? rows : kBlockM, split)))
    return DG_ERR_UNSUPPORTED;

  const int b_groups = (kind == kDense) ? 1 : G;
  const uint32_t elem = bf16 ? 2 : 1;
  dg_status s = a_mn ? make_map_mn(&pl->ta, call.a, rows, K)
                     : make_map(&pl->ta, call.a, K, rows, kind == kMasked ? G : 1,
                                args.a_box_rows, var.kps, elem);
  if (s != DG_OK) return s;
  s = b_mn ? make_map_mn(&pl->tb, call.b, N, K)
           : make_map(&pl->tb, call.b, K, N, b_groups, var.block_n, var.kps, elem);
  if (s != DG_OK) return s;
  s = is_f32_form(form)
          ? make_d_map_f32(&pl->td, call.d, N, rows, kind == kKGrouped ? G : 1)
          : make_d_map(&pl->td, call.d, N, static_cast<uint64_t>(a_rows), ldd);
  if (s != DG_OK) return s;

  if (print_configs())
    std::fprintf(stderr,
                 "[dg] form=%d rows=%d N=%d K=%d G=%d expected_m=%d -> BLOCK_N=%d stages=%d "
                 "kps=%d acc=%d split_k=%d grid=%d tile_limit=%d\n",
                 form, rows, N, K, G, call.expected_m, var.block_n, var.stages, var.kps,
                 var.num_acc, split, grid, tile_limit);
  pl->form = form;
  pl->variant = variant;
  pl->grid = grid;
  return DG_OK;
}

}  // namespace

dg_status plan_gemm(const GemmCall& call, const DeviceFacts& facts, int* error_word,
                    LaunchPlans* plans) {
  plans->n = 0;
  bool empty = false;
  dg_status s = check_gemm_call(call, &empty);
  if (s != DG_OK || empty) return s;
  const int form = call.form;
  const int kind = kind_of_form(form);
  const int layout = layout_of_form(form);
  const bool bf16 = is_bf16_form(form);
  const int rows = call.rows, N = call.N, K = call.K, G = call.G;
  // the picker and the kernel count K in 128-byte blocks of a row
  const int k_bytes = bf16 ? 2 * K : K;
  const int sms = facts.num_sms;

  PickedConfig pc = pick_config(kind, rows, N, k_bytes, G, call.expected_m, sms, facts.limits,
                                /*mn_operands=*/layout != kLayoutNT || is_f32_form(form),
                                /*f32_out=*/is_f32_form(form));
  const PickedConfig picked = pc;
  forced_config(kind, rows, N, k_bytes, G, sms, is_f32_form(form), &pc);
  const bool forced = pc.variant != picked.variant || pc.split_k != picked.split_k;

  TailPlan tp;
  if (kind == kDense && layout == kLayoutNT && !is_f32_form(form) && !forced &&
      tail_split_enabled())
    tp = plan_tail(rows, N, k_bytes, sms, pc.variant, facts.limits);
  const int main_grid = tp.main_tiles > 0 && tp.main_tiles < pc.grid ? tp.main_tiles : pc.grid;
  s = fill_plan(call, pc.variant, pc.split_k, main_grid, N, tp.main_tiles, error_word,
                &plans->plan[0]);
  if (s != DG_OK) return s;
  plans->n = 1;
  // tail launches: a rectangle of D each, A and B (and their scales) offset
  // to its first row and column
  const size_t elem = bf16 ? 2 : 1;
  const int KB = k_bytes / kBlockK;
  for (int i = 0; i < tp.n_rects; ++i) {
    const TailRect& r = tp.rect[i];
    GemmCall sub = call;
    sub.a = static_cast<const uint8_t*>(call.a) + static_cast<size_t>(r.row0) * K * elem;
    sub.b = static_cast<const uint8_t*>(call.b) + static_cast<size_t>(r.col0) * K * elem;
    if (!bf16) {
      sub.sfa = call.sfa + static_cast<size_t>(r.row0) * KB;
      sub.sfb = call.sfb + static_cast<size_t>(r.col0 / 128) * KB;
    }
    sub.d = static_cast<uint8_t*>(call.d) +
            (static_cast<size_t>(r.row0) * N + r.col0) * sizeof(__nv_bfloat16);
    sub.rows = r.rows;
    sub.N = r.cols;
    const int tiles = ceil_div(r.rows, 128) * ceil_div(r.cols, kVariants[tp.variant].block_n);
    s = fill_plan(sub, tp.variant, tp.split, tiles * tp.split, N, 0, error_word,
                  &plans->plan[plans->n]);
    if (s != DG_OK) return s;
    ++plans->n;
  }
  return DG_OK;
}

}  // namespace dg

using namespace dg;

namespace {

cudaStream_t as_stream(dg_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

dg_status dense_call(int form, const void* a, const float* sfa, const void* b, const float* sfb,
                     void* d, int M, int N, int K, dg_stream_t stream, const float* c = nullptr) {
  GemmCall call{form, a, sfa, b, sfb, d, c, nullptr, nullptr, M, N, K, 1, 0};
  return run(call, as_stream(stream));
}

}  // namespace

extern "C" {

dg_status dg_fp8_gemm_nt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return dense_call(kFormDense, a, sfa, b, sfb, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_nn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return dense_call(kFormNN, a, sfa, b, sfb, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_tn(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return dense_call(kFormTN, a, sfa, b, sfb, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_tt(const void* a, const float* sfa, const void* b, const float* sfb,
                         void* d, int M, int N, int K, dg_stream_t stream) {
  return dense_call(kFormTT, a, sfa, b, sfb, d, M, N, K, stream);
}

dg_status dg_fp8_gemm_nt_f32(const void* a, const float* sfa, const void* b, const float* sfb,
                             const float* c, float* d, int M, int N, int K, dg_stream_t stream) {
  return dense_call(kFormF32, a, sfa, b, sfb, d, M, N, K, stream, c);
}

dg_status dg_m_grouped_fp8_gemm_nt_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, void* d, const int* m_indices,
                                              int M_sum, int N, int K, int G,
                                              dg_stream_t stream) {
  GemmCall call{kFormContiguous, a, sfa, b, sfb, d, nullptr, m_indices, nullptr, M_sum, N, K, G, 0};
  return run(call, as_stream(stream));
}

dg_status dg_m_grouped_fp8_gemm_nt_masked(const void* a, const float* sfa, const void* b,
                                          const float* sfb, void* d, const int* masked_m, int G,
                                          int max_m, int N, int K, int expected_m,
                                          dg_stream_t stream) {
  GemmCall call{kFormMasked, a, sfa, b, sfb, d, nullptr, nullptr, masked_m, max_m, N, K, G,
                expected_m};
  return run(call, as_stream(stream));
}

dg_status dg_k_grouped_fp8_gemm_tn_contiguous(const void* a, const float* sfa, const void* b,
                                              const float* sfb, const float* c, float* d,
                                              const int* ks, int G, int M, int N, int K_sum,
                                              dg_stream_t stream) {
  GemmCall call{kFormKGrouped, a, sfa, b, sfb, d, c, nullptr, nullptr, M, N, K_sum, G, 0, ks};
  return run(call, as_stream(stream));
}

dg_status dg_bf16_gemm_nt(const void* a, const void* b, void* d, int M, int N, int K,
                          dg_stream_t stream) {
  return dense_call(kFormBf16Dense, a, nullptr, b, nullptr, d, M, N, K, stream);
}

dg_status dg_m_grouped_bf16_gemm_nt_contiguous(const void* a, const void* b, void* d,
                                               const int* m_indices, int M_sum, int N, int K,
                                               int G, dg_stream_t stream) {
  GemmCall call{kFormBf16Contiguous, a, nullptr, b, nullptr, d, nullptr, m_indices, nullptr,
                M_sum, N, K, G, 0};
  return run(call, as_stream(stream));
}

dg_status dg_m_grouped_bf16_gemm_nt_masked(const void* a, const void* b, void* d,
                                           const int* masked_m, int G, int max_m, int N, int K,
                                           int expected_m, dg_stream_t stream) {
  GemmCall call{kFormBf16Masked, a, nullptr, b, nullptr, d, nullptr, nullptr, masked_m, max_m,
                N, K, G, expected_m};
  return run(call, as_stream(stream));
}

dg_status dg_set_num_sms(int n) {
  std::lock_guard<std::mutex> lock(g_mutex);
  g_num_sms_cap = n > 0 ? n : 0;
  return DG_OK;
}

int dg_get_num_sms(void) {
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  if (device_state(&st) != DG_OK) return -1;
  return effective_sms(*st);
}

dg_status dg_get_last_device_error(int* code) {
  if (!code) return DG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mutex);
  DeviceState* st = nullptr;
  dg_status s = device_state(&st);
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

dg_status dg_set_wait_timeout_ns(long long ns) {
  if (ns <= 0) return DG_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  g_timeout_from_env = true;
  g_timeout_ns = static_cast<unsigned long long>(ns);
  return DG_OK;
}

dg_status dg_set_weight_preload(int enable) {
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  g_weight_preload = enable ? 1 : 0;
  return DG_OK;
}

dg_status dg_set_check_scales(int enable) {
  std::lock_guard<std::mutex> lock(g_settings_mutex);
  g_check_scales = enable ? 1 : 0;
  return DG_OK;
}

dg_status dg_set_wait_timeout_ms(int ms) {
  if (ms <= 0) return DG_ERR_INVALID_ARG;
  return dg_set_wait_timeout_ns(1000000LL * ms);
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
  if (!out || kind < 0 || kind > 3 || rows < 0 || N <= 0 || N % 16 != 0 || K <= 0 ||
      K % 128 != 0 || G < 1 || num_sms < 1)
    return DG_ERR_INVALID_ARG;
  const PickedConfig pc = pick_config(kind, rows, N, K, G, expected_m, num_sms, nullptr,
                                      /*mn_operands=*/kind == kKGrouped,
                                      /*f32_out=*/kind == kKGrouped);
  const Variant v = kVariants[pc.variant];
  out->block_m = tile_rows(v);
  out->block_n = v.block_n;
  out->stages = v.stages;
  out->num_acc = v.num_acc;
  out->split_k = pc.split_k;
  out->grid = pc.grid;
  out->smem_bytes = variant_smem_bytes(pc.variant);
  out->tmem_cols = variant_tmem_cols(pc.variant);
  out->kps = v.kps;
  TailPlan tp;
  if (kind == kDense) tp = plan_tail(rows, N, K, num_sms, pc.variant, nullptr);
  out->main_tiles = tp.main_tiles;
  out->tail_launches = tp.n_rects;
  out->tail_split = tp.n_rects ? tp.split : 0;
  if (tp.main_tiles > 0 && tp.main_tiles < out->grid) out->grid = tp.main_tiles;
  return DG_OK;
}

const char* dg_version(void) { return "0.2.0"; }

}  // extern "C"
