// FP8 (E4M3) block-scaled GEMM D = A * B^T for sm_100a, dense and MoE
// M-grouped (contiguous and masked layouts); the same kernel template also
// serves BF16 operands without scales (BF16 = true).
//
// What it computes (DeepGEMM release article, deepseek.csdn.net, part 1.2;
// DeepGEMM project card, aiproducthub.cn, "core features" and "technical
// implementation"):
//   D[m, n] = bf16( sum_kb sfa[m, kb] * sfb[n / 128, kb] * sum_{k in kb} a[m, k] * b[n, k] )
// with A [rows, K] and B [N, K] both K-major E4M3, FP32 power-of-two scales
// (A: one per row per 128-wide K block; B: one per 128 x 128 block), FP32
// accumulation and one BF16 rounding.
//
// Design (B200-first; the pages' Hopper design -- warp-specialised wgmma with
// CUDA-core promotion every K block and SASS-level FFMA interleaving -- is
// prior art only):
//  * The fine-grained scales are applied inside the tensor core: every
//    128-wide K block is four tcgen05.mma.kind::mxf8f6f4.block_scale
//    instructions (K = 32 each) whose UE8M0 scale factors sit in TMEM.  A
//    power-of-two FP32 scale is exactly a UE8M0 byte (its exponent field), so
//    this is the pages' per-block scaling with the FP32 promotion done by the
//    MMA itself; the accumulator lives in TMEM for the whole K loop.
//  * Warp roles in a 256-thread CTA: warp 0 issues TMA loads of A and B tiles
//    (128-byte swizzle) into a multi-stage shared-memory ring; warp 1 owns the
//    TMEM allocation and issues tcgen05.cp (scales) + tcgen05.mma; warp 2
//    turns the FP32 scales into the UE8M0 layout that tcgen05.cp expects,
//    loading them several stages ahead so that their latency stays hidden.
//    One set of scale words serves up to four consecutive K blocks (one per
//    byte, chosen by the MMA's scale-factor id): the two or four K blocks of
//    a decode variant's stage, or four one-block stages in the others, so the
//    copy into TMEM is not paid for every K block;
//    warps 4..7 drain the TMEM accumulator (tcgen05.ld), convert to BF16 and
//    store.
//  * Split-K (decode shapes, too few output tiles for the SMs): the CTAs that
//    share an output tile form one thread-block cluster, each computes the
//    partial sum of its K slice and parks it in its own shared memory; after
//    a cluster barrier every CTA pushes the rows each other CTA owns to that
//    CTA with one bulk copy (distributed shared memory), and every CTA sums
//    the partials of its own rows in a fixed order (deterministic), then
//    stores BF16.  No global scratch is used.
//  * Before waiting on the previous kernel (programmatic dependent launch),
//    the producer asks TMA to prefetch its first tile's operands into L2.
//  * A single-tile CTA (decode) drains its accumulator with all eight warps.
//  * Persistent CTAs walk a static tile sequence.  For the grouped layouts the
//    sequence is group-aware: contiguous tiles read their expert from
//    m_indices and skip all-padding blocks; masked tiles are enumerated over
//    the valid (group, m-block) pairs only, from masked_m read on the device.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_ptx.cuh"

namespace dg {

// kKGrouped: the reduction axis is grouped (the weight gradient of the MoE
// grouped forms in training): group g sums the K rows [k_off[g], k_off[g] +
// ks[g]) of A [K_sum, M] and B [K_sum, N] into its own FP32 output D[g].
enum GemmKind : int { kDense = 0, kContiguous = 1, kMasked = 2, kKGrouped = 3 };

// Operand layouts of the dense form (DeepGEMM project card, core features:
// NT / NN / TN / TT on SM100).  Bit 0: A is M-major ([K, M] in memory);
// bit 1: B is N-major ([K, N]).  NT, both K-major, is the grouped forms' only one.
enum GemmLayout : int { kLayoutNT = 0, kLayoutTT = 1, kLayoutNN = 2, kLayoutTN = 3 };

// Device error codes (also the values reported through the C ABI).
enum DeviceError : int {
  kDevOk = 0,
  kDevTimeoutProducer = 0x101,
  kDevTimeoutScales = 0x102,
  kDevTimeoutMma = 0x103,
  kDevTimeoutEpilogue = 0x104,
  kDevMixedExperts = 0x201,   // a 128-row block of m_indices names two experts
  kDevExpertRange = 0x202,    // an m_indices entry is >= G
  kDevKGroups = 0x203,        // K-grouped: group sizes negative, not multiples of 128, or not
                              // summing to K (nothing is computed)
  kDevBadScale = 0x301,       // a scale that is not a positive normal power of two (reported
                              // by check_scales_kernel, launched only on request)
};

struct GemmArgs {
  int rows;          // dense: M; contiguous: M_sum; masked: max_m (rows per group)
  int N, K, G;
  int num_m_blocks;  // m-blocks per group: ceil(rows / 128)
  int num_n_blocks;  // ceil(N / BLOCK_N)
  int k_blocks;      // K / 128
  int split_k;       // K slices per output tile; > 1: cluster of split_k CTAs per tile,
                     // launched with exactly one tile per CTA
  int kb_per_split;  // ceil(k_blocks / split_k)
  int nb128;         // ceil(N / 128): B scale blocks along N
  const float* sfa;  // [G * rows, k_blocks]   (dense/contiguous: G = 1 row space)
  const float* sfb;  // [G, nb128, k_blocks]
  __nv_bfloat16* d;  // [G * rows, N], rows ldd elements apart
  int ldd;           // BF16 D: row stride in elements (N; larger for a sub-block of D)
  float* d_f32;      // FP32 output form: D [rows, N] (d unused)
  const float* c_f32;  // FP32 output form: C [rows, N] added to the product, or null
  const int* m_indices;  // contiguous: [rows]
  const int* masked_m;   // masked: [G]
  const int* ks;         // K-grouped: rows of K of each group [G]
  int* error_word;
  unsigned long long timeout_ns;
  int a_box_rows;    // rows of A one TMA box brings (128, or fewer for a short dense A)
  int prefetch;      // 1: warm L2 with the first tile before waiting on the previous kernel
  int preload_b;     // 1 (dense form): B is constant while kernels run (weights), so the
                     // first ring stages of B may be loaded before that wait
  int tile_limit;    // dense form: > 0: compute only the first tile_limit output tiles of
                     // the tile order (the rest go to a launch of their own)
};

constexpr int kBlockM = 128;
constexpr int kBlockK = 128;
constexpr int kThreads = 256;
constexpr int kMaxMaskedGroups = 1024;
constexpr int kMaxSplit = 8;  // CTAs per split-K cluster (portable cluster size)

__host__ __device__ constexpr int pow2_ceil(int x) {
  int p = 32;
  while (p < x) p <<= 1;
  return p;
}

// Compile-time geometry of one kernel variant.
//   BLOCK_N  output columns (rows of B) per tile
//   STAGES   depth of the shared-memory operand ring
//   NUM_ACC  TMEM accumulator buffers (2: the epilogue of a tile overlaps the
//            next tile's main loop)
//   KPS      128-wide K blocks per ring stage: every stage is one TMA box of A
//            and one of B, each KPS K blocks deep (bigger boxes stream faster)
//   A_ROWS   rows of A a stage holds room for (64 for a dense A of at most 64
//            rows, else 128)
//   MODE     0: general (persistent CTAs, any number of tiles each);
//            1: decode (dense form, one tile per CTA, split-K capable, the
//            epilogue staged in the then idle operand ring);
//            2: small decode, as 1 but small enough (shared memory and TMEM)
//            for two CTAs per SM, so that the next kernel's CTAs can start
//            (and warm L2) while this kernel drains
//   SCALED   block-scaled E4M3 operands (scale factors staged per stage in
//            shared memory and TMEM); false for BF16 operands, whose K block
//            is 64 elements, the same 128 bytes of a row
template <int BLOCK_N, int STAGES, int NUM_ACC, int KPS = 1, int A_ROWS = 128, int MODE = 0,
          bool SCALED = true, bool F32EPI = false>
struct KernelShape {
  static constexpr bool kSmall = MODE == 2;
  static constexpr int kABytes = KPS * A_ROWS * kBlockK;  // kBlockK bytes of a row per K block
  static constexpr int kBBytes = KPS * BLOCK_N * kBlockK;
  static constexpr int kSfbChunks = (BLOCK_N + 127) / 128;
  // 128-row scale blocks of B one tile can touch (a tile that is not aligned
  // to 128 rows straddles one more)
  static constexpr int kSfbBlocks = kSfbChunks + (BLOCK_N % 128 != 0 && 128 % BLOCK_N != 0 ? 1 : 0);
  // SFA 512 B per 128 rows of A + SFB 512 B per 128 rows of B
  static constexpr int kSfBytes = SCALED ? 512 * (1 + kSfbChunks) : 0;
  static constexpr int kSfCols = SCALED ? 4 * (1 + kSfbChunks) : 0;  // TMEM columns per stage
  // stages whose K blocks share one set of scale words: four one-block
  // stages; a stage of several K blocks has words of its own (the decode
  // variants, where the per-stage scale path measured faster)
  static constexpr int kSfGroup = KPS == 1 ? 4 : 1;
  static constexpr int kAccCols = NUM_ACC * BLOCK_N;
  static constexpr int kTmemCols = pow2_ceil(kAccCols + STAGES * kSfCols);
  static constexpr int kBarBytes = 8 * (2 * STAGES + 2 * NUM_ACC + 2);
  // epilogue: each of the 4 epilogue warps stages 32 rows x kEpiCols BF16
  // columns in shared memory (16-byte chunks XOR-swizzled by row, the layout
  // of the 128-byte TMA swizzle), then stores them with one TMA box or with
  // whole row segments
  static constexpr int kEpiCols = BLOCK_N % 64 == 0 ? 64 : 32;
  static constexpr int kEpiPitch = kEpiCols * 2;        // bytes per staged row
  // Decode variants serve the dense form only and run one tile per CTA:
  // their epilogue stages in the idle operand ring (no staging region of its
  // own) and they need no masked-group prefix.
  static constexpr bool kDecode = MODE != 0;
  // (FP32-output forms: 16 KB per warp, two halves of four 2 KB boxes)
  static constexpr int kF32Bufs = 8;
  static constexpr int kEpiBytes = kDecode ? 0 : F32EPI ? 4 * kF32Bufs * 2048 : 4 * 32 * kEpiPitch;
  // tmem slot, flags, and (grouped forms) the masked or K-group prefix
  static constexpr int kMiscBytes = 16 + (kDecode ? 0 : 4 * (kMaxMaskedGroups + 1));
  // A short A tile is read by the 128-row MMA past its end (rows that only
  // feed never-stored accumulator rows); the B ring follows the A ring, so
  // that read stays inside this CTA's shared memory.
  static constexpr int kSmemBytes = 1024 /* alignment slack */ + STAGES * (kABytes + kBBytes) +
                                    STAGES * kSfBytes + kEpiBytes + kBarBytes + kMiscBytes;
  static_assert(kSmemBytes <= 232448, "shared memory budget (227 KB) exceeded");
  static_assert(!kSmall || (kSmemBytes <= 115712 && kTmemCols <= 256),
                "a small variant must leave room for a second CTA on its SM");
  static_assert(STAGES * (kABytes + kBBytes) >= 8 * BLOCK_N * 64,
                "a single-tile CTA stages its whole output tile in the ring");
  static_assert(kTmemCols <= 512, "TMEM budget exceeded");
  static_assert(BLOCK_N % 32 == 0 && BLOCK_N >= 32 && BLOCK_N <= 256, "BLOCK_N");
  static_assert(KPS >= 1 && KPS <= 4 && 4 % KPS == 0,
                "four K blocks (a whole number of stages) share one scale-factor word");
  static_assert(A_ROWS == 64 || A_ROWS == 128, "A_ROWS");
  static_assert((BLOCK_N * kBlockK) % 1024 == 0, "B sub-tiles must keep 1024-byte alignment");
};

struct Tile {
  int m_blk, n_blk, group, split, kb_begin, kb_end, out_tile;
  bool skip;
};

// A positive power-of-two FP32 value is 2^(e-127) with e its exponent field;
// UE8M0 encodes 2^(e-127) as the byte e.
__device__ __forceinline__ uint32_t ue8m0(float v) { return (__float_as_uint(v) >> 23) & 0xFFu; }

// The scales' contract: a positive normal power of two (sign 0, mantissa 0,
// exponent field neither 0 nor 255), the only values whose exponent byte is
// the whole value.
__device__ __forceinline__ bool scale_ok(float v) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t e = (u >> 23) & 0xFFu;
  return (u & 0x807FFFFFu) == 0 && e != 0 && e != 0xFFu;
}

// Expert of a 128-row block in the contiguous layout: the largest m_indices
// entry of the block (padding rows are -1).  Warp-collective.
__device__ __forceinline__ int block_expert(const int* m_indices, int row0, int rows, int lane) {
  int e = -1;
#pragma unroll
  for (int i = 0; i < kBlockM / 32; ++i) {
    int r = row0 + i * 32 + lane;
    if (r < rows) e = max(e, __ldg(m_indices + r));
  }
  return __reduce_max_sync(0xFFFFFFFFu, e);
}

// The t-th tile of the static sequence.  Warp-collective for the contiguous
// layout (all 32 lanes must call it with the same t).
template <int KIND>
__device__ __forceinline__ Tile get_tile(int t, const GemmArgs& p, const int* s_prefix, int lane) {
  Tile ti;
  const int S = p.split_k;
  ti.split = t % S;
  const int u = t / S;
  ti.out_tile = u;
  ti.skip = false;
  if (KIND == kMasked) {
    // find the group whose unit range holds u (binary search over the prefix)
    int lo = 0, hi = p.G;  // invariant: s_prefix[lo] <= u < s_prefix[hi]
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (s_prefix[mid] <= u) lo = mid; else hi = mid;
    }
    const int local = u - s_prefix[lo];
    const int mb = (s_prefix[lo + 1] - s_prefix[lo]) / p.num_n_blocks;  // m-blocks of group lo
    ti.group = lo;
    ti.n_blk = local / mb;
    ti.m_blk = local % mb;
  } else if (KIND == kDense) {
    // column-major over tiles: the CTAs of one wave share a few B column
    // tiles and read every A row block
    ti.m_blk = u % p.num_m_blocks;
    ti.n_blk = u / p.num_m_blocks;
    ti.group = 0;
  } else if (KIND == kKGrouped) {
    // every group has the same output tiles; its K range comes from the
    // prefix of the group sizes (in K blocks); a group without K rows still
    // has its output written (C, or zeros) by the epilogue
    const int tpg = p.num_m_blocks * p.num_n_blocks;
    ti.group = u / tpg;
    const int local = u - ti.group * tpg;
    ti.m_blk = local % p.num_m_blocks;
    ti.n_blk = local / p.num_m_blocks;
    ti.kb_begin = s_prefix[ti.group];
    ti.kb_end = s_prefix[ti.group + 1];
    ti.skip = ti.kb_begin >= ti.kb_end;
    return ti;
  } else {
    // row-major over tiles: the CTAs of one wave cover a few consecutive
    // 128-row blocks (one or a few experts) and all their column tiles, so
    // each expert's B streams from HBM about once and is reused from L2
    ti.m_blk = u / p.num_n_blocks;
    ti.n_blk = u % p.num_n_blocks;
    ti.group = block_expert(p.m_indices, ti.m_blk * kBlockM, p.rows, lane);
    ti.skip = (ti.group < 0) || (ti.group >= p.G);
  }
  ti.kb_begin = ti.split * p.kb_per_split;
  ti.kb_end = min(p.k_blocks, ti.kb_begin + p.kb_per_split);
  if (ti.kb_begin >= ti.kb_end) ti.skip = true;
  return ti;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Barrier over `nthreads` threads that also ANDs a predicate across them: every
// participant leaves with the same answer.
__device__ __forceinline__ bool named_bar_and(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, %2, %3, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Walks the tiles one CTA owns (t = first, first + stride, ...), skipping
// tiles with no work.  Warp-collective for the contiguous layout.
template <int KIND>
struct TileWalker {
  int t, stride, total;
  Tile ti;
  bool valid;

  __device__ __forceinline__ void seek(const GemmArgs& p, const int* s_prefix, int lane) {
    valid = false;
    while (t < total) {
      ti = get_tile<KIND>(t, p, s_prefix, lane);
      if (!ti.skip) { valid = true; return; }
      t += stride;
    }
  }
  __device__ __forceinline__ void start(int first, int stride_, int total_, const GemmArgs& p,
                                        const int* s_prefix, int lane) {
    t = first; stride = stride_; total = total_;
    seek(p, s_prefix, lane);
  }
  __device__ __forceinline__ void next(const GemmArgs& p, const int* s_prefix, int lane) {
    t += stride;
    seek(p, s_prefix, lane);
  }
};

// Walks (tile, stage) pairs in the order the pipeline consumes them; a stage
// starts at K block `kb` and covers up to STEP K blocks.
template <int KIND, int STEP>
struct StageWalker {
  TileWalker<KIND> w;
  int kb;
  bool done;

  __device__ __forceinline__ void start(int first, int stride, int total, const GemmArgs& p,
                                        const int* s_prefix, int lane) {
    w.start(first, stride, total, p, s_prefix, lane);
    done = !w.valid;
    kb = done ? 0 : w.ti.kb_begin;
  }
  __device__ __forceinline__ void next(const GemmArgs& p, const int* s_prefix, int lane) {
    kb += STEP;
    if (kb >= w.ti.kb_end) {
      w.next(p, s_prefix, lane);
      done = !w.valid;
      kb = done ? 0 : w.ti.kb_begin;
    }
  }
};

// BF16: the same GEMM forms on BF16 operands (no scales): the ring, the tile
// scheduler, split-K and the epilogue are shared; the scale-factor warp idles
// and every 128-byte K block is four kind::f16 MMAs (K = 16 each).
template <int KIND, int BLOCK_N, int STAGES, int NUM_ACC, int KPS, int A_ROWS, int MODE,
          int LAYOUT = kLayoutNT, bool OUT_F32 = false, bool BF16 = false>
__global__ void __launch_bounds__(kThreads, MODE == 2 ? 2 : 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a,
                    const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_d, const GemmArgs p) {
  using Shape = KernelShape<BLOCK_N, STAGES, NUM_ACC, KPS, A_ROWS, MODE, !BF16, OUT_F32>;
  constexpr bool SMALL = Shape::kSmall;
  constexpr int A_BYTES = Shape::kABytes;
  constexpr int B_BYTES = Shape::kBBytes;
  constexpr int SF_BYTES = Shape::kSfBytes;
  constexpr int SF_COLS = Shape::kSfCols;
  constexpr int SFB_CHUNKS = Shape::kSfbChunks;
  constexpr int SFB_BLOCKS = Shape::kSfbBlocks;
  constexpr int SF_GROUP = Shape::kSfGroup;
  constexpr int ACC_COLS = Shape::kAccCols;
  constexpr int TMEM_COLS = Shape::kTmemCols;
  static_assert((KPS == 1 && MODE == 0) || KIND == kDense,
                "decode variants and several K blocks per stage: the dense form");
  // M-major A / N-major B: 2-D maps over [K, M] / [K, N] with boxes of 128
  // MN bytes x 128 K rows; one K block per stage, whole 128-row A boxes, and B
  // tiles made of whole 128-column boxes.
  constexpr bool A_MN = (LAYOUT & 1) != 0;
  constexpr bool B_MN = (LAYOUT & 2) != 0;
  static_assert(!BF16 || (LAYOUT == kLayoutNT && !OUT_F32),
                "BF16 operands: K-major A and B, BF16 output");
  // FP32 output (D = A B^T + C): the dense form, no split-K (host-checked)
  static_assert(!OUT_F32 || ((KIND == kDense || KIND == kKGrouped) && A_ROWS == 128 && MODE == 0),
                "FP32 output form");
  static_assert(KIND != kKGrouped || (OUT_F32 && LAYOUT == kLayoutTN),
                "K-grouped: M-major A, N-major B, FP32 output");
  static_assert(LAYOUT == kLayoutNT ||
                    ((KIND == kDense || KIND == kKGrouped) && KPS == 1 && A_ROWS == 128 &&
                     MODE == 0 && BLOCK_N % 128 == 0),
                "M-/N-major operands: dense form, general variants with 128-column B boxes");

  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the 128-byte-swizzled operand tiles
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  // epilogue staging tiles (1024-aligned, swizzled): their own region, or,
  // when every CTA has a single tile (always for a small variant), the operand
  // ring, idle once that tile's MMAs are done, with one tile per warp and chunk
  // output tiles of the dense and contiguous forms (x split) this launch computes
  const int flat_tiles =
      (KIND == kDense && p.tile_limit > 0 ? p.tile_limit : p.num_m_blocks * p.num_n_blocks) *
      p.split_k;
  const int n_tiles_total = (KIND == kMasked || KIND == kKGrouped) ? -1 : flat_tiles;
  // (a decode variant always runs one tile per CTA: the host launches it so)
  const bool one_tile =
      Shape::kDecode || (n_tiles_total >= 0 && n_tiles_total <= static_cast<int>(gridDim.x));
  uint8_t* sEpi = one_tile ? sA : sB + STAGES * B_BYTES;
  uint8_t* sSF = sB + STAGES * B_BYTES + Shape::kEpiBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSF + STAGES * SF_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + NUM_ACC;
  uint64_t* drain = acc_empty + NUM_ACC;
  uint64_t* recv_bar = drain + 1;  // split-K: partial slices pushed by the other CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(recv_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_kvalid = const_cast<int*>(abort_flag + 1);  // K-grouped form: group sizes consistent
  int* s_prefix = const_cast<int*>(abort_flag + 3);  // masked and K-grouped forms
  // split-K: this CTA's FP32 partial, parked over the (by then idle) operand ring
  constexpr int RED_PITCH = BLOCK_N + 4;  // floats per row of a parked split-K partial
  // split-K: parked partial (valid rows) plus incoming slices (at most
  // valid rows + split more) live in the idle operand ring; the host only
  // picks a split for which (2 * valid rows + split) rows fit.
  static_assert(kBlockM * RED_PITCH * 4 <= STAGES * (A_BYTES + B_BYTES),
                "split-K partial must fit in the operand ring");
  float* red = reinterpret_cast<float*>(sA);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const bool split = p.split_k > 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      // producer arrive.expect_tx (+ the scale warp's arrive for E4M3 operands)
      ptx::mbar_init(&full[s], BF16 ? 1 : 2);
      ptx::mbar_init(&empty[s], 1);  // tcgen05.commit
    }
    for (int a = 0; a < NUM_ACC; ++a) {
      ptx::mbar_init(&acc_full[a], 1);     // tcgen05.commit
      ptx::mbar_init(&acc_empty[a], 128);  // every epilogue thread
    }
    ptx::mbar_init(drain, 1);
    ptx::mbar_init(recv_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmap_a);
    ptx::prefetch_tensormap(&tmap_b);
    ptx::prefetch_tensormap(&tmap_d);
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish();
  }
  if (KIND == kDense && p.prefetch && !p.preload_b && warp == 0 &&
      static_cast<int>(blockIdx.x) < flat_tiles) {
    // Warm L2 with this CTA's first tile while the previous kernel finishes
    // (the tile order of the dense form does not depend on device data).
    // A small variant prefetches the whole K range of B, the weights it
    // streams; the others the first stages of both operands.
    const Tile ti = get_tile<kDense>(blockIdx.x, p, nullptr, lane);
    if (lane == 0) {
      const int kb_end = SMALL ? ti.kb_end : min(ti.kb_end, ti.kb_begin + STAGES * KPS);
      for (int kb = ti.kb_begin; kb < kb_end; kb += KPS) {
        if constexpr (B_MN) {
          for (int h = 0; h < BLOCK_N / 128; ++h)
            ptx::tma_prefetch_l2_2d(&tmap_b, ti.n_blk * BLOCK_N + 128 * h, kb * kBlockK);
        } else {
          ptx::tma_prefetch_l2_4d(&tmap_b, 0, ti.n_blk * BLOCK_N, kb, 0);
        }
        if constexpr (A_MN) {
          ptx::tma_prefetch_l2_2d(&tmap_a, ti.m_blk * kBlockM, kb * kBlockK);
        } else {
          if (!SMALL) ptx::tma_prefetch_l2_4d(&tmap_a, 0, ti.m_blk * kBlockM, kb, 0);
        }
      }
    }
  }
  // Barriers, the abort flag and the TMEM base are published before waiting
  // on the previous kernel, so that every role starts right after the wait.
  ptx::tc_fence_before_sync();
  __syncthreads();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  // Let the next kernel start its own prologue (once every CTA of this grid
  // got here).  Everything above reads no input; the inputs may be the
  // previous kernel's outputs, so every thread waits for that kernel (a no-op
  // without programmatic dependent launch) before it reads an input, writes
  // D or starts a timed wait.  The dense form's tile sequence follows from
  // the sizes alone, so each of its roles first sets up its first stage and
  // waits only right before its first global access; the grouped forms'
  // sequence depends on device data, so every thread waits here.
  ptx::grid_launch_dependents();
  constexpr bool kLateWait = (KIND == kDense);
  if constexpr (!kLateWait) ptx::grid_dependency_wait();
  if (KIND == kMasked) {
    // the tile sequence of the masked form depends on masked_m (device data)
    if (threadIdx.x == 96) {
      int acc = 0;
      for (int g = 0; g < p.G; ++g) {
        s_prefix[g] = acc;
        int mm = min(max(p.masked_m[g], 0), p.rows);
        acc += ((mm + kBlockM - 1) / kBlockM) * p.num_n_blocks;
      }
      s_prefix[p.G] = acc;
    }
    __syncthreads();
  }
  if (KIND == kKGrouped) {
    // K-block offsets of the groups, from the group sizes (device data); an
    // inconsistent set of sizes computes nothing and says why
    if (threadIdx.x == 96) {
      int acc = 0;
      bool bad = false;
      for (int g = 0; g < p.G; ++g) {
        s_prefix[g] = acc;
        const int k = p.ks[g];
        bad |= k < 0 || k % kBlockK != 0;
        acc += max(k, 0) / kBlockK;
      }
      s_prefix[p.G] = acc;
      bad |= acc != p.k_blocks;
      if (bad) atomicCAS(p.error_word, 0, kDevKGroups);
      *s_kvalid = bad ? 0 : 1;
    }
    __syncthreads();
  }

  ptx::WaitCtl ctl{abort_flag, p.error_word, p.timeout_ns};
  const int total = KIND == kMasked     ? s_prefix[p.G] * p.split_k
                    : KIND == kKGrouped ? (*s_kvalid ? p.G : 0) * p.num_m_blocks *
                                              p.num_n_blocks * p.split_k
                                        : flat_tiles;

  // Drains TMEM accumulator buffer `a` of tile `ti`, lane quarter q (rows
  // 32q..32q+31), columns [c_begin, c_end): BF16 through the staging tiles
  // at stage0 to D, or (split-K) FP32 into the parked partial.
  constexpr int NCH_ALL = BLOCK_N / Shape::kEpiCols;
  const CUtensorMap* dmap = &tmap_d;
  int f32_chunks = 0;  // FP32-output chunks this thread's warp has stored (its staging half)
  // staging bytes of one epilogue warp in the staging region (persistent CTAs)
  constexpr int kWarpEpiBytes = Shape::kEpiBytes / 4;
  static_assert(!OUT_F32 || (Shape::kEpiBytes == 4 * Shape::kF32Bufs * 2048 &&
                             Shape::kEpiCols == 64 && Shape::kF32Bufs == 8),
                "FP32 output: two halves of four 2 KB box buffers per epilogue warp");
  static_assert(!OUT_F32 || STAGES * (A_BYTES + B_BYTES) >= Shape::kEpiBytes,
                "FP32 output, one tile per CTA: the staging buffers fit in the operand ring");
  // The output row of accumulator row 32q + lane of tile `ti` (`grow`, the
  // row of D) and whether it is written; `report` flags a contiguous row of
  // another expert.
  auto out_row = [&](const Tile& ti, int q, bool report, bool& valid, size_t& grow) {
    const int row_local = 32 * q + lane;  // accumulator row = TMEM lane
    const int m_in_group = ti.m_blk * kBlockM + row_local;
    if (KIND == kMasked) {
      const int mm = min(max(__ldg(p.masked_m + ti.group), 0), p.rows);
      valid = m_in_group < mm;
      grow = (size_t)ti.group * p.rows + m_in_group;
    } else if (KIND == kKGrouped) {
      valid = m_in_group < p.rows;
      grow = (size_t)ti.group * p.rows + m_in_group;
    } else {
      valid = m_in_group < p.rows;
      grow = m_in_group;
      if (KIND == kContiguous && valid) {
        const int e = __ldg(p.m_indices + m_in_group);
        if (report && e >= 0 && e != ti.group) atomicCAS(p.error_word, 0, kDevMixedExperts);
        valid = (e == ti.group);
      }
    }
  };

  // Stores BF16 columns [c0, c0 + 64) of this lane's output row, held as
  // packed pairs in v[0..31], through the warp's staging tile: one TMA box of
  // 32 rows x 64 columns (rows past the tensor's end and columns past N are
  // clipped by the TMA unit), or whole row segments when some of the warp's
  // rows are not written (grouped forms).  The staging tile is free again on
  // return.
  auto store_bf16_64 = [&](const uint32_t* v, uint8_t* stage, int n0, int c0, bool valid,
                           size_t grow, bool tma_store) {
    constexpr int CPR = 8;  // 16-byte chunks per staged row
    // chunk j of row `lane` at chunk position j ^ (lane % 8): the 128-byte swizzle
#pragma unroll
    for (int j = 0; j < CPR; ++j)
      *reinterpret_cast<uint4*>(stage + lane * 128 + 16 * (j ^ (lane % CPR))) =
          make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
    if (tma_store) {
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::tma_store_2d(dmap, stage, n0 + c0, static_cast<int>(grow - lane));
        ptx::bulk_commit_group();
        ptx::bulk_wait_group_read0();
      }
      __syncwarp();
      return;
    }
    __syncwarp();
    constexpr int RPI = 32 / CPR;  // rows per store instruction
    const int sub = lane % CPR;
#pragma unroll
    for (int i = 0; i < 32 / RPI; ++i) {
      const int rr = RPI * i + lane / CPR;  // row within the warp's 32
      const bool row_ok = __shfl_sync(0xFFFFFFFFu, valid, rr);
      const int n = n0 + c0 + 8 * sub;
      if (row_ok && n < p.N) {
        const size_t g_row = grow - lane + rr;  // the rows of a warp are consecutive
        *reinterpret_cast<uint4*>(p.d + g_row * p.ldd + n) =
            *reinterpret_cast<const uint4*>(stage + rr * 128 + 16 * (sub ^ (rr % CPR)));
      }
    }
    __syncwarp();
  };

  auto drain_acc = [&](const Tile& ti, int a, int q, int c_begin, int c_end, uint8_t* stage0,
                       bool report) {
    // which output row this thread owns, and whether it may be written
    const int row_local = 32 * q + lane;  // accumulator row = TMEM lane
    bool valid;
    size_t grow;
    out_row(ti, q, report, valid, grow);
    const uint32_t t_row =
        tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a * BLOCK_N;
    const int n0 = ti.n_blk * BLOCK_N;

    // A warp whose 32 rows are all outside the output (a short dense A, a
    // masked group) skips the TMEM reads; it still releases the buffer.
    if (__any_sync(0xFFFFFFFFu, valid)) {
      constexpr int CH = Shape::kEpiCols;  // columns per TMEM wait
      // TMA store of whole 32-row boxes: the dense form always (rows past M
      // are clipped); the grouped forms only when all 32 rows are written.
      const bool tma_store = CH == 64 && !split &&
                             (KIND == kDense || __all_sync(0xFFFFFFFFu, valid));
#pragma unroll 1
      for (int c0 = c_begin; c0 < c_end; c0 += CH) {
        uint32_t r[CH];
        ptx::tc_ld_32x32b_x32(t_row + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        if (CH == 64)
          ptx::tc_ld_32x32b_x32(t_row + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[CH - 32]));
        ptx::tc_wait_ld();
        if constexpr (OUT_F32) {
          // FP32 output in boxes of 32 rows x 16 columns (64 bytes a row),
          // four per 64-column chunk: each lane adds its row's C values if
          // given (C may be D: every element is read by the thread that
          // stages it, before its box is stored) and stages the row's 64
          // bytes of each box (16-byte chunk j of row l at position
          // j ^ ((l / 2) % 4): the 64-byte swizzle) in one half of the warp's
          // staging buffers; then one fence, and four TMA stores committed as
          // one bulk group (the tensor map is [groups][rows][N], so rows past
          // a group's end and columns past N are clipped).  A half is reused
          // once the group issued from it two chunks earlier has read it: the
          // form is bound by writing its output, and one chunk's stores stay
          // in flight while the next chunk is loaded from TMEM and staged.
          const int grp = (KIND == kKGrouped) ? ti.group : 0;
          const size_t off = grow * p.N + n0 + c0;
          uint8_t* half = stage0 + (f32_chunks & 1) * (Shape::kF32Bufs / 2) * 2048;
          if (lane == 0) ptx::bulk_wait_group_read<1>();
          __syncwarp();
#pragma unroll
          for (int h = 0; h < CH / 16; ++h) {
            float* v = reinterpret_cast<float*>(&r[16 * h]);
            if (p.c_f32 && valid) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                if (n0 + c0 + 16 * h + 4 * j >= p.N) break;
                const float4 cv = *reinterpret_cast<const float4*>(p.c_f32 + off + 16 * h + 4 * j);
                v[4 * j] += cv.x; v[4 * j + 1] += cv.y; v[4 * j + 2] += cv.z; v[4 * j + 3] += cv.w;
              }
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
              *reinterpret_cast<float4*>(half + h * 2048 + lane * 64 + 16 * (j ^ ((lane >> 1) & 3))) =
                  make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
#pragma unroll
            for (int h = 0; h < CH / 16; ++h)
              ptx::tma_store_3d(dmap, half + h * 2048, n0 + c0 + 16 * h,
                                ti.m_blk * kBlockM + 32 * q, grp);
            ptx::bulk_commit_group();
          }
          ++f32_chunks;
          continue;
        }
        uint8_t* stage = one_tile ? stage0 + ((c0 - c_begin) / CH) * 32 * Shape::kEpiPitch : stage0;
        if (split) {
          // park the FP32 partial; the cluster reduces it below
          if (valid) {
#pragma unroll
            for (int j = 0; j < CH / 4; ++j)
              *reinterpret_cast<float4*>(red + row_local * RED_PITCH + c0 + 4 * j) =
                  make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                              __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
          }
          continue;
        }
        // BF16 row of this lane into the warp's staging tile (chunk j of row
        // `lane` at chunk position j ^ (lane % 8): the 128-byte swizzle) ...
        constexpr int CPR = CH / 8;  // 16-byte chunks per row
#pragma unroll
        for (int j = 0; j < CPR; ++j) {
          uint4 v;
          v.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
          v.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
          v.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
          v.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
          *reinterpret_cast<uint4*>(stage + lane * Shape::kEpiPitch + 16 * (j ^ (lane % CPR))) = v;
        }
        if (tma_store) {
          // ... then one TMA box of 32 rows x 64 columns (rows past the
          // tensor's end and columns past N are clipped by the TMA unit)
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(dmap, stage, n0 + c0, static_cast<int>(grow - lane));
            ptx::bulk_commit_group();
            if (!one_tile) ptx::bulk_wait_group_read0();  // staging tile free again
          }
          __syncwarp();
          continue;
        }
        __syncwarp();
        // ... or whole row segments: a store instruction covers 32 / CPR
        // rows, CPR lanes per row, 16 bytes a lane.
        constexpr int RPI = 32 / CPR;  // rows per instruction
        const int sub = lane % CPR;
#pragma unroll
        for (int i = 0; i < 32 / RPI; ++i) {
          const int rr = RPI * i + lane / CPR;  // row within the warp's 32
          const bool row_ok = __shfl_sync(0xFFFFFFFFu, valid, rr);
          const int n = n0 + c0 + 8 * sub;
          if (row_ok && n < p.N) {
            const size_t g_row = grow - lane + rr;  // the rows of a warp are consecutive
            *reinterpret_cast<uint4*>(p.d + g_row * p.ldd + n) = *reinterpret_cast<const uint4*>(
                stage + rr * Shape::kEpiPitch + 16 * (sub ^ (rr % CPR)));
          }
        }
        __syncwarp();
      }
      if (split) ptx::fence_proxy_async_smem();  // parked rows are read by bulk copies
    }
  };
  // A persistent CTA with a single accumulator (BLOCK_N 256) would hold its
  // MMAs back for the whole epilogue.  Instead each epilogue thread reads its
  // accumulator row into registers as packed BF16 pairs, releases the
  // accumulator (the MMA warp starts the CTA's next tile), and only then
  // stages and stores the row, overlapping the next tile's MMAs.
  constexpr bool kEarlyRelease =
      NUM_ACC == 1 && MODE == 0 && !OUT_F32 && Shape::kEpiCols == 64 && BLOCK_N % 64 == 0;
  auto drain_release = [&](const Tile& ti, int a, int q, uint8_t* stage) {
    bool valid;
    size_t grow;
    out_row(ti, q, true, valid, grow);
    const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + a * BLOCK_N;
    const bool any = __any_sync(0xFFFFFFFFu, valid);
    uint32_t pk[BLOCK_N / 2];
    if (any) {
#pragma unroll
      for (int c = 0; c < BLOCK_N / 64; ++c) {
        uint32_t r[64];
        ptx::tc_ld_32x32b_x32(t_row + 64 * c, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
        ptx::tc_ld_32x32b_x32(t_row + 64 * c + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
        ptx::tc_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j)
          pk[32 * c + j] = pack_bf16x2(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
      }
    }
    ptx::tc_fence_before_sync();
    ptx::mbar_arrive(&acc_empty[a]);
    if (!any) return;
    const bool tma_store = KIND == kDense || __all_sync(0xFFFFFFFFu, valid);
#pragma unroll
    for (int c = 0; c < BLOCK_N / 64; ++c)
      store_bf16_64(pk + 32 * c, stage, ti.n_blk * BLOCK_N, 64 * c, valid, grow, tma_store);
  };

  // A single-tile CTA's warps 0-3 are idle once their roles end: they drain
  // the upper half of the columns while warps 4-7 drain the lower half.
  const bool helpers = one_tile && !split && KIND != kMasked && !OUT_F32 &&
                       BLOCK_N >= 2 * Shape::kEpiCols && (BLOCK_N / 2) % Shape::kEpiCols == 0;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    // One box of A and one of B per stage, each KPS K blocks deep (blocks
    // past K are zero-filled and still counted).  A short dense A (fewer than
    // 128 rows) is fetched with a box of only its rows; the 128-row MMA then
    // reads stale shared memory for the other rows, which only feeds
    // accumulator rows that are never stored.
    auto load_a = [&](int s, const Tile& ti, int kb) {
      if constexpr (A_MN) {
        ptx::tma_load_2d(sA + s * A_BYTES, &tmap_a, &full[s], ti.m_blk * kBlockM, kb * kBlockK);
      } else {
        ptx::tma_load_4d(sA + s * A_BYTES, &tmap_a, &full[s], 0, ti.m_blk * kBlockM, kb,
                         (KIND == kMasked) ? ti.group : 0);
      }
    };
    auto load_b = [&](int s, const Tile& ti, int kb) {
      if constexpr (B_MN) {
        // 128-column blocks of the tile, 128 x 128 bytes each
#pragma unroll
        for (int h = 0; h < BLOCK_N / 128; ++h)
          ptx::tma_load_2d(sB + s * B_BYTES + h * 128 * kBlockK, &tmap_b, &full[s],
                           ti.n_blk * BLOCK_N + 128 * h, kb * kBlockK);
      } else {
        ptx::tma_load_4d(sB + s * B_BYTES, &tmap_b, &full[s], 0, ti.n_blk * BLOCK_N, kb,
                         ti.group);
      }
    };
    const uint32_t stage_bytes = KPS * (p.a_box_rows + BLOCK_N) * kBlockK;
    int it = 0;
    bool ok = true;
    // Weight preload (dense form, on request): B does not change while
    // kernels run, so the first ring stages' B boxes go out before the wait on
    // the previous kernel (whose outputs A may be); their A boxes follow the
    // wait.  The ring is fresh, so those stages' slots are free.
    int preloaded = 0;
    if (kLateWait && p.preload_b && static_cast<int>(blockIdx.x) < total) {
      const Tile ti = get_tile<KIND>(blockIdx.x, p, s_prefix, lane);
      if (!ti.skip && lane == 0) {
        for (int kb = ti.kb_begin; kb < ti.kb_end && preloaded < STAGES; kb += KPS, ++preloaded) {
          ptx::mbar_arrive_expect_tx(&full[preloaded], stage_bytes);
          load_b(preloaded, ti, kb);
        }
      }
      preloaded = __shfl_sync(0xFFFFFFFFu, preloaded, 0);
    }
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Tile ti = get_tile<KIND>(t, p, s_prefix, lane);
      if (ti.skip) continue;
      for (int kb = ti.kb_begin; kb < ti.kb_end; kb += KPS, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (lane == 0) {
          if (it < preloaded) {
            if (it == 0) ptx::grid_dependency_wait();
            load_a(s, ti, kb);  // its B box and barrier bytes went out before the wait
          } else {
            ok = ptx::mbar_wait(&empty[s], ph ^ 1, ctl, kDevTimeoutProducer);
            if (ok) {
              ptx::mbar_arrive_expect_tx(&full[s], stage_bytes);
              if (kLateWait && it == 0) ptx::grid_dependency_wait();
              load_a(s, ti, kb);
              load_b(s, ti, kb);
            }
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
      }
    }
    if (!ok && lane == 0) {
      // wait (briefly) for loads still in flight before the CTA tears down
      for (int j = max(0, it - STAGES); j < it; ++j)
        ptx::mbar_wait_drain(&full[j % STAGES], (j / STAGES) & 1, 20000000ull);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------- MMA issuer --
    if constexpr (kLateWait) ptx::grid_dependency_wait();
    constexpr uint32_t idesc = BF16 ? ptx::idesc_bf16_f32(kBlockM, BLOCK_N)
                                    : ptx::idesc_mxf8_e4m3_ue8m0(kBlockM, BLOCK_N, A_MN, B_MN);
    // Scale words of one group, from its shared-memory slot into the TMEM
    // columns of the same slot: the SFA words of the tile's 128 rows, then
    // the SFB words of each 128-row chunk of the tile's B rows.
    auto copy_sf = [&](int slot) {
      const uint32_t sfa_tmem = tmem_base + ACC_COLS + slot * SF_COLS;
      const uint32_t sfb_tmem = sfa_tmem + 4;
      const uint32_t sf_smem = ptx::smem_addr(sSF + slot * SF_BYTES);
      ptx::tc_cp_32x128b_warpx4(sfa_tmem, ptx::sdesc_sf_32x16(sf_smem));
#pragma unroll
      for (int h = 0; h < SFB_CHUNKS; ++h)
        ptx::tc_cp_32x128b_warpx4(sfb_tmem + 4 * h, ptx::sdesc_sf_32x16(sf_smem + 512 * (1 + h)));
    };
    int it = 0, acc_it = 0;
    // scale-word groups walked, and the slot of the current group's words:
    // the slot of a group is its count modulo STAGES, in shared memory and
    // TMEM alike.  A group has at least one stage, so the slot's previous
    // group ended at least STAGES stages earlier, and its MMAs (and copy)
    // are complete once this stage's full barrier has flipped.
    int gc = 0, sf_slot = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Tile ti = get_tile<KIND>(t, p, s_prefix, lane);
      if (ti.skip) continue;
      const int a = acc_it % NUM_ACC;
      const uint32_t aph = (acc_it / NUM_ACC) & 1;
      if (lane == 0) ok = ptx::mbar_wait(&acc_empty[a], aph ^ 1, ctl, kDevTimeoutMma);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after_sync();
      const uint32_t d_tmem = tmem_base + a * BLOCK_N;
      for (int kb = ti.kb_begin; kb < ti.kb_end; kb += KPS, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int q = (kb - ti.kb_begin) / KPS;  // stage within the tile
        const bool group_first = q % SF_GROUP == 0;
        if (group_first) {
          sf_slot = gc % STAGES;
          ++gc;
        }
        if (lane == 0) ok = ptx::mbar_wait(&full[s], ph, ctl, kDevTimeoutMma);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        ptx::tc_fence_after_sync();
        if (BF16 && lane == 0) {
          // BF16 operands: four K = 16 MMAs per 128-byte K block, no scales
          const uint32_t a_base = ptx::smem_addr(sA + s * A_BYTES);
          const uint32_t b_base = ptx::smem_addr(sB + s * B_BYTES);
#pragma unroll
          for (int j = 0; j < KPS; ++j) {
            if (kb + j >= ti.kb_end) break;
            const uint64_t db = ptx::sdesc_kmajor_sw128(b_base + j * BLOCK_N * kBlockK);
            const uint64_t da = ptx::sdesc_kmajor_sw128(a_base + j * p.a_box_rows * kBlockK);
#pragma unroll
            for (int ks = 0; ks < kBlockK / 32; ++ks)
              ptx::tc_mma_bf16(d_tmem, da + (32 >> 4) * ks, db + (32 >> 4) * ks, idesc,
                               kb + j > ti.kb_begin || ks > 0);
          }
          ptx::tc_commit(&empty[s]);
        } else if (!BF16 && lane == 0) {
          const uint32_t sfa_tmem = tmem_base + ACC_COLS + sf_slot * SF_COLS;
          const uint32_t sfb_tmem = sfa_tmem + 4;
          if (group_first) copy_sf(sf_slot);
          const uint32_t a_base = ptx::smem_addr(sA + s * A_BYTES);
          const uint32_t b_base = ptx::smem_addr(sB + s * B_BYTES);
#pragma unroll
          for (int j = 0; j < KPS; ++j) {
            if (kb + j >= ti.kb_end) break;
            // K block j of the stage is K block sb of its group: its scale
            // factors are byte sb of every TMEM scale word (selected by the
            // scale-factor id)
            const uint32_t sb = static_cast<uint32_t>((q % SF_GROUP) * KPS + j);
            // a K step of 32 moves 32 bytes along a K-major row, or 4 swizzle
            // atoms (4096 bytes) down an M-/N-major tile
            constexpr uint32_t kStepA = A_MN ? 4096 >> 4 : 32 >> 4;
            constexpr uint32_t kStepB = B_MN ? 4096 >> 4 : 32 >> 4;
            const uint64_t db =
                B_MN ? ptx::sdesc_mnmajor_sw128(b_base, 128 * kBlockK)
                     : ptx::sdesc_kmajor_sw128(b_base + j * BLOCK_N * kBlockK);
            const uint32_t id = idesc | (sb << 29) | (sb << 4);
            const uint32_t byte_sel = sb << 30;
            const uint64_t da = A_MN ? ptx::sdesc_mnmajor_sw128(a_base, 128 * kBlockK)
                                     : ptx::sdesc_kmajor_sw128(a_base + j * p.a_box_rows * kBlockK);
#pragma unroll
            for (int ks = 0; ks < kBlockK / 32; ++ks)
              ptx::tc_mma_mxf8_block_scale(d_tmem, da + kStepA * ks, db + kStepB * ks, id,
                                           sfa_tmem | byte_sel, sfb_tmem | byte_sel,
                                           kb + j > ti.kb_begin || ks > 0);
          }
          ptx::tc_commit(&empty[s]);
        }
        __syncwarp();
      }
      if (!ok) break;
      if (lane == 0) ptx::tc_commit(&acc_full[a]);
      __syncwarp();
      ++acc_it;
    }
    // all MMAs this thread issued have completed once `drain` flips
    if (lane == 0) {
      ptx::tc_commit(drain);
      ptx::mbar_wait_drain(drain, 0, 50000000ull);
    }
    __syncwarp();
  } else if (warp == 2 && !BF16) {
    if constexpr (SF_GROUP == 1) {
      // --------------------------------------------- scale-factor producer --
      // The FP32 scales of a stage are loaded PF stages before they are
      // written, so the global-load latency overlaps several pipeline stages.
      // Scale words pack the stage's K blocks: byte j belongs to K block j.
      constexpr int PF = (8 + KPS - 1) / KPS;
      const int KB = p.k_blocks;
      float va[PF][4][KPS];
      float vb[PF][SFB_BLOCKS][KPS];
      StageWalker<KIND, KPS> ld, wr;
      ld.start(blockIdx.x, gridDim.x, total, p, s_prefix, lane);
      wr.start(blockIdx.x, gridDim.x, total, p, s_prefix, lane);
      if constexpr (kLateWait) ptx::grid_dependency_wait();

      auto issue = [&](float (&a)[4][KPS], float (&b)[SFB_BLOCKS][KPS]) {
        const Tile& ti = ld.w.ti;
        const int m0 = ti.m_blk * kBlockM;  // first row of the tile
        const int row_base = (KIND == kMasked ? ti.group * p.rows : 0) + m0;
        const int rows_left = p.rows - m0;  // rows of the tile that exist
  #pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int r = 32 * c + lane;
  #pragma unroll
          for (int j = 0; j < KPS; ++j)
            a[c][j] = (r < rows_left && ld.kb + j < ti.kb_end)
                          ? __ldg(p.sfa + (size_t)(row_base + r) * KB + ld.kb + j)
                          : 1.0f;
        }
        // B scale blocks are 128 rows: the tile's rows touch blocks b0, b0 + 1, ...
        // (K-grouped: one sfb for all groups, indexed by the global K block)
        const float* sfb_g = p.sfb + (KIND == kKGrouped ? 0 : (size_t)ti.group * p.nb128 * KB);
        const int b0 = ti.n_blk * BLOCK_N / 128;
  #pragma unroll
        for (int i = 0; i < SFB_BLOCKS; ++i) {
          const int nb = min(b0 + i, p.nb128 - 1);
  #pragma unroll
          for (int j = 0; j < KPS; ++j)
            b[i][j] = (ld.kb + j < ti.kb_end) ? __ldg(sfb_g + (size_t)nb * KB + ld.kb + j) : 1.0f;
        }
        ld.next(p, s_prefix, lane);
      };

  #pragma unroll
      for (int j = 0; j < PF; ++j)
        if (!ld.done) issue(va[j], vb[j]);

      int it = 0;
      bool ok = true;
      while (!wr.done && ok) {
  #pragma unroll
        for (int slot = 0; slot < PF; ++slot) {
          if (wr.done || !ok) break;
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (lane == 0) ok = ptx::mbar_wait(&empty[s], ph ^ 1, ctl, kDevTimeoutScales);
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (!ok) break;
          uint8_t* sf = sSF + s * SF_BYTES;
          // A scales: TMEM lane l, column c holds row 32c + l of the tile.
          {
            uint32_t w[4];
  #pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t x = 0x7F7F7F7Fu;  // unused bytes: scale 1
  #pragma unroll
              for (int j = 0; j < KPS; ++j)
                x = (x & ~(0xFFu << (8 * j))) | (ue8m0(va[slot][c][j]) << (8 * j));
              w[c] = x;
            }
            *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          // B scales, same layout per 128-row chunk of the tile's B rows: row
          // r of the tile takes the scale of its own 128-row block of B
          const int n_off = (wr.w.ti.n_blk * BLOCK_N) % 128;  // tile start within its block
  #pragma unroll
          for (int h = 0; h < SFB_CHUNKS; ++h) {
            uint32_t w[4];
  #pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int idx = min((n_off + 128 * h + 32 * c + lane) / 128, SFB_BLOCKS - 1);
              uint32_t x = 0x7F7F7F7Fu;
  #pragma unroll
              for (int j = 0; j < KPS; ++j) {
                float v = vb[slot][0][j];
  #pragma unroll
                for (int i = 1; i < SFB_BLOCKS; ++i)
                  if (idx == i) v = vb[slot][i][j];
                x = (x & ~(0xFFu << (8 * j))) | (ue8m0(v) << (8 * j));
              }
              w[c] = x;
            }
            *reinterpret_cast<uint4*>(sf + 512 * (1 + h) + 16 * lane) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&full[s]);
          if (!ld.done) issue(va[slot], vb[slot]);
          wr.next(p, s_prefix, lane);
          ++it;
        }
      }
    } else {
      // --------------------------------------------- scale-factor producer --
      // A tile's K blocks form groups of up to four (SF_GROUP stages of KPS
      // blocks), and one set of scale words serves a whole group: byte b of a
      // word is the group's K block b, selected by the MMA's scale-factor id,
      // so a group costs one tcgen05.cp instead of one per stage.  A group's
      // words go to the shared-memory slot of the group counter modulo STAGES
      // at the group's first stage; every stage still takes its empty slot and
      // arrives on its full barrier.  The FP32 scales of a group are loaded
      // two groups ahead (a float4 per row when the rows allow it).
      constexpr int GK = SF_GROUP * KPS;  // K blocks of a full group (4)
      const int KB = p.k_blocks;
      float va[2][4][GK];
      float vb[2][SFB_BLOCKS][GK];
      StageWalker<KIND, GK> ld;    // walks the groups
      StageWalker<KIND, KPS> wr;   // walks the stages
      ld.start(blockIdx.x, gridDim.x, total, p, s_prefix, lane);
      wr.start(blockIdx.x, gridDim.x, total, p, s_prefix, lane);
      if constexpr (kLateWait) ptx::grid_dependency_wait();
      // rows of sfa and sfb start on 16-byte boundaries: whole float4s per group
      const bool vec = GK == 4 && KB % 4 == 0 &&
                       (reinterpret_cast<uintptr_t>(p.sfa) & 15) == 0 &&
                       (reinterpret_cast<uintptr_t>(p.sfb) & 15) == 0;

      auto issue = [&](float (&a)[4][GK], float (&b)[SFB_BLOCKS][GK]) {
        const Tile& ti = ld.w.ti;
        const int kb0 = ld.kb;                       // first K block of the group
        const bool v4 = vec && (kb0 & 3) == 0;       // then kb0 + 4 <= KB as well
        const int m0 = ti.m_blk * kBlockM;           // first row of the tile
        const int row_base = (KIND == kMasked ? ti.group * p.rows : 0) + m0;
        const int rows_left = p.rows - m0;           // rows of the tile that exist
  #pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int r = 32 * c + lane;
          const float* src = p.sfa + (size_t)(row_base + r) * KB + kb0;
          if (r < rows_left && v4) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(src));
            a[c][0] = x.x; a[c][1] = x.y; a[c][2] = x.z; a[c][3] = x.w;
          } else {
  #pragma unroll
            for (int j = 0; j < GK; ++j)
              a[c][j] = (r < rows_left && kb0 + j < ti.kb_end) ? __ldg(src + j) : 1.0f;
          }
        }
        // B scale blocks are 128 rows: the tile's rows touch blocks b0, b0 + 1, ...
        // (K-grouped: one sfb for all groups, indexed by the global K block)
        const float* sfb_g = p.sfb + (KIND == kKGrouped ? 0 : (size_t)ti.group * p.nb128 * KB);
        const int b0 = ti.n_blk * BLOCK_N / 128;
  #pragma unroll
        for (int i = 0; i < SFB_BLOCKS; ++i) {
          const int nb = min(b0 + i, p.nb128 - 1);
          const float* src = sfb_g + (size_t)nb * KB + kb0;
          if (v4) {
            const float4 x = __ldg(reinterpret_cast<const float4*>(src));
            b[i][0] = x.x; b[i][1] = x.y; b[i][2] = x.z; b[i][3] = x.w;
          } else {
  #pragma unroll
            for (int j = 0; j < GK; ++j)
              b[i][j] = (kb0 + j < ti.kb_end) ? __ldg(src + j) : 1.0f;
          }
        }
        ld.next(p, s_prefix, lane);
      };

      if (!ld.done) issue(va[0], vb[0]);
      if (!ld.done) issue(va[1], vb[1]);

      int it = 0, gc = 0;  // stages and groups walked
      bool ok = true;
      // one stage: take its empty slot, (at a group's first stage) write the
      // group's words, arrive on its full barrier
      auto stage = [&](bool first, const float (&a)[4][GK],
                       const float (&b)[SFB_BLOCKS][GK]) -> bool {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        bool good = true;
        if (lane == 0) good = ptx::mbar_wait(&empty[s], ph ^ 1, ctl, kDevTimeoutScales);
        good = __shfl_sync(0xFFFFFFFFu, good, 0);
        if (!good) return false;
        if (first) {
          uint8_t* sf = sSF + (gc % STAGES) * SF_BYTES;
          const int n_valid = min(GK, wr.w.ti.kb_end - wr.kb);  // K blocks of this group
          // A scales: TMEM lane l, column c holds row 32c + l of the tile.
          {
            uint32_t w[4];
  #pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint32_t x = 0x7F7F7F7Fu;  // unused bytes: scale 1
  #pragma unroll
              for (int j = 0; j < GK; ++j)
                if (j < n_valid) x = (x & ~(0xFFu << (8 * j))) | (ue8m0(a[c][j]) << (8 * j));
              w[c] = x;
            }
            *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          // B scales, same layout per 128-row chunk of the tile's B rows: row
          // r of the tile takes the scale of its own 128-row block of B
          const int n_off = (wr.w.ti.n_blk * BLOCK_N) % 128;  // tile start within its block
  #pragma unroll
          for (int h = 0; h < SFB_CHUNKS; ++h) {
            uint32_t w[4];
  #pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int idx = min((n_off + 128 * h + 32 * c + lane) / 128, SFB_BLOCKS - 1);
              uint32_t x = 0x7F7F7F7Fu;
  #pragma unroll
              for (int j = 0; j < GK; ++j) {
                float v = b[0][j];
  #pragma unroll
                for (int i = 1; i < SFB_BLOCKS; ++i)
                  if (idx == i) v = b[i][j];
                if (j < n_valid) x = (x & ~(0xFFu << (8 * j))) | (ue8m0(v) << (8 * j));
              }
              w[c] = x;
            }
            *reinterpret_cast<uint4*>(sf + 512 * (1 + h) + 16 * lane) =
                make_uint4(w[0], w[1], w[2], w[3]);
          }
          ptx::fence_proxy_async_smem();
          __syncwarp();
          ++gc;
        }
        if (lane == 0) ptx::mbar_arrive(&full[s]);
        wr.next(p, s_prefix, lane);
        ++it;
        return true;
      };

      while (!wr.done && ok) {
  #pragma unroll
        for (int buf = 0; buf < 2; ++buf) {
          if (wr.done || !ok) break;
          // the group's first stage (walking always stops at one), then the rest
          ok = stage(true, va[buf], vb[buf]);
          if (!ok) break;
          if (!ld.done) issue(va[buf], vb[buf]);  // the group after next
          while (ok && !wr.done && ((wr.kb - wr.w.ti.kb_begin) / KPS) % SF_GROUP != 0)
            ok = stage(false, va[buf], vb[buf]);
        }
      }
    }
  } else if (warp >= 4) {
    // --------------------------------------------------------- epilogue --
    if constexpr (kLateWait) ptx::grid_dependency_wait();
    const int q = warp & 3;                // TMEM lane quarter of this warp
    const int row_local = 32 * q + lane;   // accumulator row = TMEM lane
    const int ep_tid = threadIdx.x - 128;  // 0..127
    int acc_it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
      const Tile ti = get_tile<KIND>(t, p, s_prefix, lane);
      if (ti.skip) {
        if (KIND == kContiguous && ti.group >= p.G && ep_tid == 0)
          atomicCAS(p.error_word, 0, kDevExpertRange);
        if constexpr (KIND == kKGrouped && OUT_F32) {
          // a group without K rows: its output is C (or zeros), no product
          const int m = ti.m_blk * kBlockM + row_local;
          if (m < p.rows) {
            const size_t off = ((size_t)ti.group * p.rows + m) * p.N;
            for (int n = ti.n_blk * BLOCK_N; n < min(p.N, (ti.n_blk + 1) * BLOCK_N); n += 4) {
              const float4 v = p.c_f32 ? *reinterpret_cast<const float4*>(p.c_f32 + off + n)
                                       : make_float4(0.f, 0.f, 0.f, 0.f);
              *reinterpret_cast<float4*>(p.d_f32 + off + n) = v;
            }
          }
        }
        if (split) {
          // an empty K slice still contributes (zeros) to the cluster's sum
          const int valid_rows = min(p.rows - ti.m_blk * kBlockM, kBlockM);
          if (row_local < valid_rows)
            for (int c = 0; c < BLOCK_N; c += 4)
              *reinterpret_cast<float4*>(red + row_local * RED_PITCH + c) = make_float4(0, 0, 0, 0);
          ptx::fence_proxy_async_smem();  // parked rows are read by bulk copies
        }
        continue;
      }
      const int a = acc_it % NUM_ACC;
      const uint32_t aph = (acc_it / NUM_ACC) & 1;
      if (lane == 0) ok = ptx::mbar_wait(&acc_full[a], aph, ctl, kDevTimeoutEpilogue);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      // all four epilogue warps take the same branch
      ok = named_bar_and(2, 128, ok);
      if (!ok) break;
      ptx::tc_fence_after_sync();

      if (kEarlyRelease && !one_tile && !split) {
        drain_release(ti, a, q, sEpi + q * kWarpEpiBytes);  // releases the buffer
      } else {
        const int split_col = helpers ? BLOCK_N / 2 : BLOCK_N;
        // staging: the warp's own slice of the staging region, or in one_tile
        // mode of the idle operand ring (BF16: warp w owns tiles
        // [w * NCH_ALL, (w + 1) * NCH_ALL); FP32: 16 KB per warp)
        uint8_t* stage0 = (OUT_F32 || !one_tile) ? sEpi + q * kWarpEpiBytes
                                                 : sEpi + warp * NCH_ALL * 32 * Shape::kEpiPitch;
        drain_acc(ti, a, q, 0, split_col, stage0, true);
        ptx::tc_fence_before_sync();
        ptx::mbar_arrive(&acc_empty[a]);
      }
      ++acc_it;
    }
    // this warp's TMA stores have read their staging tiles (the writes
    // themselves are part of the grid's completion)
    if (lane == 0) ptx::bulk_wait_group_read0();
  }

  // the threads that have not waited yet (the producer's other lanes, warp 3)
  // do so before the helper drain and the split-K reduction write D
  if constexpr (kLateWait) ptx::grid_dependency_wait();

  if (helpers && warp < 4 && !*abort_flag) {
    if (static_cast<int>(blockIdx.x) < total) {
      const Tile ti = get_tile<KIND>(blockIdx.x, p, s_prefix, lane);
      if (!ti.skip) {
        bool ok = true;
        if (lane == 0) ok = ptx::mbar_wait(&acc_full[0], 0, ctl, kDevTimeoutEpilogue);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (ok) {
          ptx::tc_fence_after_sync();
          drain_acc(ti, 0, warp, BLOCK_N / 2, BLOCK_N,
                    sEpi + (warp * NCH_ALL + NCH_ALL / 2) * 32 * Shape::kEpiPitch, false);
        }
      }
    }
    // this warp's TMA stores have read their staging tiles (the writes
    // themselves are part of the grid's completion)
    if (lane == 0) ptx::bulk_wait_group_read0();
  }

  if (split) {
    // ---------------------------------------- split-K cluster reduction --
    // One output tile per cluster, one K slice per CTA (rank = slice).  The
    // tile's valid rows are cut into one slice per CTA; every CTA pushes the
    // rows of each other CTA's slice of its parked partial to that CTA with
    // one bulk copy (distributed shared memory), then sums the partials of
    // its own slice in rank order and stores BF16.
    const int S = p.split_k;
    const uint32_t rank = ptx::cluster_ctarank();
    const Tile ti = get_tile<KIND>(blockIdx.x, p, s_prefix, lane);
    const int valid_rows = min(p.rows - ti.m_blk * kBlockM, kBlockM);
    const int rows_per = (valid_rows + S - 1) / S;
    auto slice_rows = [&](int r) { return max(0, min(valid_rows, (r + 1) * rows_per) - r * rows_per); };
    // incoming slices land after the parked rows: slot `src` holds CTA src's rows
    float* recv = red + valid_rows * RED_PITCH;
    static_assert(RED_PITCH % 4 == 0, "16-byte rows");
    __syncwarp();
    ptx::cluster_sync();  // every CTA has parked its partial and is done with its ring
    if (threadIdx.x == 0) {
      const uint32_t mine = static_cast<uint32_t>(slice_rows(rank) * RED_PITCH * 4);
      ptx::mbar_arrive_expect_tx(recv_bar, (S - 1) * mine);
      const uint32_t bar_local = ptx::smem_addr(recv_bar);
      const uint32_t slot_local = ptx::smem_addr(recv + rank * rows_per * RED_PITCH);
      for (int dst = 0; dst < S; ++dst) {
        const int n_rows = slice_rows(dst);
        if (dst == static_cast<int>(rank) || n_rows == 0) continue;
        ptx::bulk_copy_to_peer(ptx::map_shared_rank(slot_local, dst),
                               red + dst * rows_per * RED_PITCH,
                               static_cast<uint32_t>(n_rows * RED_PITCH * 4),
                               ptx::map_shared_rank(bar_local, dst));
      }
      ptx::bulk_commit_group();
    }
    {
      __syncwarp();
      bool ok = true;
      if (lane == 0) ok = ptx::mbar_wait(recv_bar, 0, ctl, kDevTimeoutEpilogue);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      // every copy into this CTA has landed: the cluster barrier that keeps
      // CTAs alive for incoming copies can complete while this CTA reduces
      ptx::cluster_arrive_relaxed();
      const int r0 = rank * rows_per;
      constexpr int C8 = BLOCK_N / 8;
      const int items = ok ? slice_rows(rank) * C8 : 0;
      const int n0 = ti.n_blk * BLOCK_N;
      for (int item = threadIdx.x; item < items; item += kThreads) {
        const int lr = item / C8;  // row within the slice
        const int c = 8 * (item % C8);
        if (n0 + c >= p.N) continue;
        float4 lo = make_float4(0, 0, 0, 0), hi = make_float4(0, 0, 0, 0);
#pragma unroll
        for (int src = 0; src < kMaxSplit; ++src) {  // fixed order: deterministic
          if (src >= S) break;
          const float* part = (src == static_cast<int>(rank))
                                  ? red + (r0 + lr) * RED_PITCH + c
                                  : recv + (src * rows_per + lr) * RED_PITCH + c;
          const float4 x = *reinterpret_cast<const float4*>(part);
          const float4 y = *reinterpret_cast<const float4*>(part + 4);
          lo.x += x.x; lo.y += x.y; lo.z += x.z; lo.w += x.w;
          hi.x += y.x; hi.y += y.y; hi.z += y.z; hi.w += y.w;
        }
        uint4 v;
        v.x = pack_bf16x2(lo.x, lo.y);
        v.y = pack_bf16x2(lo.z, lo.w);
        v.z = pack_bf16x2(hi.x, hi.y);
        v.w = pack_bf16x2(hi.z, hi.w);
        const size_t grow = (size_t)ti.m_blk * kBlockM + r0 + lr;
        *reinterpret_cast<uint4*>(p.d + grow * p.ldd + n0 + c) = v;
      }
    }
    if (threadIdx.x == 0) ptx::bulk_wait_group_read0();  // outgoing copies done reading
    __syncwarp();
    ptx::cluster_wait();  // no CTA leaves while a copy into it may still land
  }

  ptx::tc_fence_before_sync();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace dg
