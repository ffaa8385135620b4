// Shape-keyed configuration picker (host only).
//
// The pages choose a kernel per shape and per GPU at run time (DeepGEMM
// release article, part 1.3 and part 4.1: the JIT "automatically picks the
// best kernel"; youleyou.com article, features: code generated "by hardware
// configuration and input size").  Here every variant is compiled ahead of
// time and this picker maps (form, rows, N, K, groups, SM count) to one of
// them: BLOCK_N, pipeline depth, accumulator buffers, split-K and grid size.
#pragma once

#include <cmath>

namespace dg {

struct Variant {
  int block_n;
  int stages;
  int num_acc;
  int kps;      // 128-wide K blocks per ring stage (one TMA box of each operand)
  int a_rows;   // rows of A a stage holds (64: dense A of at most 64 rows)
  bool decode;  // built for dense problems of at most one 128-row block
  bool small;   // two CTAs fit per SM; one tile per CTA
  bool f32 = false;  // for the FP32-output forms only: 8 KB of epilogue staging per
                     // epilogue warp, four output boxes in flight
};

// The compiled variants: general ones first (every form), then
// the decode-shaped dense ones, whose stages are several K blocks deep so
// that each TMA box moves 32-64 KB, then the small decode ones (at most
// ~100 KB of shared memory and 256 TMEM columns, so that the next kernel's
// CTAs can be resident and warm L2 with their weights while this kernel
// drains), then the FP32-output ones (a shallower ring, room for four
// output boxes in flight per epilogue warp: those forms are bound by writing
// their FP32 output).
constexpr Variant kVariants[] = {
    {256, 4, 1, 1, 128, false, false},
    {128, 6, 2, 1, 128, false, false},
    {64, 8, 2, 1, 128, false, false},
    {32, 9, 2, 1, 128, false, false},
    {128, 2, 1, 4, 64, true, false},
    {64, 3, 2, 4, 64, true, false},
    {256, 2, 1, 2, 64, true, false},
    {128, 3, 1, 2, 128, true, false},
    {64, 4, 2, 2, 128, true, false},
    {256, 2, 1, 2, 128, true, false},
    {128, 2, 1, 2, 64, true, true},
    {64, 3, 1, 2, 64, true, true},
    {128, 3, 1, 1, 128, true, true},
    {64, 2, 1, 2, 128, true, true},
    {256, 3, 1, 1, 128, false, false, true},
    {128, 4, 2, 1, 128, false, false, true},
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);
constexpr int kMaxSplitK = 8;  // portable cluster size

struct PickedConfig {
  int variant;   // index into kVariants
  int split_k;   // K slices per output tile (> 1: one cluster of split_k CTAs per tile)
  int grid;      // CTAs to launch
  int out_tiles; // output tiles (upper bound for masked)
};

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// Output rows of one tile (every variant: one 128-row MMA block).
inline int tile_rows(const Variant&) { return 128; }

// How many split-K clusters of `cluster` CTAs of variant `variant` the device
// can run at once.  max_clusters[v][s] for s in 1..kMaxSplitK; a value <= 0 means
// "not known": then the SM count divided by the cluster size is assumed.
struct ClusterLimits {
  int max_clusters[kNumVariants][kMaxSplitK + 1];
};

inline int cluster_limit(const ClusterLimits* lim, int v, int s, int num_sms) {
  int n = lim ? lim->max_clusters[v][s] : 0;
  return n > 0 ? n : num_sms / s;
}

// Split-K parks each CTA's FP32 partial and the slices the other CTAs push to
// it in the (then idle) operand ring: (2 * rows + split) rows of BLOCK_N + 4
// floats must fit.
inline bool split_fits(const Variant& var, int rows, int split) {
  const long long ring = static_cast<long long>(var.stages) * var.kps * (var.a_rows + var.block_n) * 128;
  const long long need = static_cast<long long>(2 * rows + split) * (var.block_n + 4) * 4;
  return need <= ring;
}

// Decode-shaped dense problems (at most one 128-row block): HBM-bound.  Pick
// the variant and K split (one cluster of `split` CTAs per output tile, all in
// one wave) that minimise an estimate of the time:
//   fixed cost + smooth max(HBM time of B, busiest CTA's streaming time)
//   + split tail (growing with the CTAs of a cluster)
// where a CTA streams its B slice plus (at a discount: it is read from L2) its
// A slice at a rate that grows with the bytes one ring stage moves (both
// boxes).  The constants were fitted to three sweeps of every (variant,
// split) on the six decode-shaped workloads, each on a different B200: in
// every sweep the pick is the fastest measured configuration, or within
// 0.35 us of it, for each shape.  Returns false if no one-wave configuration
// exists.
inline bool pick_decode(int rows, int N, int K, int num_sms, const ClusterLimits* lim,
                        PickedConfig* out) {
  const int KB = K / 128;
  constexpr double kHbmBytesPerUs = 4.5e6;  // effective, whole GPU
  constexpr double kRate16KB = 20.0;        // KB per microsecond per CTA, 16 KB stages
  constexpr double kRateCap = 70.0;         // KB per microsecond per CTA, large stages
  constexpr double kAWeight = 0.35;         // A slices come from L2
  constexpr double kFixedUs = 6.0;
  constexpr double kSplitUs = 1.0;          // cluster barriers, pushes, reduction ...
  constexpr double kSplitPerCtaUs = 0.1;    // ... growing with the CTAs of a cluster
  double best = 1e30;
  bool found = false;
  for (int v = 0; v < kNumVariants; ++v) {
    const Variant& var = kVariants[v];
    if (!var.decode || var.small || rows > var.a_rows) continue;
    const int bn = var.block_n;
    const int nt = ceil_div(N, bn);
    const double stage_kb = var.kps * (bn + var.a_rows) * 128 / 1024.0;
    double r_cta = kRate16KB * stage_kb / 16.0;
    if (r_cta > kRateCap) r_cta = kRateCap;
    for (int s = 1; s <= kMaxSplitK && s <= KB; ++s) {
      if (nt * s > num_sms) break;
      const int per = ceil_div(KB, s);
      if ((s - 1) * per >= KB) continue;          // an empty slice
      if (s > 1 && cluster_limit(lim, v, s, num_sms) < nt) continue;
      if (s > 1 && !split_fits(var, rows, s)) continue;
      const double b_cta = static_cast<double>(bn) * per * 128 / 1024.0;    // KB
      const double a_cta = static_cast<double>(rows) * per * 128 / 1024.0;  // KB
      const double t_cta = (b_cta + kAWeight * a_cta) / r_cta;             // us
      const double t_hbm = static_cast<double>(N) * K / kHbmBytesPerUs;     // us
      const double t_stream = std::pow(std::pow(t_cta, 8.0) + std::pow(t_hbm, 8.0), 0.125);
      const double t = kFixedUs + t_stream + (s > 1 ? kSplitUs + kSplitPerCtaUs * s : 0.0);
      if (t < best - 1e-9) {
        best = t;
        found = true;
        out->variant = v;
        out->split_k = s;
        out->out_tiles = nt;
        out->grid = nt * s;
      }
    }
  }
  return found;
}

// kind: 0 dense, 1 contiguous, 2 masked, 3 K-grouped.  rows: M, M_sum, max_m,
// or M (the output rows of each group of the K-grouped form).
inline PickedConfig pick_config(int kind, int rows, int N, int K, int G, int expected_m,
                                int num_sms, const ClusterLimits* lim = nullptr,
                                bool mn_operands = false, bool f32_out = false) {
  PickedConfig best{1, 1, 1, 1};
  if (kind == 0 && rows <= 128 && !mn_operands && !f32_out &&
      pick_decode(rows, N, K, num_sms, lim, &best))
    return best;

  // Everything else: persistent CTAs, no split.  Tile time is set by the
  // bytes the SM must pull through TMA per K block (A 16 KB + B BLOCK_N x
  // 128 B; measured on B200 to bound these compute-bound tiles), so choose
  // the variant minimising waves x bytes per K block.  The FP32-output forms
  // are bound by writing their output instead: waves x output columns per
  // tile (on a tie, the 256-column variant: 0.866 against 0.881 ms for the
  // 128-column one with two accumulators on the K-grouped workload).
  int eff_rows = rows;
  int groups = 1;
  if (kind == 2) {
    eff_rows = expected_m > 0 ? (expected_m < rows ? expected_m : rows) : rows;
    groups = G;
  } else if (kind == 3) {
    groups = G;  // every group has all of its output tiles
  }
  double best_cost = 1e30;
  for (int v = 0; v < kNumVariants; ++v) {
    const Variant& var = kVariants[v];
    if (var.small || var.a_rows < 128 || var.f32 != f32_out) continue;
    // M-/N-major operands: one K block per stage and whole 128-column B boxes
    if (mn_operands && (var.decode || var.kps != 1 || var.block_n % 128 != 0)) continue;
    // decode variants run one tile per CTA; several K blocks per stage: dense only
    if (var.decode || (var.kps != 1 && kind != 0)) continue;
    const int bn = var.block_n;
    if (bn > 128 && N <= 128) continue;
    const int tm = tile_rows(var);
    const int m_blocks = groups * ceil_div(eff_rows > 0 ? eff_rows : 1, tm);
    const int n_tiles = ceil_div(N, bn);
    const long long tiles = static_cast<long long>(m_blocks) * n_tiles;
    const int waves = ceil_div(tiles, num_sms);
    double cost = f32_out ? static_cast<double>(waves) * bn : waves * (tm / 8.0 + bn / 8.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.variant = v;
    }
  }
  const int bn = kVariants[best.variant].block_n;
  const int tm = tile_rows(kVariants[best.variant]);
  const int n_tiles = ceil_div(N, bn);
  long long tiles;
  if (kind == 2 || kind == 3) {
    tiles = static_cast<long long>(G) * ceil_div(rows, tm) * n_tiles;  // masked: upper bound
  } else {
    tiles = static_cast<long long>(ceil_div(rows, tm)) * n_tiles;
  }
  best.split_k = 1;
  best.out_tiles = tiles > 0x7fffffff ? 0x7fffffff : static_cast<int>(tiles);
  best.grid = tiles < num_sms ? static_cast<int>(tiles) : num_sms;
  if (best.grid < 1) best.grid = 1;
  return best;
}

}  // namespace dg

namespace dg {

// Last-wave split of a dense GEMM.  The persistent kernel walks the output
// tiles column by column (m fastest), one tile per SM per wave.  When the
// last wave would hold at most a quarter as many tiles as there are SMs, each
// of them a whole K loop while the other SMs idle, the first launch stops
// after the whole waves (`main_tiles`) and the remaining tiles, one or two
// rectangles of D (the last m-blocks of one column, then whole columns), run
// as further launches of 128 x 128 tiles of a decode variant, split along K
// across thread-block clusters so that they fill the SMs.
struct TailRect {
  int row0, rows;  // rows of D (and of A)
  int col0, cols;  // columns of D (rows of B); col0 is a multiple of 128
};
struct TailPlan {
  int main_tiles = 0;  // tiles of the first launch (0: no split)
  int n_rects = 0;
  TailRect rect[2] = {};
  int variant = -1;    // decode variant of the tail launches
  int split = 1;       // K slices per tail tile (CTAs per cluster)
};

inline TailPlan plan_tail(int rows, int N, int K, int num_sms, int main_variant,
                          const ClusterLimits* lim) {
  TailPlan tp;
  const Variant& mv = kVariants[main_variant];
  const int KB = K / 128;
  // only the general variants with whole 128-column B scale blocks per tile
  // (a rectangle then starts on a scale block), and long enough K loops that
  // a wave is worth saving
  if (mv.decode || mv.small || mv.block_n % 128 != 0 || KB < 32 || num_sms < 2) return tp;
  const int mb = ceil_div(rows, 128), nb = ceil_div(N, mv.block_n);
  const long long tiles = static_cast<long long>(mb) * nb;
  if (tiles <= num_sms) return tp;
  const int rem = static_cast<int>(tiles % num_sms);
  if (rem == 0 || 2 * rem > num_sms) return tp;
  int tail_v = -1;
  for (int v = 0; v < kNumVariants; ++v) {
    const Variant& x = kVariants[v];
    if (x.decode && !x.small && x.block_n == 128 && x.a_rows == 128) tail_v = v;
  }
  if (tail_v < 0) return tp;
  const int main_tiles = static_cast<int>(tiles) - rem;
  const int c0 = main_tiles / mb, m0 = main_tiles % mb;
  TailPlan out;
  out.main_tiles = main_tiles;
  out.variant = tail_v;
  int c_next = c0;
  if (m0 > 0) {
    out.rect[out.n_rects++] = TailRect{m0 * 128, rows - m0 * 128, c0 * mv.block_n,
                                       (N < (c0 + 1) * mv.block_n ? N : (c0 + 1) * mv.block_n) -
                                           c0 * mv.block_n};
    c_next = c0 + 1;
  }
  if (c_next < nb)
    out.rect[out.n_rects++] = TailRect{0, rows, c_next * mv.block_n, N - c_next * mv.block_n};
  int tail_tiles = 0;
  for (int i = 0; i < out.n_rects; ++i)
    tail_tiles += ceil_div(out.rect[i].rows, 128) * ceil_div(out.rect[i].cols, 128);
  // the largest split whose clusters all fit in one wave, each CTA keeping at
  // least four K blocks.  Unsplit, the tail's 128-column tiles would stream
  // their whole K loop with every SM busy, while the partial wave they
  // replace runs with few SMs contending for L2 (measured: 4096 x 4096 x 7168,
  // 68 tiles past three waves, took 12 us longer as 136 unsplit tail tiles),
  // so a split of at least 2 is required.
  const Variant& tv = kVariants[tail_v];
  for (int s = kMaxSplitK; s >= 2; s >>= 1) {
    if (static_cast<long long>(tail_tiles) * s > num_sms || KB < 4 * s) continue;
    if (s > 1 && (!split_fits(tv, 128, s) || cluster_limit(lim, tail_v, s, num_sms) < tail_tiles))
      continue;
    out.split = s;
    return out;
  }
  return tp;  // the tail does not fit one wave even unsplit: keep one launch
}

}  // namespace dg
