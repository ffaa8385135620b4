// Shape-keyed configuration picker (host only).
//
// The pages choose a kernel per shape and per GPU at run time (DeepGEMM
// release article, part 1.3 and part 4.1: the JIT "automatically picks the
// best kernel"; youleyou.com article, features: code generated "by hardware
// configuration and input size").  Here every variant is compiled ahead of
// time and this picker maps (form, rows, N, K, groups, SM count) to one of
// them: BLOCK_N, pipeline depth, accumulator buffers, split-K and grid size.
#pragma once

namespace dg {

struct Variant {
  int block_n;
  int stages;
  int num_acc;
};

// The compiled variants, largest tile first.
constexpr Variant kVariants[] = {
    {256, 4, 1},
    {128, 6, 2},
    {64, 8, 2},
    {32, 9, 2},
};
constexpr int kNumVariants = sizeof(kVariants) / sizeof(kVariants[0]);

struct PickedConfig {
  int variant;   // index into kVariants
  int split_k;   // K slices per output tile
  int grid;      // CTAs to launch
  int out_tiles; // output tiles (upper bound for masked)
};

inline int ceil_div(long long a, long long b) { return static_cast<int>((a + b - 1) / b); }

// kind: 0 dense, 1 contiguous, 2 masked.  rows: M, M_sum or max_m.
inline PickedConfig pick_config(int kind, int rows, int N, int K, int G, int expected_m,
                                int num_sms) {
  PickedConfig best{1, 1, 1, 1};
  const int KB = K / 128;
  // Rows that will actually carry tokens, per group, for the estimate.
  int eff_rows = rows;
  int groups = 1;
  if (kind == 2) {
    eff_rows = expected_m > 0 ? (expected_m < rows ? expected_m : rows) : rows;
    groups = G;
  }
  const int m_blocks = groups * ceil_div(eff_rows > 0 ? eff_rows : 1, 128);

  // Decode-shaped dense problems (one 128-row block): memory-bound.  Keep a
  // 128-wide tile and split K until the tiles fill the SMs in one wave.
  if (kind == 0 && rows <= 128) {
    const int v = 1;  // BLOCK_N = 128
    const int n_tiles = ceil_div(N, kVariants[v].block_n);
    int split = 1;
    for (int s = 2; s <= KB && n_tiles * s <= num_sms; ++s) {
      if (KB / s < 2) break;  // keep at least two K blocks per slice
      split = s;
    }
    // prefer a split that divides the K blocks evenly, if one nearly as large exists
    for (int s = split; s >= 2 && s * 4 >= split * 3; --s) {
      if (KB % s == 0) { split = s; break; }
    }
    best.variant = v;
    best.split_k = split;
    best.out_tiles = n_tiles;
    const int tiles = n_tiles * split;
    best.grid = tiles < num_sms ? tiles : num_sms;
    return best;
  }

  // Everything else: choose the tile width minimising (waves x tile width),
  // a proxy for the time of the busiest SM, preferring wider tiles on ties.
  double best_cost = 1e30;
  for (int v = 0; v < kNumVariants; ++v) {
    const int bn = kVariants[v].block_n;
    if (bn > 128 && N <= 128) continue;
    const int n_tiles = ceil_div(N, bn);
    const long long tiles = static_cast<long long>(m_blocks) * n_tiles;
    const int waves = ceil_div(tiles, num_sms);
    const double cost = waves * (bn + 32.0);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.variant = v;
    }
  }
  const int bn = kVariants[best.variant].block_n;
  const int n_tiles = ceil_div(N, bn);
  long long tiles;
  if (kind == 2) {
    tiles = static_cast<long long>(G) * ceil_div(rows, 128) * n_tiles;  // upper bound
  } else {
    tiles = static_cast<long long>(ceil_div(rows, 128)) * n_tiles;
  }
  best.split_k = 1;
  best.out_tiles = tiles > 0x7fffffff ? 0x7fffffff : static_cast<int>(tiles);
  best.grid = tiles < num_sms ? static_cast<int>(tiles) : num_sms;
  if (best.grid < 1) best.grid = 1;
  return best;
}

}  // namespace dg
