// Dense FP8 block-scaled GEMM on SM pairs: the compute-bound variant.
//
// Same operation as sm100_fp8_gemm.cuh (DeepGEMM release article,
// deepseek.csdn.net, part 1.2; DeepGEMM project card, aiproducthub.cn,
// "technical implementation"): D = bf16(sum_kb sfa * sfb * A_kb * B_kb^T),
// dense form only.
//
// Why pairs: the single-SM kernel keeps about 192 KB of operands in flight
// per SM (four 48 KB stages of a 128 x 256 tile) and, at the ~1.8 us a stage
// takes from its TMA request to landing inside the running GEMM, that bounds
// it near 2 PFLOP/s while the tensor core idles half the time.  Here two CTAs
// of a cluster (one per SM) compute one 256 x 256 output tile with
// tcgen05.mma.cta_group::2: each CTA holds 128 rows of A and 128 rows of B per
// stage (32 KB), and the pair's leader issues one MMA of M = 256, N = 256 that
// reads both CTAs' shared memory, each CTA accumulating its own 128 rows x 256
// columns in its own TMEM, so the same in-flight bytes carry 1.5x the work.
// Measured on B200 it is correct but not faster (1.6-1.7 PFLOP/s on the
// prefill shapes): a stage's round trip through the pair (commit to both
// CTAs, loads completing on the leader's barrier, remote arrives) is longer.
// The library runs it only when it is forced (DG_FORCE_CONFIG).
//
// Pair protocol (rank 0 = leader, rank 1 = peer; barriers at the same
// shared-memory offsets in both CTAs):
//  * full[s] (leader's only): the leader's producer arrives with the whole
//    stage's transaction bytes (both CTAs), both CTAs' TMA loads complete on
//    it (cta_group::2 form; each CTA loads its own boxes), and both CTAs'
//    scale warps arrive
//    after writing their UE8M0 words (the peer remotely);
//  * empty[s] (both): the leader's MMA warp commits once to each CTA's;
//  * acc_full (both): the leader's commits at the end of a tile, one each;
//  * acc_empty (leader's): one arrive per epilogue warp of both CTAs.
// Scale factors: each CTA's scale warp writes the SFA words of its 128 rows
// and the SFB words of all 256 B rows of the tile; the leader's
// tcgen05.cp.cta_group::2 copies each CTA's words into that CTA's TMEM.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "sm100_fp8_gemm.cuh"
#include "sm100_ptx.cuh"

namespace dg {

// Geometry of the pair variant: BLOCK_N output columns per pair tile (each CTA
// loads BLOCK_N / 2 rows of B), STAGES ring stages, one TMEM accumulator.
template <int BLOCK_N, int STAGES>
struct PairShape {
  static constexpr int kTileM = 2 * kBlockM;                 // output rows per pair tile
  static constexpr int kBHalf = BLOCK_N / 2;                 // B rows per CTA per stage
  static constexpr int kABytes = kBlockM * kBlockK;          // 16 KB
  static constexpr int kBBytes = kBHalf * kBlockK;
  static constexpr int kSfbChunks = (BLOCK_N + 127) / 128;   // 128-row SFB chunks of the tile
  static constexpr int kSfBytes = 512 * (1 + kSfbChunks);
  static constexpr int kSfCols = 4 * (1 + kSfbChunks);
  static constexpr int kAccCols = BLOCK_N;
  static constexpr int kTmemCols = pow2_ceil(kAccCols + STAGES * kSfCols);
  static constexpr int kEpiCols = 64;
  static constexpr int kEpiPitch = kEpiCols * 2;
  static constexpr int kEpiBytes = 4 * 32 * kEpiPitch;
  static constexpr int kBarBytes = 8 * (2 * STAGES + 3);
  static constexpr int kSmemBytes = 1024 + STAGES * (kABytes + kBBytes) + kEpiBytes +
                                    STAGES * kSfBytes + kBarBytes + 16;
  static_assert(BLOCK_N % 128 == 0 && BLOCK_N <= 256, "pair tiles are 128 or 256 columns");
  static_assert(kSmemBytes <= 232448, "shared memory budget (227 KB) exceeded");
  static_assert(kTmemCols <= 512, "TMEM budget exceeded");
};

template <int BLOCK_N, int STAGES>
__global__ void __launch_bounds__(kThreads, 1)
    fp8_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a,
                         const __grid_constant__ CUtensorMap tmap_b,
                         const __grid_constant__ CUtensorMap tmap_d, const GemmArgs p) {
  using Shape = PairShape<BLOCK_N, STAGES>;
  constexpr int A_BYTES = Shape::kABytes;
  constexpr int B_BYTES = Shape::kBBytes;
  constexpr int SF_BYTES = Shape::kSfBytes;
  constexpr int SF_COLS = Shape::kSfCols;
  constexpr int SFB_CHUNKS = Shape::kSfbChunks;
  constexpr int TMEM_COLS = Shape::kTmemCols;
  constexpr int B_HALF = Shape::kBHalf;
  constexpr int TILE_M = Shape::kTileM;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = ptx::smem_addr(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_addr & 1023u)) & 1023u);
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * A_BYTES;
  uint8_t* sEpi = sB + STAGES * B_BYTES;
  uint8_t* sSF = sEpi + Shape::kEpiBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSF + STAGES * SF_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = ptx::cluster_ctarank();  // 0: leader of the pair
  const bool leader = rank == 0;
  const int pair = blockIdx.x / 2;
  const int num_pairs = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      ptx::mbar_init(&full[s], 3);   // leader producer (+ tx bytes) + two scale warps
      ptx::mbar_init(&empty[s], 1);  // leader's MMA commit
    }
    ptx::mbar_init(acc_full, 1);     // leader's MMA commit
    ptx::mbar_init(acc_empty, 8);    // one lane of each epilogue warp of both CTAs
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
    ptx::prefetch_tensormap(&tmap_a);
    ptx::prefetch_tensormap(&tmap_b);
    ptx::prefetch_tensormap(&tmap_d);
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, TMEM_COLS);
    ptx::tmem_relinquish_pair();
  }
  // barriers of both CTAs initialised and TMEM allocated before any role of
  // either CTA touches them
  ptx::tc_fence_before_sync();
  ptx::cluster_sync();
  ptx::tc_fence_after_sync();
  const uint32_t tmem_base = *tmem_slot;
  ptx::grid_launch_dependents();
  ptx::grid_dependency_wait();

  ptx::WaitCtl ctl{abort_flag, p.error_word, p.timeout_ns};
  const int total = p.num_m_blocks * p.num_n_blocks;  // pair tiles
  auto tile_mn = [&](int t, int& mt, int& nt) {
    mt = t % p.num_m_blocks;  // column-major over tiles, as the single-SM kernel
    nt = t / p.num_m_blocks;
  };
  // the leader's copy of a barrier, as a cluster address
  auto leader_bar = [&](uint64_t* bar) { return ptx::map_shared_rank(ptx::smem_addr(bar), 0); };
  // MMA completion, signalled on the barrier at this offset in both CTAs
  auto commit_both = [&](uint64_t* bar) {
    ptx::tc_commit_pair(ptx::map_shared_rank(ptx::smem_addr(bar), 0));
    ptx::tc_commit_pair(ptx::map_shared_rank(ptx::smem_addr(bar), 1));
  };

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer --
    int it = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += num_pairs) {
      int mt, nt;
      tile_mn(t, mt, nt);
      const int a_row = mt * TILE_M + kBlockM * rank;
      const int b_row = nt * BLOCK_N + B_HALF * rank;
      for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
        const int s = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (lane == 0) {
          ok = ptx::mbar_wait(&empty[s], ph ^ 1, ctl, kDevTimeoutProducer);
          if (ok) {
            if (leader) ptx::mbar_arrive_expect_tx(&full[s], 2 * (A_BYTES + B_BYTES));
            const uint32_t bar = leader_bar(&full[s]);
            ptx::tma_load_4d_pair(sA + s * A_BYTES, &tmap_a, bar, 0, a_row, kb, 0);
            ptx::tma_load_4d_pair(sB + s * B_BYTES, &tmap_b, bar, 0, b_row, kb, 0);
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (leader only) --
    if (leader) {
      constexpr uint32_t idesc = ptx::idesc_mxf8_e4m3_ue8m0(TILE_M, BLOCK_N);
      int it = 0, acc_it = 0;
      bool ok = true;
      for (int t = pair; t < total && ok; t += num_pairs, ++acc_it) {
        // both CTAs' epilogues have drained the accumulator
        if (lane == 0) ok = ptx::mbar_wait(acc_empty, (acc_it & 1) ^ 1, ctl, kDevTimeoutMma);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        ptx::tc_fence_after_sync();
        for (int kb = 0; kb < p.k_blocks; ++kb, ++it) {
          const int s = it % STAGES;
          const uint32_t ph = (it / STAGES) & 1;
          if (lane == 0) ok = ptx::mbar_wait(&full[s], ph, ctl, kDevTimeoutMma);
          ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
          if (!ok) break;
          ptx::tc_fence_after_sync();
          if (lane == 0) {
            const uint32_t sfa_tmem = tmem_base + BLOCK_N + s * SF_COLS;
            const uint32_t sfb_tmem = sfa_tmem + 4;
            const uint32_t sf_smem = ptx::smem_addr(sSF + s * SF_BYTES);
            ptx::tc_cp_pair_32x128b_warpx4(sfa_tmem, ptx::sdesc_sf_32x16(sf_smem));
#pragma unroll
            for (int h = 0; h < SFB_CHUNKS; ++h)
              ptx::tc_cp_pair_32x128b_warpx4(sfb_tmem + 4 * h,
                                             ptx::sdesc_sf_32x16(sf_smem + 512 * (1 + h)));
            const uint64_t da = ptx::sdesc_kmajor_sw128(ptx::smem_addr(sA + s * A_BYTES));
            const uint64_t db = ptx::sdesc_kmajor_sw128(ptx::smem_addr(sB + s * B_BYTES));
#pragma unroll
            for (int ks = 0; ks < kBlockK / 32; ++ks)
              ptx::tc_mma_pair_mxf8_block_scale(tmem_base, da + 2 * ks, db + 2 * ks, idesc,
                                                sfa_tmem, sfb_tmem, kb > 0 || ks > 0);
            commit_both(&empty[s]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (lane == 0) commit_both(acc_full);
        __syncwarp();
      }
      // every MMA this thread issued has completed once `drain` flips
      if (lane == 0) {
        ptx::tc_commit_pair(ptx::map_shared_rank(ptx::smem_addr(drain), 0));
        ptx::mbar_wait_drain(drain, 0, 50000000ull);
      }
      __syncwarp();
    }
  } else if (warp == 2) {
    // --------------------------------------------- scale-factor producer --
    // Stage i of this pair's sequence is K block i % KB of its (i / KB)-th
    // tile; its scales are loaded in batches of PF stages, one batch ahead of
    // their writes, so the global-load latency overlaps several stages.
    constexpr int PF = 8;
    const int KB = p.k_blocks;
    const int n_stages = total > pair ? ((total - pair + num_pairs - 1) / num_pairs) * KB : 0;
    const uint32_t full_leader0 = leader_bar(&full[0]);
    float va[PF][4], vb[PF][SFB_CHUNKS];
    auto load = [&](int i, float (&a)[4], float (&b)[SFB_CHUNKS]) {
      int mt, nt;
      tile_mn(pair + (i / KB) * num_pairs, mt, nt);
      const int kb = i % KB;
      const int m0 = mt * TILE_M + kBlockM * rank;  // this CTA's 128 rows
      const int rows_left = p.rows - m0;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = 32 * c + lane;
        a[c] = r < rows_left ? __ldg(p.sfa + (size_t)(m0 + r) * KB + kb) : 1.0f;
      }
#pragma unroll
      for (int h = 0; h < SFB_CHUNKS; ++h) {
        const int nb = min(nt * (BLOCK_N / 128) + h, p.nb128 - 1);
        b[h] = __ldg(p.sfb + (size_t)nb * KB + kb);
      }
    };
#pragma unroll
    for (int j = 0; j < PF; ++j)
      if (j < n_stages) load(j, va[j], vb[j]);
    bool ok = true;
    for (int i0 = 0; i0 < n_stages && ok; i0 += PF) {
#pragma unroll
      for (int slot = 0; slot < PF; ++slot) {
        const int i = i0 + slot;
        if (i >= n_stages) break;
        const int s = i % STAGES;
        const uint32_t ph = (i / STAGES) & 1;
        if (lane == 0) ok = ptx::mbar_wait(&empty[s], ph ^ 1, ctl, kDevTimeoutScales);
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        uint8_t* sf = sSF + s * SF_BYTES;
        // one K block per stage: byte 0 of every word; the other bytes scale 1
        *reinterpret_cast<uint4*>(sf + 16 * lane) = make_uint4(
            0x7F7F7F00u | ue8m0(va[slot][0]), 0x7F7F7F00u | ue8m0(va[slot][1]),
            0x7F7F7F00u | ue8m0(va[slot][2]), 0x7F7F7F00u | ue8m0(va[slot][3]));
#pragma unroll
        for (int h = 0; h < SFB_CHUNKS; ++h) {
          const uint32_t x = 0x7F7F7F00u | ue8m0(vb[slot][h]);
          *reinterpret_cast<uint4*>(sf + 512 * (1 + h) + 16 * lane) = make_uint4(x, x, x, x);
        }
        ptx::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (leader) ptx::mbar_arrive(&full[s]);
          else ptx::mbar_arrive_cluster(full_leader0 + 8u * s);
        }
      }
      // The next batch of loads goes out only now: an arrive releases this
      // thread's earlier memory accesses, so it would otherwise wait for
      // loads still in flight for later stages.
#pragma unroll
      for (int slot = 0; slot < PF; ++slot)
        if (i0 + PF + slot < n_stages) load(i0 + PF + slot, va[slot], vb[slot]);
    }
  } else if (warp >= 4) {
    // --------------------------------------------------------- epilogue --
    const int q = warp & 3;  // TMEM lane quarter of this warp
    const uint32_t acc_empty_leader = leader_bar(acc_empty);
    uint8_t* stage = sEpi + q * 32 * Shape::kEpiPitch;
    int acc_it = 0;
    bool ok = true;
    for (int t = pair; t < total && ok; t += num_pairs, ++acc_it) {
      int mt, nt;
      tile_mn(t, mt, nt);
      if (lane == 0) ok = ptx::mbar_wait(acc_full, acc_it & 1, ctl, kDevTimeoutEpilogue);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      ptx::tc_fence_after_sync();
      const int row0 = mt * TILE_M + kBlockM * rank + 32 * q;  // first row of this warp
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      if (row0 < p.rows) {
#pragma unroll 1
        for (int c0 = 0; c0 < BLOCK_N; c0 += 64) {
          uint32_t r[64];
          ptx::tc_ld_32x32b_x32(t_row + c0, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
          ptx::tc_ld_32x32b_x32(t_row + c0 + 32, *reinterpret_cast<uint32_t(*)[32]>(&r[32]));
          ptx::tc_wait_ld();
          // BF16 row of this lane into the staging tile, 16-byte chunk j at
          // position j ^ (lane % 8) (the 128-byte swizzle of the D map) ...
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint4 v;
            v.x = pack_bf16x2(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
            v.y = pack_bf16x2(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
            v.z = pack_bf16x2(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
            v.w = pack_bf16x2(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
            *reinterpret_cast<uint4*>(stage + lane * Shape::kEpiPitch + 16 * (j ^ (lane % 8))) = v;
          }
          // ... then one TMA store of 32 rows x 64 columns (rows past M and
          // columns past N are clipped by the TMA unit)
          ptx::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            ptx::tma_store_2d(&tmap_d, stage, nt * BLOCK_N + c0, row0);
            ptx::bulk_commit_group();
            ptx::bulk_wait_group_read0();  // staging tile free again
          }
          __syncwarp();
        }
      }
      // this warp is done with the accumulator: tell the leader's MMA warp
      ptx::tc_fence_before_sync();
      __syncwarp();
      if (lane == 0) {
        if (leader) ptx::mbar_arrive(acc_empty);
        else ptx::mbar_arrive_cluster(acc_empty_leader);
      }
    }
    if (lane == 0) ptx::bulk_wait_group_read0();
  }

  // No CTA of the pair leaves (or frees TMEM) while the other may still use
  // its shared memory or TMEM: the leader's MMAs read both CTAs' operands and
  // write both CTAs' TMEM, and the peer arrives on the leader's barriers.
  ptx::tc_fence_before_sync();
  __syncwarp();
  ptx::cluster_sync();
  if (warp == 1) {
    ptx::tc_fence_after_sync();
    ptx::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
}

}  // namespace dg
