"""Seeded synthetic inputs for the FP8 block-scaled GEMM, shared by the tests, the
oracle checks and the benchmark.

This module only *produces inputs*: random FP32 matrices, their quantisation to
FP8 E4M3 with power-of-two block scales (or, for the BF16-operand GEMM, their
rounding to BF16 operands by ``ml_dtypes``), and the MoE group structure
(per-expert token counts, ``m_indices``, ``masked_m``).  It holds none of the
GEMM's own arithmetic: no decoding of operands, no scale application, no
accumulation and no rounding of the result.  Those live, independently, in
``oracle/`` (CPU) and in the CUDA library.

Input recipe (the pages' workloads are DeepSeek-V3/R1 inference GEMMs, prefill
and decode, dense and MoE-grouped; see the DeepGEMM release articles, sections on
performance and on the MoE grouped layouts):

* values: i.i.d. N(0, 1) in FP32 from numpy's PCG64, one child stream per tensor;
* quantisation: per block, ``scale = 2**e`` with ``e`` the smallest integer such
  that ``amax <= 448 * 2**e`` (an all-zero block gets scale 1); the block is then
  divided by the scale (exact, a power of two) and rounded to E4M3 ("fn" variant,
  max 448) with round-to-nearest-even by ``ml_dtypes``;
* A blocks are 1 x 128 (one scale per row per 128-wide K block); B blocks are
  128 x 128 (the last N block may be partial and then covers its real rows only);
* contiguous grouped layout: expert probabilities proportional to rank**-1.1 for
  ranks 1..G in a seeded random order, token counts from a seeded multinomial,
  each expert's segment padded up to a multiple of 128 rows, padding rows marked
  ``-1`` in ``m_indices`` and filled with random FP8 bytes (so that a kernel that
  forgets to skip them is caught);
* masked grouped layout: ``masked_m[g]`` uniform in ``[0, max_m]``;
* K-grouped layout (weight gradient): the contiguous layout's token counts,
  each expert's rows padded with zero rows to a multiple of 128; A (output
  gradients) and B (layer inputs) stored one row per token;
* BF16 operands: the same N(0, 1) values (same streams) rounded to BF16 with
  round-to-nearest-even, and the same group structure; no scales.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import ml_dtypes
import numpy as np

E4M3_MAX = 448.0
BLOCK_K = 128          # K extent of every scale block (A and B)
BLOCK_N_SCALE = 128    # N extent of a B scale block
SENTINEL_BF16 = 0x7FBF  # a quiet-NaN BF16 pattern no computed value can take

# Stream tags: each tensor of a problem gets its own child generator.
_TAG_A, _TAG_B, _TAG_GROUPS, _TAG_PAD = 0, 1, 2, 3


def _rng(seed: int, tag: int, sub: int = 0) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(tag), int(sub)]))


def pow2_block_scale(amax: np.ndarray) -> np.ndarray:
    """Smallest power of two ``s`` with ``amax <= 448 * s`` (1 where amax == 0).

    Computed with exact exponent arithmetic (frexp/ldexp), not a float log2.
    """
    amax = np.asarray(amax, dtype=np.float64)
    ratio = amax / E4M3_MAX
    _, p = np.frexp(ratio)            # ratio = f * 2**p, f in [0.5, 1)
    e = p.astype(np.int64)            # 2**p >= ratio always
    # step down while the next smaller power of two still covers amax
    lower = np.ldexp(E4M3_MAX, e - 1) >= amax
    e = np.where(lower, e - 1, e)
    e = np.where(amax == 0, 0, e)
    s = np.ldexp(1.0, e)
    assert np.all(amax <= E4M3_MAX * s)
    assert np.all((amax == 0) | (amax > E4M3_MAX * s / 2))
    return s.astype(np.float32)


def quantize_rows(x: np.ndarray, rows_per_block: int) -> tuple[np.ndarray, np.ndarray]:
    """Quantise FP32 ``x[R, K]`` to E4M3 bytes with one power-of-two scale per
    ``rows_per_block x 128`` block.  Returns ``(q uint8 [R, K], s float32
    [ceil(R / rows_per_block), K / 128])``."""
    R, K = x.shape
    assert K % BLOCK_K == 0
    KB = K // BLOCK_K
    RB = -(-R // rows_per_block)
    pad = RB * rows_per_block - R
    ax = np.abs(x).reshape(R, KB, BLOCK_K).max(axis=2)           # [R, KB]
    if pad:
        ax = np.concatenate([ax, np.zeros((pad, KB), ax.dtype)], axis=0)
    amax = ax.reshape(RB, rows_per_block, KB).max(axis=1)          # [RB, KB]
    s = pow2_block_scale(amax)                                     # [RB, KB]
    srow = np.repeat(s, rows_per_block, axis=0)[:R]                # [R, KB]
    y = x.reshape(R, KB, BLOCK_K) / srow[:, :, None]
    q = y.reshape(R, K).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    return q, s


def _normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _quantized_b(seed: int, G: int, N: int, K: int) -> tuple[np.ndarray, np.ndarray]:
    """B[G, N, K] quantised per group with 128x128 blocks (generated group by
    group to bound host memory)."""
    NB = -(-N // BLOCK_N_SCALE)
    qb = np.empty((G, N, K), np.uint8)
    sb = np.empty((G, NB, K // BLOCK_K), np.float32)
    for g in range(G):
        qb[g], sb[g] = quantize_rows(_normal(_rng(seed, _TAG_B, g), (N, K)), BLOCK_N_SCALE)
    return qb, sb


@dataclasses.dataclass
class DenseProblem:
    a: np.ndarray     # uint8 [M, K]  E4M3 bytes, K-major
    sfa: np.ndarray   # float32 [M, K/128]
    b: np.ndarray     # uint8 [N, K]  E4M3 bytes, K-major
    sfb: np.ndarray   # float32 [ceil(N/128), K/128]
    M: int
    N: int
    K: int

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def bytes(self) -> float:
        return float(self.a.nbytes + self.sfa.nbytes + self.b.nbytes + self.sfb.nbytes
                     + 2 * self.M * self.N)


def dense_problem(M: int, N: int, K: int, seed: int = 0) -> DenseProblem:
    qa, sa = quantize_rows(_normal(_rng(seed, _TAG_A), (M, K)), 1)
    qb, sb = _quantized_b(seed, 1, N, K)
    return DenseProblem(qa, sa, qb[0], sb[0], M, N, K)


@dataclasses.dataclass
class ContiguousProblem:
    a: np.ndarray          # uint8 [M_sum, K]
    sfa: np.ndarray        # float32 [M_sum, K/128]
    b: np.ndarray          # uint8 [G, N, K]
    sfb: np.ndarray        # float32 [G, ceil(N/128), K/128]
    m_indices: np.ndarray  # int32 [M_sum]; expert id or -1 for padding rows
    counts: np.ndarray     # int64 [G] real tokens per expert
    M_sum: int
    N: int
    K: int
    G: int

    def valid_rows(self) -> int:
        return int((self.m_indices >= 0).sum())

    def flops(self) -> float:
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        used = int((self.counts > 0).sum())
        v = self.valid_rows()
        KB = self.K // BLOCK_K
        NB = -(-self.N // BLOCK_N_SCALE)
        return float(v * self.K + v * KB * 4 + used * (self.N * self.K + NB * KB * 4)
                     + 2 * v * self.N + 4 * self.M_sum)


def zipf_counts(total: int, G: int, s: float, seed: int) -> np.ndarray:
    rng = _rng(seed, _TAG_GROUPS)
    ranks = rng.permutation(G) + 1
    p = ranks.astype(np.float64) ** (-s)
    p /= p.sum()
    return rng.multinomial(total, p)


def contiguous_problem(G: int = 32, N: int = 4096, K: int = 7168, total_tokens: int = 8192,
                       zipf_s: float = 1.1, align: int = 128, seed: int = 0,
                       counts: Optional[np.ndarray] = None) -> ContiguousProblem:
    if counts is None:
        counts = zipf_counts(total_tokens, G, zipf_s, seed)
    counts = np.asarray(counts, dtype=np.int64)
    assert counts.shape == (G,)
    padded = -(-counts // align) * align
    M_sum = int(padded.sum())
    m_indices = np.full(M_sum, -1, np.int32)
    off = 0
    for g in range(G):
        m_indices[off:off + counts[g]] = g
        off += int(padded[g])
    qa, sa = quantize_rows(_normal(_rng(seed, _TAG_A), (M_sum, K)), 1)
    qb, sb = _quantized_b(seed, G, N, K)
    return ContiguousProblem(qa, sa, qb, sb, m_indices, counts, M_sum, N, K, G)


@dataclasses.dataclass
class MaskedProblem:
    a: np.ndarray         # uint8 [G, max_m, K]
    sfa: np.ndarray       # float32 [G, max_m, K/128]
    b: np.ndarray         # uint8 [G, N, K]
    sfb: np.ndarray       # float32 [G, ceil(N/128), K/128]
    masked_m: np.ndarray  # int32 [G]
    G: int
    max_m: int
    N: int
    K: int
    expected_m: int

    def valid_rows(self) -> int:
        return int(np.clip(self.masked_m, 0, self.max_m).sum())

    def flops(self) -> float:
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        mm = np.clip(self.masked_m, 0, self.max_m)
        used = int((mm > 0).sum())
        v = int(mm.sum())
        KB = self.K // BLOCK_K
        NB = -(-self.N // BLOCK_N_SCALE)
        return float(v * self.K + v * KB * 4 + used * (self.N * self.K + NB * KB * 4)
                     + 2 * v * self.N + 4 * self.G)


def masked_problem(G: int = 32, max_m: int = 256, N: int = 4096, K: int = 7168, seed: int = 0,
                   masked_m: Optional[np.ndarray] = None, expected_m: Optional[int] = None
                   ) -> MaskedProblem:
    if masked_m is None:
        masked_m = _rng(seed, _TAG_GROUPS).integers(0, max_m + 1, G)
    masked_m = np.asarray(masked_m, dtype=np.int32)
    assert masked_m.shape == (G,)
    qa, sa = quantize_rows(_normal(_rng(seed, _TAG_A), (G * max_m, K)), 1)
    qb, sb = _quantized_b(seed, G, N, K)
    if expected_m is None:
        expected_m = max(1, int(round(float(np.clip(masked_m, 0, max_m).mean()))))
    return MaskedProblem(qa.reshape(G, max_m, K), sa.reshape(G, max_m, K // BLOCK_K), qb, sb,
                         masked_m, G, max_m, N, K, int(expected_m))


@dataclasses.dataclass
class KGroupedProblem:
    """The weight gradient of an M-grouped layer: per expert g,
    dW[g] = dY_g^T X_g, the reduction running over the expert's tokens.  In the
    K-grouped call's terms: A = dY as [K_sum, M] (one row per token), B = X as
    [K_sum, N], group g owning ks[g] consecutive rows (its tokens, then zero
    rows up to a multiple of 128)."""
    a: np.ndarray        # uint8 [K_sum, M]  E4M3 bytes, M-major
    sfa: np.ndarray      # float32 [M, K_sum/128]
    b: np.ndarray        # uint8 [K_sum, N]  E4M3 bytes, N-major
    sfb: np.ndarray      # float32 [ceil(N/128), K_sum/128]
    ks: np.ndarray       # int32 [G]: rows of K of each group (multiples of 128)
    counts: np.ndarray   # tokens of each group (the rest of its rows are zero)
    G: int
    M: int
    N: int
    K_sum: int

    def valid_rows(self) -> int:
        return int(self.counts.sum())

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.valid_rows()

    def bytes(self) -> float:
        v = self.valid_rows()
        KB = self.K_sum // BLOCK_K
        NB = -(-self.N // BLOCK_N_SCALE)
        return float(v * (self.M + self.N) + 4 * (self.M + NB) * KB + 4 * self.G
                     + 4 * self.G * self.M * self.N)


def k_grouped_problem(G: int = 32, M: int = 4096, N: int = 7168, total_tokens: int = 8192,
                      zipf_s: float = 1.1, align: int = 128, seed: int = 0,
                      counts: Optional[np.ndarray] = None) -> KGroupedProblem:
    """Token counts as in the contiguous layout (Zipf over the experts), each
    expert's segment padded with zero rows to a multiple of ``align``; N(0, 1)
    values for the real rows, quantised in 1 x 128 blocks along the tokens for
    A (one scale per column of dY per 128 tokens) and 128 x 128 blocks for B."""
    if counts is None:
        counts = zipf_counts(total_tokens, G, zipf_s, seed)
    counts = np.asarray(counts, dtype=np.int64)
    ks = (-(-counts // align) * align).astype(np.int32)
    K_sum = int(ks.sum())
    real = np.zeros(K_sum, bool)
    off = 0
    for g in range(G):
        real[off:off + counts[g]] = True
        off += int(ks[g])
    xa = _normal(_rng(seed, _TAG_A), (M, K_sum)) * real[None, :]
    xb = _normal(_rng(seed, _TAG_B), (N, K_sum)) * real[None, :]
    qa, sa = quantize_rows(xa, 1)
    qb, sb = quantize_rows(xb, BLOCK_N_SCALE)
    return KGroupedProblem(np.ascontiguousarray(qa.T), sa, np.ascontiguousarray(qb.T), sb, ks,
                           counts, G, M, N, K_sum)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """FP32 values -> BF16 operand bit patterns (round to nearest even, ml_dtypes)."""
    return np.asarray(x, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


@dataclasses.dataclass
class Bf16DenseProblem:
    a: np.ndarray     # uint16 [M, K]  BF16 bits, K-major
    b: np.ndarray     # uint16 [N, K]  BF16 bits, K-major
    M: int
    N: int
    K: int

    def flops(self) -> float:
        return 2.0 * self.M * self.N * self.K

    def bytes(self) -> float:
        return float(self.a.nbytes + self.b.nbytes + 2 * self.M * self.N)


def bf16_dense_problem(M: int, N: int, K: int, seed: int = 0) -> Bf16DenseProblem:
    a = to_bf16_bits(_normal(_rng(seed, _TAG_A), (M, K)))
    b = to_bf16_bits(_normal(_rng(seed, _TAG_B, 0), (N, K)))
    return Bf16DenseProblem(a, b, M, N, K)


@dataclasses.dataclass
class Bf16ContiguousProblem:
    a: np.ndarray          # uint16 [M_sum, K]
    b: np.ndarray          # uint16 [G, N, K]
    m_indices: np.ndarray  # int32 [M_sum]; expert id or -1 for padding rows
    counts: np.ndarray     # int64 [G]
    M_sum: int
    N: int
    K: int
    G: int

    def valid_rows(self) -> int:
        return int((self.m_indices >= 0).sum())

    def flops(self) -> float:
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        used = int((self.counts > 0).sum())
        v = self.valid_rows()
        return float(2 * v * self.K + used * 2 * self.N * self.K + 2 * v * self.N + 4 * self.M_sum)


def bf16_contiguous_problem(G: int, N: int, K: int, counts: np.ndarray, align: int = 128,
                            seed: int = 0) -> Bf16ContiguousProblem:
    counts = np.asarray(counts, dtype=np.int64)
    assert counts.shape == (G,)
    padded = -(-counts // align) * align
    M_sum = int(padded.sum())
    m_indices = np.full(M_sum, -1, np.int32)
    off = 0
    for g in range(G):
        m_indices[off:off + counts[g]] = g
        off += int(padded[g])
    a = to_bf16_bits(_normal(_rng(seed, _TAG_A), (M_sum, K)))
    b = np.stack([to_bf16_bits(_normal(_rng(seed, _TAG_B, g), (N, K))) for g in range(G)])
    return Bf16ContiguousProblem(a, b, m_indices, counts, M_sum, N, K, G)


@dataclasses.dataclass
class Bf16MaskedProblem:
    a: np.ndarray         # uint16 [G, max_m, K]
    b: np.ndarray         # uint16 [G, N, K]
    masked_m: np.ndarray  # int32 [G]
    G: int
    max_m: int
    N: int
    K: int
    expected_m: int

    def valid_rows(self) -> int:
        return int(np.clip(self.masked_m, 0, self.max_m).sum())

    def flops(self) -> float:
        return 2.0 * self.valid_rows() * self.N * self.K

    def bytes(self) -> float:
        mm = np.clip(self.masked_m, 0, self.max_m)
        v = int(mm.sum())
        used = int((mm > 0).sum())
        return float(2 * v * self.K + used * 2 * self.N * self.K + 2 * v * self.N + 4 * self.G)


def bf16_masked_problem(G: int, max_m: int, N: int, K: int, masked_m: np.ndarray,
                        seed: int = 0) -> Bf16MaskedProblem:
    masked_m = np.asarray(masked_m, dtype=np.int32)
    assert masked_m.shape == (G,)
    a = to_bf16_bits(_normal(_rng(seed, _TAG_A), (G * max_m, K))).reshape(G, max_m, K)
    b = np.stack([to_bf16_bits(_normal(_rng(seed, _TAG_B, g), (N, K))) for g in range(G)])
    expected_m = max(1, int(round(float(np.clip(masked_m, 0, max_m).mean()))))
    return Bf16MaskedProblem(a, b, masked_m, G, max_m, N, K, expected_m)


def sentinel_d(*shape: int) -> np.ndarray:
    """A BF16 output buffer (as uint16 bits) filled with the sentinel pattern."""
    return np.full(shape, SENTINEL_BF16, np.uint16)


# The workloads, by name and size.
SMOKE_SHAPE = (64, 512, 1024)                                   # dense M, N, K
DECODE_SHAPES = [(m, n, k) for m in (64, 128)
                 for (n, k) in ((2112, 7168), (32768, 512), (7168, 2048))]
PREFILL_SHAPES = [(4096, n, k) for (n, k) in ((2112, 7168), (24576, 1536), (7168, 16384),
                                              (4096, 7168))]
CONTIGUOUS_MOE = dict(G=32, N=4096, K=7168, total_tokens=8192, zipf_s=1.1, align=128)
MASKED_MOE = dict(G=32, max_m=256, N=4096, K=7168)
# the masked layer in decode: few tokens per expert (masked_m uniform in [0, 64])
MASKED_DECODE_MOE = dict(G=32, max_m=64, N=4096, K=7168)
# the weight gradient of the contiguous MoE layer: dW[g] [4096, 7168] per expert
K_GROUPED_MOE = dict(G=32, M=4096, N=7168, total_tokens=8192, zipf_s=1.1, align=128)
