"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each pin is a plain function taking an ``oracle.Oracle`` and raising
``AssertionError`` on a mismatch, so the same checks serve the normal test run
(``test_oracle.py``) and the mutation check (``test_oracle_mutants.py``), which
compiles deliberately broken copies of the oracle and requires that some pin
fails for each of them.

What each pin compares against:

* the E4M3 table: the format definition (hand-derived golden values) and two
  independent implementations (``ml_dtypes.float8_e4m3fn``, ``torch.float8_e4m3fn``);
* the BF16 rounding: hand-worked cases (golden file), and torch's FP32->BF16
  conversion for values that are exactly FP32 (where one rounding from double
  equals one rounding from FP32);
* the BF16 operand GEMM: every one of the 65536 operand patterns against the
  FP32 widening and ml_dtypes; numpy float64 matmul; Python-float loops (bit
  for bit); exact integer results; an empty K; the grouped forms row by row;
* the K-grouped (weight-gradient) form: numpy float64 per group plus C, the
  dense oracle on each group's slice (bit for bit) and over all of K (the sum
  over groups), exact integer results, an empty group leaving C;
* the GEMM: a hand-worked tiny example (golden file); brute force with numpy's
  float64 matmul on ml_dtypes-decoded operands; exact integer results; one-hot
  selection; power-of-two scale invariance; and for the grouped forms, the same
  brute force applied row by row with the sentinel left in every row that must
  stay untouched.
"""
from __future__ import annotations

import os

import ml_dtypes
import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
SENTINEL = 0x7FBF


# ----------------------------------------------------------------- helpers --

def _golden_rows(name: str, sep=None):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            yield [c.strip() for c in (line.split(sep) if sep else line.split())]


def decode_ml(q: np.ndarray) -> np.ndarray:
    """E4M3 bytes -> float64 through ml_dtypes (independent of the oracle)."""
    return np.asarray(q, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def bf16_nearest_even(x: np.ndarray) -> np.ndarray:
    """Round float64 values to BF16 bit patterns by comparing candidates.

    Written differently from the oracle on purpose: it takes the FP32
    neighbours' upper halves and the next pattern up, measures the exact
    distance in float64, and breaks exact ties towards an even pattern."""
    x = np.asarray(x, np.float64).ravel()
    out = np.empty(x.shape, np.uint16)
    for i, v in enumerate(x):
        if np.isnan(v):
            out[i] = 0x7FC0
            continue
        sign = 0x8000 if np.signbit(v) else 0
        a = abs(v)
        if a >= 2.0 ** 128:
            out[i] = sign | 0x7F80
            continue
        f = np.float32(a)
        if float(f) > a:
            f = np.nextafter(f, np.float32(0))
        lo = int(np.array(f, np.float32).view(np.uint32)) >> 16   # truncated pattern <= a
        best, best_d = None, None
        for cand in (lo, lo + 1):
            cv = float(np.array(cand << 16, np.uint32).view(np.float32))
            if cand >= 0x7F80:
                cv = float("inf")
            d = abs(cv - a)
            if best is None or d < best_d or (d == best_d and cand % 2 == 0):
                best, best_d = cand, d
        out[i] = sign | best
    return out


def brute_acc(a, sfa, b, sfb) -> np.ndarray:
    """Dequantise with ml_dtypes and expanded scales, then numpy float64 matmul."""
    M, K = a.shape
    N = b.shape[0]
    ah = decode_ml(a) * np.repeat(np.asarray(sfa, np.float64), 128, axis=1)
    sfb_rows = np.repeat(np.asarray(sfb, np.float64), 128, axis=0)[:N]
    bh = decode_ml(b) * np.repeat(sfb_rows, 128, axis=1)
    return ah @ bh.T


def random_pow2_scales(rng, shape, lo=-10, hi=10) -> np.ndarray:
    return np.ldexp(1.0, rng.integers(lo, hi + 1, size=shape)).astype(np.float32)


def random_e4m3(rng, shape) -> np.ndarray:
    q = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((q & 0x7F) == 0x7F, q & 0xF7, q).astype(np.uint8)  # no NaNs


# ------------------------------------------------------------------- pins --

def pin_e4m3_golden(o):
    t = o.e4m3_table()
    for byte_s, val_s in _golden_rows("e4m3_spot_values.txt"):
        byte = int(byte_s, 16)
        if val_s == "nan":
            assert np.isnan(t[byte]), byte_s
        else:
            want = float(val_s)
            assert t[byte] == want and np.signbit(t[byte]) == np.signbit(want), (byte_s, t[byte])


def pin_e4m3_structure(o):
    t = o.e4m3_table()
    pos = t[:0x7F]
    assert np.all(np.diff(pos) > 0), "not strictly increasing over 0x00..0x7E"
    for b in range(128):
        if b == 0x7F:
            continue
        assert t[b | 0x80] == -t[b] and np.signbit(t[b | 0x80]), b
    assert np.isnan(t[0x7F]) and np.isnan(t[0xFF]) and np.sum(np.isnan(t)) == 2


def pin_e4m3_libraries(o):
    t = o.e4m3_table()
    ref_ml = decode_ml(np.arange(256, dtype=np.uint8))
    ref_torch = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    for ref in (ref_ml, ref_torch):
        same = (t == ref) | (np.isnan(t) & np.isnan(ref))
        assert np.all(same), np.nonzero(~same)


def pin_bf16_golden(o):
    for expr, bits, why in _golden_rows("bf16_rounding_cases.txt", sep="|"):
        v = float(eval(expr, {"__builtins__": {}}))
        got = o.bf16_from_double(v)
        assert got == int(bits, 16), (expr, hex(got), bits, why)


def pin_bf16_vs_torch_on_fp32_values(o, n=20000, seed=7):
    rng = np.random.default_rng(seed)
    bits = rng.integers(0, 2 ** 32, size=n, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    extra = np.array([0.0, -0.0, 1.0, 3.0e38, -3.4e38, 1e-40, -1e-45, 65504.0], np.float32)
    f = np.concatenate([f, extra])
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([o.bf16_from_double(float(v)) for v in f], np.uint16)
    assert np.array_equal(got, ref), np.nonzero(got != ref)[0][:5]


def pin_bf16_vs_candidates_on_wide_values(o, n=3000, seed=8):
    """Values carrying bits below FP32 precision, where a float intermediate
    would round twice."""
    rng = np.random.default_rng(seed)
    base = rng.standard_normal(n) * np.ldexp(1.0, rng.integers(-30, 30, n))
    ties = np.ldexp(rng.integers(1 << 8, 1 << 9, n).astype(np.float64) + 0.5, rng.integers(-20, 20, n))
    wide = ties * (1 + np.ldexp(1.0, -40) * rng.choice([-1.0, 0.0, 1.0], n))
    vals = np.concatenate([base, ties, wide])
    got = np.array([o.bf16_from_double(float(v)) for v in vals], np.uint16)
    assert np.array_equal(got, bf16_nearest_even(vals))


def pin_tiny_worked_gemm(o):
    vals = {(0, 0): 0x38, (0, 1): 0x40, (1, 0): 0xB8, (1, 1): 0x30}
    a = np.zeros((2, 256), np.uint8)
    for (m, kb), byte in vals.items():
        a[m, kb * 128:(kb + 1) * 128] = byte
    bvals = {(0, 0): 0x38, (0, 1): 0x38, (1, 0): 0x3C, (1, 1): 0x00, (2, 0): 0x01, (2, 1): 0x7E}
    b = np.zeros((3, 256), np.uint8)
    for (n, kb), byte in bvals.items():
        b[n, kb * 128:(kb + 1) * 128] = byte
    sfa = np.array([[1, 0.5], [4, 0.25]], np.float32)
    sfb = np.array([[0.125, 2]], np.float32)
    d, acc = o.gemm_nt(a, sfa, b, sfb)
    for m, n, exact, bits in _golden_rows("tiny_worked_gemm.txt"):
        m, n = int(m), int(n)
        assert acc[m, n] == float(exact), (m, n, acc[m, n], exact)
        assert d[m, n] == int(bits, 16), (m, n, hex(d[m, n]), bits)


BRUTE_SHAPES = [(1, 1, 128), (3, 5, 128), (8, 8, 256), (5, 130, 256), (7, 200, 384), (4, 257, 128)]


def pin_dense_brute_force(o, seed=11):
    rng = np.random.default_rng(seed)
    for (M, N, K) in BRUTE_SHAPES:
        a = random_e4m3(rng, (M, K))
        b = random_e4m3(rng, (N, K))
        sfa = random_pow2_scales(rng, (M, K // 128))
        sfb = random_pow2_scales(rng, (-(-N // 128), K // 128))
        d, acc = o.gemm_nt(a, sfa, b, sfb)
        ref = brute_acc(a, sfa, b, sfb)
        assert np.allclose(acc, ref, rtol=1e-12, atol=0), (M, N, K, np.abs(acc - ref).max())
        assert np.array_equal(d, bf16_nearest_even(acc).reshape(M, N)), (M, N, K)
        assert np.array_equal(d, bf16_nearest_even(ref).reshape(M, N)), (M, N, K)


def pin_dense_integer_exact(o, seed=12):
    rng = np.random.default_rng(seed)
    for (M, N, K) in [(4, 6, 128), (9, 17, 256), (3, 140, 256)]:
        ia = rng.integers(-1, 2, (M, K))
        ib = rng.integers(-1, 2, (N, K))
        enc = {-1: 0xB8, 0: 0x00, 1: 0x38}
        a = np.vectorize(enc.get)(ia).astype(np.uint8)
        b = np.vectorize(enc.get)(ib).astype(np.uint8)
        sfa = np.ones((M, K // 128), np.float32)
        sfb = np.ones((-(-N // 128), K // 128), np.float32)
        d, acc = o.gemm_nt(a, sfa, b, sfb)
        exact = ia @ ib.T                                   # int64, |.| <= 256
        assert np.array_equal(acc, exact.astype(np.float64))
        want = torch.from_numpy(exact.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
        assert np.array_equal(d, want.numpy().view(np.uint16))


def pin_dense_one_hot(o, seed=13):
    rng = np.random.default_rng(seed)
    M, N, K = 6, 150, 384
    ks = rng.integers(0, K, M)
    a = np.zeros((M, K), np.uint8)
    a[np.arange(M), ks] = 0x38
    b = random_e4m3(rng, (N, K))
    sfa = np.ones((M, K // 128), np.float32)
    sfb = random_pow2_scales(rng, (2, K // 128))
    d, acc = o.gemm_nt(a, sfa, b, sfb)
    for m in range(M):
        k = ks[m]
        want = decode_ml(b[:, k]) * sfb[np.arange(N) // 128, k // 128].astype(np.float64)
        assert np.array_equal(acc[m], want), m
        # an exact zero sum is +0 in IEEE arithmetic whatever the sign of the
        # selected byte, so compare with negative zero folded to positive zero
        want = np.where(want == 0, 0.0, want)
        wbits = torch.from_numpy(want.astype(np.float32)).to(torch.bfloat16).view(torch.int16)
        assert np.array_equal(d[m], wbits.numpy().view(np.uint16)), m


def pin_dense_scale_invariance(o, seed=14):
    rng = np.random.default_rng(seed)
    M, N, K = 5, 140, 384
    a = random_e4m3(rng, (M, K))
    b = random_e4m3(rng, (N, K))
    sfa = random_pow2_scales(rng, (M, K // 128), -4, 4)
    sfb = random_pow2_scales(rng, (2, K // 128), -4, 4)
    _, acc = o.gemm_nt(a, sfa, b, sfb)
    # whole row scaled by 2^3: acc row scales exactly
    s2 = sfa.copy()
    s2[2] *= 8
    _, acc2 = o.gemm_nt(a, s2, b, sfb)
    assert np.array_equal(acc2[2], acc[2] * 8) and np.array_equal(np.delete(acc2, 2, 0), np.delete(acc, 2, 0))
    # one K block of one row scaled by 2^2: the change is 3x that block's partial sum
    s3 = sfa.copy()
    s3[1, 1] *= 4
    _, acc3 = o.gemm_nt(a, s3, b, sfb)
    part = brute_acc(a[1:2, 128:256], sfa[1:2, 1:2], b[:, 128:256], sfb[:, 1:2])[0]
    assert np.allclose(acc3[1] - acc[1], 3 * part, rtol=1e-12, atol=1e-300)
    # one B scale block changed: only columns of that 128-row N block move
    s4 = sfb.copy()
    s4[1, 0] *= 2
    _, acc4 = o.gemm_nt(a, sfa, b, s4)
    assert np.array_equal(acc4[:, :128], acc[:, :128])
    part_b = brute_acc(a[:, :128], sfa[:, :1], b[128:, :128], sfb[1:, :1])
    assert np.allclose(acc4[:, 128:] - acc[:, 128:], part_b, rtol=1e-12, atol=1e-300)


def pin_contiguous(o, seed=15):
    rng = np.random.default_rng(seed)
    G, N, K = 4, 140, 256
    counts = [3, 0, 130, 1]
    padded = [(-(-c // 128)) * 128 for c in counts]
    M_sum = sum(padded)
    m_idx = np.full(M_sum, -1, np.int32)
    off = 0
    for g, c in enumerate(counts):
        m_idx[off:off + c] = g
        off += padded[g]
    a = random_e4m3(rng, (M_sum, K))
    b = random_e4m3(rng, (G, N, K))
    sfa = random_pow2_scales(rng, (M_sum, K // 128))
    sfb = random_pow2_scales(rng, (G, 2, K // 128))
    d = np.full((M_sum, N), SENTINEL, np.uint16)
    o.grouped_contiguous(a, sfa, b, sfb, m_idx, d=d)
    for r in range(M_sum):
        e = m_idx[r]
        if e < 0:
            assert np.all(d[r] == SENTINEL), r
        else:
            ref = brute_acc(a[r:r + 1], sfa[r:r + 1], b[e], sfb[e])[0]
            assert np.array_equal(d[r], bf16_nearest_even(ref)), r
    # the grouped result equals the per-expert dense GEMMs on that expert's rows
    off = 0
    for g, c in enumerate(counts):
        if c:
            dg, _ = o.gemm_nt(a[off:off + c], sfa[off:off + c], b[g], sfb[g], want_acc=False)
            assert np.array_equal(d[off:off + c], dg), g
        off += padded[g]


def pin_masked(o, seed=16):
    rng = np.random.default_rng(seed)
    G, max_m, N, K = 5, 7, 136, 256
    masked_m = np.array([0, 7, 3, 9, -2], np.int32)      # 9 clamps to 7, -2 to 0
    a = random_e4m3(rng, (G, max_m, K))
    b = random_e4m3(rng, (G, N, K))
    sfa = random_pow2_scales(rng, (G, max_m, K // 128))
    sfb = random_pow2_scales(rng, (G, 2, K // 128))
    d = np.full((G, max_m, N), SENTINEL, np.uint16)
    o.grouped_masked(a, sfa, b, sfb, masked_m, d=d)
    for g in range(G):
        valid = min(max(int(masked_m[g]), 0), max_m)
        for m in range(max_m):
            if m < valid:
                ref = brute_acc(a[g, m:m + 1], sfa[g, m:m + 1], b[g], sfb[g])[0]
                assert np.array_equal(d[g, m], bf16_nearest_even(ref)), (g, m)
            else:
                assert np.all(d[g, m] == SENTINEL), (g, m)


# ------------------------------------------------------ BF16 operand GEMM --

def decode_bf16_np(bits) -> np.ndarray:
    """BF16 bit patterns -> float64 by widening to FP32 bit patterns
    (independent of the oracle's table)."""
    with np.errstate(invalid="ignore"):  # NaN patterns widen to NaN
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def random_bf16(rng, shape, scale=1.0) -> np.ndarray:
    x = torch.from_numpy((rng.standard_normal(shape) * scale).astype(np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_of_ints(ints: np.ndarray) -> np.ndarray:
    """Exact BF16 patterns of small integers (|i| <= 256), through torch."""
    x = torch.from_numpy(np.asarray(ints, np.float32))
    return x.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def pin_bf16_operand_table(o):
    """All 65536 patterns against the FP32 widening and ml_dtypes' bfloat16."""
    bits = np.arange(65536, dtype=np.uint32)
    ref = decode_bf16_np(bits.astype(np.uint16))
    with np.errstate(invalid="ignore"):
        ref2 = bits.astype(np.uint16).view(ml_dtypes.bfloat16).astype(np.float64)
    got = np.array([o.bf16_decode(i) for i in range(65536)])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and np.array_equal(np.isnan(ref2), nan)
    assert np.array_equal(got[~nan], ref[~nan]) and np.array_equal(ref2[~nan], ref[~nan])
    assert np.array_equal(np.signbit(got[~nan]), np.signbit(ref[~nan]))
    # spot values from the format definition
    assert o.bf16_decode(0x3F80) == 1.0 and o.bf16_decode(0xC040) == -3.0
    assert o.bf16_decode(0x0001) == 2.0 ** -133 and o.bf16_decode(0x0080) == 2.0 ** -126
    assert o.bf16_decode(0x7F7F) == (2 - 2.0 ** -7) * 2.0 ** 127
    assert o.bf16_decode(0xFF80) == -np.inf


BF16_BRUTE_SHAPES = [(1, 1, 1), (3, 5, 7), (8, 9, 64), (5, 130, 200), (2, 257, 64)]


def pin_bf16_gemm_brute_force(o, seed=17):
    rng = np.random.default_rng(seed)
    for (M, N, K) in BF16_BRUTE_SHAPES:
        a = random_bf16(rng, (M, K))
        b = random_bf16(rng, (N, K), scale=4.0)
        d, acc = o.bf16_gemm_nt(a, b)
        ref = decode_bf16_np(a) @ decode_bf16_np(b).T
        assert np.allclose(acc, ref, rtol=1e-12, atol=1e-300), (M, N, K)
        assert np.array_equal(d, bf16_nearest_even(acc).reshape(M, N)), (M, N, K)


def pin_bf16_gemm_python_loops(o, seed=18):
    """Tiny case summed with Python floats in k order: the same IEEE double
    operations, so the accumulator must match bit for bit."""
    rng = np.random.default_rng(seed)
    M, N, K = 2, 3, 11
    a = random_bf16(rng, (M, K))
    b = random_bf16(rng, (N, K))
    d, acc = o.bf16_gemm_nt(a, b)
    da, db = decode_bf16_np(a), decode_bf16_np(b)
    for m in range(M):
        for n in range(N):
            s = 0.0
            for k in range(K):
                s += float(da[m, k]) * float(db[n, k])
            assert acc[m, n] == s, (m, n)
            assert d[m, n] == bf16_nearest_even(np.array([s]))[0], (m, n)


def pin_bf16_gemm_integer_exact(o, seed=19):
    rng = np.random.default_rng(seed)
    for (M, N, K) in [(4, 6, 64), (9, 17, 256), (3, 140, 192)]:
        ia = rng.integers(-8, 9, (M, K))
        ib = rng.integers(-8, 9, (N, K))
        d, acc = o.bf16_gemm_nt(bf16_of_ints(ia), bf16_of_ints(ib))
        exact = ia @ ib.T                                   # |.| <= 64 K, exact in FP32
        assert np.array_equal(acc, exact.astype(np.float64))
        assert np.array_equal(d, bf16_of_ints(exact.astype(np.float32)))


def pin_bf16_gemm_empty_k(o):
    d, acc = o.bf16_gemm_nt(np.zeros((3, 0), np.uint16), np.zeros((5, 0), np.uint16))
    assert np.array_equal(acc, np.zeros((3, 5))) and np.all(d == 0)


def pin_bf16_grouped(o, seed=20):
    rng = np.random.default_rng(seed)
    # contiguous: padding rows keep the sentinel; expert rows equal the
    # per-expert dense GEMM on the same rows
    G, N, K = 3, 136, 128
    counts = [2, 0, 129]
    padded = [(-(-c // 128)) * 128 for c in counts]
    m_idx = np.full(sum(padded), -1, np.int32)
    off = 0
    for g, c in enumerate(counts):
        m_idx[off:off + c] = g
        off += padded[g]
    a = random_bf16(rng, (len(m_idx), K))
    b = random_bf16(rng, (G, N, K))
    d = np.full((len(m_idx), N), SENTINEL, np.uint16)
    o.bf16_grouped_contiguous(a, b, m_idx, d=d)
    for r in range(len(m_idx)):
        e = m_idx[r]
        if e < 0:
            assert np.all(d[r] == SENTINEL), r
        else:
            ref = decode_bf16_np(a[r]) @ decode_bf16_np(b[e]).T
            assert np.array_equal(d[r], bf16_nearest_even(ref)), r
    # masked: rows m >= masked_m[g] (clamped to [0, max_m]) keep the sentinel
    G, max_m, N, K = 4, 5, 72, 64
    masked_m = np.array([5, 0, 2, 8], np.int32)
    a = random_bf16(rng, (G, max_m, K))
    b = random_bf16(rng, (G, N, K))
    d = np.full((G, max_m, N), SENTINEL, np.uint16)
    o.bf16_grouped_masked(a, b, masked_m, d=d)
    for g in range(G):
        valid = min(max(int(masked_m[g]), 0), max_m)
        for m in range(max_m):
            if m < valid:
                ref = decode_bf16_np(a[g, m]) @ decode_bf16_np(b[g]).T
                assert np.array_equal(d[g, m], bf16_nearest_even(ref)), (g, m)
            else:
                assert np.all(d[g, m] == SENTINEL), (g, m)


# ------------------------------------------------- K-grouped (weight grad) --

def _k_grouped_case(rng, ks, M, N, with_c=True):
    K_sum = int(np.sum(ks))
    a = random_e4m3(rng, (K_sum, M))           # [K_sum, M], M-major
    b = random_e4m3(rng, (K_sum, N))           # [K_sum, N], N-major
    sfa = random_pow2_scales(rng, (M, K_sum // 128))
    sfb = random_pow2_scales(rng, (-(-N // 128), K_sum // 128))
    c = rng.standard_normal((len(ks), M, N)).astype(np.float32) * 64 if with_c else None
    return a, sfa, b, sfb, np.asarray(ks, np.int32), c


def pin_k_grouped_brute_force(o, seed=21):
    """Per group, numpy float64 on ml_dtypes-decoded operands over the group's
    rows of K only, plus C; an empty group leaves exactly C."""
    rng = np.random.default_rng(seed)
    ks = [256, 0, 128, 384]
    M, N = 24, 136
    a, sfa, b, sfb, ks, c = _k_grouped_case(rng, ks, M, N)
    acc = o.k_grouped_tn(a, sfa, b, sfb, ks, c)
    k0 = 0
    for g, kg in enumerate(ks):
        kb = slice(k0 // 128, (k0 + kg) // 128)
        ah = decode_ml(a[k0:k0 + kg]).T * np.repeat(sfa[:, kb].astype(np.float64), 128, axis=1)
        sfb_rows = np.repeat(sfb[:, kb].astype(np.float64), 128, axis=0)[:N]
        bh = decode_ml(b[k0:k0 + kg]).T * np.repeat(sfb_rows, 128, axis=1)
        ref = c[g].astype(np.float64) + ah @ bh.T
        tol = 1e-12 * (np.abs(c[g]).astype(np.float64) + np.abs(ah) @ np.abs(bh).T) + 1e-300
        assert np.all(np.abs(acc[g] - ref) <= tol), g
        if kg == 0:
            assert np.array_equal(acc[g], c[g].astype(np.float64)), g
        k0 += kg


def pin_k_grouped_is_per_group_dense(o, seed=22):
    """Without C, group g's result is bit for bit the dense NT oracle run on
    that group's rows of K (transposed to K-major) with that group's scale
    columns; and the sum over groups equals the dense GEMM over all of K."""
    rng = np.random.default_rng(seed)
    ks = [128, 512, 0, 256]
    M, N = 40, 264
    a, sfa, b, sfb, ks, _ = _k_grouped_case(rng, ks, M, N, with_c=False)
    acc = o.k_grouped_tn(a, sfa, b, sfb, ks, None)
    k0 = 0
    for g, kg in enumerate(ks):
        if kg == 0:
            assert np.all(acc[g] == 0.0), g
            continue
        kb = slice(k0 // 128, (k0 + kg) // 128)
        _, dense = o.gemm_nt(np.ascontiguousarray(a[k0:k0 + kg].T), sfa[:, kb],
                             np.ascontiguousarray(b[k0:k0 + kg].T), sfb[:, kb])
        assert np.array_equal(acc[g], dense), g
        k0 += kg
    _, full = o.gemm_nt(np.ascontiguousarray(a.T), sfa, np.ascontiguousarray(b.T), sfb)
    total = acc.sum(axis=0)
    assert np.allclose(total, full, rtol=1e-12, atol=1e-9 * np.abs(full).max())


def pin_k_grouped_integer_exact(o, seed=23):
    """Values in {-1, 0, 1}, unit scales: every group's result is the integer
    product of its slices exactly."""
    rng = np.random.default_rng(seed)
    ks = np.array([128, 256, 0, 128], np.int32)
    M, N = 16, 48
    K_sum = int(ks.sum())
    enc = np.array([0xB8, 0x00, 0x38], np.uint8)
    ia, ib = rng.integers(-1, 2, (K_sum, M)), rng.integers(-1, 2, (K_sum, N))
    acc = o.k_grouped_tn(enc[ia + 1], np.ones((M, K_sum // 128), np.float32), enc[ib + 1],
                         np.ones((1, K_sum // 128), np.float32), ks, None)
    k0 = 0
    for g, kg in enumerate(ks):
        assert np.array_equal(acc[g], (ia[k0:k0 + kg].T @ ib[k0:k0 + kg]).astype(np.float64)), g
        k0 += kg


ALL_PINS = [
    pin_e4m3_golden, pin_e4m3_structure, pin_e4m3_libraries,
    pin_bf16_golden, pin_bf16_vs_torch_on_fp32_values, pin_bf16_vs_candidates_on_wide_values,
    pin_tiny_worked_gemm, pin_dense_brute_force, pin_dense_integer_exact, pin_dense_one_hot,
    pin_dense_scale_invariance, pin_contiguous, pin_masked,
    pin_bf16_operand_table, pin_bf16_gemm_brute_force, pin_bf16_gemm_python_loops,
    pin_bf16_gemm_integer_exact, pin_bf16_gemm_empty_k, pin_bf16_grouped,
    pin_k_grouped_brute_force, pin_k_grouped_is_per_group_dense, pin_k_grouped_integer_exact,
]


def run_all(o) -> list[str]:
    """Run every pin; return the names of those that failed (or crashed)."""
    failed = []
    for pin in ALL_PINS:
        try:
            pin(o)
        except Exception as exc:  # noqa: BLE001 - a crash counts as a failure
            failed.append(f"{pin.__name__}: {type(exc).__name__}: {str(exc)[:120]}")
    return failed
