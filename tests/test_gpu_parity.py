"""GPU parity: the CUDA library, called through its C ABI (via the Python
binding), against the CPU oracle on the same seeded inputs.

Small shapes are compared element by element over the whole output; the
full-size workloads (the pages' DeepSeek-V3/R1-shaped decode and prefill GEMMs
and the two MoE layouts) are compared on every row where the oracle finishes in
seconds, else on sampled rows that cover every 128-row tile boundary.  Rows the
method must leave untouched (contiguous padding, masked rows) are checked to
still hold the sentinel bit pattern.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import (check_close, d_bits, dev, oracle_contiguous_rows, oracle_dense_rows,
                    sample_rows, sentinel_like)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as lib
    lib.set_num_sms(0)
    assert lib.get_last_device_error() == 0
    return lib


def run_dense(dg, p: workloads.DenseProblem):
    d = sentinel_like((p.M, p.N))
    dg.fp8_gemm_nt(dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    return d_bits(d)


SMALL_DENSE = [
    (1, 16, 128), (64, 512, 1024), (127, 144, 256), (128, 128, 128), (129, 272, 384),
    (200, 2112, 512), (256, 256, 640), (300, 96, 128), (64, 48, 896), (16, 4112, 256),
]


@pytest.mark.parametrize("M,N,K", SMALL_DENSE)
def test_dense_small(dg, M, N, K):
    p = workloads.dense_problem(M, N, K, seed=1)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, f"dense {M}x{N}x{K}")


def test_dense_integer_exact(dg):
    """Values in {-1, 0, 1} with unit scales: every output is an integer of
    magnitude <= K = 256, exact in FP32 and BF16, so the result is bit-exact."""
    rng = np.random.default_rng(5)
    M, N, K = 200, 272, 256
    enc = np.array([0xB8, 0x00, 0x38], np.uint8)
    ia, ib = rng.integers(-1, 2, (M, K)), rng.integers(-1, 2, (N, K))
    p = workloads.DenseProblem(enc[ia + 1], np.ones((M, 2), np.float32), enc[ib + 1],
                               np.ones((3, 2), np.float32), M, N, K)
    got = run_dense(dg, p)
    want = torch.from_numpy((ia @ ib.T).astype(np.float32)).to(torch.bfloat16)
    assert np.array_equal(got, want.view(torch.int16).numpy().view(np.uint16))


def test_dense_scale_layout(dg):
    """Every row of A and every 128x128 block of B gets its own power-of-two
    scale, so a scale read from the wrong row, column block or K block shows."""
    rng = np.random.default_rng(6)
    M, N, K = 256, 384, 512
    p = workloads.dense_problem(M, N, K, seed=2)
    p.sfa = np.ldexp(1.0, rng.integers(-12, 4, p.sfa.shape)).astype(np.float32)
    p.sfb = np.ldexp(1.0, rng.integers(-12, 4, p.sfb.shape)).astype(np.float32)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, "scale layout")


def test_dense_scales_not_16_byte_aligned(dg):
    """Scale tensors that start 4 bytes past a 16-byte boundary (the ABI asks
    only for 4-byte alignment): the kernels must fall back from whole-float4
    scale loads and still read every row's own scales."""
    rng = np.random.default_rng(7)
    M, N, K = 300, 400, 1024
    p = workloads.dense_problem(M, N, K, seed=4)
    p.sfa = np.ldexp(1.0, rng.integers(-8, 4, p.sfa.shape)).astype(np.float32)
    p.sfb = np.ldexp(1.0, rng.integers(-8, 4, p.sfb.shape)).astype(np.float32)
    sfa_buf = torch.empty(p.sfa.size + 4, dtype=torch.float32, device="cuda")
    sfb_buf = torch.empty(p.sfb.size + 4, dtype=torch.float32, device="cuda")
    sfa = sfa_buf[1:1 + p.sfa.size].view(p.sfa.shape)
    sfb = sfb_buf[1:1 + p.sfb.size].view(p.sfb.shape)
    sfa.copy_(dev(p.sfa))
    sfb.copy_(dev(p.sfb))
    assert sfa.data_ptr() % 16 == 4 and sfb.data_ptr() % 16 == 4
    d = sentinel_like((M, N))
    dg.fp8_gemm_nt(dev(p.a), sfa, dev(p.b), sfb, d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(d_bits(d), ref, "unaligned scales")


# Every general variant, forced, on one ragged shape with a random power-of-two
# scale per A row and per B block (the picker would choose only some of them
# for this shape).
FORCED_GENERAL = ["256:1:1:128:0", "128:1", "64:1", "32:1"]


@pytest.mark.parametrize("cfg", FORCED_GENERAL)
def test_dense_forced_variant(dg, cfg, monkeypatch):
    rng = np.random.default_rng(11)
    M, N, K = 300, 400, 384
    p = workloads.dense_problem(M, N, K, seed=7)
    p.sfa = np.ldexp(1.0, rng.integers(-10, 4, p.sfa.shape)).astype(np.float32)
    p.sfb = np.ldexp(1.0, rng.integers(-10, 4, p.sfb.shape)).astype(np.float32)
    monkeypatch.setenv("DG_FORCE_CONFIG", cfg)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, f"forced {cfg}")


# Every decode variant ("block_n:split_k:kps:a_rows:mode", mode 1 decode, 2
# small decode), forced, with and
# without split-K clusters, on a short A (one 128-row block) with a ragged N
# and random power-of-two scales per A row and per B block.
FORCED_DECODE = [
    (100, "128:1:2:128:1"), (64, "128:4:2:128:1"), (100, "64:2:2:128:1"), (100, "64:8:2:128:1"),
    (128, "64:4:2:128:1"), (64, "256:2:2:64:1"), (64, "256:8:2:64:1"), (100, "128:1:1:128:2"),
    (40, "64:4:2:128:2"), (64, "128:1:4:64:1"), (64, "128:8:4:64:1"), (40, "64:8:4:64:1"),
    (48, "128:2:2:64:2"), (17, "64:2:2:64:2"),
]


@pytest.mark.parametrize("M,cfg", FORCED_DECODE)
def test_dense_forced_decode_variant(dg, M, cfg, monkeypatch):
    rng = np.random.default_rng(M + len(cfg))
    N, K = 400, 1024
    p = workloads.dense_problem(M, N, K, seed=13)
    p.sfa = np.ldexp(1.0, rng.integers(-10, 4, p.sfa.shape)).astype(np.float32)
    p.sfb = np.ldexp(1.0, rng.integers(-10, 4, p.sfb.shape)).astype(np.float32)
    monkeypatch.setenv("DG_FORCE_CONFIG", cfg)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, f"forced decode {cfg}")


# The other operand layouts: the same problem handed over with A M-major
# ([K, M]) and/or B N-major ([K, N]); random power-of-two scales per A row and
# per B block; ragged N and several tiles.
LAYOUT_CASES = [(256, 384, 512), (208, 272, 384), (64, 256, 1024), (512, 640, 256)]


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
@pytest.mark.parametrize("M,N,K", LAYOUT_CASES)
def test_dense_operand_layouts(dg, layout, M, N, K):
    rng = np.random.default_rng(M + N + K)
    p = workloads.dense_problem(M, N, K, seed=8)
    p.sfa = np.ldexp(1.0, rng.integers(-10, 4, p.sfa.shape)).astype(np.float32)
    p.sfb = np.ldexp(1.0, rng.integers(-10, 4, p.sfb.shape)).astype(np.float32)
    a = dev(np.ascontiguousarray(p.a.T) if layout[0] == "t" else p.a)
    b = dev(np.ascontiguousarray(p.b.T) if layout[1] == "n" else p.b)
    d = sentinel_like((M, N))
    getattr(dg, f"fp8_gemm_{layout}")(a, dev(p.sfa), b, dev(p.sfb), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(d_bits(d), ref, f"{layout} {M}x{N}x{K}")


@pytest.mark.parametrize("layout", ["nn", "tn", "tt"])
def test_dense_operand_layouts_prefill_sampled(dg, layout):
    M, N, K = 4096, 2112, 7168
    p = workloads.dense_problem(M, N, K, seed=9)
    a = dev(np.ascontiguousarray(p.a.T) if layout[0] == "t" else p.a)
    b = dev(np.ascontiguousarray(p.b.T) if layout[1] == "n" else p.b)
    d = sentinel_like((M, N))
    getattr(dg, f"fp8_gemm_{layout}")(a, dev(p.sfa), b, dev(p.sfb), d)
    torch.cuda.synchronize()
    got = d_bits(d)
    rows = sample_rows(M, 24, seed=K)
    check_close(got[rows], oracle_dense_rows(p, rows), f"{layout} prefill")


# FP32 output, D = A B^T + C.  The FP32 tensor-core accumulation against the
# oracle's exact double sum plus C: per element within 1e-4 of
# |ref| + rms(ref) (K/32 FP32 additions of exact products), and the global
# 1 - 2 sum(xy) / sum(x^2 + y^2) within 1e-9.
@pytest.mark.parametrize("mode", ["none", "c", "in_place"])
@pytest.mark.parametrize("M,N,K", [(300, 400, 384), (64, 2112, 1024), (512, 256, 2048),
                                   (1040, 4864, 512)])   # the last: persistent, 171 tiles
def test_dense_f32_output(dg, mode, M, N, K):
    rng = np.random.default_rng(M * 3 + N + K)
    p = workloads.dense_problem(M, N, K, seed=10)
    _, acc = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=True)
    c_host = rng.standard_normal((M, N)).astype(np.float32) * 8
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    if mode == "none":
        d = dg.fp8_gemm_nt_f32(a, sfa, b, sfb)
        ref = acc
    elif mode == "c":
        c = dev(c_host)
        d = dg.fp8_gemm_nt_f32(a, sfa, b, sfb, c=c)
        assert np.array_equal(c.cpu().numpy(), c_host)  # C is read only
        ref = acc + c_host.astype(np.float64)
    else:
        d = dev(c_host)
        dg.fp8_gemm_nt_f32(a, sfa, b, sfb, c=d, d=d)
        ref = acc + c_host.astype(np.float64)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    got = d.cpu().numpy().astype(np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    viol = np.abs(got - ref) / (1e-4 * (np.abs(ref) + rms))
    assert viol.max() <= 1.0, f"f32 {mode} {M}x{N}x{K}: worst {viol.max():.3f}"
    diff = 1 - 2 * np.sum(got * ref) / np.sum(got * got + ref * ref)
    assert diff <= 1e-9, diff


@pytest.mark.parametrize("M,N,K", [(64, 2112, 1024), (512, 384, 512)])
def test_dependent_launches_in_a_graph(dg, M, N, K):
    """Four launches captured back to back in one CUDA graph, each adding
    A B^T to the FP32 D the previous one wrote (programmatic dependent launch
    lets a launch start before the previous one ends; it must not read D
    before that one has finished writing it): D = 4 A B^T exactly as four
    separate accumulations."""
    p = workloads.dense_problem(M, N, K, seed=12)
    _, acc = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=True)
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    d = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    dg.fp8_gemm_nt_f32(a, sfa, b, sfb, c=d, d=d)  # eager warm-up (device set-up)
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(4):
            dg.fp8_gemm_nt_f32(a, sfa, b, sfb, c=d, d=d)
    for rep in range(3):
        d.zero_()
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            g.replay()
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0
        got = d.cpu().numpy().astype(np.float64)
        ref = 4 * acc
        rms = np.sqrt(np.mean(ref * ref))
        viol = np.abs(got - ref) / (1e-4 * (np.abs(ref) + rms))
        assert viol.max() <= 1.0, f"replay {rep}: worst {viol.max():.3f}"


@pytest.mark.parametrize("M,N,K", workloads.DECODE_SHAPES)
def test_dense_decode_full(dg, M, N, K):
    """The decode-shaped workloads, whole output (split-K path)."""
    p = workloads.dense_problem(M, N, K, seed=0)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, f"decode {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", workloads.PREFILL_SHAPES)
def test_dense_prefill_sampled(dg, M, N, K):
    p = workloads.dense_problem(M, N, K, seed=0)
    got = run_dense(dg, p)
    rows = sample_rows(M, 48, seed=M + N)
    check_close(got[rows], oracle_dense_rows(p, rows), f"prefill {M}x{N}x{K}")


def test_dense_prefill_full(dg):
    """One prefill-shaped GEMM (4096 x 2112 x 7168: 288 output tiles, two
    waves, a ragged last column tile) compared on every output element."""
    M, N, K = workloads.PREFILL_SHAPES[0]
    p = workloads.dense_problem(M, N, K, seed=0)
    got = run_dense(dg, p)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(got, ref, f"prefill full {M}x{N}x{K}")


def test_dense_deterministic(dg):
    p = workloads.dense_problem(64, 2112, 7168, seed=3)   # split-K path
    a, b = run_dense(dg, p), run_dense(dg, p)
    assert np.array_equal(a, b)


def test_dense_zero_rows(dg):
    dg.fp8_gemm_nt(torch.empty((0, 128), dtype=torch.uint8, device="cuda"),
                   torch.empty((0, 1), device="cuda"),
                   torch.zeros((16, 128), dtype=torch.uint8, device="cuda"),
                   torch.ones((1, 1), device="cuda"))
    torch.cuda.synchronize()


def test_num_sms_cap(dg):
    p = workloads.dense_problem(300, 1024, 512, seed=4)
    ref = run_dense(dg, p)
    try:
        dg.set_num_sms(7)
        assert dg.get_num_sms() == 7
        got = run_dense(dg, p)
    finally:
        dg.set_num_sms(0)
    assert np.array_equal(got, ref)


# --------------------------------------------------------------- contiguous --

def run_contiguous(dg, p: workloads.ContiguousProblem):
    d = sentinel_like((p.M_sum, p.N))
    dg.m_grouped_fp8_gemm_nt_contiguous(dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb),
                                        dev(p.m_indices), d)
    torch.cuda.synchronize()
    return d_bits(d)


def test_contiguous_small(dg):
    p = workloads.contiguous_problem(G=4, N=144, K=256, seed=1, counts=np.array([3, 0, 130, 1]))
    got = run_contiguous(dg, p)
    assert dg.get_last_device_error() == 0
    ref = np.full((p.M_sum, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().grouped_contiguous(p.a, p.sfa, p.b, p.sfb, p.m_indices, d=ref)
    pad = p.m_indices < 0
    assert np.all(got[pad] == workloads.SENTINEL_BF16), "padding rows were written"
    check_close(got[~pad], ref[~pad], "contiguous small")


def test_contiguous_full(dg):
    """The contiguous MoE workload (32 experts, Zipf-skewed token counts),
    every valid row against the oracle and every padding row untouched."""
    p = workloads.contiguous_problem(**workloads.CONTIGUOUS_MOE, seed=0)
    got = run_contiguous(dg, p)
    assert dg.get_last_device_error() == 0
    pad = p.m_indices < 0
    assert np.all(got[pad] == workloads.SENTINEL_BF16), "padding rows were written"
    ref = np.full((p.M_sum, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().grouped_contiguous(p.a, p.sfa, p.b, p.sfb, p.m_indices, d=ref)
    check_close(got[~pad], ref[~pad], "contiguous full")


def test_contiguous_mixed_block_reports(dg):
    """A 128-row block naming two experts: the block belongs to the largest
    index in it, rows naming another expert stay untouched, and the device
    error word says why."""
    p = workloads.contiguous_problem(G=3, N=128, K=128, seed=2, counts=np.array([100, 128, 0]))
    p.m_indices[200] = 0  # inside expert 1's block
    got = run_contiguous(dg, p)
    assert dg.get_last_device_error() == 0x201
    assert np.all(got[200] == workloads.SENTINEL_BF16)
    block_expert = np.repeat(p.m_indices.reshape(-1, 128).max(axis=1), 128)
    ok = np.nonzero((p.m_indices >= 0) & (p.m_indices == block_expert))[0]
    check_close(got[ok], oracle_contiguous_rows(p, ok), "mixed block, other rows")


# ------------------------------------------------------------------- masked --

def run_masked(dg, p: workloads.MaskedProblem):
    d = sentinel_like((p.G, p.max_m, p.N))
    dg.m_grouped_fp8_gemm_nt_masked(dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb),
                                    dev(p.masked_m), p.expected_m, d)
    torch.cuda.synchronize()
    return d_bits(d)


def test_masked_small(dg):
    p = workloads.masked_problem(G=5, max_m=200, N=144, K=256, seed=1,
                                 masked_m=np.array([0, 200, 3, 129, 250]))
    got = run_masked(dg, p)
    assert dg.get_last_device_error() == 0
    ref = np.full((p.G, p.max_m, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().grouped_masked(p.a, p.sfa, p.b, p.sfb, p.masked_m, d=ref)
    for g in range(p.G):
        v = min(max(int(p.masked_m[g]), 0), p.max_m)
        assert np.all(got[g, v:] == workloads.SENTINEL_BF16), f"group {g}: masked rows written"
        if v:
            check_close(got[g, :v], ref[g, :v], f"masked group {g}")


def test_masked_out_of_range_counts_are_clamped(dg):
    """masked_m outside [0, max_m] is clamped on the device, as in the oracle:
    a negative count writes no row of its group, one above max_m writes all
    of them; the other rows keep the sentinel."""
    p = workloads.masked_problem(G=4, max_m=128, N=272, K=384, seed=6,
                                 masked_m=np.array([-7, 64, 300, 1]))
    got = run_masked(dg, p)
    assert dg.get_last_device_error() == 0
    ref = np.full((p.G, p.max_m, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().grouped_masked(p.a, p.sfa, p.b, p.sfb, p.masked_m, d=ref)
    for g, v in enumerate([0, 64, 128, 1]):
        assert np.all(got[g, v:] == workloads.SENTINEL_BF16), f"group {g}: masked rows written"
        assert np.all(ref[g, v:] == workloads.SENTINEL_BF16), f"oracle group {g}"
        if v:
            check_close(got[g, :v], ref[g, :v], f"clamped masked group {g}")


def test_masked_full(dg):
    """The masked MoE workload (32 groups, masked_m uniform in [0, 256]),
    every valid row against the oracle and every masked row untouched."""
    p = workloads.masked_problem(**workloads.MASKED_MOE, seed=0)
    got = run_masked(dg, p)
    assert dg.get_last_device_error() == 0
    ref = np.full((p.G, p.max_m, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().grouped_masked(p.a, p.sfa, p.b, p.sfb, p.masked_m, d=ref)
    valid = np.arange(p.max_m)[None, :] < p.masked_m[:, None]
    assert np.all(got[~valid] == workloads.SENTINEL_BF16), "masked rows were written"
    check_close(got[valid], ref[valid], "masked full")


def test_masked_expected_m_does_not_change_results(dg):
    p = workloads.masked_problem(G=4, max_m=256, N=256, K=256, seed=3)
    a = run_masked(dg, p)
    p.expected_m = 1
    b = run_masked(dg, p)
    p.expected_m = 256
    c = run_masked(dg, p)
    assert np.array_equal(a, b) and np.array_equal(a, c)


@pytest.mark.parametrize("M,N,K", [(64, 2112, 1024), (300, 400, 1024)])
def test_scale_contract_check(dg, M, N, K):
    """With the scale check on, valid scales run clean and match the oracle;
    one A scale and one B scale with mantissa bits (1.5, 0.75: not powers of
    two) record device error 0x301.  With the check off the same call records
    nothing (the contract is the caller's)."""
    p = workloads.dense_problem(M, N, K, seed=14)
    a, b = dev(p.a), dev(p.b)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    bad_sfa, bad_sfb = p.sfa.copy(), p.sfb.copy()
    bad_sfa[M // 2, K // 256] = 1.5
    bad_sfb[-1, 0] = 0.75
    try:
        dg.set_check_scales(True)
        d = sentinel_like((M, N))
        dg.fp8_gemm_nt(a, dev(p.sfa), b, dev(p.sfb), d)
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0
        check_close(d_bits(d), ref, "valid scales, check on")
        dg.fp8_gemm_nt(a, dev(bad_sfa), b, dev(p.sfb), sentinel_like((M, N)))
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0x301
        dg.fp8_gemm_nt(a, dev(p.sfa), b, dev(bad_sfb), sentinel_like((M, N)))
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0x301
    finally:
        dg.set_check_scales(False)
    dg.fp8_gemm_nt(a, dev(bad_sfa), b, dev(bad_sfb), sentinel_like((M, N)))
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0


@pytest.mark.parametrize("M,N,K", workloads.DECODE_SHAPES + [(300, 400, 1024), (4096, 2112, 1024),
                                                              (1280, 4096, 4096)])
def test_weight_preload_gives_the_same_results(dg, M, N, K):
    """With the weight preload on (B loaded before the wait on the previous
    kernel), every decode shape (split-K clusters included), persistent tiles
    and a call whose last wave is split off into split-K tail launches (each
    loading its B sub-block early) give bit-identical results to the preload
    off, and match the oracle."""
    p = workloads.dense_problem(M, N, K, seed=15)
    try:
        dg.set_weight_preload(True)
        on = run_dense(dg, p)
    finally:
        dg.set_weight_preload(False)
    off = run_dense(dg, p)
    assert np.array_equal(on, off)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(on, ref, f"preload {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(64, 2112, 1024), (512, 384, 512)])
def test_dependent_launches_with_weight_preload(dg, M, N, K):
    """The graph of four dependent in-place FP32 accumulations with the
    weight preload on: B is loaded early, but each launch still reads the D
    the previous one wrote only after that launch has finished."""
    try:
        dg.set_weight_preload(True)
        test_dependent_launches_in_a_graph(dg, M, N, K)
    finally:
        dg.set_weight_preload(False)
