"""GPU parity of the BF16-operand GEMM forms (dense, contiguous, masked)
against the CPU oracle on the same seeded inputs, through the C ABI.

The kernels are the FP8 kernels' template built without scale factors, so
these cases cover the paths that differ (the kind::f16 MMA, 64-element K
blocks, BF16 tensor maps, the idle scale warp) over the same tile shapes,
ragged tails, split-K clusters, small and general variants, and the grouped
layouts' untouched rows.  Tolerance as for FP8 (``parity.check_close``).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_close, d_bits, sample_rows, sentinel_like

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as lib
    lib.set_num_sms(0)
    assert lib.get_last_device_error() == 0
    return lib


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """BF16 bit patterns (uint16) -> a bfloat16 CUDA tensor with those bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to("cuda")
    return t.view(torch.bfloat16)


def run_dense(dg, p: workloads.Bf16DenseProblem) -> np.ndarray:
    d = sentinel_like((p.M, p.N))
    dg.bf16_gemm_nt(bf16_dev(p.a), bf16_dev(p.b), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    return d_bits(d)


SMALL_DENSE = [
    (1, 16, 64), (64, 512, 1024), (127, 144, 192), (128, 128, 64), (129, 272, 448),
    (200, 2112, 512), (256, 256, 640), (300, 96, 128), (64, 48, 896), (16, 4112, 256),
]


@pytest.mark.parametrize("M,N,K", SMALL_DENSE)
def test_bf16_dense_small(dg, M, N, K):
    p = workloads.bf16_dense_problem(M, N, K, seed=1)
    got = run_dense(dg, p)
    ref, _ = oracle.default().bf16_gemm_nt(p.a, p.b, want_acc=False)
    check_close(got, ref, f"bf16 dense {M}x{N}x{K}")


def test_bf16_dense_integer_exact(dg):
    """Integers in [-4, 4]: every sum is an integer of magnitude <= 16 K, exact
    in FP32 and, at K = 192, in BF16 after one rounding: bit-exact."""
    rng = np.random.default_rng(6)
    M, N, K = 130, 272, 192
    ia = rng.integers(-4, 5, (M, K)).astype(np.float32)
    ib = rng.integers(-4, 5, (N, K)).astype(np.float32)
    p = workloads.Bf16DenseProblem(workloads.to_bf16_bits(ia), workloads.to_bf16_bits(ib), M, N, K)
    got = run_dense(dg, p)
    ref, acc = oracle.default().bf16_gemm_nt(p.a, p.b)
    assert np.array_equal(acc, ia.astype(np.float64) @ ib.astype(np.float64).T)
    assert np.array_equal(got, ref)


# (config, M): general variants (persistent, several tiles per CTA), decode
# variants with split-K clusters, and a small variant (two CTAs per SM)
FORCED = [("256:1:1:128:0", 300), ("128:1", 300), ("64:1", 300), ("32:1", 300),
          ("128:4:4:64:1", 64), ("64:2:2:128:1", 128), ("128:2:2:64:2", 48)]


@pytest.mark.parametrize("cfg,M", FORCED)
def test_bf16_dense_forced_variant(dg, cfg, M, monkeypatch):
    monkeypatch.setenv("DG_FORCE_CONFIG", cfg)
    p = workloads.bf16_dense_problem(M, 400, 1024, seed=2)
    got = run_dense(dg, p)
    ref, _ = oracle.default().bf16_gemm_nt(p.a, p.b, want_acc=False)
    check_close(got, ref, f"bf16 forced {cfg}")


@pytest.mark.parametrize("M,N,K", [(64, 2112, 7168), (128, 7168, 2048), (64, 32768, 512)])
def test_bf16_dense_decode_full(dg, M, N, K):
    """Decode-shaped problems (the picker's split-K and one-wave paths)."""
    p = workloads.bf16_dense_problem(M, N, K, seed=0)
    got = run_dense(dg, p)
    ref, _ = oracle.default().bf16_gemm_nt(p.a, p.b, want_acc=False)
    check_close(got, ref, f"bf16 decode {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", [(4096, 2112, 7168), (4096, 24576, 1536)])
def test_bf16_dense_prefill_sampled(dg, M, N, K):
    p = workloads.bf16_dense_problem(M, N, K, seed=0)
    got = run_dense(dg, p)
    rows = sample_rows(M, 40, seed=M + N)
    ref, _ = oracle.default().bf16_gemm_nt(p.a[rows], p.b, want_acc=False)
    check_close(got[rows], ref, f"bf16 prefill {M}x{N}x{K}")


def test_bf16_dense_deterministic(dg):
    p = workloads.bf16_dense_problem(64, 2112, 7168, seed=3)   # split-K path
    assert np.array_equal(run_dense(dg, p), run_dense(dg, p))


def test_bf16_dense_zero_rows(dg):
    a = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    b = torch.zeros((128, 256), dtype=torch.bfloat16, device="cuda")
    d = dg.bf16_gemm_nt(a, b)
    assert d.shape == (0, 128)


# ---------------------------------------------------------------- grouped --

def run_contiguous(dg, p: workloads.Bf16ContiguousProblem) -> np.ndarray:
    d = sentinel_like((p.M_sum, p.N))
    dg.m_grouped_bf16_gemm_nt_contiguous(bf16_dev(p.a), bf16_dev(p.b),
                                         torch.from_numpy(p.m_indices).cuda(), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    return d_bits(d)


@pytest.mark.parametrize("G,N,K,counts", [
    (4, 144, 256, [3, 0, 130, 1]),
    (8, 1024, 2048, None),
])
def test_bf16_contiguous(dg, G, N, K, counts):
    if counts is None:
        counts = workloads.zipf_counts(2048, G, 1.1, seed=5)
    p = workloads.bf16_contiguous_problem(G, N, K, np.asarray(counts), seed=1)
    got = run_contiguous(dg, p)
    pad = p.m_indices < 0
    assert np.all(got[pad] == workloads.SENTINEL_BF16), "padding rows were written"
    valid = np.nonzero(~pad)[0]
    rows = valid[sample_rows(len(valid), 96, seed=7)]
    ref = np.full((len(rows), p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().bf16_grouped_contiguous(p.a[rows], p.b, p.m_indices[rows], d=ref)
    check_close(got[rows], ref, f"bf16 contiguous G={G}")


def run_masked(dg, p: workloads.Bf16MaskedProblem) -> np.ndarray:
    d = sentinel_like((p.G, p.max_m, p.N))
    dg.m_grouped_bf16_gemm_nt_masked(bf16_dev(p.a), bf16_dev(p.b),
                                     torch.from_numpy(p.masked_m).cuda(), p.expected_m, d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    return d_bits(d)


@pytest.mark.parametrize("G,max_m,N,K,masked_m", [
    (5, 200, 144, 256, [0, 200, 3, 129, 250]),
    (16, 256, 1024, 2048, None),
])
def test_bf16_masked(dg, G, max_m, N, K, masked_m):
    if masked_m is None:
        masked_m = np.random.default_rng(8).integers(0, max_m + 1, G)
    p = workloads.bf16_masked_problem(G, max_m, N, K, np.asarray(masked_m), seed=1)
    got = run_masked(dg, p)
    ref = np.full((p.G, p.max_m, p.N), workloads.SENTINEL_BF16, np.uint16)
    oracle.default().bf16_grouped_masked(p.a, p.b, p.masked_m, d=ref)
    for g in range(p.G):
        v = min(max(int(p.masked_m[g]), 0), p.max_m)
        assert np.all(got[g, v:] == workloads.SENTINEL_BF16), f"group {g}: masked rows written"
        if v:
            check_close(got[g, :v], ref[g, :v], f"bf16 masked group {g}")
