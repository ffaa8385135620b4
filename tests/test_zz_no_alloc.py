"""GPU test of dg_fp8_gemm_nt_noalloc, the dense GEMM for callers that cannot
allocate device memory (a pool or caching allocator owns it, or the process
must not grow after start-up).  Its scratch is a fixed array inside the
library.  The test calls it through the C ABI and checks its output against
dg_fp8_gemm_nt's, within the parity tolerance, on two calls in a row -- the
second call finds the array holding the first call's contents.

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads
from parity import check_close, d_bits, dev, sentinel_like

pytestmark = pytest.mark.gpu

# split-K decode shapes (they use the scratch) and one that needs none
SHAPES = [(64, 2112, 7168), (128, 7168, 2048), (64, 512, 1024), (300, 384, 512)]


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as dg
    return dg


def _call_noalloc(dg, a, sfa, b, sfb, d, M, N, K):
    c = ctypes.CDLL(dg.LIB_PATH)
    fn = c.dg_fp8_gemm_nt_noalloc
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 3 + [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    return fn(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(), d.data_ptr(), M, N, K,
              stream)


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_noalloc_matches_regular_entry_point(lib, M, N, K):
    p = workloads.dense_problem(M, N, K, seed=21)
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    ref = sentinel_like((M, N))
    lib.fp8_gemm_nt(a, sfa, b, sfb, ref)
    torch.cuda.synchronize()
    ref_bits = d_bits(ref)
    for call in range(2):
        d = sentinel_like((M, N))
        rc = _call_noalloc(lib, a, sfa, b, sfb, d, M, N, K)
        assert rc == 0, lib.status_string(rc)
        torch.cuda.synchronize()
        got = d_bits(d)
        check_close(got, ref_bits, f"no-alloc call {call} {M}x{N}x{K}")


def test_noalloc_rejects_bad_sizes(lib):
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    f = torch.ones(16, device="cuda")
    o = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, z, f, z, f, o, 4, 15, 128) == 1     # N % 16 != 0
    assert _call_noalloc(lib, z, f, z, f, o, 4, 16, 100) == 1     # K % 128 != 0
