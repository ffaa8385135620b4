"""GPU test of dg_fp8_gemm_nt_noalloc, the dense GEMM for callers that cannot
allocate device memory (a pool or caching allocator owns it, or the process
must not grow after start-up).  Its only scratch, the device error word, is a
fixed array inside the library.  The test calls it through the C ABI, checks
its output against the oracle and against dg_fp8_gemm_nt's, within the parity
tolerance, on two calls in a row, and reads the array's error word after each
call through dg_fp8_gemm_nt_noalloc_get_last_device_error: it must be 0 (the
array keeps the last call's contents, so a code left by the first call would
still show after the second).

This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test; it also passes on its own in a
fresh process.
"""
import ctypes

import pytest
import torch

import oracle
import workloads
from parity import check_close, d_bits, dev, sentinel_like

pytestmark = pytest.mark.gpu

# split-K decode shapes (cluster reduction in shared memory), a short one, a
# ragged general one, a prefill-sized one (persistent CTAs, many tiles each)
# and one whose last wave is split off (a first launch and two split-K tails)
SHAPES = [(64, 2112, 7168), (128, 7168, 2048), (64, 512, 1024), (300, 384, 512),
          (4096, 2112, 1024), (1280, 4096, 4096)]


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as dg
    return dg


def _c(dg):
    c = ctypes.CDLL(dg.LIB_PATH)
    fn = c.dg_fp8_gemm_nt_noalloc
    fn.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 3 + [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    err = c.dg_fp8_gemm_nt_noalloc_get_last_device_error
    err.argtypes = [ctypes.POINTER(ctypes.c_int)]
    err.restype = ctypes.c_int
    return fn, err


def _call_noalloc(dg, a, sfa, b, sfb, d, M, N, K):
    fn, _ = _c(dg)
    stream = torch.cuda.current_stream().cuda_stream
    return fn(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(), d.data_ptr(), M, N, K,
              stream)


def _noalloc_error(dg) -> int:
    _, err = _c(dg)
    code = ctypes.c_int(-1)
    assert err(ctypes.byref(code)) == 0
    return code.value


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_noalloc_matches_oracle_and_regular_entry_point(lib, M, N, K):
    p = workloads.dense_problem(M, N, K, seed=21)
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    want, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    regular = sentinel_like((M, N))
    lib.fp8_gemm_nt(a, sfa, b, sfb, regular)
    torch.cuda.synchronize()
    assert lib.get_last_device_error() == 0
    regular_bits = d_bits(regular)
    for call in range(2):
        d = sentinel_like((M, N))
        rc = _call_noalloc(lib, a, sfa, b, sfb, d, M, N, K)
        assert rc == 0, lib.status_string(rc)
        torch.cuda.synchronize()
        assert _noalloc_error(lib) == 0, f"call {call}: error word set"
        got = d_bits(d)
        check_close(got, want, f"no-alloc call {call} {M}x{N}x{K} vs oracle")
        check_close(got, regular_bits, f"no-alloc call {call} {M}x{N}x{K} vs dg_fp8_gemm_nt")


def test_noalloc_rejects_bad_sizes(lib):
    z = torch.zeros(16, dtype=torch.uint8, device="cuda")
    f = torch.ones(16, device="cuda")
    o = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    assert _call_noalloc(lib, z, f, z, f, o, 4, 15, 128) == 1     # N % 16 != 0
    assert _call_noalloc(lib, z, f, z, f, o, 4, 16, 100) == 1     # K % 128 != 0
