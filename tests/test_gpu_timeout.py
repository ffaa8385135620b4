"""GPU test of the kernels' bounded waits: a wait that runs out of time records
a device error code and the kernel returns, leaving the context usable.

No fault is injected and nothing is left unsignalled: the wait limit is set to
one microsecond, well below the time the pipeline's own waits take on a long-K
problem (the epilogue waits for the whole K loop, tens of microseconds), so a
wait runs out during an ordinary launch.  The kernel then records a timeout
code (0x101..0x104), raises its abort flag, drains its in-flight copies and
tensor-core work, frees its tensor memory and returns.  The test checks that
the stream synchronises, that the code is reported, and that the next launch
at the default limit is correct against the oracle, for a single-CTA tile and
for a split-K cluster of two CTAs.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_close, d_bits, dev, sentinel_like

pytestmark = pytest.mark.gpu

DEFAULT_LIMIT_NS = 1_000_000_000
TIMEOUT_CODES = {0x101, 0x102, 0x103, 0x104}


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as lib
    assert lib.get_last_device_error() == 0
    yield lib
    lib.set_wait_timeout_ns(DEFAULT_LIMIT_NS)


# (force config "block_n:split_k:kps:a_rows:mode", M, N, K): one output tile of
# a decode variant, so one CTA without split and a cluster of two CTAs with
# split 2
CASES = [("64:1:2:128:1", 64, 64, 16384), ("64:2:2:128:1", 64, 64, 16384)]


@pytest.mark.parametrize("cfg,M,N,K", CASES)
def test_wait_runs_out_then_recovers(dg, cfg, M, N, K, monkeypatch):
    monkeypatch.setenv("DG_FORCE_CONFIG", cfg)
    p = workloads.dense_problem(M, N, K, seed=31)
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)

    try:
        dg.set_wait_timeout_ns(1000)
        d = sentinel_like((M, N))
        dg.fp8_gemm_nt(a, sfa, b, sfb, d)
        torch.cuda.synchronize()          # the aborted launch returned
        code = dg.get_last_device_error()
    finally:
        dg.set_wait_timeout_ns(DEFAULT_LIMIT_NS)
    assert code in TIMEOUT_CODES, hex(code)

    for _ in range(2):                     # the context is still usable
        d = sentinel_like((M, N))
        dg.fp8_gemm_nt(a, sfa, b, sfb, d)
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0
        check_close(d_bits(d), ref, f"after timeout {cfg}")
