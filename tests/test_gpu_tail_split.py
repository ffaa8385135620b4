"""GPU parity of the last-wave split of the dense forms: when the last wave of
output tiles would occupy at most half of the SMs, the call computes the whole
waves in one launch and the remaining tiles (one or two rectangles of D) in
split-K launches of 128 x 128 tiles.  Every output element is compared with
the oracle, for shapes whose tail is one rectangle or two, with ragged last
row and column blocks, on E4M3 and BF16 operands; D's untouched-row rule does
not apply to the dense form, so a sentinel fill checks that every element is
written exactly by one of the launches."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_close, d_bits, dev, oracle_dense_rows, sample_rows, sentinel_like

pytestmark = pytest.mark.gpu


def bf16_dev(bits: np.ndarray) -> torch.Tensor:
    """BF16 bit patterns (uint16) -> a bfloat16 CUDA tensor with those bits."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to("cuda")
    return t.view(torch.bfloat16)


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as lib
    assert lib.get_last_device_error() == 0
    return lib


def _tail(dg, M, N, k_bytes):
    c = dg.query_config(dg.KIND_DENSE, M, N, k_bytes, num_sms=dg.get_num_sms())
    return c["tail_launches"], c["tail_split"], c["main_tiles"]


# (M, N, K): the tail is the last m-blocks of one column plus whole columns
# (1280 x 4096: 160 tiles, 12 past the first wave; split 4), the same with
# ragged rows and columns (1200 x 4000), the last m-blocks of one column only
# (1024 x 4864: 152 tiles, 4 past the wave; split 8), and whole columns only
# (512 x 10240: 160 tiles, the last three columns; split 4).
SHAPES = [(1280, 4096, 4096), (1200, 4000, 4096), (1024, 4864, 4096), (512, 10240, 4096)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_tail_split_matches_oracle(dg, M, N, K):
    if dg.get_num_sms() != 148:
        pytest.skip("tile counts assume 148 SMs")
    launches, split, main = _tail(dg, M, N, K)
    assert launches >= 1, "the shape must take the last-wave split"
    p = workloads.dense_problem(M, N, K, seed=M + N)
    d = sentinel_like((M, N))
    dg.fp8_gemm_nt(dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    ref, _ = oracle.default().gemm_nt(p.a, p.sfa, p.b, p.sfb, want_acc=False)
    check_close(d_bits(d), ref, f"tail split {M}x{N}x{K} ({launches} tail launches, split {split})")


def test_tail_split_prefill_shape(dg):
    """4096 x 7168 x 16384 (896 tiles: six waves, then 8 tiles of the last
    column, split 8 ways as 16 tiles of 128 x 128): sampled rows, among them
    rows of the tail rectangle, every column."""
    if dg.get_num_sms() != 148:
        pytest.skip("tile counts assume 148 SMs")
    M, N, K = 4096, 7168, 16384
    assert _tail(dg, M, N, K) == (1, 8, 888)
    p = workloads.dense_problem(M, N, K, seed=2)
    d = sentinel_like((M, N))
    dg.fp8_gemm_nt(dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    rows = np.union1d(sample_rows(M, 24, seed=3), [0, 3071, 3072, 3500, 4095])
    check_close(d_bits(d)[rows], oracle_dense_rows(p, rows), "tail split 4096x7168x16384")


def test_tail_split_deterministic(dg):
    if dg.get_num_sms() != 148:
        pytest.skip("tile counts assume 148 SMs")
    M, N, K = SHAPES[0]
    p = workloads.dense_problem(M, N, K, seed=5)
    a, sfa, b, sfb = dev(p.a), dev(p.sfa), dev(p.b), dev(p.sfb)
    outs = []
    for _ in range(2):
        d = sentinel_like((M, N))
        dg.fp8_gemm_nt(a, sfa, b, sfb, d)
        torch.cuda.synchronize()
        outs.append(d_bits(d))
    assert np.array_equal(outs[0], outs[1])


def test_tail_split_bf16(dg):
    if dg.get_num_sms() != 148:
        pytest.skip("tile counts assume 148 SMs")
    M, N, K = 1280, 4096, 2048           # 4096 bytes of K per row, as the E4M3 case
    assert _tail(dg, M, N, 2 * K)[0] >= 1
    p = workloads.bf16_dense_problem(M, N, K, seed=9)
    d = sentinel_like((M, N))
    dg.bf16_gemm_nt(bf16_dev(p.a), bf16_dev(p.b), d)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    ref, _ = oracle.default().bf16_gemm_nt(p.a, p.b, want_acc=False)
    check_close(d_bits(d), ref, f"bf16 tail split {M}x{N}x{K}")
