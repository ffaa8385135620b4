"""GPU parity of the K-grouped GEMM (the weight gradient of the MoE grouped
forms in training): dg_k_grouped_fp8_gemm_tn_contiguous against the oracle.

D[g] = C[g] + A_g^T B_g over group g's rows of K, in FP32.  The tolerance is
the FP32-output one of the dense FP32 form: the tensor core adds K/32 exact
products per element in FP32, the oracle sums them exactly in double, so per
element |gpu - ref| <= 1e-4 * (|ref| + rms(ref)) and globally
1 - 2 sum(xy) / sum(x^2 + y^2) <= 1e-9.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def dg():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import moe_grouped_gemm_09_b200 as lib
    assert lib.get_last_device_error() == 0
    return lib


def make_case(seed, ks, M, N):
    """Per-token rows of A [K_sum, M] (e.g. output gradients) and B [K_sum, N]
    (e.g. layer inputs): N(0, 1) values quantised in 1 x 128 blocks along K
    for A (one scale per output row per 128 tokens) and 128 x 128 blocks for
    B, the scale conventions of the dense call."""
    rng = np.random.default_rng(seed)
    K_sum = int(np.sum(ks))
    xa = rng.standard_normal((M, K_sum), dtype=np.float32)
    xb = rng.standard_normal((N, K_sum), dtype=np.float32)
    qa, sfa = workloads.quantize_rows(xa, 1)            # [M, K_sum], [M, K_sum/128]
    qb, sfb = workloads.quantize_rows(xb, 128)          # [N, K_sum], [N/128, K_sum/128]
    a = np.ascontiguousarray(qa.T)                      # [K_sum, M]
    b = np.ascontiguousarray(qb.T)                      # [K_sum, N]
    c = (rng.standard_normal((len(ks), M, N)) * 16).astype(np.float32)
    return a, sfa, b, sfb, np.asarray(ks, np.int32), c


def check_f32(got, ref, what):
    got = np.asarray(got, np.float64)
    rms = np.sqrt(np.mean(ref * ref))
    viol = np.abs(got - ref) / (1e-4 * (np.abs(ref) + rms))
    assert viol.max() <= 1.0, f"{what}: worst {viol.max():.3f}"
    diff = 1 - 2 * np.sum(got * ref) / np.sum(got * got + ref * ref)
    assert diff <= 1e-9, f"{what}: global {diff:.3e}"


CASES = [
    ([256, 0, 128, 384], 144, 272),            # an empty group, ragged N, several tiles
    ([128] * 3 + [1024, 0, 640], 512, 640),    # uneven groups, many tiles per group
]


@pytest.mark.parametrize("mode", ["none", "c", "in_place"])
@pytest.mark.parametrize("ks,M,N", CASES)
def test_k_grouped_matches_oracle(dg, ks, M, N, mode):
    a, sfa, b, sfb, ks, c = make_case(len(ks) + M, ks, M, N)
    G = len(ks)
    ta, tsfa, tb, tsfb, tks = dev(a), dev(sfa), dev(b), dev(sfb), dev(ks)
    if mode == "none":
        d = dg.k_grouped_fp8_gemm_tn_contiguous(ta, tsfa, tb, tsfb, tks)
        ref = oracle.default().k_grouped_tn(a, sfa, b, sfb, ks, None)
    elif mode == "c":
        tc = dev(c)
        d = dg.k_grouped_fp8_gemm_tn_contiguous(ta, tsfa, tb, tsfb, tks, c=tc)
        assert np.array_equal(tc.cpu().numpy(), c)     # C is read only
        ref = oracle.default().k_grouped_tn(a, sfa, b, sfb, ks, c)
    else:
        d = dev(c)
        dg.k_grouped_fp8_gemm_tn_contiguous(ta, tsfa, tb, tsfb, tks, c=d, d=d)
        ref = oracle.default().k_grouped_tn(a, sfa, b, sfb, ks, c)
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    got = d.cpu().numpy()
    for g in range(G):
        if ks[g] == 0:   # an empty group: exactly C (or zeros)
            want = c[g] if mode != "none" else np.zeros((M, N), np.float32)
            assert np.array_equal(got[g], want), g
    check_f32(got, ref, f"k-grouped {list(ks)} {M}x{N} {mode}")


def test_k_grouped_moe_shaped(dg):
    """32 groups with Zipf-skewed token counts (the contiguous MoE recipe: 8192
    tokens, each expert's segment padded to 128), the gradient of a
    768 x 1024 expert weight; every element compared."""
    counts = workloads.zipf_counts(8192, 32, 1.1, seed=5)
    ks = (-(-counts // 128) * 128).astype(np.int32)
    a, sfa, b, sfb, ks, _ = make_case(7, ks, 768, 1024)
    d = dg.k_grouped_fp8_gemm_tn_contiguous(dev(a), dev(sfa), dev(b), dev(sfb), dev(ks))
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    ref = oracle.default().k_grouped_tn(a, sfa, b, sfb, ks, None)
    check_f32(d.cpu().numpy(), ref, "k-grouped MoE-shaped")


def test_k_grouped_bad_group_sizes_write_nothing(dg):
    """Group sizes that do not tile K in multiples of 128 are found on the
    device: device error 0x203, and D is left untouched."""
    a, sfa, b, sfb, ks, c = make_case(3, [256, 128], 32, 128)
    for bad in ([256, 64], [256, 256], [384, -128]):
        d = torch.full((2, 32, 128), 7.0, device="cuda")
        dg.k_grouped_fp8_gemm_tn_contiguous(dev(a), dev(sfa), dev(b), dev(sfb),
                                            dev(np.asarray(bad, np.int32)), d=d)
        torch.cuda.synchronize()
        assert dg.get_last_device_error() == 0x203, bad
        assert torch.all(d == 7.0), bad


@pytest.mark.parametrize("cfg", ["256:1", "128:1"])
def test_k_grouped_each_fp32_output_variant(dg, cfg, monkeypatch):
    """Both FP32-output variants (256 columns, one accumulator; 128 columns,
    two), forced, on uneven groups with an empty one and an addend."""
    monkeypatch.setenv("DG_FORCE_CONFIG", cfg)
    ks, M, N = [128] * 3 + [1024, 0, 640], 384, 528
    a, sfa, b, sfb, ks, c = make_case(11, ks, M, N)
    d = dg.k_grouped_fp8_gemm_tn_contiguous(dev(a), dev(sfa), dev(b), dev(sfb), dev(ks), c=dev(c))
    torch.cuda.synchronize()
    assert dg.get_last_device_error() == 0
    got = d.cpu().numpy()
    assert np.array_equal(got[4], c[4])
    check_f32(got, oracle.default().k_grouped_tn(a, sfa, b, sfb, ks, c), f"k-grouped forced {cfg}")
