"""Helpers shared by the GPU parity tests: moving seeded problems to the device,
running the oracle on all or on sampled rows, and the tolerance check.

Tolerance (FP32 accumulation in a different order than the oracle's exact
double sum, then one BF16 rounding on each side): per element
``|gpu - ref| <= 8e-3 * |ref| + 1e-3 * rms(ref)`` and, over the compared set,
``1 - 2 * sum(x*y) / sum(x*x + y*y) <= 1e-5``.  One BF16 unit in the last place
is 2**-8 relative, so the per-element bound admits the two results landing on
neighbouring BF16 values; the rms term covers values that cancel to near zero.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

REL_TOL = 8e-3
RMS_TOL = 1e-3
GLOBAL_TOL = 1e-5


def bits_to_f64(bits) -> np.ndarray:
    if isinstance(bits, torch.Tensor):
        bits = bits.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return oracle.bf16_bits_to_float(np.asarray(bits, np.uint16)).astype(np.float64)


def check_close(gpu_bits, ref_bits, what: str = "") -> dict:
    x = bits_to_f64(gpu_bits).ravel()
    y = bits_to_f64(ref_bits).ravel()
    assert x.shape == y.shape, (x.shape, y.shape)
    assert np.all(np.isfinite(x)), f"{what}: non-finite GPU output"
    rms = float(np.sqrt(np.mean(y * y))) if y.size else 0.0
    bound = REL_TOL * np.abs(y) + RMS_TOL * rms
    err = np.abs(x - y)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if y.size else 0.0
    den = float(np.sum(x * x + y * y))
    gdiff = 1.0 - 2.0 * float(np.sum(x * y)) / den if den > 0 else 0.0
    stats = {"max_err_over_bound": ratio, "global_diff": gdiff,
             "exact_fraction": float(np.mean(x == y)) if y.size else 1.0}
    assert ratio <= 1.0, f"{what}: element error {ratio:.3f}x the bound"
    assert gdiff <= GLOBAL_TOL, f"{what}: global difference {gdiff:.3e}"
    return stats


def dev(x: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(device)


def sentinel_like(shape, device="cuda") -> torch.Tensor:
    t = torch.full(shape, workloads.SENTINEL_BF16, dtype=torch.int16, device=device)
    return t.view(torch.bfloat16)


def d_bits(d: torch.Tensor) -> np.ndarray:
    return d.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def sample_rows(total: int, n: int, seed: int = 0) -> np.ndarray:
    """Rows spread over every 128-row tile, always including the first and last."""
    if total <= n:
        return np.arange(total)
    rng = np.random.default_rng(seed)
    picks = set([0, total - 1, min(127, total - 1), min(128, total - 1)])
    picks.update(rng.choice(total, n - len(picks), replace=False).tolist())
    return np.array(sorted(picks))


def oracle_dense_rows(p: workloads.DenseProblem, rows: np.ndarray) -> np.ndarray:
    d, _ = oracle.default().gemm_nt(p.a[rows], p.sfa[rows], p.b, p.sfb, want_acc=False)
    return d


def oracle_contiguous_rows(p: workloads.ContiguousProblem, rows: np.ndarray) -> np.ndarray:
    sentinel = np.full((len(rows), p.N), workloads.SENTINEL_BF16, np.uint16)
    d, _ = oracle.default().grouped_contiguous(p.a[rows], p.sfa[rows], p.b, p.sfb,
                                               p.m_indices[rows], d=sentinel)
    return d


def oracle_masked_rows(p: workloads.MaskedProblem, pairs: list[tuple[int, int]]) -> np.ndarray:
    """Reference rows (g, m) of the masked problem, one row at a time."""
    o = oracle.default()
    out = np.full((len(pairs), p.N), workloads.SENTINEL_BF16, np.uint16)
    for i, (g, m) in enumerate(pairs):
        valid = min(max(int(p.masked_m[g]), 0), p.max_m)
        if m < valid:
            d, _ = o.gemm_nt(p.a[g, m:m + 1], p.sfa[g, m:m + 1], p.b[g], p.sfb[g], want_acc=False)
            out[i] = d[0]
    return out
