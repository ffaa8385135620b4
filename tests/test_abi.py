"""The C ABI without a GPU: the library loads, exports every entry point that
include/dg.h declares, rejects bad arguments before touching a device, and its
configuration picker (host code) makes sane choices."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dg.h")


@pytest.fixture(scope="module")
def dg():
    from conftest import ensure_library_built
    ensure_library_built()
    import moe_grouped_gemm_09_b200 as lib
    return lib


def declared_functions() -> list[str]:
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(dg_\w+)\s*\(", text)
    return sorted(set(n for n in names if n not in ("dg_status", "dg_stream_t", "dg_config")))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
                     "dg_m_grouped_fp8_gemm_nt_masked", "dg_set_num_sms"):
        assert required in names


def test_every_declared_symbol_is_exported(dg):
    lib = ctypes.CDLL(dg.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(dg.EXPORTED_SYMBOLS) == set(declared_functions())


def test_version_and_status_strings(dg):
    assert re.fullmatch(r"\d+\.\d+\.\d+", dg.version())
    assert dg.status_string(0) == "DG_OK"
    assert dg.status_string(1) == "DG_ERR_INVALID_ARG"
    assert dg.status_string(99) == "DG_ERR_UNKNOWN"


FAKE = 0x10000  # never dereferenced: the checks below fail before any device work


@pytest.mark.parametrize("M,N,K", [(4, 15, 128), (4, 16, 100), (4, 16, 0), (-1, 16, 128), (4, 0, 128)])
def test_dense_bad_sizes_rejected(dg, M, N, K):
    rc = dg._gemm_nt(FAKE, FAKE, FAKE, FAKE, FAKE, M, N, K, None)
    assert rc == 1  # DG_ERR_INVALID_ARG


def test_dense_null_and_misaligned_rejected(dg):
    assert dg._gemm_nt(FAKE, FAKE, None, FAKE, FAKE, 4, 16, 128, None) == 1
    assert dg._gemm_nt(FAKE + 8, FAKE, FAKE, FAKE, FAKE, 4, 16, 128, None) == 1
    assert dg._gemm_nt(FAKE, FAKE + 2, FAKE, FAKE, FAKE, 4, 16, 128, None) == 1


def test_layout_forms_reject_bad_arguments(dg):
    # an M-major A needs M % 16 == 0; all three forms share the dense checks
    assert dg._gemm_tn(FAKE, FAKE, FAKE, FAKE, FAKE, 20, 16, 128, None) == 1
    assert dg._gemm_tt(FAKE, FAKE, FAKE, FAKE, FAKE, 20, 16, 128, None) == 1
    for fn in (dg._gemm_nn, dg._gemm_tn, dg._gemm_tt):
        assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 32, 15, 128, None) == 1
        assert fn(FAKE, FAKE, FAKE, FAKE, FAKE, 32, 16, 100, None) == 1
        assert fn(FAKE + 8, FAKE, FAKE, FAKE, FAKE, 32, 16, 128, None) == 1
        assert fn(None, None, None, None, None, 0, 16, 128, None) == 0


def test_f32_form_rejects_bad_arguments(dg):
    assert dg._gemm_nt_f32(FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, 32, 16, 128, None) == 1  # c
    assert dg._gemm_nt_f32(FAKE, FAKE, FAKE, FAKE, None, FAKE + 4, 32, 16, 128, None) == 1  # d
    assert dg._gemm_nt_f32(FAKE, FAKE, FAKE, FAKE, None, FAKE, 32, 15, 128, None) == 1
    assert dg._gemm_nt_f32(None, None, None, None, None, None, 0, 16, 128, None) == 0


def test_bf16_forms_reject_bad_arguments(dg):
    # K must be a whole number of 64-element (128-byte) blocks; no scales needed
    assert dg._bf16_gemm_nt(FAKE, FAKE, FAKE, 4, 16, 96, None) == 1
    assert dg._bf16_gemm_nt(FAKE, FAKE, FAKE, 4, 15, 64, None) == 1
    assert dg._bf16_gemm_nt(None, FAKE, FAKE, 4, 16, 64, None) == 1
    assert dg._bf16_gemm_nt(FAKE, FAKE, FAKE + 8, 4, 16, 64, None) == 1
    assert dg._bf16_gemm_nt(None, None, None, 0, 16, 64, None) == 0
    assert dg._bf16_gemm_contig(FAKE, FAKE, FAKE, FAKE, 100, 16, 64, 2, None) == 1
    assert dg._bf16_gemm_contig(FAKE, FAKE, FAKE, None, 128, 16, 64, 2, None) == 1
    assert dg._bf16_gemm_masked(FAKE, FAKE, FAKE, None, 2, 64, 16, 64, 1, None) == 1
    assert dg._bf16_gemm_masked(FAKE, FAKE, FAKE, FAKE, 5000, 64, 16, 64, 1, None) == 2
    assert dg._bf16_gemm_masked(None, None, None, None, 0, 64, 16, 64, 1, None) == 0


def test_zero_rows_is_a_noop(dg):
    # no device is touched for an empty problem, even with null pointers
    assert dg._gemm_nt(None, None, None, None, None, 0, 16, 128, None) == 0
    assert dg._gemm_masked(None, None, None, None, None, None, 0, 64, 16, 128, 1, None) == 0


def test_grouped_bad_arguments_rejected(dg):
    # contiguous: M_sum not a multiple of 128, missing m_indices
    assert dg._gemm_contig(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 100, 16, 128, 2, None) == 1
    assert dg._gemm_contig(FAKE, FAKE, FAKE, FAKE, FAKE, None, 128, 16, 128, 2, None) == 1
    # masked: missing masked_m; too many groups
    assert dg._gemm_masked(FAKE, FAKE, FAKE, FAKE, FAKE, None, 2, 64, 16, 128, 1, None) == 1
    assert dg._gemm_masked(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 5000, 64, 16, 128, 1, None) == 2


def test_timeout_setter(dg):
    with pytest.raises(dg.DgError):
        dg.set_wait_timeout_ms(0)
    dg.set_wait_timeout_ms(1000)


# ------------------------------------------------------------- the picker --

def test_decode_shapes_run_in_one_wave_of_deep_stages(dg):
    """Decode-shaped dense problems use a decode variant (several K blocks per
    stage) and exactly one wave of CTAs; split-K tiles are whole clusters."""
    for (m, n, k) in [(64, 2112, 7168), (128, 2112, 7168), (64, 7168, 2048), (128, 7168, 2048),
                      (64, 32768, 512), (128, 32768, 512), (64, 512, 1024)]:
        c = dg.query_config(0, m, n, k, num_sms=148)
        n_tiles = -(-n // c["block_n"])
        assert c["kps"] >= 2, (m, n, k, c)
        assert c["grid"] == n_tiles * c["split_k"] <= 148, (m, n, k, c)
        kb = k // 128
        per = -(-kb // c["split_k"])
        assert (c["split_k"] - 1) * per < kb            # no empty K slice
        assert c["smem_bytes"] <= 232448 and c["tmem_cols"] <= 512


def test_decode_split_is_a_portable_cluster(dg):
    for n in (512, 2112, 4096, 7168):
        for k in (512, 1024, 2048, 7168, 16384):
            c = dg.query_config(0, 64, n, k, num_sms=148)
            assert 1 <= c["split_k"] <= 8


def test_prefill_is_persistent(dg):
    for (m, n, k) in [(4096, 2112, 7168), (4096, 24576, 1536), (4096, 7168, 16384)]:
        c = dg.query_config(0, m, n, k, num_sms=148)
        assert c["split_k"] == 1 and c["grid"] == 148
        assert c["smem_bytes"] <= 232448 and c["tmem_cols"] <= 512


def test_sm_cap_bounds_the_grid(dg):
    for kind, rows, g in ((0, 4096, 1), (1, 10112, 32), (2, 256, 32)):
        c = dg.query_config(kind, rows, 4096, 7168, G=g, expected_m=128, num_sms=48)
        assert c["grid"] <= 48


def test_small_problem_grid_is_its_tile_count(dg):
    c = dg.query_config(0, 300, 96, 128, num_sms=148)
    assert c["grid"] == (-(-300 // 128)) * (-(-96 // c["block_n"]))


def test_k_grouped_plan_covers_every_group(dg):
    """The K-grouped form (kind 3) takes persistent general tiles with whole
    128-column B boxes, and its tiles are every group's output tiles."""
    c = dg.query_config(3, 256, 384, 4096, G=8, num_sms=148)
    assert c["block_n"] % 128 == 0 and c["split_k"] == 1 and c["kps"] == 1
    assert c["grid"] == min(148, 8 * 2 * (-(-384 // c["block_n"])))


def test_k_grouped_bad_arguments_rejected(dg):
    fn = dg._k_grouped
    # a, sfa, b, sfb, c, d, ks, G, M, N, K_sum, stream
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 24, 128, 256, None) == 1   # M % 16
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 32, 120, 256, None) == 1   # N % 16
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2, 32, 128, 200, None) == 1   # K % 128
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, None, 2, 32, 128, 256, None) == 1   # no ks
    assert fn(FAKE, FAKE, FAKE, FAKE, FAKE + 4, FAKE, FAKE, 2, 32, 128, 256, None) == 1  # c align
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 2000, 32, 128, 256, None) == 2  # G > 1024
    assert fn(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, 0, 32, 128, 256, None) == 0     # no groups


def test_last_wave_split_plan(dg):
    """The dense form's last-wave split (host planning, no GPU): taken when
    the tiles past the whole waves, as 128-column tiles split at least 2
    ways, fit one wave and K is at least 4096 bytes, with the largest split
    whose clusters fit one wave."""
    q = dg.query_config
    # 896 tiles = 6 waves + 8 tiles in one column: one rectangle, 16 tiles x 8
    c = q(0, 4096, 7168, 16384)
    assert (c["main_tiles"], c["tail_launches"], c["tail_split"]) == (888, 1, 8)
    # 160 tiles = 1 wave + 12: two rectangles of 24 tiles, split 4
    c = q(0, 1280, 4096, 4096)
    assert (c["main_tiles"], c["tail_launches"], c["tail_split"]) == (148, 2, 4)
    # no split: the last wave is more than half full (288 = 148 + 140), K is
    # short, the problem fits one wave, the tiles divide into whole waves
    # (4096 x 4096 x 7168: 3 waves + 68 tiles, 136 tail tiles, no split of 2 fits)
    for shape in [(4096, 2112, 7168), (4096, 4096, 2048), (1024, 4096, 7168), (4736, 1024, 7168),
                  (4096, 4096, 7168)]:
        c = q(0, *shape)
        assert (c["main_tiles"], c["tail_launches"], c["tail_split"]) == (0, 0, 0), shape
    # the grouped forms never split their last wave
    c = q(1, 10112, 4096, 7168, G=32)
    assert c["tail_launches"] == 0
    # fewer SMs: 512 tiles on 132 SMs = 3 waves + 116 (more than half): none
    assert q(0, 4096, 4096, 7168, num_sms=132)["tail_launches"] == 0


def test_query_rejects_bad_input(dg):
    with pytest.raises(dg.DgError):
        dg.query_config(4, 64, 128, 128)
    with pytest.raises(dg.DgError):
        dg.query_config(0, 64, 100, 128)


# ------------------------------------------------ the Python binding's checks --

def test_binding_rejects_wrong_dtypes_and_host_tensors(dg):
    """The binding validates tensors before any call into the library: wrong
    element types raise TypeError, host (CPU) tensors ValueError."""
    import torch
    a8 = torch.zeros((4, 128), dtype=torch.uint8)
    sfa = torch.ones((4, 1), dtype=torch.float32)
    b8 = torch.zeros((16, 128), dtype=torch.uint8)
    sfb = torch.ones((1, 1), dtype=torch.float32)
    with pytest.raises(TypeError):
        dg.fp8_gemm_nt(a8.float(), sfa, b8, sfb)
    with pytest.raises(ValueError):
        dg.fp8_gemm_nt(a8, sfa, b8, sfb)                  # not on a CUDA device
    a16 = torch.zeros((4, 64), dtype=torch.bfloat16)
    b16 = torch.zeros((16, 64), dtype=torch.bfloat16)
    with pytest.raises(TypeError):
        dg.bf16_gemm_nt(a16.float(), b16)
    with pytest.raises(TypeError):
        dg.m_grouped_bf16_gemm_nt_contiguous(a8, b16.unsqueeze(0), torch.zeros(4, dtype=torch.int32))
    with pytest.raises(ValueError):
        dg.bf16_gemm_nt(a16, b16)                         # not on a CUDA device
