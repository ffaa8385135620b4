"""FP8 (E4M3) block-scaled GEMM for NVIDIA B200 (sm_100a): dense and MoE
M-grouped (contiguous and masked layouts), and the same forms on BF16 operands.

This module is a thin binding over the C ABI of ``libdg.so`` (declared in
``include/dg.h``): it checks tensor types and devices, passes raw device
pointers, sizes and the current CUDA stream, and raises on a non-zero status.
Every step of the computation runs in the library's CUDA kernels; there is no
Python or CPU fallback, and importing this package fails if the library has not
been built (``python moe_grouped_gemm_09_b200/build.py``).

The calls mirror the DeepGEMM API named on the pages (``fp8_gemm_nt``,
``m_grouped_fp8_gemm_nt_contiguous``, a masked grouped call and
``set_num_sms``), with the scale factors passed next to their operand.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with "
                      "`python moe_grouped_gemm_09_b200/build.py` (nvcc, sm_100a)")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I = ctypes.c_int


def _decl(name, args, res=ctypes.c_int):
    f = getattr(_lib, name)
    f.argtypes = args
    f.restype = res
    return f


_gemm_nt = _decl("dg_fp8_gemm_nt", [_P, _P, _P, _P, _P, _I, _I, _I, _P])
_gemm_nn = _decl("dg_fp8_gemm_nn", [_P, _P, _P, _P, _P, _I, _I, _I, _P])
_gemm_tn = _decl("dg_fp8_gemm_tn", [_P, _P, _P, _P, _P, _I, _I, _I, _P])
_gemm_tt = _decl("dg_fp8_gemm_tt", [_P, _P, _P, _P, _P, _I, _I, _I, _P])
_gemm_nt_f32 = _decl("dg_fp8_gemm_nt_f32", [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P])
_gemm_contig = _decl("dg_m_grouped_fp8_gemm_nt_contiguous", [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P])
_gemm_masked = _decl("dg_m_grouped_fp8_gemm_nt_masked", [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P])
_k_grouped = _decl("dg_k_grouped_fp8_gemm_tn_contiguous",
                   [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P])
_bf16_gemm_nt = _decl("dg_bf16_gemm_nt", [_P, _P, _P, _I, _I, _I, _P])
_bf16_gemm_contig = _decl("dg_m_grouped_bf16_gemm_nt_contiguous", [_P, _P, _P, _P, _I, _I, _I, _I, _P])
_bf16_gemm_masked = _decl("dg_m_grouped_bf16_gemm_nt_masked", [_P, _P, _P, _P, _I, _I, _I, _I, _I, _P])
_set_num_sms = _decl("dg_set_num_sms", [_I])
_get_num_sms = _decl("dg_get_num_sms", [])
_get_last_err = _decl("dg_get_last_device_error", [ctypes.POINTER(ctypes.c_int)])
_set_timeout = _decl("dg_set_wait_timeout_ms", [_I])
_set_timeout_ns = _decl("dg_set_wait_timeout_ns", [ctypes.c_longlong])
_set_check_scales = _decl("dg_set_check_scales", [_I])
_set_weight_preload = _decl("dg_set_weight_preload", [_I])
_gemm_nt_noalloc = _decl("dg_fp8_gemm_nt_noalloc", [_P, _P, _P, _P, _P, _I, _I, _I, _P])
_noalloc_err = _decl("dg_fp8_gemm_nt_noalloc_get_last_device_error", [ctypes.POINTER(ctypes.c_int)])
_status_string = _decl("dg_status_string", [_I], ctypes.c_char_p)
_version = _decl("dg_version", [], ctypes.c_char_p)


class DgConfig(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("block_m", "block_n", "stages", "num_acc", "split_k", "grid", "smem_bytes", "tmem_cols",
                 "kps", "main_tiles", "tail_launches", "tail_split")]


_query = _decl("dg_query_config", [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(DgConfig)])

EXPORTED_SYMBOLS = ("dg_fp8_gemm_nt", "dg_m_grouped_fp8_gemm_nt_contiguous",
                    "dg_m_grouped_fp8_gemm_nt_masked", "dg_set_num_sms", "dg_get_num_sms",
                    "dg_get_last_device_error", "dg_set_wait_timeout_ms", "dg_status_string",
                    "dg_query_config", "dg_version", "dg_fp8_gemm_nt_noalloc", "dg_fp8_gemm_nn",
                    "dg_fp8_gemm_tn", "dg_fp8_gemm_tt", "dg_fp8_gemm_nt_f32", "dg_bf16_gemm_nt",
                    "dg_m_grouped_bf16_gemm_nt_contiguous", "dg_m_grouped_bf16_gemm_nt_masked",
                    "dg_set_wait_timeout_ns", "dg_fp8_gemm_nt_noalloc_get_last_device_error",
                    "dg_set_check_scales", "dg_k_grouped_fp8_gemm_tn_contiguous",
                    "dg_set_weight_preload")

DEVICE_ERRORS = {
    0x101: "wait timeout in the TMA producer",
    0x102: "wait timeout in the scale-factor producer",
    0x103: "wait timeout in the MMA issuer",
    0x104: "wait timeout in the epilogue",
    0x201: "a 128-row block of m_indices names two experts",
    0x202: "an m_indices entry is >= the number of groups",
    0x203: "K-grouped group sizes that do not tile K in multiples of 128",
    0x301: "a scale that is not a positive normal power of two",
}


class DgError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def status_string(status: int) -> str:
    return _status_string(int(status)).decode()


def version() -> str:
    return _version().decode()


def _check(status: int, where: str):
    if status != 0:
        raise DgError(status, where)


def _fp8_bytes(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype not in (torch.float8_e4m3fn, torch.uint8):
        raise TypeError(f"{name}: expected float8_e4m3fn or uint8 (E4M3 bytes), got {t.dtype}")
    return t


def _need(t: torch.Tensor, name: str, dtype: Optional[torch.dtype], shape: tuple, device) -> None:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _stream_ptr(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def fp8_gemm_nt(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense ``D[M,N] = A[M,K] B[N,K]^T`` (BF16), A/B E4M3 K-major, ``sfa [M, K/128]`` and
    ``sfb [ceil(N/128), K/128]`` float32 power-of-two scales.  Runs on the current stream."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    M, K = a.shape
    N = b.shape[0]
    dev = a.device
    _need(a, "a", None, (M, K), dev)
    _need(b, "b", None, (N, K), dev)
    _need(sfa, "sfa", torch.float32, (M, K // 128), dev)
    _need(sfb, "sfb", torch.float32, ((N + 127) // 128, K // 128), dev)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (M, N), dev)
    with torch.cuda.device(dev):
        _check(_gemm_nt(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(), d.data_ptr(),
                        M, N, K, _stream_ptr(dev)), "dg_fp8_gemm_nt")
    return d


def _gemm_layout(name, fn, a_m_major: bool, b_n_major: bool, a, sfa, b, sfb, d):
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    K, M = a.shape if a_m_major else a.shape[::-1]
    N = b.shape[1] if b_n_major else b.shape[0]
    dev = a.device
    _need(a, "a", None, (K, M) if a_m_major else (M, K), dev)
    _need(b, "b", None, (K, N) if b_n_major else (N, K), dev)
    _need(sfa, "sfa", torch.float32, (M, K // 128), dev)
    _need(sfb, "sfb", torch.float32, ((N + 127) // 128, K // 128), dev)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (M, N), dev)
    with torch.cuda.device(dev):
        _check(fn(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(), d.data_ptr(),
                  M, N, K, _stream_ptr(dev)), name)
    return d


def fp8_gemm_nn(a, sfa, b, sfb, d=None):
    """``D[M,N] = A B^T`` with A ``[M, K]`` (K-major) and B given N-major as
    ``b [K, N]``; scales and D as in :func:`fp8_gemm_nt`."""
    return _gemm_layout("dg_fp8_gemm_nn", _gemm_nn, False, True, a, sfa, b, sfb, d)


def fp8_gemm_tn(a, sfa, b, sfb, d=None):
    """``D[M,N] = A B^T`` with A given M-major as ``a [K, M]`` (M % 16 == 0) and
    B N-major as ``b [K, N]``."""
    return _gemm_layout("dg_fp8_gemm_tn", _gemm_tn, True, True, a, sfa, b, sfb, d)


def fp8_gemm_tt(a, sfa, b, sfb, d=None):
    """``D[M,N] = A B^T`` with A given M-major as ``a [K, M]`` (M % 16 == 0) and
    B ``[N, K]`` (K-major)."""
    return _gemm_layout("dg_fp8_gemm_tt", _gemm_tt, True, False, a, sfa, b, sfb, d)


def fp8_gemm_nt_f32(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                    c: Optional[torch.Tensor] = None,
                    d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``D = A B^T + C`` in float32 (``C`` optional; ``c`` may be ``d`` itself to
    accumulate in place); A, B, scales as in :func:`fp8_gemm_nt`."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    M, K = a.shape
    N = b.shape[0]
    dev = a.device
    _need(a, "a", None, (M, K), dev)
    _need(b, "b", None, (N, K), dev)
    _need(sfa, "sfa", torch.float32, (M, K // 128), dev)
    _need(sfb, "sfb", torch.float32, ((N + 127) // 128, K // 128), dev)
    if c is not None:
        _need(c, "c", torch.float32, (M, N), dev)
    if d is None:
        d = torch.empty((M, N), dtype=torch.float32, device=dev)
    _need(d, "d", torch.float32, (M, N), dev)
    with torch.cuda.device(dev):
        _check(_gemm_nt_f32(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(),
                            None if c is None else c.data_ptr(), d.data_ptr(), M, N, K,
                            _stream_ptr(dev)), "dg_fp8_gemm_nt_f32")
    return d


def fp8_gemm_nt_noalloc(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor, sfb: torch.Tensor,
                        d: torch.Tensor) -> torch.Tensor:
    """Dense GEMM through the entry point that allocates no device memory (its
    scratch is a fixed array inside the library), for callers that cannot
    allocate.  ``d`` must be given.  Calls must not overlap on the GPU.  Its
    device error codes are read with :func:`noalloc_get_last_device_error`."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    M, K = a.shape
    N = b.shape[0]
    dev = a.device
    _need(a, "a", None, (M, K), dev)
    _need(b, "b", None, (N, K), dev)
    _need(sfa, "sfa", torch.float32, (M, K // 128), dev)
    _need(sfb, "sfb", torch.float32, ((N + 127) // 128, K // 128), dev)
    _need(d, "d", torch.bfloat16, (M, N), dev)
    with torch.cuda.device(dev):
        _check(_gemm_nt_noalloc(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(),
                                d.data_ptr(), M, N, K, _stream_ptr(dev)), "dg_fp8_gemm_nt_noalloc")
    return d


def m_grouped_fp8_gemm_nt_contiguous(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                                     sfb: torch.Tensor, m_indices: torch.Tensor,
                                     d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Contiguous grouped GEMM: ``D[r] = A[r] B[m_indices[r]]^T``; rows with index -1 are
    left untouched.  ``a [M_sum,K]``, ``b [G,N,K]``, ``sfb [G,ceil(N/128),K/128]``."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    M_sum, K = a.shape
    G, N, _ = b.shape
    dev = a.device
    _need(a, "a", None, (M_sum, K), dev)
    _need(b, "b", None, (G, N, K), dev)
    _need(sfa, "sfa", torch.float32, (M_sum, K // 128), dev)
    _need(sfb, "sfb", torch.float32, (G, (N + 127) // 128, K // 128), dev)
    _need(m_indices, "m_indices", torch.int32, (M_sum,), dev)
    if d is None:
        d = torch.empty((M_sum, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (M_sum, N), dev)
    with torch.cuda.device(dev):
        _check(_gemm_contig(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(),
                            d.data_ptr(), m_indices.data_ptr(), M_sum, N, K, G, _stream_ptr(dev)),
               "dg_m_grouped_fp8_gemm_nt_contiguous")
    return d


def m_grouped_fp8_gemm_nt_masked(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                                 sfb: torch.Tensor, masked_m: torch.Tensor, expected_m: int,
                                 d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Masked grouped GEMM: ``D[g, m] = A[g, m] B[g]^T`` for ``m < masked_m[g]``; other rows
    are never written.  ``a [G,max_m,K]``, ``masked_m`` int32 [G] on the device."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    G, max_m, K = a.shape
    N = b.shape[1]
    dev = a.device
    _need(a, "a", None, (G, max_m, K), dev)
    _need(b, "b", None, (G, N, K), dev)
    _need(sfa, "sfa", torch.float32, (G, max_m, K // 128), dev)
    _need(sfb, "sfb", torch.float32, (G, (N + 127) // 128, K // 128), dev)
    _need(masked_m, "masked_m", torch.int32, (G,), dev)
    if d is None:
        d = torch.empty((G, max_m, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (G, max_m, N), dev)
    with torch.cuda.device(dev):
        _check(_gemm_masked(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(),
                            d.data_ptr(), masked_m.data_ptr(), G, max_m, N, K, int(expected_m),
                            _stream_ptr(dev)), "dg_m_grouped_fp8_gemm_nt_masked")
    return d


def k_grouped_fp8_gemm_tn_contiguous(a: torch.Tensor, sfa: torch.Tensor, b: torch.Tensor,
                                     sfb: torch.Tensor, ks: torch.Tensor,
                                     c: Optional[torch.Tensor] = None,
                                     d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """K-grouped GEMM (MoE weight gradient): ``D[g] = C[g] + A_g^T B_g`` over the
    K rows of group g.  ``a [K_sum, M]`` and ``b [K_sum, N]`` E4M3 (M-/N-major,
    one row per token), ``sfa [M, K_sum/128]``, ``sfb [ceil(N/128), K_sum/128]``,
    ``ks`` int32 [G] on the device (multiples of 128 summing to K_sum), ``c`` and
    ``d`` float32 [G, M, N] (``c`` optional, may be ``d``)."""
    _fp8_bytes(a, "a"); _fp8_bytes(b, "b")
    K_sum, M = a.shape
    N = b.shape[1]
    G = ks.shape[0]
    dev = a.device
    _need(a, "a", None, (K_sum, M), dev)
    _need(b, "b", None, (K_sum, N), dev)
    _need(sfa, "sfa", torch.float32, (M, K_sum // 128), dev)
    _need(sfb, "sfb", torch.float32, ((N + 127) // 128, K_sum // 128), dev)
    _need(ks, "ks", torch.int32, (G,), dev)
    if c is not None:
        _need(c, "c", torch.float32, (G, M, N), dev)
    if d is None:
        d = torch.empty((G, M, N), dtype=torch.float32, device=dev)
    _need(d, "d", torch.float32, (G, M, N), dev)
    with torch.cuda.device(dev):
        _check(_k_grouped(a.data_ptr(), sfa.data_ptr(), b.data_ptr(), sfb.data_ptr(),
                          None if c is None else c.data_ptr(), d.data_ptr(), ks.data_ptr(), G, M,
                          N, K_sum, _stream_ptr(dev)), "dg_k_grouped_fp8_gemm_tn_contiguous")
    return d


def _bf16(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name}: expected bfloat16, got {t.dtype}")
    return t


def bf16_gemm_nt(a: torch.Tensor, b: torch.Tensor, d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Dense ``D[M,N] = A[M,K] B[N,K]^T`` on BF16 operands (K-major, K % 64 == 0),
    FP32 accumulation, BF16 output.  Runs on the current stream."""
    _bf16(a, "a"); _bf16(b, "b")
    M, K = a.shape
    N = b.shape[0]
    dev = a.device
    _need(a, "a", torch.bfloat16, (M, K), dev)
    _need(b, "b", torch.bfloat16, (N, K), dev)
    if d is None:
        d = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (M, N), dev)
    with torch.cuda.device(dev):
        _check(_bf16_gemm_nt(a.data_ptr(), b.data_ptr(), d.data_ptr(), M, N, K, _stream_ptr(dev)),
               "dg_bf16_gemm_nt")
    return d


def m_grouped_bf16_gemm_nt_contiguous(a: torch.Tensor, b: torch.Tensor, m_indices: torch.Tensor,
                                      d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Contiguous grouped GEMM on BF16 operands: ``D[r] = A[r] B[m_indices[r]]^T``;
    rows with index -1 are left untouched.  ``a [M_sum,K]``, ``b [G,N,K]``."""
    _bf16(a, "a"); _bf16(b, "b")
    M_sum, K = a.shape
    G, N, _ = b.shape
    dev = a.device
    _need(a, "a", torch.bfloat16, (M_sum, K), dev)
    _need(b, "b", torch.bfloat16, (G, N, K), dev)
    _need(m_indices, "m_indices", torch.int32, (M_sum,), dev)
    if d is None:
        d = torch.empty((M_sum, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (M_sum, N), dev)
    with torch.cuda.device(dev):
        _check(_bf16_gemm_contig(a.data_ptr(), b.data_ptr(), d.data_ptr(), m_indices.data_ptr(),
                                 M_sum, N, K, G, _stream_ptr(dev)),
               "dg_m_grouped_bf16_gemm_nt_contiguous")
    return d


def m_grouped_bf16_gemm_nt_masked(a: torch.Tensor, b: torch.Tensor, masked_m: torch.Tensor,
                                  expected_m: int, d: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Masked grouped GEMM on BF16 operands: ``D[g, m] = A[g, m] B[g]^T`` for
    ``m < masked_m[g]``; other rows are never written."""
    _bf16(a, "a"); _bf16(b, "b")
    G, max_m, K = a.shape
    N = b.shape[1]
    dev = a.device
    _need(a, "a", torch.bfloat16, (G, max_m, K), dev)
    _need(b, "b", torch.bfloat16, (G, N, K), dev)
    _need(masked_m, "masked_m", torch.int32, (G,), dev)
    if d is None:
        d = torch.empty((G, max_m, N), dtype=torch.bfloat16, device=dev)
    _need(d, "d", torch.bfloat16, (G, max_m, N), dev)
    with torch.cuda.device(dev):
        _check(_bf16_gemm_masked(a.data_ptr(), b.data_ptr(), d.data_ptr(), masked_m.data_ptr(),
                                 G, max_m, N, K, int(expected_m), _stream_ptr(dev)),
               "dg_m_grouped_bf16_gemm_nt_masked")
    return d


def set_num_sms(n: int) -> None:
    """Use at most ``n`` SMs in later calls (``n <= 0``: all of them)."""
    _check(_set_num_sms(int(n)), "dg_set_num_sms")


def get_num_sms() -> int:
    return int(_get_num_sms())


def get_last_device_error() -> int:
    """Synchronise, then read and clear the device-side error code (0: none)."""
    code = ctypes.c_int(0)
    _check(_get_last_err(ctypes.byref(code)), "dg_get_last_device_error")
    return code.value


def noalloc_get_last_device_error() -> int:
    """Synchronise, then read and clear the error word of the no-alloc entry
    point (0: none since the last read)."""
    code = ctypes.c_int(0)
    _check(_noalloc_err(ctypes.byref(code)), "dg_fp8_gemm_nt_noalloc_get_last_device_error")
    return code.value


def set_wait_timeout_ms(ms: int) -> None:
    _check(_set_timeout(int(ms)), "dg_set_wait_timeout_ms")


def set_check_scales(enable: bool) -> None:
    """Make later launches check every scale against the contract (a positive
    normal power of two; device error 0x301 otherwise)."""
    _check(_set_check_scales(1 if enable else 0), "dg_set_check_scales")


def set_weight_preload(enable: bool) -> None:
    """Let later dense launches load B (weights) before waiting on the previous
    kernel of their stream; the caller declares that no kernel that may still
    run writes B."""
    _check(_set_weight_preload(1 if enable else 0), "dg_set_weight_preload")


def set_wait_timeout_ns(ns: int) -> None:
    """Time limit of every wait inside later launches, in nanoseconds."""
    _check(_set_timeout_ns(int(ns)), "dg_set_wait_timeout_ns")


def query_config(kind: int, rows: int, N: int, K: int, G: int = 1, expected_m: int = 0,
                 num_sms: int = 148) -> dict:
    """The configuration the picker would choose (no GPU needed)."""
    c = DgConfig()
    _check(_query(int(kind), int(rows), int(N), int(K), int(G), int(expected_m), int(num_sms),
                  ctypes.byref(c)), "dg_query_config")
    return {n: getattr(c, n) for n, _ in DgConfig._fields_}


KIND_DENSE, KIND_CONTIGUOUS, KIND_MASKED, KIND_K_GROUPED = 0, 1, 2, 3
