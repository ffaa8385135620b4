"""CPU oracle for the FP8 block-scaled GEMM (dense, contiguous grouped, masked
grouped) and for the same three forms with BF16 operands: a plain, slow,
obviously correct restatement of what the method computes, in double
precision, rounded once to BF16.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares nothing with
the CUDA library in ``moe_grouped_gemm_09_b200/`` and never imports it.

The arithmetic is in ``dg_oracle.c`` (see its header for the passages of the
DeepGEMM pages each step follows); this module compiles it with gcc on first use
and wraps it with ctypes.  Every function here takes numpy arrays and returns
numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "dg_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(lib_path: str = _LIB_PATH, extra_flags: tuple = ()) -> str:
    """Compile the oracle with gcc (OpenMP) into ``lib_path``."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", *extra_flags,
           _SRC, "-o", lib_path, "-lm"]
    subprocess.run(cmd, check=True)
    return lib_path


def _needs_build(lib_path: str) -> bool:
    return (not os.path.exists(lib_path)
            or os.path.getmtime(lib_path) < os.path.getmtime(_SRC))


def load(lib_path: str = _LIB_PATH):
    """Load (building if missing or stale) and declare the oracle library."""
    if lib_path == _LIB_PATH and _needs_build(lib_path):
        build(lib_path)
    lib = ctypes.CDLL(lib_path)
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_table.restype = None
    lib.oracle_e4m3_table.argtypes = [P]
    lib.oracle_bf16_from_double.restype = ctypes.c_uint16
    lib.oracle_bf16_from_double.argtypes = [ctypes.c_double]
    lib.oracle_gemm_nt.restype = ctypes.c_int
    lib.oracle_gemm_nt.argtypes = [P, P, P, P, I64, I64, I64, P, P]
    lib.oracle_grouped_contiguous.restype = ctypes.c_int
    lib.oracle_grouped_contiguous.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, P]
    lib.oracle_grouped_masked.restype = ctypes.c_int
    lib.oracle_grouped_masked.argtypes = [P, P, P, P, P, I64, I64, I64, I64, P, P]
    lib.oracle_k_grouped_tn.restype = ctypes.c_int
    lib.oracle_k_grouped_tn.argtypes = [P, P, P, P, P, P, I64, I64, I64, I64, P]
    lib.oracle_bf16_decode.restype = ctypes.c_double
    lib.oracle_bf16_decode.argtypes = [ctypes.c_uint16]
    lib.oracle_bf16_gemm_nt.restype = ctypes.c_int
    lib.oracle_bf16_gemm_nt.argtypes = [P, P, I64, I64, I64, P, P]
    lib.oracle_bf16_grouped_contiguous.restype = ctypes.c_int
    lib.oracle_bf16_grouped_contiguous.argtypes = [P, P, P, I64, I64, I64, I64, P, P]
    lib.oracle_bf16_grouped_masked.restype = ctypes.c_int
    lib.oracle_bf16_grouped_masked.argtypes = [P, P, P, I64, I64, I64, I64, P, P]
    lib.oracle_num_threads.restype = ctypes.c_int
    lib.oracle_num_threads.argtypes = []
    lib.oracle_set_num_threads.restype = None
    lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
    return lib


def _get():
    global _lib
    with _lock:
        if _lib is None:
            _lib = load()
    return _lib


def _ptr(x: np.ndarray | None):
    return None if x is None else x.ctypes.data


def _c(x: np.ndarray, dtype) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=dtype)


class Oracle:
    """The oracle's functions bound to one compiled library (the default one, or
    another build of the same source, e.g. with different compiler flags)."""

    def __init__(self, lib=None):
        self.lib = lib if lib is not None else _get()

    # -- element-level definitions --
    def e4m3_table(self) -> np.ndarray:
        t = np.empty(256, np.float64)
        self.lib.oracle_e4m3_table(_ptr(t))
        return t

    def bf16_from_double(self, x: float) -> int:
        return int(self.lib.oracle_bf16_from_double(float(x)))

    # -- GEMMs --
    def gemm_nt(self, a, sfa, b, sfb, want_acc: bool = True):
        """Dense D = A B^T.  Returns ``(d uint16 [M,N] BF16 bits, acc float64 [M,N] or None)``."""
        a = _c(a, np.uint8); b = _c(b, np.uint8)
        sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32)
        M, K = a.shape
        N = b.shape[0]
        assert b.shape[1] == K and sfa.shape == (M, K // 128)
        assert sfb.shape == (-(-N // 128), K // 128)
        d = np.empty((M, N), np.uint16)
        acc = np.empty((M, N), np.float64) if want_acc else None
        rc = self.lib.oracle_gemm_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), M, N, K,
                                     _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_gemm_nt: bad arguments (rc={rc})")
        return d, acc

    def grouped_contiguous(self, a, sfa, b, sfb, m_indices, d=None, acc=None):
        """Contiguous grouped GEMM.  ``d``/``acc`` (optional) are updated in
        place on valid rows only; padding rows keep what they held."""
        a = _c(a, np.uint8); b = _c(b, np.uint8)
        sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32)
        m_indices = _c(m_indices, np.int32)
        M_sum, K = a.shape
        G, N, _ = b.shape
        assert sfb.shape == (G, -(-N // 128), K // 128) and m_indices.shape == (M_sum,)
        if d is None:
            d = np.zeros((M_sum, N), np.uint16)
        assert d.dtype == np.uint16 and d.shape == (M_sum, N) and d.flags.c_contiguous
        if acc is not None:
            assert acc.dtype == np.float64 and acc.shape == (M_sum, N) and acc.flags.c_contiguous
        rc = self.lib.oracle_grouped_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb),
                                                _ptr(m_indices), M_sum, N, K, G,
                                                _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_grouped_contiguous: bad arguments (rc={rc})")
        return d, acc

    def grouped_masked(self, a, sfa, b, sfb, masked_m, d=None, acc=None):
        """Masked grouped GEMM.  ``d``/``acc`` (optional) are updated in place on
        rows ``m < masked_m[g]`` only."""
        a = _c(a, np.uint8); b = _c(b, np.uint8)
        sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32)
        masked_m = _c(masked_m, np.int32)
        G, max_m, K = a.shape
        N = b.shape[1]
        assert b.shape == (G, N, K) and sfa.shape == (G, max_m, K // 128)
        assert sfb.shape == (G, -(-N // 128), K // 128) and masked_m.shape == (G,)
        if d is None:
            d = np.zeros((G, max_m, N), np.uint16)
        assert d.dtype == np.uint16 and d.shape == (G, max_m, N) and d.flags.c_contiguous
        if acc is not None:
            assert acc.dtype == np.float64 and acc.shape == (G, max_m, N)
        rc = self.lib.oracle_grouped_masked(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb),
                                            _ptr(masked_m), G, max_m, N, K,
                                            _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_grouped_masked: bad arguments (rc={rc})")
        return d, acc

    # -- BF16 operands (no scales) --
    def k_grouped_tn(self, a, sfa, b, sfb, ks, c=None):
        """K-grouped GEMM (weight gradient): ``acc[g] = C[g] + A_g^T B_g`` over
        the K rows of group g.  ``a [K_sum, M]`` and ``b [K_sum, N]`` E4M3 bytes
        (M-/N-major), ``sfa [M, K_sum/128]``, ``sfb [ceil(N/128), K_sum/128]``,
        ``ks`` int32 [G] (multiples of 128 summing to K_sum), ``c`` float32
        [G, M, N] or None.  Returns ``acc`` float64 [G, M, N]."""
        a = _c(a, np.uint8); b = _c(b, np.uint8)
        sfa = _c(sfa, np.float32); sfb = _c(sfb, np.float32)
        ks = _c(ks, np.int32)
        K_sum, M = a.shape
        N = b.shape[1]
        G = ks.shape[0]
        assert b.shape[0] == K_sum and sfa.shape == (M, K_sum // 128)
        assert sfb.shape == (-(-N // 128), K_sum // 128)
        if c is not None:
            c = _c(c, np.float32)
            assert c.shape == (G, M, N)
        acc = np.empty((G, M, N), np.float64)
        rc = self.lib.oracle_k_grouped_tn(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(ks),
                                          _ptr(c), G, M, N, K_sum, _ptr(acc))
        if rc != 0:
            raise ValueError(f"oracle_k_grouped_tn: bad arguments (rc={rc})")
        return acc

    def bf16_decode(self, bits: int) -> float:
        return float(self.lib.oracle_bf16_decode(int(bits)))

    def bf16_gemm_nt(self, a, b, want_acc: bool = True):
        """Dense D = A B^T with BF16 operands given as uint16 bit patterns.
        Returns ``(d uint16 [M,N], acc float64 [M,N] or None)``."""
        a = _c(a, np.uint16); b = _c(b, np.uint16)
        M, K = a.shape
        N = b.shape[0]
        assert b.shape[1] == K
        d = np.empty((M, N), np.uint16)
        acc = np.empty((M, N), np.float64) if want_acc else None
        rc = self.lib.oracle_bf16_gemm_nt(_ptr(a), _ptr(b), M, N, K, _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_bf16_gemm_nt: failed (rc={rc})")
        return d, acc

    def bf16_grouped_contiguous(self, a, b, m_indices, d=None, acc=None):
        """Contiguous grouped GEMM with BF16 operands; ``d``/``acc`` are
        updated in place on valid rows only."""
        a = _c(a, np.uint16); b = _c(b, np.uint16)
        m_indices = _c(m_indices, np.int32)
        M_sum, K = a.shape
        G, N, _ = b.shape
        assert b.shape[2] == K and m_indices.shape == (M_sum,)
        if d is None:
            d = np.zeros((M_sum, N), np.uint16)
        assert d.dtype == np.uint16 and d.shape == (M_sum, N) and d.flags.c_contiguous
        if acc is not None:
            assert acc.dtype == np.float64 and acc.shape == (M_sum, N) and acc.flags.c_contiguous
        rc = self.lib.oracle_bf16_grouped_contiguous(_ptr(a), _ptr(b), _ptr(m_indices),
                                                     M_sum, N, K, G, _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_bf16_grouped_contiguous: failed (rc={rc})")
        return d, acc

    def bf16_grouped_masked(self, a, b, masked_m, d=None, acc=None):
        """Masked grouped GEMM with BF16 operands; ``d``/``acc`` are updated in
        place on rows ``m < masked_m[g]`` only."""
        a = _c(a, np.uint16); b = _c(b, np.uint16)
        masked_m = _c(masked_m, np.int32)
        G, max_m, K = a.shape
        N = b.shape[1]
        assert b.shape == (G, N, K) and masked_m.shape == (G,)
        if d is None:
            d = np.zeros((G, max_m, N), np.uint16)
        assert d.dtype == np.uint16 and d.shape == (G, max_m, N) and d.flags.c_contiguous
        if acc is not None:
            assert acc.dtype == np.float64 and acc.shape == (G, max_m, N)
        rc = self.lib.oracle_bf16_grouped_masked(_ptr(a), _ptr(b), _ptr(masked_m),
                                                 G, max_m, N, K, _ptr(acc), _ptr(d))
        if rc != 0:
            raise ValueError(f"oracle_bf16_grouped_masked: failed (rc={rc})")
        return d, acc

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    def set_num_threads(self, n: int) -> None:
        self.lib.oracle_set_num_threads(int(n))


def default() -> Oracle:
    return Oracle()


def bf16_bits_to_float(bits: np.ndarray) -> np.ndarray:
    """Reinterpret BF16 bit patterns as float32 values (exact widening)."""
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)
