"""CPU fp64 oracle for exact softmax attention (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline leg may import this package.  The product path (the C-ABI library and
its Python binding) never does: the two share no code.

The arithmetic lives in ``oracle.c`` (plain C, double precision, one thread per
work item); this module only builds it with gcc and marshals numpy arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

# -ffp-contract=off keeps every multiply and add separately rounded (no FMA
# contraction), so the result is the textbook fp64 evaluation order.
GCC_FLAGS = ["-O2", "-ffp-contract=off", "-fno-fast-math", "-std=c11", "-fPIC",
             "-shared", "-pthread"]


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    """Compile ``oracle.c`` into a shared library (idempotent unless ``force``)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, src, "-lm"], check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes handle on one compiled oracle library."""

    def __init__(self, so_path: str):
        lib = ctypes.CDLL(so_path)
        f = lib.oracle_attention
        f.restype = ctypes.c_int
        f.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 9 + [ctypes.c_double] + \
                     [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int] + \
                     [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_default_threads.restype = ctypes.c_int
        b = lib.oracle_attention_backward
        b.restype = ctypes.c_int
        b.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int] * 9 + [ctypes.c_double] + \
                     [ctypes.c_void_p] * 3 + [ctypes.c_int]
        self._lib = lib

    def default_threads(self) -> int:
        return int(self._lib.oracle_default_threads())

    def attention(self, q, k, v, causal: bool, scale: float, rows=None, k_range=None,
                  nthreads: int = 0, window=(-1, -1)):
        """Exact attention in fp64.

        q: uint16 [B,Nq,Hq,d] (bf16 bit patterns); k, v: uint16 [B,Nk,Hkv,d].
        rows: optional int sequence of query rows; k_range: optional (k_begin, k_end).
        window: (left, right) widths of a local window around each row's
        diagonal key i + Nk - Nq; a negative width leaves that side open.
        Returns (o [B,R,Hq,d] float64, lse [B,Hq,R] float64).
        """
        q = np.ascontiguousarray(q, dtype=np.uint16)
        k = np.ascontiguousarray(k, dtype=np.uint16)
        v = np.ascontiguousarray(v, dtype=np.uint16)
        B, Nq, Hq, d = q.shape
        Bk, Nk, Hkv, dk = k.shape
        if v.shape != k.shape or Bk != B or dk != d:
            raise ValueError("shape mismatch between q, k, v")
        if rows is None:
            rows_arr, n_rows, rows_ptr = None, Nq, None
        else:
            rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int32))
            n_rows = int(rows_arr.size)
            rows_ptr = rows_arr.ctypes.data
        kb, ke = (0, Nk) if k_range is None else (int(k_range[0]), int(k_range[1]))
        o = np.empty((B, n_rows, Hq, d), dtype=np.float64)
        lse = np.empty((B, Hq, n_rows), dtype=np.float64)
        rc = self._lib.oracle_attention(q.ctypes.data, k.ctypes.data, v.ctypes.data,
                                        B, Hq, Hkv, Nq, Nk, d, int(bool(causal)),
                                        int(window[0]), int(window[1]), float(scale),
                                        rows_ptr, n_rows, kb, ke,
                                        o.ctypes.data, lse.ctypes.data, int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_attention rejected its arguments (status {rc})")
        return o, lse


    def backward(self, q, k, v, dout, causal: bool, scale: float, window=(-1, -1),
                 nthreads: int = 0):
        """Gradients of the attention output against an upstream gradient, in fp64.

        q, dout: uint16 [B,Nq,Hq,d] (bf16 bit patterns); k, v: uint16 [B,Nk,Hkv,d].
        Returns (dq [B,Nq,Hq,d], dk [B,Nk,Hkv,d], dv [B,Nk,Hkv,d]) float64.
        """
        q, k, v, dout = (np.ascontiguousarray(t, dtype=np.uint16) for t in (q, k, v, dout))
        B, Nq, Hq, d = q.shape
        Bk, Nk, Hkv, dk_ = k.shape
        if v.shape != k.shape or dout.shape != q.shape or Bk != B or dk_ != d:
            raise ValueError("shape mismatch between q, k, v, dout")
        dq = np.empty((B, Nq, Hq, d), dtype=np.float64)
        dk = np.empty((B, Nk, Hkv, d), dtype=np.float64)
        dv = np.empty((B, Nk, Hkv, d), dtype=np.float64)
        rc = self._lib.oracle_attention_backward(
            q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data, B, Hq, Hkv, Nq, Nk, d,
            int(bool(causal)), int(window[0]), int(window[1]), float(scale), dq.ctypes.data,
            dk.ctypes.data, dv.ctypes.data, int(nthreads))
        if rc != 0:
            raise ValueError(f"oracle_attention_backward rejected its arguments (status {rc})")
        return dq, dk, dv


_default: Oracle | None = None


def _get() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def attention(q, k, v, causal: bool, scale: float, rows=None, k_range=None, nthreads: int = 0,
              window=(-1, -1)):
    """Module-level convenience over the default oracle build; see ``Oracle.attention``."""
    return _get().attention(q, k, v, causal, scale, rows=rows, k_range=k_range, nthreads=nthreads,
                            window=window)


def backward(q, k, v, dout, causal: bool, scale: float, window=(-1, -1), nthreads: int = 0):
    """Module-level convenience over the default oracle build; see ``Oracle.backward``."""
    return _get().backward(q, k, v, dout, causal, scale, window=window, nthreads=nthreads)


def default_threads() -> int:
    return _get().default_threads()
