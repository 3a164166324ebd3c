"""Python front end of the fp64 CPU attention oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the CPU-baseline leg of
the benchmark use it; the library under test never does.  It imports nothing
from the CUDA package and the CUDA package imports nothing from here.

The C source defines the operation (textbook masked softmax attention with GQA
head sharing, forward and analytic backward; see its header for the passages of
the pages it follows).  This module only builds it with gcc/OpenMP, marshals
float64 numpy arrays in and out, and converts (b, h, i) row samples.

All arrays are float64, C-contiguous, in the [B, S, H, D] layout; LSE and the
row sums Dr are [B, Hq, S].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "libattn_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libattn_oracle.so`` (gcc, -O2, OpenMP).

    No fast-math: the oracle keeps IEEE double semantics."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _f64(a) -> np.ndarray:
    """float64 C-contiguous copy/view of a numpy array or CPU torch tensor."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu")
        import torch  # only for the dtype conversion of torch inputs

        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(_dp)


def _dims(q, k, causal, scale):
    B, S, Hq, D = q.shape
    Bk, Sk, Hkv, Dk = k.shape
    if (B, S, D) != (Bk, Sk, Dk) or Hq % Hkv:
        raise ValueError(f"incompatible shapes q{q.shape} k{k.shape}")
    return (B, Hq, Hkv, S, D, float(scale), int(bool(causal)))


def _rows(rows) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1, 3))


class Oracle:
    """The oracle's entry points bound to one compiled library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        i, d = ctypes.c_int, ctypes.c_double
        dims = [i, i, i, i, i, d, i]
        lib.oracle_attn_fwd.argtypes = [_dp] * 5 + dims
        lib.oracle_attn_fwd_rows.argtypes = [_dp] * 3 + dims + [i, _ip, _dp, _dp]
        lib.oracle_attn_probs_row.argtypes = [_dp] * 2 + dims + [i, i, i, _dp]
        lib.oracle_attn_bwd.argtypes = [_dp] * 8 + dims
        lib.oracle_attn_bwd_dq_rows.argtypes = [_dp] * 4 + dims + [i, _ip, _dp, _dp]
        lib.oracle_attn_bwd_dkdv_rows.argtypes = [_dp] * 4 + dims + [i, _ip, _dp, _dp]
        lib.oracle_rope.argtypes = [_dp, i, i, i, i, d, i]
        lib.oracle_attn_decode.argtypes = [_dp] * 3 + [_ip] + [_dp] * 2 + [i] * 5 + [d]
        lib.oracle_attn_decode_q.argtypes = [_dp] * 3 + [_ip] + [_dp] * 2 + [i] * 6 + [d]
        for f in ("oracle_attn_fwd", "oracle_attn_fwd_rows", "oracle_attn_probs_row",
                  "oracle_attn_bwd", "oracle_attn_bwd_dq_rows", "oracle_attn_bwd_dkdv_rows",
                  "oracle_rope", "oracle_attn_decode", "oracle_attn_decode_q", "oracle_max_threads"):
            getattr(lib, f).restype = ctypes.c_int
        self.lib = lib

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def rope(self, x, base: float = 10000.0, inverse: bool = False):
        """Rotary position embedding of x [B, S, H, D] (a rotated float64 copy);
        inverse=True applies the transposed rotation (for gradients)."""
        y = _f64(x).copy()
        B, S, H, D = y.shape
        if self.lib.oracle_rope(_ptr(y), B, S, H, D, float(base), int(bool(inverse))):
            raise ValueError("oracle_rope rejected the arguments")
        return y

    def attn_decode(self, q, k, v, lens, scale: float):
        """Decode step: q [B, Hq, D] (one new row per sequence), cache k, v
        [B, Smax, Hkv, D] of which sequence b uses its first lens[b] rows.
        Returns (O [B, Hq, D], LSE [B, Hq]), float64."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, Hq, D = q.shape
        Bk, Smax, Hkv, Dk = k.shape
        if (B, D) != (Bk, Dk) or v.shape != k.shape:
            raise ValueError(f"incompatible shapes q{q.shape} k{k.shape} v{v.shape}")
        ln = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1))
        o = np.empty((B, Hq, D))
        lse = np.empty((B, Hq))
        rc = self.lib.oracle_attn_decode(_ptr(q), _ptr(k), _ptr(v), ln.ctypes.data_as(_ip), _ptr(o), _ptr(lse),
                                         B, Hq, Hkv, Smax, D, float(scale))
        if rc:
            raise ValueError("oracle_attn_decode rejected the arguments")
        return o, lse

    def attn_decode_q(self, q, k, v, lens, scale: float):
        """Decode step with several new tokens per sequence: q [B, q_len, Hq, D]
        (the last q_len positions of each sequence), cache k, v [B, Smax, Hkv,
        D] of which sequence b uses its first lens[b] rows (the new tokens'
        included).  Returns (O [B, q_len, Hq, D], LSE [B, Hq, q_len]), float64."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, q_len, Hq, D = q.shape
        Bk, Smax, Hkv, Dk = k.shape
        if (B, D) != (Bk, Dk) or v.shape != k.shape:
            raise ValueError(f"incompatible shapes q{q.shape} k{k.shape} v{v.shape}")
        ln = np.ascontiguousarray(np.asarray(lens, dtype=np.int32).reshape(-1))
        o = np.empty((B, q_len, Hq, D))
        lse = np.empty((B, Hq, q_len))
        rc = self.lib.oracle_attn_decode_q(_ptr(q), _ptr(k), _ptr(v), ln.ctypes.data_as(_ip), _ptr(o), _ptr(lse),
                                           B, q_len, Hq, Hkv, Smax, D, float(scale))
        if rc:
            raise ValueError("oracle_attn_decode_q rejected the arguments")
        return o, lse

    def attn_fwd(self, q, k, v, scale: float, causal: bool = True):
        """Full forward.  Returns (O [B,S,Hq,D], LSE [B,Hq,S]), float64."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        dims = _dims(q, k, causal, scale)
        B, Hq, _, S, D = dims[:5]
        o = np.empty((B, S, Hq, D))
        lse = np.empty((B, Hq, S))
        rc = self.lib.oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), *dims)
        if rc:
            raise ValueError("oracle_attn_fwd rejected the dimensions")
        return o, lse

    def attn_bwd(self, q, k, v, dout, scale: float, causal: bool = True):
        """Full backward.  Returns (dQ, dK, dV, Dr) with Dr = rowsum(dO*O) [B,Hq,S]."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        dims = _dims(q, k, causal, scale)
        dq, dk, dv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
        B, Hq, _, S, _ = dims[:5]
        dr = np.empty((B, Hq, S))
        rc = self.lib.oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(dq),
                                      _ptr(dk), _ptr(dv), _ptr(dr), *dims)
        if rc:
            raise ValueError("oracle_attn_bwd rejected the dimensions")
        return dq, dk, dv, dr

    def attn_fwd_rows(self, q, k, v, scale: float, causal: bool, rows):
        """O and LSE of selected query rows; rows = iterable of (b, h, i)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        dims = _dims(q, k, causal, scale)
        r = _rows(rows)
        n, D = r.shape[0], dims[4]
        o = np.empty((n, D))
        lse = np.empty((n,))
        rc = self.lib.oracle_attn_fwd_rows(_ptr(q), _ptr(k), _ptr(v), *dims, n,
                                          r.ctypes.data_as(_ip), _ptr(o), _ptr(lse))
        if rc:
            raise ValueError("oracle_attn_fwd_rows rejected the dimensions")
        return o, lse

    def probs_row(self, q, k, scale: float, causal: bool, b: int, h: int, i: int):
        """The probability row P[b, h, i, :] (length S)."""
        q, k = _f64(q), _f64(k)
        dims = _dims(q, k, causal, scale)
        p = np.empty((dims[3],))
        rc = self.lib.oracle_attn_probs_row(_ptr(q), _ptr(k), *dims, int(b), int(h), int(i), _ptr(p))
        if rc:
            raise ValueError("oracle_attn_probs_row rejected the dimensions")
        return p

    def attn_bwd_dq_rows(self, q, k, v, dout, scale: float, causal: bool, rows):
        """dQ (and Dr) of selected query rows; rows = iterable of (b, h, i)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        dims = _dims(q, k, causal, scale)
        r = _rows(rows)
        n, D = r.shape[0], dims[4]
        dq = np.empty((n, D))
        dr = np.empty((n,))
        rc = self.lib.oracle_attn_bwd_dq_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), *dims, n,
                                             r.ctypes.data_as(_ip), _ptr(dq), _ptr(dr))
        if rc:
            raise ValueError("oracle_attn_bwd_dq_rows rejected the dimensions")
        return dq, dr

    def attn_bwd_dkdv_rows(self, q, k, v, dout, scale: float, causal: bool, rows):
        """dK and dV of selected key rows; rows = iterable of (b, kv, j)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        dims = _dims(q, k, causal, scale)
        r = _rows(rows)
        n, D = r.shape[0], dims[4]
        dk = np.empty((n, D))
        dv = np.empty((n, D))
        rc = self.lib.oracle_attn_bwd_dkdv_rows(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), *dims, n,
                                               r.ctypes.data_as(_ip), _ptr(dk), _ptr(dv))
        if rc:
            raise ValueError("oracle_attn_bwd_dkdv_rows rejected the dimensions")
        return dk, dv


def default() -> Oracle:
    """The oracle built from ``attn_oracle.c`` in this directory."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def _forward(name):
    def f(*a, **kw):
        return getattr(default(), name)(*a, **kw)

    f.__name__ = name
    f.__doc__ = getattr(Oracle, name).__doc__
    return f


max_threads = _forward("max_threads")
attn_fwd = _forward("attn_fwd")
attn_bwd = _forward("attn_bwd")
attn_fwd_rows = _forward("attn_fwd_rows")
probs_row = _forward("probs_row")
attn_bwd_dq_rows = _forward("attn_bwd_dq_rows")
attn_bwd_dkdv_rows = _forward("attn_bwd_dkdv_rows")
rope = _forward("rope")
attn_decode = _forward("attn_decode")
attn_decode_q = _forward("attn_decode_q")
