"""ctypes binding of ``libaxis_attn.so`` (C ABI in ``include/axis_attn.h``).

The functions named like the C entry points marshal arguments only: they take
device pointers (ints) and sizes and return the C status code.  The helpers
``attention_forward`` / ``attention_backward`` take torch tensors, allocate the
outputs and the workspace with torch (device memory is PyTorch's job here) and
raise on a non-zero status.  All arithmetic runs in the library's kernels;
there is no fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libaxis_attn.so")

# The symbols include/axis_attn.h declares.
EXPORTS = (
    "axis_attn_fwd",
    "axis_attn_bwd_workspace_bytes",
    "axis_attn_bwd",
    "axis_attn_bwd_prepare",
    "axis_attn_bwd_main",
    "axis_attn_bwd_finalize",
    "axis_attn_bwd_noalloc",
    "axis_attn_bwd_det_workspace_bytes",
    "axis_attn_bwd_det",
    "axis_attn_get_status",
    "axis_attn_last_status_word",
    "axis_attn_strerror",
)

STATUS = {
    0: "AXIS_ATTN_OK",
    1: "AXIS_ATTN_ERR_NULL",
    2: "AXIS_ATTN_ERR_ALIGN",
    3: "AXIS_ATTN_ERR_SHAPE",
    4: "AXIS_ATTN_ERR_UNSUPPORTED",
    5: "AXIS_ATTN_ERR_WORKSPACE",
    6: "AXIS_ATTN_ERR_CUDA",
    7: "AXIS_ATTN_ERR_TIMEOUT",
}

_lock = threading.Lock()
_lib = None


class AxisAttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({strerror(code)})")


def library_path() -> str:
    return LIB_PATH


def load():
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m causal_attention_fwd_b200.build` (no CPU fallback exists)")
            lib = ctypes.CDLL(LIB_PATH)
            vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
            lib.axis_attn_fwd.argtypes = [vp] * 5 + [i] * 5 + [f, i, vp]
            lib.axis_attn_fwd.restype = i
            lib.axis_attn_bwd_workspace_bytes.argtypes = [i] * 5
            lib.axis_attn_bwd_workspace_bytes.restype = sz
            lib.axis_attn_bwd.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp, sz, vp]
            lib.axis_attn_bwd.restype = i
            lib.axis_attn_bwd_prepare.argtypes = [vp] * 3 + [i] * 5 + [vp, sz, vp]
            lib.axis_attn_bwd_prepare.restype = i
            lib.axis_attn_bwd_main.argtypes = [vp] * 6 + [i] * 5 + [f, i, vp, sz, vp]
            lib.axis_attn_bwd_main.restype = i
            lib.axis_attn_bwd_finalize.argtypes = [vp] + [i] * 5 + [vp, sz, vp]
            lib.axis_attn_bwd_finalize.restype = i
            lib.axis_attn_bwd_noalloc.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp]
            lib.axis_attn_bwd_noalloc.restype = i
            lib.axis_attn_bwd_det_workspace_bytes.argtypes = [i] * 5
            lib.axis_attn_bwd_det_workspace_bytes.restype = sz
            lib.axis_attn_bwd_det.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp, sz, vp]
            lib.axis_attn_bwd_det.restype = i
            lib.axis_attn_get_status.argtypes = [vp]
            lib.axis_attn_get_status.restype = i
            lib.axis_attn_last_status_word.argtypes = []
            lib.axis_attn_last_status_word.restype = ctypes.c_uint
            lib.axis_attn_strerror.argtypes = [i]
            lib.axis_attn_strerror.restype = ctypes.c_char_p
            _lib = lib
    return _lib


# ------------------------------------------------------------------ raw C ABI
def axis_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, scale, causal, stream) -> int:
    return load().axis_attn_fwd(q, k, v, o, lse, B, Hq, Hkv, S, D, scale, causal, stream)


def axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D) -> int:
    return int(load().axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D))


def axis_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                  workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                                workspace, workspace_bytes, stream)


def axis_attn_bwd_prepare(o, dO, lse, B, Hq, Hkv, S, D, workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd_prepare(o, dO, lse, B, Hq, Hkv, S, D, workspace, workspace_bytes, stream)


def axis_attn_bwd_main(q, k, v, dO, dk, dv, B, Hq, Hkv, S, D, scale, causal, workspace,
                       workspace_bytes, stream) -> int:
    return load().axis_attn_bwd_main(q, k, v, dO, dk, dv, B, Hq, Hkv, S, D, scale, causal, workspace,
                                     workspace_bytes, stream)


def axis_attn_bwd_finalize(dq, B, Hq, Hkv, S, D, workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd_finalize(dq, B, Hq, Hkv, S, D, workspace, workspace_bytes, stream)


def axis_attn_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                          stream) -> int:
    """Backward with the library's built-in 32 MiB scratch instead of a workspace,
    for callers that cannot allocate device memory (see include/axis_attn.h)."""
    return load().axis_attn_bwd_noalloc(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                                        stream)


def axis_attn_bwd_det_workspace_bytes(B, Hq, Hkv, S, D) -> int:
    return int(load().axis_attn_bwd_det_workspace_bytes(B, Hq, Hkv, S, D))


def axis_attn_bwd_det(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                      workspace, workspace_bytes, stream) -> int:
    """Backward whose results are bitwise reproducible run to run (dQ summed over
    the key tiles in a fixed order; see include/axis_attn.h)."""
    return load().axis_attn_bwd_det(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                                    workspace, workspace_bytes, stream)


def axis_attn_get_status(stream) -> int:
    return load().axis_attn_get_status(stream)


def axis_attn_last_status_word() -> int:
    return int(load().axis_attn_last_status_word())


def axis_attn_strerror(code: int) -> str:
    return load().axis_attn_strerror(code).decode()


def strerror(code: int) -> str:
    try:
        return axis_attn_strerror(code)
    except Exception:  # library not loadable: still produce a message
        return STATUS.get(code, "unknown")


# ------------------------------------------------------------ torch helpers
def _dims(q, k):
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    return B, Hq, Hkv, S, D


def _stream(stream):
    import torch

    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def attention_forward(q, k, v, causal: bool = True, scale: float | None = None, out=None,
                      lse=None, stream=None):
    """O, LSE for bf16 CUDA tensors q [B,S,Hq,D], k/v [B,S,Hkv,D]."""
    import torch

    B, Hq, Hkv, S, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    o = torch.empty_like(q) if out is None else out
    l = torch.empty((B, Hq, S), device=q.device, dtype=torch.float32) if lse is None else lse
    rc = axis_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                       B, Hq, Hkv, S, D, scale, int(causal), _stream(stream))
    if rc:
        raise AxisAttnError(rc, "axis_attn_fwd")
    return o, l


def attention_backward(q, k, v, o, lse, dout, causal: bool = True, scale: float | None = None,
                       workspace=None, grads=None, stream=None, deterministic: bool = False):
    """dQ, dK, dV (bf16) of sum(dO * O).  deterministic=True: axis_attn_bwd_det
    (bitwise reproducible, larger workspace)."""
    import torch

    B, Hq, Hkv, S, D = _dims(q, k)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    size_fn, call, name = ((axis_attn_bwd_det_workspace_bytes, axis_attn_bwd_det, "axis_attn_bwd_det")
                           if deterministic else
                           (axis_attn_bwd_workspace_bytes, axis_attn_bwd, "axis_attn_bwd"))
    need = size_fn(B, Hq, Hkv, S, D)
    if workspace is None:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k),
                                                  torch.empty_like(v))
    rc = call(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
              lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
              B, Hq, Hkv, S, D, scale, int(causal), workspace.data_ptr(),
              workspace.numel() * workspace.element_size(), _stream(stream))
    if rc:
        raise AxisAttnError(rc, name)
    return dq, dk, dv


def check_status(stream=None):
    """Synchronise and raise if a kernel reported a timed-out device wait."""
    rc = axis_attn_get_status(_stream(stream))
    if rc:
        w = axis_attn_last_status_word()
        raise AxisAttnError(rc, f"axis_attn_get_status (status word {w:#x}, wait site {(w >> 8) & 0xff})")
