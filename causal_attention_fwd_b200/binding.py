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
    "axis_attn_bwd_head_split",
    "axis_attn_bwd",
    "axis_attn_bwd_prepare",
    "axis_attn_bwd_main",
    "axis_attn_bwd_finalize",
    "axis_attn_bwd_noalloc",
    "axis_attn_bwd_det_workspace_bytes",
    "axis_attn_bwd_det",
    "axis_attn_rope_table",
    "axis_attn_rope",
    "axis_attn_fwd_rope",
    "axis_attn_bwd_rope",
    "axis_attn_decode_workspace_bytes",
    "axis_attn_decode",
    "axis_attn_decode_hnd",
    "axis_attn_decode_q",
    "axis_attn_decode_q_workspace_bytes",
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
    8: "AXIS_ATTN_ERR_INDEX",
}

_lock = threading.Lock()
_lib = None


class AxisAttnError(RuntimeError):
    def __init__(self, code: int, where: str, detail: str | None = None):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({detail or strerror(code)})")


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
            lib.axis_attn_bwd_head_split.argtypes = [i] * 5
            lib.axis_attn_bwd_head_split.restype = i
            lib.axis_attn_bwd.argtypes = [vp] * 9 + [i] * 5 + [f, i, vp, sz, vp]
            lib.axis_attn_bwd.restype = i
            lib.axis_attn_bwd_prepare.argtypes = [vp] * 3 + [i] * 5 + [f, vp, sz, vp]
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
            lib.axis_attn_rope_table.argtypes = [vp, i, i, ctypes.c_double, vp]
            lib.axis_attn_rope_table.restype = i
            lib.axis_attn_rope.argtypes = [vp] * 3 + [i] * 5 + [vp]
            lib.axis_attn_rope.restype = i
            lib.axis_attn_fwd_rope.argtypes = [vp] * 8 + [i] * 5 + [f, i, vp]
            lib.axis_attn_fwd_rope.restype = i
            lib.axis_attn_bwd_rope.argtypes = [vp] * 10 + [i] * 5 + [f, i, i, vp, sz, vp]
            lib.axis_attn_bwd_rope.restype = i
            lib.axis_attn_decode_workspace_bytes.argtypes = [i] * 6
            lib.axis_attn_decode_workspace_bytes.restype = sz
            lib.axis_attn_decode.argtypes = [vp] * 7 + [i] * 7 + [f, vp, sz, vp]
            lib.axis_attn_decode.restype = i
            lib.axis_attn_decode_hnd.argtypes = [vp] * 7 + [i] * 7 + [f, vp, sz, vp]
            lib.axis_attn_decode_hnd.restype = i
            lib.axis_attn_decode_q.argtypes = [vp] * 7 + [i] * 8 + [f, i, vp, sz, vp]
            lib.axis_attn_decode_q.restype = i
            lib.axis_attn_decode_q_workspace_bytes.argtypes = [i] * 7
            lib.axis_attn_decode_q_workspace_bytes.restype = sz
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


def axis_attn_bwd_head_split(B, Hq, Hkv, S, D) -> int:
    return int(load().axis_attn_bwd_head_split(B, Hq, Hkv, S, D))


def axis_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                  workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd(q, k, v, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                                workspace, workspace_bytes, stream)


def axis_attn_bwd_prepare(o, dO, lse, B, Hq, Hkv, S, D, scale, workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd_prepare(o, dO, lse, B, Hq, Hkv, S, D, scale, workspace, workspace_bytes, stream)


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


def axis_attn_rope_table(cs, S, D, base, stream) -> int:
    return load().axis_attn_rope_table(cs, S, D, base, stream)


def axis_attn_rope(x, y, cs, B, S, H, D, inverse, stream) -> int:
    return load().axis_attn_rope(x, y, cs, B, S, H, D, inverse, stream)


def axis_attn_fwd_rope(q, k, v, cs, o, lse, q_rot, k_rot, B, Hq, Hkv, S, D, scale, causal, stream) -> int:
    return load().axis_attn_fwd_rope(q, k, v, cs, o, lse, q_rot, k_rot, B, Hq, Hkv, S, D, scale, causal, stream)


def axis_attn_bwd_rope(q_rot, k_rot, v, cs, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal, deterministic,
                       workspace, workspace_bytes, stream) -> int:
    return load().axis_attn_bwd_rope(q_rot, k_rot, v, cs, o, dO, lse, dq, dk, dv, B, Hq, Hkv, S, D, scale, causal,
                                     deterministic, workspace, workspace_bytes, stream)


def axis_attn_decode_workspace_bytes(B, Hq, Hkv, D, page_size, max_pages) -> int:
    return int(load().axis_attn_decode_workspace_bytes(B, Hq, Hkv, D, page_size, max_pages))


def axis_attn_decode(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size, max_pages,
                     num_pages, scale, workspace, workspace_bytes, stream) -> int:
    """Decode step against a paged KV cache (see include/axis_attn.h)."""
    return load().axis_attn_decode(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                                   max_pages, num_pages, scale, workspace, workspace_bytes, stream)


def axis_attn_decode_hnd(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size, max_pages,
                         num_pages, scale, workspace, workspace_bytes, stream) -> int:
    """Decode step against a head-major paged KV cache (see include/axis_attn.h)."""
    return load().axis_attn_decode_hnd(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, Hq, Hkv, D, page_size,
                                       max_pages, num_pages, scale, workspace, workspace_bytes, stream)


def axis_attn_decode_q_workspace_bytes(B, q_len, Hq, Hkv, D, page_size, max_pages) -> int:
    return int(load().axis_attn_decode_q_workspace_bytes(B, q_len, Hq, Hkv, D, page_size, max_pages))


def axis_attn_decode_q(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, q_len, Hq, Hkv, D, page_size,
                       max_pages, num_pages, scale, head_major, workspace, workspace_bytes, stream) -> int:
    """Decode step with q_len new tokens per sequence (see include/axis_attn.h)."""
    return load().axis_attn_decode_q(q, k_cache, v_cache, block_table, seq_lens, o, lse, B, q_len, Hq, Hkv, D,
                                     page_size, max_pages, num_pages, scale, head_major, workspace, workspace_bytes,
                                     stream)


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
ERR_SHAPE, ERR_UNSUPPORTED = 3, 4


def _require(cond: bool, code: int, where: str, detail: str):
    if not cond:
        raise AxisAttnError(code, where, detail)


def _check_tensor(t, name: str, shape, dtype, where: str):
    """Shape, then dtype, then layout: everything the C ABI cannot see."""
    import torch

    _require(isinstance(t, torch.Tensor), ERR_SHAPE, where, f"{name} must be a torch.Tensor")
    _require(tuple(t.shape) == tuple(shape), ERR_SHAPE, where,
             f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    _require(t.dtype == dtype, ERR_UNSUPPORTED, where, f"{name} is {t.dtype}, expected {dtype}")
    _require(t.is_contiguous(), ERR_SHAPE, where, f"{name} must be contiguous (row-major)")


def _check_device(tensors: dict, where: str):
    import torch

    devs = {n: t.device for n, t in tensors.items()}
    first = next(iter(devs.values()))
    _require(first.type == "cuda", ERR_UNSUPPORTED, where, f"tensors must be on a CUDA device, got {first}")
    bad = [n for n, d in devs.items() if d != first]
    _require(not bad, ERR_SHAPE, where, f"{', '.join(bad)} not on {first}")
    return torch.device(first)


def _dims(q, k, v, where: str):
    import torch

    _require(isinstance(q, torch.Tensor) and q.dim() == 4, ERR_SHAPE, where, "q must be a 4-D tensor [B, S, Hq, D]")
    _require(isinstance(k, torch.Tensor) and k.dim() == 4, ERR_SHAPE, where, "k must be a 4-D tensor [B, S, Hkv, D]")
    B, S, Hq, D = q.shape
    Hkv = k.shape[2]
    _require(Hkv >= 1 and Hq % Hkv == 0, ERR_SHAPE, where, f"Hq = {Hq} is not a multiple of Hkv = {Hkv}")
    for name, t in (("q", q), ("k", k), ("v", v)):
        _check_tensor(t, name, (B, S, Hq if name == "q" else Hkv, D), torch.bfloat16, where)
    return B, Hq, Hkv, S, D


def _stream(stream, device=None):
    """The caller's stream, else the current stream of `device` (the tensors'
    device; the current device if None)."""
    import torch

    s = torch.cuda.current_stream(device) if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def attention_forward(q, k, v, causal: bool = True, scale: float | None = None, out=None,
                      lse=None, stream=None):
    """O, LSE for bf16 CUDA tensors q [B,S,Hq,D], k/v [B,S,Hkv,D] (contiguous,
    one device).  Raises AxisAttnError before any launch on a wrong dtype,
    shape, layout or device."""
    import torch

    where = "attention_forward"
    B, Hq, Hkv, S, D = _dims(q, k, v, where)
    if out is not None:
        _check_tensor(out, "out", (B, S, Hq, D), torch.bfloat16, where)
    if lse is not None:
        _check_tensor(lse, "lse", (B, Hq, S), torch.float32, where)
    dev = _check_device({n: t for n, t in (("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse))
                         if t is not None}, where)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    with torch.cuda.device(dev):
        o = torch.empty_like(q) if out is None else out
        l = torch.empty((B, Hq, S), device=dev, dtype=torch.float32) if lse is None else lse
        rc = axis_attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), l.data_ptr(),
                           B, Hq, Hkv, S, D, scale, int(causal), _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, "axis_attn_fwd")
    return o, l


def attention_backward(q, k, v, o, lse, dout, causal: bool = True, scale: float | None = None,
                       workspace=None, grads=None, stream=None, deterministic: bool = False):
    """dQ, dK, dV (bf16) of sum(dO * O).  deterministic=True: axis_attn_bwd_det
    (bitwise reproducible, larger workspace).  Every tensor is checked (dtype,
    shape, contiguity, one CUDA device) before any launch."""
    import torch

    where = "attention_backward"
    B, Hq, Hkv, S, D = _dims(q, k, v, where)
    _check_tensor(o, "o", (B, S, Hq, D), torch.bfloat16, where)
    _check_tensor(dout, "dout", (B, S, Hq, D), torch.bfloat16, where)
    _check_tensor(lse, "lse", (B, Hq, S), torch.float32, where)
    named = {"q": q, "k": k, "v": v, "o": o, "lse": lse, "dout": dout}
    if grads is not None:
        _require(len(grads) == 3, ERR_SHAPE, where, "grads must be (dq, dk, dv)")
        for name, t, shp in zip(("dq", "dk", "dv"), grads, ((B, S, Hq, D), (B, S, Hkv, D), (B, S, Hkv, D))):
            _check_tensor(t, name, shp, torch.bfloat16, where)
            named[name] = t
    if workspace is not None:
        _require(isinstance(workspace, torch.Tensor) and workspace.is_contiguous(), ERR_SHAPE, where,
                 "workspace must be a contiguous tensor")
        named["workspace"] = workspace
    dev = _check_device(named, where)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    size_fn, call, name = ((axis_attn_bwd_det_workspace_bytes, axis_attn_bwd_det, "axis_attn_bwd_det")
                           if deterministic else
                           (axis_attn_bwd_workspace_bytes, axis_attn_bwd, "axis_attn_bwd"))
    need = size_fn(B, Hq, Hkv, S, D)
    with torch.cuda.device(dev):
        if workspace is None:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        dq, dk, dv = grads if grads is not None else (torch.empty_like(q), torch.empty_like(k),
                                                      torch.empty_like(v))
        rc = call(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                  lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                  B, Hq, Hkv, S, D, scale, int(causal), workspace.data_ptr(),
                  workspace.numel() * workspace.element_size(), _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, name)
    return dq, dk, dv


def rope_table(S: int, D: int, base: float = 10000.0, device=None, stream=None):
    """The (cos, sin) table [S, D/2, 2] fp64 of the rotary embedding (freqs_cis)."""
    import torch

    dev = torch.device("cuda") if device is None else torch.device(device)
    cs = torch.empty((S, D // 2, 2), device=dev, dtype=torch.float64)
    with torch.cuda.device(dev):
        rc = axis_attn_rope_table(cs.data_ptr(), S, D, base, _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, "axis_attn_rope_table")
    return cs


def _check_cs(cs, S, D, where):
    import torch

    _require(isinstance(cs, torch.Tensor) and cs.dim() == 3 and cs.shape[0] >= S and cs.shape[1:] == (D // 2, 2),
             ERR_SHAPE, where, f"the RoPE table must be [>= {S}, {D // 2}, 2]")
    _check_tensor(cs[:S], "cs", (S, D // 2, 2), torch.float64, where)


def attention_forward_rope(q, k, v, cs, causal: bool = True, scale: float | None = None, stream=None):
    """Forward with RoPE: (o, lse, q_rot, k_rot) for unrotated bf16 q, k and the
    table cs of rope_table(); q_rot, k_rot (the rotated inputs) feed
    attention_backward_rope."""
    import torch

    where = "attention_forward_rope"
    B, Hq, Hkv, S, D = _dims(q, k, v, where)
    _check_cs(cs, S, D, where)
    dev = _check_device({"q": q, "k": k, "v": v, "cs": cs}, where)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    with torch.cuda.device(dev):
        o = torch.empty_like(q)
        l = torch.empty((B, Hq, S), device=dev, dtype=torch.float32)
        q_rot, k_rot = torch.empty_like(q), torch.empty_like(k)
        rc = axis_attn_fwd_rope(q.data_ptr(), k.data_ptr(), v.data_ptr(), cs.data_ptr(), o.data_ptr(), l.data_ptr(),
                                q_rot.data_ptr(), k_rot.data_ptr(), B, Hq, Hkv, S, D, scale, int(causal),
                                _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, "axis_attn_fwd_rope")
    return o, l, q_rot, k_rot


def attention_backward_rope(q_rot, k_rot, v, cs, o, lse, dout, causal: bool = True, scale: float | None = None,
                            deterministic: bool = False, stream=None):
    """Gradients (dq, dk, dv) with respect to the unrotated q, k of
    attention_forward_rope, from its rotated inputs q_rot, k_rot."""
    import torch

    where = "attention_backward_rope"
    q = q_rot
    B, Hq, Hkv, S, D = _dims(q, k_rot, v, where)
    _check_cs(cs, S, D, where)
    _check_tensor(o, "o", (B, S, Hq, D), torch.bfloat16, where)
    _check_tensor(dout, "dout", (B, S, Hq, D), torch.bfloat16, where)
    _check_tensor(lse, "lse", (B, Hq, S), torch.float32, where)
    dev = _check_device({"q": q, "k_rot": k_rot, "v": v, "cs": cs, "o": o, "lse": lse, "dout": dout}, where)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    need = (axis_attn_bwd_det_workspace_bytes if deterministic else axis_attn_bwd_workspace_bytes)(B, Hq, Hkv, S, D)
    with torch.cuda.device(dev):
        ws = torch.empty(need, device=dev, dtype=torch.uint8)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k_rot), torch.empty_like(v)
        rc = axis_attn_bwd_rope(q.data_ptr(), k_rot.data_ptr(), v.data_ptr(), cs.data_ptr(), o.data_ptr(),
                                dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                B, Hq, Hkv, S, D, scale, int(causal), int(deterministic), ws.data_ptr(), need,
                                _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, "axis_attn_bwd_rope")
    return dq, dk, dv


def attention_decode(q, k_cache, v_cache, block_table, seq_lens, scale: float | None = None, out=None,
                     lse=None, workspace=None, stream=None, layout: str = "NHD"):
    """Decode step: q [B, Hq, D] bf16 (one new token per sequence) or
    [B, q_len, Hq, D] (the last q_len positions of each sequence),
    k_cache / v_cache [num_pages, page_size, Hkv, D] bf16 (layout "NHD") or
    [num_pages, Hkv, page_size, D] (layout "HND"), block_table [B, max_pages]
    int32, seq_lens [B] int32 (the new tokens included), all on one CUDA
    device.  Returns (o shaped like q, bf16; lse [B, Hq] or [B, Hq, q_len],
    fp32)."""
    import torch

    where = "attention_decode"
    _require(layout in ("NHD", "HND"), ERR_SHAPE, where, "layout must be 'NHD' or 'HND'")
    hnd = layout == "HND"
    dims = "[num_pages, Hkv, page_size, D]" if hnd else "[num_pages, page_size, Hkv, D]"
    _require(isinstance(q, torch.Tensor) and q.dim() in (3, 4), ERR_SHAPE, where,
             "q must be a 3-D tensor [B, Hq, D] or a 4-D tensor [B, q_len, Hq, D]")
    _require(isinstance(k_cache, torch.Tensor) and k_cache.dim() == 4, ERR_SHAPE, where,
             f"k_cache must be a 4-D tensor {dims}")
    multi = q.dim() == 4
    if multi:
        B, q_len, Hq, D = q.shape
    else:
        (B, Hq, D), q_len = q.shape, 1
    if hnd:
        num_pages, Hkv, page_size, _ = k_cache.shape
        cache_shape = (num_pages, Hkv, page_size, D)
    else:
        num_pages, page_size, Hkv, _ = k_cache.shape
        cache_shape = (num_pages, page_size, Hkv, D)
    _check_tensor(q, "q", tuple(q.shape), torch.bfloat16, where)
    _check_tensor(k_cache, "k_cache", cache_shape, torch.bfloat16, where)
    _check_tensor(v_cache, "v_cache", cache_shape, torch.bfloat16, where)
    _require(isinstance(block_table, torch.Tensor) and block_table.dim() == 2, ERR_SHAPE, where,
             "block_table must be a 2-D tensor [B, max_pages]")
    max_pages = block_table.shape[1]
    _check_tensor(block_table, "block_table", (B, max_pages), torch.int32, where)
    _check_tensor(seq_lens, "seq_lens", (B,), torch.int32, where)
    named = {"q": q, "k_cache": k_cache, "v_cache": v_cache, "block_table": block_table, "seq_lens": seq_lens}
    lse_shape = (B, Hq, q_len) if multi else (B, Hq)
    if out is not None:
        _check_tensor(out, "out", tuple(q.shape), torch.bfloat16, where)
        named["out"] = out
    if lse is not None:
        _check_tensor(lse, "lse", lse_shape, torch.float32, where)
        named["lse"] = lse
    dev = _check_device(named, where)
    scale = 1.0 / math.sqrt(D) if scale is None else scale
    need = (axis_attn_decode_q_workspace_bytes(B, q_len, Hq, Hkv, D, page_size, max_pages) if multi
            else axis_attn_decode_workspace_bytes(B, Hq, Hkv, D, page_size, max_pages))
    with torch.cuda.device(dev):
        o = torch.empty_like(q) if out is None else out
        l = torch.empty(lse_shape, device=dev, dtype=torch.float32) if lse is None else lse
        if workspace is None and need > 0:
            workspace = torch.empty(need, device=dev, dtype=torch.uint8)
        wp = workspace.data_ptr() if workspace is not None else None
        wb = workspace.numel() * workspace.element_size() if workspace is not None else 0
        ptrs = (q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(), seq_lens.data_ptr(),
                o.data_ptr(), l.data_ptr())
        if multi:
            call = axis_attn_decode_q
            rc = call(*ptrs, B, q_len, Hq, Hkv, D, page_size, max_pages, num_pages, scale, int(hnd), wp, wb,
                      _stream(stream, dev))
        else:
            call = axis_attn_decode_hnd if hnd else axis_attn_decode
            rc = call(*ptrs, B, Hq, Hkv, D, page_size, max_pages, num_pages, scale, wp, wb, _stream(stream, dev))
    if rc:
        raise AxisAttnError(rc, call.__name__)
    return o, l


def check_status(stream=None):
    """Synchronise and raise if a kernel reported a timed-out device wait."""
    rc = axis_attn_get_status(_stream(stream))
    if rc:
        w = axis_attn_last_status_word()
        raise AxisAttnError(rc, f"axis_attn_get_status (status word {w:#x}, wait site {(w >> 8) & 0xff})")
