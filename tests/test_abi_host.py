"""Host-side checks of the C ABI (CPU only; nothing here launches a kernel).

The library must load, export every function include/axis_attn.h declares,
size the backward workspace, and reject every invalid argument with its status
code before touching the device.
"""
import ctypes
import os
import re

import pytest

import causal_attention_fwd_b200 as aa
from causal_attention_fwd_b200 import build as build_mod

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "axis_attn.h")


@pytest.fixture(scope="module")
def lib():
    build_mod.build()
    return aa.load()


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(axis_attn_\w+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(aa.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in _declared():
        assert hasattr(lib, name), name
    nm = os.popen(f"nm -D --defined-only {aa.library_path()}").read()
    for name in _declared():
        assert re.search(rf"\bT {name}\b", nm), name


def test_strerror_covers_every_status(lib):
    texts = {aa.axis_attn_strerror(c) for c in range(9)}
    assert len(texts) == 9 and "ok" in texts
    assert aa.axis_attn_strerror(99) == "unknown status"


def head_split(B, Hq, Hkv, S):
    """The header's rule: with fewer than 148 (b, kv head, 128-key tile) CTAs
    and G = Hq / Hkv > 1, the smallest divisor of G reaching 148 CTAs, else G."""
    G, ctas = Hq // Hkv, -(-S // 128) * B * Hkv
    if G == 1 or ctas >= 148:
        return 1
    return next((d for d in range(2, G) if G % d == 0 and ctas * d >= 148), G)


def test_head_split_rule(lib):
    for B, Hq, Hkv, S, want in ((4, 32, 8, 2048, 1),      # llm1b: 512 CTAs
                                (2, 12, 4, 1024, 3),      # gpt2s_gqa: 64 CTAs, G = 3
                                (1, 1, 1, 128, 1),        # G = 1: nothing to split
                                (1, 8, 1, 1000, 8),       # 8 CTAs: every head its own CTA
                                (2, 16, 2, 2048, 4),      # 64 CTAs x 2 = 128 < 148: the next divisor
                                (3, 16, 2, 2048, 2)):     # 96 x 2 = 192 >= 148
        got = aa.axis_attn_bwd_head_split(B, Hq, Hkv, S, 64)
        assert got == head_split(B, Hq, Hkv, S) == want, (B, Hq, Hkv, S)
    assert aa.axis_attn_bwd_head_split(1, 3, 2, 128, 64) == 0  # invalid sizes


def test_workspace_bytes(lib):
    # lse2 + dr rows padded to 128, each section rounded to 256 bytes, + fp32 dQ accumulator
    # (+ two fp32 partial dK, dV sections when the backward splits the heads)
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    B, Hq, Hkv, S, D = 4, 32, 8, 1000, 64  # 256 CTAs: no head split
    rows = B * Hq * 1024
    assert aa.axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D) == 2 * r256(rows * 4) + r256(B * Hq * S * D * 4)
    B, Hq, Hkv, S, D = 2, 12, 4, 1000, 64  # 64 CTAs, G = 3: split in 3
    rows = B * Hq * 1024
    assert aa.axis_attn_bwd_workspace_bytes(B, Hq, Hkv, S, D) == (
        2 * r256(rows * 4) + r256(B * Hq * S * D * 4) + 2 * r256(3 * B * S * Hkv * D * 4))
    assert aa.axis_attn_bwd_workspace_bytes(1, 3, 2, 128, 64) == 0      # Hq % Hkv != 0
    assert aa.axis_attn_bwd_workspace_bytes(1, 1, 1, 128, 96) == 0      # unsupported D
    assert aa.axis_attn_bwd_workspace_bytes(1, 1, 1, 0, 64) == 0        # empty sequence


def test_det_workspace_bytes(lib):
    # only the two row sections: dQ stays on chip in the deterministic pass
    B, Hq, Hkv, S, D = 4, 12, 4, 5000, 64  # 320 CTAs: no head split
    rows = B * Hq * 5120
    r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
    assert aa.axis_attn_bwd_det_workspace_bytes(B, Hq, Hkv, S, D) == 2 * r256(rows * 4)
    # a head split adds the partial dK, dV sections (2 x 12 x 1000: 64 CTAs, split in 3)
    B, Hq, Hkv, S, D = 2, 12, 4, 1000, 64
    assert aa.axis_attn_bwd_det_workspace_bytes(B, Hq, Hkv, S, D) == (
        2 * r256(B * Hq * 1024 * 4) + 2 * r256(3 * B * S * Hkv * D * 4))
    # the header's example: B=4, Hq=32, S=2048 needs about 2.1 MB, flat in D
    assert aa.axis_attn_bwd_det_workspace_bytes(4, 32, 8, 2048, 64) == 2 * r256(4 * 32 * 2048 * 4)
    assert aa.axis_attn_bwd_det_workspace_bytes(4, 32, 8, 2048, 128) == 2 * r256(4 * 32 * 2048 * 4)
    # the longest workload: 1 x 16 heads x 32768 -> 4 MB (no S^2 term)
    assert aa.axis_attn_bwd_det_workspace_bytes(1, 16, 16, 32768, 128) == 2 * r256(16 * 32768 * 4)
    assert aa.axis_attn_bwd_det_workspace_bytes(1, 3, 2, 128, 64) == 0
    assert aa.axis_attn_bwd_det_workspace_bytes(1, 1, 1, 128, 96) == 0


A = 1 << 20  # a fake, 16-byte aligned "device" address; never dereferenced


def _fwd(**over):
    args = dict(q=A, k=A, v=A, o=A, lse=A, B=1, Hq=2, Hkv=1, S=128, D=64, scale=0.125, causal=1,
                stream=None)
    args.update(over)
    return aa.axis_attn_fwd(*args.values())


def _bwd(**over):
    args = dict(q=A, k=A, v=A, o=A, dO=A, lse=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=1, S=128, D=64,
                scale=0.125, causal=1, workspace=A, workspace_bytes=1 << 30, stream=None)
    args.update(over)
    return aa.axis_attn_bwd(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(lse=None), 1), (dict(v=0), 1),
    (dict(k=A + 8), 2), (dict(o=A + 2), 2), (dict(lse=A + 4), 2),
    (dict(B=0), 3), (dict(S=0), 3), (dict(Hq=3, Hkv=2), 3), (dict(Hkv=0), 3),
    (dict(scale=0.0), 3), (dict(scale=-1.0), 3), (dict(scale=float("nan")), 3),
    (dict(scale=float("inf")), 3),
    (dict(B=1 << 16, S=1 << 16), 3),
    (dict(D=32), 4), (dict(D=96), 4), (dict(D=256), 4),
])
def test_fwd_rejects(lib, over, code):
    assert _fwd(**over) == code


@pytest.mark.parametrize("over,code", [
    (dict(dO=None), 1), (dict(dq=None), 1), (dict(dv=None), 1),
    (dict(dk=A + 8), 2), (dict(dO=A + 1), 2),
    (dict(S=0), 3), (dict(Hq=4, Hkv=3), 3), (dict(scale=0.0), 3), (dict(D=80), 4),
    (dict(workspace=None), 5), (dict(workspace=A + 16), 5), (dict(workspace_bytes=1000), 5),
])
def test_bwd_rejects(lib, over, code):
    assert _bwd(**over) == code


@pytest.mark.parametrize("over,code", [
    (dict(dO=None), 1), (dict(dq=None), 1), (dict(dk=A + 8), 2), (dict(S=0), 3), (dict(D=80), 4),
    (dict(workspace=None), 5), (dict(workspace=A + 16), 5),
    # one byte short of the two row sections and the two partial sections (split in 2)
    (dict(S=1000, workspace_bytes=2 * 1024 * 2 * 4 + 2 * 2 * 1000 * 64 * 4 - 1), 5),
])
def test_bwd_det_rejects(lib, over, code):
    args = dict(q=A, k=A, v=A, o=A, dO=A, lse=A, dq=A, dk=A, dv=A, B=1, Hq=2, Hkv=1, S=128, D=64,
                scale=0.125, causal=1, workspace=A, workspace_bytes=1 << 30, stream=None)
    args.update(over)
    if "S" in over and over["S"] == 1000:
        assert aa.axis_attn_bwd_det_workspace_bytes(1, 2, 1, 1000, 64) == args["workspace_bytes"] + 1
    assert aa.axis_attn_bwd_det(*args.values()) == code


def test_torch_helpers_raise_without_valid_args(lib):
    import torch

    q = torch.zeros(1, 128, 2, 32, dtype=torch.bfloat16)  # CPU tensors, D = 32: rejected
    with pytest.raises(aa.AxisAttnError) as e:
        aa.attention_forward(q, q[:, :, :1].contiguous(), q[:, :, :1].contiguous(),
                             stream=type("S", (), {"cuda_stream": 0})())
    assert e.value.code == 4  # CPU tensors: rejected by the helper before the library is called


def test_no_cpu_fallback(tmp_path, monkeypatch):
    """With the library absent, the first call raises instead of computing on the CPU."""
    import causal_attention_fwd_b200.binding as bnd

    monkeypatch.setattr(bnd, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(bnd, "_lib", None)
    with pytest.raises(RuntimeError, match="no CPU fallback"):
        bnd.axis_attn_bwd_workspace_bytes(1, 1, 1, 128, 64)


def test_valid_args_without_gpu_report_cuda_error(lib):
    """Valid arguments on a machine with no usable GPU: a status, not a crash."""
    import torch

    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _fwd() in (4, 6)


def _dec(fn="axis_attn_decode", **over):
    args = dict(q=A, k_cache=A, v_cache=A, block_table=A, seq_lens=A, o=A, lse=A, B=1, Hq=32, Hkv=8, D=128,
                page_size=64, max_pages=128, num_pages=128, scale=0.088, workspace=A, workspace_bytes=1 << 30,
                stream=None)
    args.update(over)
    return getattr(aa, fn)(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(block_table=None), 1), (dict(seq_lens=None), 1), (dict(lse=None), 1),
    (dict(k_cache=A + 8), 2), (dict(o=A + 2), 2), (dict(block_table=A + 2), 2), (dict(seq_lens=A + 1), 2),
    (dict(B=0), 3), (dict(Hq=12, Hkv=5), 3), (dict(max_pages=0), 3), (dict(num_pages=0), 3),
    (dict(scale=0.0), 3), (dict(scale=float("nan")), 3),
    (dict(D=96), 4), (dict(Hq=72, Hkv=8), 4), (dict(page_size=24), 4), (dict(page_size=4), 4),
    (dict(page_size=512), 4),
    (dict(workspace=None), 5), (dict(workspace=A + 16), 5), (dict(workspace_bytes=100), 5),
])
@pytest.mark.parametrize("fn", ["axis_attn_decode", "axis_attn_decode_hnd"])
def test_decode_rejects(lib, fn, over, code):
    assert _dec(fn, **over) == code


def test_decode_workspace_bytes(lib):
    # B=1, 8 kv heads, 8192 keys: ceil(296 / 8) = 37 splits wanted, at least 256 keys each -> 32 splits
    n = aa.axis_attn_decode_workspace_bytes(1, 32, 8, 128, 64, 128)
    assert n == 1 * 32 * 32 * (128 + 2) * 4
    assert aa.axis_attn_decode_workspace_bytes(64, 32, 8, 128, 16, 38) == 0  # 512 units: no split
    assert aa.axis_attn_decode_workspace_bytes(1, 32, 8, 96, 64, 128) == 0


@pytest.mark.parametrize("fn,args,code", [
    ("axis_attn_rope_table", (None, 128, 64, 10000.0, None), 1),
    ("axis_attn_rope_table", (A + 8, 128, 64, 10000.0, None), 2),
    ("axis_attn_rope_table", (A, 0, 64, 10000.0, None), 3),
    ("axis_attn_rope_table", (A, 128, 60, 10000.0, None), 3),
    ("axis_attn_rope_table", (A, 128, 64, 1.0, None), 3),
    ("axis_attn_rope", (A, A, None, 1, 128, 2, 64, 0, None), 1),
    ("axis_attn_rope", (A, A + 4, A, 1, 128, 2, 64, 0, None), 2),
    ("axis_attn_rope", (A, A, A, 1, 128, 2, 12, 0, None), 3),
    ("axis_attn_fwd_rope", (A, A, A, None, A, A, A, A, 1, 2, 1, 128, 64, 0.125, 1, None), 1),
    ("axis_attn_fwd_rope", (A, A, A, A, A, A, A, None, 1, 2, 1, 128, 64, 0.125, 1, None), 1),
    ("axis_attn_fwd_rope", (A, A, A, A, A, A, A, A + 8, 1, 2, 1, 128, 64, 0.125, 1, None), 2),
    ("axis_attn_fwd_rope", (A, A, A, A, A, A, A, A, 1, 3, 2, 128, 64, 0.125, 1, None), 3),
    ("axis_attn_fwd_rope", (A, A, A, A, A, A, A, A, 1, 2, 1, 128, 96, 0.125, 1, None), 4),
    ("axis_attn_bwd_rope", (A,) * 3 + (None,) + (A,) * 6 + (1, 2, 1, 128, 64, 0.125, 1, 0, A, 1 << 30, None), 1),
    ("axis_attn_bwd_rope", (A,) * 3 + (A + 8,) + (A,) * 6 + (1, 2, 1, 128, 64, 0.125, 1, 0, A, 1 << 30, None), 2),
    ("axis_attn_bwd_rope", (A,) * 10 + (1, 2, 1, 128, 64, 0.125, 1, 0, A, 1000, None), 5),
])
def test_rope_rejects(lib, fn, args, code):
    assert getattr(aa, fn)(*args) == code


def _decq(**over):
    args = dict(q=A, k_cache=A, v_cache=A, block_table=A, seq_lens=A, o=A, lse=A, B=1, q_len=4, Hq=32, Hkv=8, D=128,
                page_size=64, max_pages=128, num_pages=128, scale=0.088, head_major=0, workspace=A,
                workspace_bytes=1 << 30, stream=None)
    args.update(over)
    return aa.axis_attn_decode_q(*args.values())


@pytest.mark.parametrize("over,code", [
    (dict(q=None), 1), (dict(seq_lens=A + 2), 2), (dict(q_len=0), 3), (dict(q_len=65), 4),
    (dict(max_pages=1, page_size=8, q_len=9), 3), (dict(Hq=72, Hkv=8), 4), (dict(workspace=None), 5),
])
def test_decode_q_rejects(lib, over, code):
    assert _decq(**over) == code


def test_decode_q_workspace_bytes(lib):
    # q_len = 1 is the one-token query; 4 tokens x G = 4 heads = 16 rows: one tile per kv head,
    # so the same splits (B=1, 8 kv heads, 8192 keys: 32), and 4x the partial rows
    one = aa.axis_attn_decode_workspace_bytes(1, 32, 8, 128, 64, 128)
    assert aa.axis_attn_decode_q_workspace_bytes(1, 1, 32, 8, 128, 64, 128) == one
    assert aa.axis_attn_decode_q_workspace_bytes(1, 4, 32, 8, 128, 64, 128) == 4 * one
    assert aa.axis_attn_decode_q_workspace_bytes(1, 65, 32, 8, 128, 64, 128) == 0  # unsupported q_len


def _dec_q_rule(B, q_len, Hq, Hkv, D, page_size, max_pages):
    """The documented rule: one tile of rows when a kv head has at most 8 (token, head) rows, else
    tiles of 16; splits give at least 296 items of at least 256 keys; partial rows are (b, token, h)."""
    G = Hq // Hkv
    n_rt = 1 if G * q_len <= 8 else -(-(G * q_len) // 16)
    keys = max_pages * page_size
    units = B * Hkv * n_rt
    n = min(-(-296 // units), -(-keys // 256))
    n = max(n, 1)
    kps = -(-(-(-keys // n)) // 32) * 32
    n = -(-keys // kps)
    return B * q_len * Hq * n * (D + 2) * 4 if n > 1 else 0


@pytest.mark.parametrize("B,q_len,Hq,Hkv,D,ps,mp", [
    (1, 2, 32, 8, 128, 64, 128),    # 8 rows: one tile, as for one token
    (1, 3, 32, 8, 128, 64, 128),    # 12 rows: one tile of 16
    (1, 8, 64, 8, 128, 64, 128),    # 64 rows: four tiles, fewer splits
    (2, 16, 8, 8, 64, 16, 512),     # G = 1: 16 rows
    (64, 4, 32, 8, 128, 16, 38),    # many units: no split
    (3, 64, 24, 8, 64, 8, 2048),    # the largest q_len
])
def test_decode_q_workspace_follows_the_rule(lib, B, q_len, Hq, Hkv, D, ps, mp):
    assert aa.axis_attn_decode_q_workspace_bytes(B, q_len, Hq, Hkv, D, ps, mp) == _dec_q_rule(
        B, q_len, Hq, Hkv, D, ps, mp)
