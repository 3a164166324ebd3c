"""Pins of the oracle's decode step (oracle_attn_decode), against facts that do
not come from the function itself.

The decode step is the last query row of causal attention over the cached
sequence (axiomlm page, Key Features: the state-cached KV decode engine;
Quick Start section 4, the paged KV-cache engine), so:
  - it equals the last row of the oracle's full forward (a separate, already
    pinned code path) on every sequence length of a ragged batch;
  - it equals torch's float64 scaled_dot_product_attention (a library routine);
  - one cached key gives O = V_0 and LSE = s_00 exactly;
  - identical keys give the mean of the visible V rows and LSE = s + ln L;
  - shifting every key by c changes LSE by scale q.c and leaves O;
  - planted mistakes (wrong kv head, one row too many or too few, scale
    dropped, log2 LSE) each break one of these.
"""
import math
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import oracle
from oracle.oracle import Oracle


def _case(B=3, Hq=6, Hkv=2, Smax=40, D=16, seed=3):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, Hq, D))
    k = g.standard_normal((B, Smax, Hkv, D))
    v = g.standard_normal((B, Smax, Hkv, D))
    lens = np.array([1, Smax, 17][:B], np.int32)
    return q, k, v, lens


def _check_all(orc, q, k, v, lens, sc):
    """Raise AssertionError if any pin fails (used on the clean and mutant builds)."""
    B, Hq, D = q.shape
    Hkv = k.shape[2]
    o, lse = orc.attn_decode(q, k, v, lens, sc)
    for b in range(B):
        L = int(lens[b])
        qf = np.zeros((1, L, Hq, D))
        qf[0, L - 1] = q[b]
        fo, fl = orc.attn_fwd(qf, k[b:b + 1, :L], v[b:b + 1, :L], sc, True)
        np.testing.assert_allclose(o[b], fo[0, L - 1], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b], fl[0, :, L - 1], rtol=0, atol=1e-13)
    # library routine
    G = Hq // Hkv
    for b in range(B):
        L = int(lens[b])
        qt = torch.from_numpy(q[b]).reshape(Hq, 1, D)
        kt = torch.from_numpy(k[b, :L]).permute(1, 0, 2).repeat_interleave(G, 0)
        vt = torch.from_numpy(v[b, :L]).permute(1, 0, 2).repeat_interleave(G, 0)
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=sc)
        np.testing.assert_allclose(o[b], ref[:, 0].numpy(), rtol=0, atol=1e-12)
    # one key
    o1, l1 = orc.attn_decode(q, k, v, np.ones(B, np.int32), sc)
    for b in range(B):
        for h in range(Hq):
            assert np.array_equal(o1[b, h], v[b, 0, h // G])
            assert abs(l1[b, h] - sc * q[b, h] @ k[b, 0, h // G]) <= 1e-13
    # identical keys
    kk = np.repeat(k[:, :1], k.shape[1], axis=1)
    oi, li = orc.attn_decode(q, kk, v, lens, sc)
    for b in range(B):
        L = int(lens[b])
        for h in range(Hq):
            np.testing.assert_allclose(oi[b, h], v[b, :L, h // G].mean(0), atol=1e-12)
            assert abs(li[b, h] - (sc * q[b, h] @ k[b, 0, h // G] + math.log(L))) <= 1e-12
    # key shift
    c = np.linspace(-1, 1, D)
    os_, ls_ = orc.attn_decode(q, k + c, v, lens, sc)
    np.testing.assert_allclose(os_, o, atol=1e-12)
    np.testing.assert_allclose(ls_ - lse, sc * q @ c, atol=1e-12)


def test_decode_pins():
    q, k, v, lens = _case()
    from oracle.oracle import default

    _check_all(default(), q, k, v, lens, 0.3)


def test_decode_rejects_bad_lengths():
    q, k, v, lens = _case()
    with pytest.raises(ValueError):
        oracle.attn_decode(q, k, v, np.array([0, 3, 3], np.int32), 0.25)
    with pytest.raises(ValueError):
        oracle.attn_decode(q, k, v, np.array([1, 41, 3], np.int32), 0.25)


MUTANTS = [
    ("kv head", "const int kv = h / G, L = lens[b];", "const int kv = h % Hkv, L = lens[b];"),
    ("one row short", "for (int j = 0; j < L; ++j) {\n                    s[j]",
     "for (int j = 0; j < L - 1; ++j) {\n                    s[j]"),
    ("scale dropped", "\n                    s[j] = scale * dot(qh,", "\n                    s[j] = dot(qh,"),
    ("log2 lse", "lse[(size_t)b * Hq + h] = m + log(l);", "lse[(size_t)b * Hq + h] = m + log2(l);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS)
def test_decode_mutants_are_caught(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    assert src.count(old) == 1, name
    mut = tmp_path / "m.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "m.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(mut), "-lm"])
    q, k, v, lens = _case()
    with pytest.raises(AssertionError):
        _check_all(Oracle(str(lib)), q, k, v, lens, 0.3)


# ---- several new tokens per sequence (oracle_attn_decode_q)
#
# Token t of q_len new tokens sits at position lens[b] - q_len + t and sees the
# keys up to and including its own position.  Pins:
#   - the last q_len rows of the oracle's full causal forward (a separately
#     pinned code path) on every sequence of a ragged batch;
#   - torch's float64 scaled_dot_product_attention with the causal mask
#     aligned to the end of the keys (a library routine);
#   - q_len = 1 is the one-token decode step;
#   - planted mistakes (the mask one key too wide or too narrow, the tokens'
#     positions counted from the front, the LSE laid out token-major) each
#     break one of these.


def _case_q(B=3, q_len=4, Hq=6, Hkv=2, Smax=40, D=16, seed=5):
    g = np.random.default_rng(seed)
    q = g.standard_normal((B, q_len, Hq, D))
    k = g.standard_normal((B, Smax, Hkv, D))
    v = g.standard_normal((B, Smax, Hkv, D))
    lens = np.array([q_len, Smax, 17][:B], np.int32)
    return q, k, v, lens


def _check_all_q(orc, q, k, v, lens, sc):
    B, T, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    o, lse = orc.attn_decode_q(q, k, v, lens, sc)
    assert o.shape == (B, T, Hq, D) and lse.shape == (B, Hq, T)
    for b in range(B):
        L = int(lens[b])
        qf = np.zeros((1, L, Hq, D))
        qf[0, L - T:] = q[b]
        fo, fl = orc.attn_fwd(qf, k[b:b + 1, :L], v[b:b + 1, :L], sc, True)
        np.testing.assert_allclose(o[b], fo[0, L - T:], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b], fl[0, :, L - T:], rtol=0, atol=1e-13)
        # library routine: mask[t, j] = j <= L - T + t
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)                       # [Hq, T, D]
        kt = torch.from_numpy(k[b, :L]).permute(1, 0, 2).repeat_interleave(G, 0)
        vt = torch.from_numpy(v[b, :L]).permute(1, 0, 2).repeat_interleave(G, 0)
        mask = torch.arange(L)[None, :] <= (L - T + torch.arange(T))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=sc)
        np.testing.assert_allclose(o[b], ref.permute(1, 0, 2).numpy(), rtol=0, atol=1e-12)
    # one new token: the one-token step
    o1, l1 = orc.attn_decode_q(q[:, -1:], k, v, lens, sc)
    d1, dl1 = orc.attn_decode(q[:, -1], k, v, lens, sc)
    np.testing.assert_allclose(o1[:, 0], d1, rtol=0, atol=1e-13)
    np.testing.assert_allclose(l1[:, :, 0], dl1, rtol=0, atol=1e-13)


def test_decode_q_pins():
    from oracle.oracle import default

    q, k, v, lens = _case_q()
    _check_all_q(default(), q, k, v, lens, 0.3)
    q, k, v, lens = _case_q(B=2, q_len=1, Hq=4, Hkv=4, Smax=9, D=8, seed=6)
    _check_all_q(default(), q, k, v, lens, 0.5)


def test_decode_q_rejects_short_sequences():
    q, k, v, lens = _case_q()
    with pytest.raises(ValueError):  # a sequence must hold its q_len new tokens
        oracle.attn_decode_q(q, k, v, np.array([3, 40, 17], np.int32), 0.25)
    with pytest.raises(ValueError):
        oracle.attn_decode_q(q, k, v, np.array([4, 41, 17], np.int32), 0.25)


MUTANTS_Q = [
    ("mask one key too wide", "p = lens[b] - q_len + t;  /* this token's position */",
     "p = lens[b] - q_len + t + (t + 1 < q_len);  /* this token's position */"),
    ("mask one key too narrow", "for (int j = 0; j <= p; ++j) l += exp", "for (int j = 0; j < p; ++j) l += exp"),
    ("positions from the front", "p = lens[b] - q_len + t;  /* this token's position */",
     "p = t + (lens[b] - q_len) * (t == q_len - 1);  /* this token's position */"),
    ("token-major lse", "lse[((size_t)b * Hq + h) * q_len + t] = m + log(l);",
     "lse[((size_t)b * q_len + t) * Hq + h] = m + log(l);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS_Q)
def test_decode_q_mutants_are_caught(tmp_path, name, old, new):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")).read()
    assert src.count(old) == 1, name
    mut = tmp_path / "m.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "m.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(lib), str(mut), "-lm"])
    q, k, v, lens = _case_q()
    with pytest.raises(AssertionError):
        _check_all_q(Oracle(str(lib)), q, k, v, lens, 0.3)
