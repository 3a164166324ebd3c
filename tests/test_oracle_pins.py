"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test checks the oracle against something it does not compute itself: a
hand-worked example, central finite differences of its own forward (which pin
the analytic backward), closed forms, invariances of softmax attention, and the
library routine torch.nn.functional.scaled_dot_product_attention in float64
with autograd.  The checks are chosen so that a dropped term, a wrong sign, a
wrong GQA index or a transposed operand in the oracle fails at least one.
(``test_oracle_mutants.py`` plants such mistakes and checks that they fail.)

Sources: Axis (zyoralabs.com/axis), feature list (fused flash attention, fwd
and bwd; bf16 storage, fp32 accumulation) and shape fuzz (KV groups);
furkanhaney/axis README, Training building blocks (causal attention,
prefix-mean learning, central differences) and Conformance with PyTorch
(independent oracles; running PyTorch alongside); axiomlm (PyPI), Quick Start
section 8 ([B,S,H,D] tensors, GQA).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from causal_attention_fwd_b200.synthetic import make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_worked_s2_gqa.json")


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------ hand-worked example
@pytest.mark.parametrize("mode", ["causal", "noncausal"])
def test_hand_worked_example(oracle_mod, mode):
    g = json.load(open(GOLDEN))
    sc = g["dims"]["scale"]
    q, k, v, do = (np.array(g["inputs"][n], dtype=np.float64) for n in ("q", "k", "v", "dout"))
    causal = mode == "causal"
    o, lse = oracle_mod.attn_fwd(q, k, v, sc, causal)
    dq, dk, dv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, causal)
    exp = g[mode]
    for name, got in (("o", o), ("lse", lse), ("dq", dq), ("dk", dk), ("dv", dv)):
        np.testing.assert_allclose(got, np.array(exp[name]), rtol=0, atol=1e-14, err_msg=name)


# ------------------------------------------------------------ P1 finite differences
@pytest.mark.parametrize("Hq,Hkv", [(2, 1), (2, 2), (3, 1)])
@pytest.mark.parametrize("S,D", [(1, 2), (3, 4), (6, 2)])
@pytest.mark.parametrize("causal", [True, False])
def test_central_differences(oracle_mod, Hq, Hkv, S, D, causal):
    """L = sum(dO * O): central differences (h = 1e-6) of the forward against
    the analytic dQ, dK, dV.  Also d(sum_i w_i LSE_i)/dQ against the softmax
    weights: the gradient of log-sum-exp is P, so dLSE_i/dq_i = scale sum_j P_ij k_j."""
    B = 1
    seed = 10 * S + D + 100 * Hq + 1000 * Hkv + int(causal)
    q = _rand((B, S, Hq, D), seed)
    k = _rand((B, S, Hkv, D), seed + 1)
    v = _rand((B, S, Hkv, D), seed + 2)
    do = _rand((B, S, Hq, D), seed + 3)
    w = _rand((B, Hq, S), seed + 4)
    sc = 0.7
    dq, dk, dv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, causal)

    def loss(qq, kk, vv):
        o, lse = oracle_mod.attn_fwd(qq, kk, vv, sc, causal)
        return float((o * do).sum()), float((lse * w).sum())

    h = 1e-6
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        fd = np.zeros_like(x)
        fd_lse = np.zeros_like(x)
        for idx in np.ndindex(*x.shape):
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            args_p = {"q": q, "k": k, "v": v, name: xp}
            args_m = {"q": q, "k": k, "v": v, name: xm}
            lp, sp = loss(args_p["q"], args_p["k"], args_p["v"])
            lm, sm = loss(args_m["q"], args_m["k"], args_m["v"])
            fd[idx] = (lp - lm) / (2 * h)
            fd_lse[idx] = (sp - sm) / (2 * h)
        err = np.abs(fd - g).max() / max(1.0, np.abs(g).max())
        assert err < 1e-7, (name, err)
        if name == "q":
            # dLSE/dq_i = scale * sum_j P_ij k_j, weighted by w
            ref = np.zeros_like(q)
            G = Hq // Hkv
            for hh in range(Hq):
                for i in range(S):
                    p = oracle_mod.probs_row(q, k, sc, causal, 0, hh, i)
                    ref[0, i, hh] = w[0, hh, i] * sc * (p[:, None] * k[0, :, hh // G]).sum(0)
            assert np.abs(fd_lse - ref).max() < 1e-7


# ------------------------------------------------------------ P2 rows sum to one
def test_rows_sum_to_one_and_causal_zeros(oracle_mod):
    B, S, Hq, Hkv, D = 2, 37, 4, 2, 8
    q, k = _rand((B, S, Hq, D), 1), _rand((B, S, Hkv, D), 2)
    for b, h, i in [(0, 0, 0), (0, 3, 5), (1, 2, 36), (1, 1, 17)]:
        p = oracle_mod.probs_row(q, k, 0.5, True, b, h, i)
        assert abs(p.sum() - 1.0) < 1e-14
        assert np.all(p[i + 1:] == 0.0) and np.all(p[: i + 1] > 0.0)
        pn = oracle_mod.probs_row(q, k, 0.5, False, b, h, i)
        assert abs(pn.sum() - 1.0) < 1e-14 and np.all(pn > 0.0)


# ------------------------------------------------------------ P3 first row
def test_first_row_is_v0(oracle_mod):
    B, S, Hq, Hkv, D = 2, 9, 6, 3, 5
    q, k, v = _rand((B, S, Hq, D), 3), _rand((B, S, Hkv, D), 4), _rand((B, S, Hkv, D), 5)
    sc = 0.3
    o, lse = oracle_mod.attn_fwd(q, k, v, sc, True)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            np.testing.assert_array_equal(o[b, 0, h], v[b, 0, h // G])
            assert abs(lse[b, h, 0] - sc * float(q[b, 0, h] @ k[b, 0, h // G])) < 1e-14


# ------------------------------------------------------------ P4/P5 identical keys
def test_identical_keys_prefix_mean(oracle_mod):
    """All keys equal: causal row i is the mean of V_0..V_i, LSE_i = s + ln(i+1),
    and dQ = 0 because each row of dS sums to zero (its keys are all the same)."""
    B, S, Hq, Hkv, D = 1, 20, 4, 2, 6
    q, v, do = _rand((B, S, Hq, D), 6), _rand((B, S, Hkv, D), 7), _rand((B, S, Hq, D), 8)
    k = np.broadcast_to(_rand((B, 1, Hkv, D), 9), (B, S, Hkv, D)).copy()
    sc = 0.4
    o, lse = oracle_mod.attn_fwd(q, k, v, sc, True)
    dq, dk, _, _ = oracle_mod.attn_bwd(q, k, v, do, sc, True)
    G = Hq // Hkv
    for h in range(Hq):
        mean = np.cumsum(v[0, :, h // G], axis=0) / np.arange(1, S + 1)[:, None]
        np.testing.assert_allclose(o[0, :, h], mean, atol=1e-13)
        s = sc * q[0, :, h] @ k[0, 0, h // G]
        np.testing.assert_allclose(lse[0, h], s + np.log(np.arange(1, S + 1)), atol=1e-13)
    assert np.abs(dq).max() < 1e-13
    # Non-causal: every row is the mean of all V rows (also the S = 1 case).
    on, _ = oracle_mod.attn_fwd(q, k, v, sc, False)
    for h in range(Hq):
        np.testing.assert_allclose(on[0, :, h], np.broadcast_to(v[0, :, h // G].mean(0), (S, D)),
                                   atol=1e-13)
    o1, lse1 = oracle_mod.attn_fwd(q[:, :1], k[:, :1], v[:, :1], sc, False)
    np.testing.assert_array_equal(o1[0, 0], v[0, 0, np.arange(Hq) // G])


# ------------------------------------------------------------ P6 shift invariance
def test_key_shift_invariance(oracle_mod):
    """Adding one vector c to every key multiplies every exp(s_ij) of a row by
    the same factor exp(scale q_i.c): O is unchanged, LSE_i moves by scale q_i.c."""
    B, S, Hq, Hkv, D = 2, 15, 4, 2, 4
    q, k, v = _rand((B, S, Hq, D), 10), _rand((B, S, Hkv, D), 11), _rand((B, S, Hkv, D), 12)
    c = _rand((D,), 13)
    sc = 0.6
    for causal in (True, False):
        o, lse = oracle_mod.attn_fwd(q, k, v, sc, causal)
        o2, lse2 = oracle_mod.attn_fwd(q, k + c, v, sc, causal)
        np.testing.assert_allclose(o2, o, atol=1e-12)
        shift = sc * np.einsum("bshd,d->bhs", q, c)
        np.testing.assert_allclose(lse2 - lse, shift, atol=1e-12)


# ------------------------------------------------------------ P7 GQA reduction
def test_gqa_equals_expanded_mha(oracle_mod):
    B, S, Hq, Hkv, D = 2, 11, 6, 2, 4
    G = Hq // Hkv
    q, k, v, do = (_rand((B, S, h, D), 20 + n) for n, h in enumerate((Hq, Hkv, Hkv, Hq)))
    ke, ve = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    for causal in (True, False):
        o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, causal)
        oe, lsee = oracle_mod.attn_fwd(q, ke, ve, 0.5, causal)
        np.testing.assert_allclose(o, oe, atol=1e-14)
        np.testing.assert_allclose(lse, lsee, atol=1e-14)
        dq, dk, dv, _ = oracle_mod.attn_bwd(q, k, v, do, 0.5, causal)
        dqe, dke, dve, _ = oracle_mod.attn_bwd(q, ke, ve, do, 0.5, causal)
        np.testing.assert_allclose(dq, dqe, atol=1e-13)
        np.testing.assert_allclose(dk, dke.reshape(B, S, Hkv, G, D).sum(3), atol=1e-13)
        np.testing.assert_allclose(dv, dve.reshape(B, S, Hkv, G, D).sum(3), atol=1e-13)


# ------------------------------------------------------------ P8 identities
def test_rowsum_identity_and_zero_sum(oracle_mod):
    """Dr_i = sum_d dO_id O_id equals sum_j P_ij dP_ij; each row of dS sums to
    zero, so the key rows of dK of one (b, kv) unit sum to zero."""
    B, S, Hq, Hkv, D = 1, 13, 4, 2, 5
    q, k, v, do = (_rand((B, S, h, D), 40 + n) for n, h in enumerate((Hq, Hkv, Hkv, Hq)))
    G = Hq // Hkv
    for causal in (True, False):
        dq, dk, dv, dr = oracle_mod.attn_bwd(q, k, v, do, 0.8, causal)
        for h in range(Hq):
            for i in range(S):
                p = oracle_mod.probs_row(q, k, 0.8, causal, 0, h, i)
                dp = v[0, :, h // G] @ do[0, i, h]
                assert abs(dr[0, h, i] - float(p @ dp)) < 1e-12
        assert np.abs(dk.sum(axis=1)).max() < 1e-12


# ------------------------------------------------------------ P9 library routine
@pytest.mark.parametrize("B,S,Hq,Hkv,D", [(1, 64, 2, 1, 16), (2, 100, 4, 2, 32), (1, 256, 4, 1, 64)])
@pytest.mark.parametrize("causal", [True, False])
def test_torch_float64_sdpa(oracle_mod, B, S, Hq, Hkv, D, causal):
    """Against torch's float64 CPU scaled_dot_product_attention with autograd
    (a library routine, written independently of the oracle)."""
    qb, kb, vb, dob = make_inputs(B, Hq, Hkv, S, D, seed=77 + S)
    sc = 1.0 / math.sqrt(D)
    q, k, v = (t.double().permute(0, 2, 1, 3).contiguous().requires_grad_() for t in (qb, kb, vb))
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=causal, scale=sc,
                                                         enable_gqa=True)
    o.backward(dob.double().permute(0, 2, 1, 3))
    ro, rl = oracle_mod.attn_fwd(qb, kb, vb, sc, causal)
    rdq, rdk, rdv, _ = oracle_mod.attn_bwd(qb, kb, vb, dob, sc, causal)
    tp = lambda t: t.detach().permute(0, 2, 1, 3).numpy()  # noqa: E731
    np.testing.assert_allclose(ro, tp(o), atol=1e-12)
    np.testing.assert_allclose(rdq, tp(q.grad), atol=1e-11)
    np.testing.assert_allclose(rdk, tp(k.grad), atol=1e-11)
    np.testing.assert_allclose(rdv, tp(v.grad), atol=1e-11)
    # LSE: logsumexp of the masked, scaled scores (torch's own logsumexp)
    G = Hq // Hkv
    s = sc * torch.einsum("bhid,bhjd->bhij", q.detach(), k.detach().repeat_interleave(G, 1))
    if causal:
        s = s.masked_fill(torch.ones(S, S, dtype=torch.bool).triu(1), float("-inf"))
    np.testing.assert_allclose(rl, torch.logsumexp(s, -1).numpy(), atol=1e-12)


# ------------------------------------------------------------ row samplers agree with full
def test_row_samplers_match_full(oracle_mod):
    B, S, Hq, Hkv, D = 2, 33, 6, 2, 8
    qb, kb, vb, dob = make_inputs(B, Hq, Hkv, S, D, seed=5)
    sc = 1 / math.sqrt(D)
    o, lse = oracle_mod.attn_fwd(qb, kb, vb, sc, True)
    dq, dk, dv, _ = oracle_mod.attn_bwd(qb, kb, vb, dob, sc, True)
    rows = [(0, 0, 0), (1, 5, 32), (0, 3, 17), (1, 1, 1)]
    ro, rl = oracle_mod.attn_fwd_rows(qb, kb, vb, sc, True, rows)
    rdq, _ = oracle_mod.attn_bwd_dq_rows(qb, kb, vb, dob, sc, True, rows)
    for n, (b, h, i) in enumerate(rows):
        np.testing.assert_allclose(ro[n], o[b, i, h], atol=1e-14)
        assert abs(rl[n] - lse[b, h, i]) < 1e-14
        np.testing.assert_allclose(rdq[n], dq[b, i, h], atol=1e-13)
    krows = [(0, 0, 0), (1, 1, 32), (0, 1, 16), (1, 0, 5)]
    rdk, rdv = oracle_mod.attn_bwd_dkdv_rows(qb, kb, vb, dob, sc, True, krows)
    for n, (b, kv, j) in enumerate(krows):
        np.testing.assert_allclose(rdk[n], dk[b, j, kv], atol=1e-13)
        np.testing.assert_allclose(rdv[n], dv[b, j, kv], atol=1e-13)
