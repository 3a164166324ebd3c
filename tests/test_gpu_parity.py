"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small shapes are compared element by element over every output; the shape
fuzz spans several tiles, ragged tails (S not a multiple of 64/128), S = 1,
GQA group sizes 1..8, both head dims and both mask modes.  The five named
workloads run at their full sizes in the launch configuration the benchmark
times; the three large ones are checked on sampled rows that the oracle
computes one by one (160 query rows for O, LSE, dQ; about 30 key rows in each
of two (b, kv) units for dK, dV).
"""
import math

import numpy as np
import pytest
import torch

from causal_attention_fwd_b200.synthetic import WORKLOADS, make_inputs, workload_inputs

from gpu_util import assert_close, rel_l2, run_gpu, TOL_GRAD, TOL_LSE, TOL_O, max_abs, f64

pytestmark = pytest.mark.gpu

FUZZ = [
    # B, Hq, Hkv, S, D, causal
    (1, 1, 1, 1, 64, True),
    (1, 2, 1, 2, 128, True),
    (1, 1, 1, 17, 64, False),
    (2, 4, 2, 127, 64, True),
    (1, 3, 1, 128, 128, True),
    (3, 2, 2, 129, 64, True),
    (1, 8, 1, 255, 128, False),
    (2, 4, 4, 256, 64, False),
    (1, 4, 1, 257, 128, True),
    (2, 6, 3, 384, 64, True),
    (1, 2, 2, 640, 128, True),
    (1, 8, 2, 1000, 64, True),
    (2, 2, 1, 1000, 128, False),
    (1, 16, 2, 513, 64, False),
    (1, 4, 2, 777, 128, True),
    # more work items than SMs: every CTA of the persistent forward walks several
    # items, some without a second query tile (S = 300: rows 256-299 are one tile)
    (8, 40, 8, 300, 64, True),
    (4, 40, 5, 300, 128, False),
]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()


@pytest.mark.parametrize("B,Hq,Hkv,S,D,causal", FUZZ)
def test_fuzz_full_outputs(oracle_mod, B, Hq, Hkv, S, D, causal):
    seed = 2000 + B * 7 + Hq * 13 + S + D + int(causal)
    q, k, v, do = make_inputs(B, Hq, Hkv, S, D, seed)
    sc = 1.0 / math.sqrt(D)
    got = run_gpu(q, k, v, do, causal, sc)
    ro, rl = oracle_mod.attn_fwd(q, k, v, sc, causal)
    rdq, rdk, rdv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, causal)
    print(assert_close(*got, ro, rl, rdq, rdk, rdv, tag=f"B{B} Hq{Hq} Hkv{Hkv} S{S} D{D} c{int(causal)}",
                       S=S))


@pytest.mark.parametrize("name", ["tiny", "gpt2s_gqa"])
def test_small_workloads_full(oracle_mod, name):
    w = WORKLOADS[name]
    q, k, v, do = workload_inputs(w)
    got = run_gpu(q, k, v, do, w.causal, w.scale)
    ro, rl = oracle_mod.attn_fwd(q, k, v, w.scale, w.causal)
    rdq, rdk, rdv, _ = oracle_mod.attn_bwd(q, k, v, do, w.scale, w.causal)
    print(assert_close(*got, ro, rl, rdq, rdk, rdv, tag=name))


def _sample_rows(w, n, seed, heads):
    g = np.random.default_rng(seed)
    rows = [(0, 0, 0), (w.B - 1, heads - 1, w.S - 1)]
    # rows at and around tile edges, plus random ones
    for i in (63, 64, 127, 128, 129, w.S // 2):
        rows.append((int(g.integers(w.B)), int(g.integers(heads)), min(i, w.S - 1)))
    while len(rows) < n:
        rows.append((int(g.integers(w.B)), int(g.integers(heads)), int(g.integers(w.S))))
    return rows


@pytest.mark.parametrize("name", ["llm1b", "llm8b_gqa", "longseq"])
def test_large_workloads_sampled(oracle_mod, name):
    w = WORKLOADS[name]
    q, k, v, do = workload_inputs(w)
    o, lse, dq, dk, dv = run_gpu(q, k, v, do, w.causal, w.scale)
    for t in (o, lse, dq, dk, dv):
        assert torch.isfinite(t.float()).all()
    qrows = _sample_rows(w, 160, 7, w.Hq)
    ro, rl = oracle_mod.attn_fwd_rows(q, k, v, w.scale, w.causal, qrows)
    rdq, _ = oracle_mod.attn_bwd_dq_rows(q, k, v, do, w.scale, w.causal, qrows)
    go = np.stack([f64(o[b, i, h]) for b, h, i in qrows])
    gl = np.array([float(lse[b, h, i]) for b, h, i in qrows])
    gdq = np.stack([f64(dq[b, i, h]) for b, h, i in qrows])
    # key rows in two (b, kv) units: the first unit over the whole key range
    # (key 0 sums over every query row: the longest dK/dV accumulation), the
    # second, for the longest sequence, among the last 1024 keys (their dK/dV
    # need the oracle's statistics of fewer query rows).  The oracle's cost is
    # the statistics of the unit's query rows, not the number of key rows, so
    # each unit samples 24 random keys besides the tile edges.
    g = np.random.default_rng(11)
    krows = []
    for unit, lo in (((0, 0), 0), ((w.B - 1, w.Hkv - 1), w.S - 1024 if w.S > 8192 else 0)):
        js = [int(j) for j in g.integers(lo, w.S, 24)] + [w.S - 1, max(lo, w.S - 129)]
        if lo == 0:
            js += [0, 127, 128]
        krows += [(unit[0], unit[1], j) for j in js]
    rdk, rdv = oracle_mod.attn_bwd_dkdv_rows(q, k, v, do, w.scale, w.causal, krows)
    gdk = np.stack([f64(dk[b, j, kv]) for b, kv, j in krows])
    gdv = np.stack([f64(dv[b, j, kv]) for b, kv, j in krows])
    msg = (f"{name}: O {max_abs(go, ro):.2e} LSE {max_abs(gl, rl):.2e} dQ {rel_l2(gdq, rdq):.2e} "
           f"dK {rel_l2(gdk, rdk):.2e} dV {rel_l2(gdv, rdv):.2e}")
    print(msg)
    assert max_abs(go, ro) <= TOL_O and max_abs(gl, rl) <= TOL_LSE, msg
    assert rel_l2(gdq, rdq) <= TOL_GRAD, msg
    assert rel_l2(gdk, rdk) <= TOL_GRAD and rel_l2(gdv, rdv) <= TOL_GRAD, msg


def test_prefix_mean_property_at_scale():
    """Identical keys make every causal row the mean of the visible V rows
    (a property that holds at any size), checked at the headline size."""
    w = WORKLOADS["llm1b"]
    q, k, v, _ = workload_inputs(w)
    k = k[:, :1].expand_as(k).contiguous()
    dev = torch.device("cuda:0")
    import causal_attention_fwd_b200 as aa

    o, lse = aa.attention_forward(q.to(dev), k.to(dev), v.to(dev), causal=True, scale=w.scale)
    aa.check_status()
    G = w.Hq // w.Hkv
    vm = torch.cumsum(v.double(), 1) / torch.arange(1, w.S + 1, dtype=torch.float64)[None, :, None, None]
    assert (o.cpu().double() - vm.repeat_interleave(G, 2)).abs().max() <= TOL_O
    # row i sees i+1 equal scores scale * q_i . k, so LSE_i = that score + ln(i+1)
    s_all = w.scale * torch.einsum("bshd,bhd->bhs", q.double(), k.double()[:, 0].repeat_interleave(G, 1))
    ref_lse = s_all + torch.log(torch.arange(1, w.S + 1, dtype=torch.float64))
    assert (lse.cpu().double() - ref_lse).abs().max() <= TOL_LSE


@pytest.mark.parametrize("S", list(range(1, 17)))
def test_short_sequences_over_seeds(oracle_mod, S):
    """Every short length, several seeds and shapes, against the per-S bounds
    (the measured worst case x 1.5; see gpu_util.GRAD_TOL_SHORT)."""
    for seed in range(3):
        for Hq, Hkv, D, causal in ((1, 1, 64, True), (4, 2, 64, True), (2, 1, 128, True), (4, 4, 64, False),
                                   (8, 2, 128, False)):
            q, k, v, do = make_inputs(1, Hq, Hkv, S, D, 7000 + 97 * seed + S)
            sc = 1.0 / math.sqrt(D)
            got = run_gpu(q, k, v, do, causal, sc)
            ro, rl = oracle_mod.attn_fwd(q, k, v, sc, causal)
            rdq, rdk, rdv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, causal)
            assert_close(*got, ro, rl, rdq, rdk, rdv, tag=f"S{S} seed{seed} Hq{Hq} Hkv{Hkv} D{D} c{int(causal)}",
                         S=S)


@pytest.mark.parametrize("D,causal", [(64, True), (64, False), (128, True)])
def test_rising_scores_move_the_running_max(oracle_mod, D, causal):
    """Scores that rise along the keys by about 6 (log2 units) per 64 keys:
    from the second kv tile on, the running max of a row moves in almost
    every tile, mostly because of the second half of the tile's columns.
    That drives the forward's rare paths: the O rescale, and the rescale of
    P and the partial row sum when the exponentials started with the old
    max.  Parity with the oracle as everywhere else."""
    B, Hq, Hkv, S = 1, 4, 2, 1000
    q, k, v, do = make_inputs(B, Hq, Hkv, S, D, 8100 + D + int(causal))
    sc = 1.0 / math.sqrt(D)
    # score_ij ~ scale * A * delta * j = 0.065 j natural-log units, ~12 in
    # log2 units per 128 keys (the rest of q, k stays random, smaller).  The
    # ramp's size sits in q (A = 512), not in k: a large k component would
    # make dQ = scale sum_j dS_ij K_j a cancellation (the dS_ij of a row sum
    # to zero) that amplifies the bf16 rounding of dS far beyond any bound.
    A = 512.0
    delta = 0.065 / (sc * A)
    q = q.float() * 0.3
    q[..., 0] = A
    k = k.float() * 0.3
    k[..., 0] = delta * torch.arange(S, dtype=torch.float32)[None, :, None]
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    got = run_gpu(q, k, v, do, causal, sc)
    ro, rl = oracle_mod.attn_fwd(q, k, v, sc, causal)
    rdq, rdk, rdv, _ = oracle_mod.attn_bwd(q, k, v, do, sc, causal)
    print(assert_close(*got, ro, rl, rdq, rdk, rdv, tag=f"rising D{D} c{int(causal)}", S=S))
