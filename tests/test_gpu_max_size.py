"""GPU parity at the largest size the ABI accepts.

The header admits B * S * max(Hq, Hkv) * D < 2^31 elements per tensor.  This
test runs B = 8191, S = 128, Hq = 16, Hkv = 8, D = 128 (2,147,221,504
elements in q, 4.3 GB, about 36 GB on the device with the gradients and the
workspace): every element offset, TMA coordinate, grid size and workspace
section is at its largest, while each (b, kv head) unit stays small enough
for the oracle to check in full.  Inputs are drawn on the GPU (seeded); the
units the oracle checks are copied back bit for bit.  The forward has one
query tile per (b, h) and the backward 65,528 CTAs.
"""
import math

import pytest
import torch

import causal_attention_fwd_b200 as aa

from gpu_util import assert_close

pytestmark = pytest.mark.gpu

B, S, HQ, HKV, D = 8191, 128, 16, 8, 128


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()


def test_largest_accepted_problem_matches_oracle_on_whole_units(oracle_mod):
    assert B * S * max(HQ, HKV) * D < 2 ** 31 <= (B + 1) * S * max(HQ, HKV) * D
    dev = torch.device("cuda:0")
    g = torch.Generator(device=dev)
    g.manual_seed(9100)
    shape_q, shape_k = (B, S, HQ, D), (B, S, HKV, D)
    q = torch.randn(shape_q, generator=g, device=dev, dtype=torch.bfloat16)
    k = torch.randn(shape_k, generator=g, device=dev, dtype=torch.bfloat16)
    v = torch.randn(shape_k, generator=g, device=dev, dtype=torch.bfloat16)
    do = torch.randn(shape_q, generator=g, device=dev, dtype=torch.bfloat16)
    sc = 1.0 / math.sqrt(D)
    o, lse = aa.attention_forward(q, k, v, causal=True, scale=sc)
    dq, dk, dv = aa.attention_backward(q, k, v, o, lse, do, causal=True, scale=sc)
    aa.check_status()
    torch.cuda.synchronize()
    G = HQ // HKV
    # first and last units (smallest and largest offsets) and two in between
    for b, kv in ((0, 0), (B - 1, HKV - 1), (B // 2, 3), (4095, 7)):
        hs = slice(kv * G, (kv + 1) * G)
        unit = (q[:, :, hs], k[:, :, kv:kv + 1], v[:, :, kv:kv + 1], do[:, :, hs])
        qu, ku, vu, dou = (t[b:b + 1].contiguous().cpu() for t in unit)
        ro, rl = oracle_mod.attn_fwd(qu, ku, vu, sc, True)
        rdq, rdk, rdv, _ = oracle_mod.attn_bwd(qu, ku, vu, dou, sc, True)
        got = (o[b:b + 1, :, hs].cpu(), lse[b:b + 1, hs].cpu(), dq[b:b + 1, :, hs].cpu(),
               dk[b:b + 1, :, kv:kv + 1].cpu(), dv[b:b + 1, :, kv:kv + 1].cpu())
        print(assert_close(*got, ro, rl, rdq, rdk, rdv, tag=f"max size unit b={b} kv={kv}", S=S))
