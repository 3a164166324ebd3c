"""GPU parity of the fused rotary embedding (RoPE) against the oracle.

The oracle side is oracle_rope (fp64) followed by the oracle's attention: the
rotated q and k are the attention's inputs and are stored in bf16, so the
test rounds the oracle's fp64 rotation to bf16 once (gpu_util.bf16_rn_from_f64)
before the oracle's attention, and the gradients with respect to the
unrotated inputs come back through oracle_rope(inverse=True).  The kernels
compute the rotation in fp64 and round once as well, so the rotated Q and K
they write are compared bit for bit; O, LSE and the gradients use the tolerances of
the other parity tests.  Shapes: the axiomlm Quick Start's own RoPE example
(q of shape (2, 1024, 12, 64), k of shape (2, 1024, 4, 64)), a ragged length,
head dim 128, and the non-causal mask.
"""
import math

import numpy as np
import pytest
import torch

import causal_attention_fwd_b200 as aa
from causal_attention_fwd_b200.synthetic import make_inputs

from gpu_util import assert_close, bf16_rn_from_f64

pytestmark = pytest.mark.gpu

BASE = 10000.0


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from causal_attention_fwd_b200 import build

    build.build()


def test_table_matches_fp64_definition():
    S, D = 4096, 128
    cs = aa.rope_table(S, D, BASE).cpu().numpy()
    s = np.arange(S, dtype=np.float64)[:, None]
    theta = BASE ** (-2.0 * np.arange(D // 2) / D)[None, :]
    assert np.abs(cs[..., 0] - np.cos(s * theta)).max() <= 1e-11
    assert np.abs(cs[..., 1] - np.sin(s * theta)).max() <= 1e-11


def test_rotation_is_the_correctly_rounded_oracle_rotation(oracle_mod):
    B, S, H, D = 2, 333, 3, 64
    g = torch.Generator().manual_seed(12)
    x = torch.randn((B, S, H, D), generator=g).to(torch.bfloat16)
    dev = torch.device("cuda:0")
    cs = aa.rope_table(S, D, BASE, device=dev)
    y = torch.empty_like(x, device=dev)
    sp = aa.binding._stream(None, dev)
    assert aa.axis_attn_rope(x.to(dev).data_ptr(), y.data_ptr(), cs.data_ptr(), B, S, H, D, 0, sp) == 0
    want = bf16_rn_from_f64(oracle_mod.rope(x, BASE))
    assert torch.equal(y.cpu().view(torch.int16), want.view(torch.int16))
    # the transposed rotation (fp32 math) brings it back to within bf16 rounding
    z = torch.empty_like(y)
    assert aa.axis_attn_rope(y.data_ptr(), z.data_ptr(), cs.data_ptr(), B, S, H, D, 1, sp) == 0
    back = oracle_mod.rope(want, BASE, inverse=True)
    assert np.abs(z.cpu().double().numpy() - back).max() <= 2.0 ** -8 * np.abs(back).max()
    aa.check_status()


SHAPES = [
    # B, Hq, Hkv, S, D, causal
    (2, 12, 4, 1024, 64, True),    # the axiomlm Quick Start's apply_rope example
    (1, 4, 2, 300, 64, True),
    (2, 2, 1, 257, 128, True),
    (1, 4, 4, 200, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,S,D,causal", SHAPES)
@pytest.mark.parametrize("det", [False, True])
def test_rope_attention_matches_oracle(oracle_mod, B, Hq, Hkv, S, D, causal, det):
    q, k, v, do = make_inputs(B, Hq, Hkv, S, D, seed=5000 + S + D + Hq)
    sc = 1.0 / math.sqrt(D)
    dev = torch.device("cuda:0")
    cs = aa.rope_table(S, D, BASE, device=dev)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    o, lse, q_rot, k_rot = aa.attention_forward_rope(qd, kd, vd, cs, causal=causal, scale=sc)
    dq, dk, dv = aa.attention_backward_rope(q_rot, k_rot, vd, cs, o, lse, dod, causal=causal, scale=sc,
                                            deterministic=det)
    aa.check_status()
    # oracle: rotate in fp64, store in bf16, attend, gradients back through R^T
    qr = bf16_rn_from_f64(oracle_mod.rope(q, BASE))
    kr = bf16_rn_from_f64(oracle_mod.rope(k, BASE))
    assert torch.equal(k_rot.cpu().view(torch.int16), kr.view(torch.int16))
    assert torch.equal(q_rot.cpu().view(torch.int16), qr.view(torch.int16))
    ro, rl = oracle_mod.attn_fwd(qr, kr, v, sc, causal)
    rdq_r, rdk_r, rdv, _ = oracle_mod.attn_bwd(qr, kr, v, do, sc, causal)
    rdq = oracle_mod.rope(rdq_r, BASE, inverse=True)
    rdk = oracle_mod.rope(rdk_r, BASE, inverse=True)
    print(assert_close(o.cpu(), lse.cpu(), dq.cpu(), dk.cpu(), dv.cpu(), ro, rl, rdq, rdk, rdv,
                       tag=f"rope B{B} Hq{Hq} Hkv{Hkv} S{S} D{D} c{int(causal)} det{int(det)}", S=S))
