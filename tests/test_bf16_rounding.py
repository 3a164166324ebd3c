"""CPU pin of the test-side fp64 -> bf16 rounding (gpu_util.bf16_rn_from_f64)
that turns the oracle's fp64 rotary embedding into the bf16 inputs of the
oracle's attention: it must agree with torch's round-to-nearest-even on every
value that float32 holds exactly, and round exact ties to even."""
import numpy as np
import torch

from gpu_util import bf16_rn_from_f64


def test_matches_torch_on_float32_values():
    g = np.random.default_rng(1)
    x32 = np.concatenate([g.standard_normal(200000), g.uniform(-1e3, 1e3, 50000),
                          g.standard_normal(50000) * 1e-20]).astype(np.float32)
    got = bf16_rn_from_f64(x32.astype(np.float64))
    ref = torch.from_numpy(x32).to(torch.bfloat16)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_ties_go_to_even_and_sticky_bits_break_ties():
    one = 1.0
    ulp = 2.0 ** -7  # bf16 spacing in [1, 2)
    vals = np.array([one + ulp / 2, one + 3 * ulp / 2, one + ulp / 2 + 2.0 ** -40, one + ulp / 2 - 2.0 ** -40,
                     -(one + ulp / 2), 2.0 - ulp / 4])
    want = np.array([one, one + 2 * ulp, one + ulp, one, -one, 2.0])  # last: a quarter ulp below 2 rounds up
    got = bf16_rn_from_f64(vals).double().numpy()
    assert np.array_equal(got, want)


def test_values_between_float32_neighbours_round_once():
    # x lies just above a bf16 tie by less than a float32 ulp: one rounding
    # from fp64 goes up, a detour through float32 would land on the tie and
    # go to even (down)
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert float(bf16_rn_from_f64(np.array([x]))[0]) == 1.0 + 2.0 ** -7
    assert float(torch.tensor([x], dtype=torch.float64).float().to(torch.bfloat16)[0]) == 1.0
