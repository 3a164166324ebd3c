"""Pins of the oracle's rotary position embedding (CPU only).

The axiomlm page names the calls (precompute_rope_frequencies, apply_rope)
but prints no formula; the oracle takes the complex-pair reading (see
``oracle_rope`` in attn_oracle.c).  Nothing here retypes that formula as its
own check: the pins are properties every correct implementation has (identity
at position 0, an inverse, norms per pair, dependence of q.k on the position
difference only), a closed form (a base chosen so that the second pair turns
by exactly a quarter turn per position), numpy's complex arithmetic on
adjacent pairs as a second formulation, and central differences of attention
applied after the rotation, whose gradient needs the transposed rotation.
The second half of the file plants mistakes in copies of the C source and
checks that a pin catches each one.
"""
import math
import os
import subprocess

import numpy as np
import pytest

import oracle.oracle as orc

RNG = np.random.default_rng(7)


def _x(B=1, S=5, H=2, D=8):
    return RNG.standard_normal((B, S, H, D))


def check_position_zero_is_identity(o):
    x = _x()
    y = o.rope(x)
    assert np.array_equal(y[:, 0], x[:, 0])
    assert not np.allclose(y[:, 1:], x[:, 1:])


def check_inverse_undoes(o):
    x = _x(S=9, D=16)
    assert np.allclose(o.rope(o.rope(x), inverse=True), x, atol=1e-12, rtol=0)
    assert np.allclose(o.rope(o.rope(x, inverse=True)), x, atol=1e-12, rtol=0)


def check_pair_norms_preserved(o):
    x = _x(S=7, D=8)
    y = o.rope(x)
    nx = np.hypot(x[..., 0::2], x[..., 1::2])
    ny = np.hypot(y[..., 0::2], y[..., 1::2])
    assert np.allclose(nx, ny, atol=1e-12, rtol=0)


def check_quarter_turn(o):
    # D = 4: the second pair turns by base^(-1/2) per position; base = (2/pi)^2
    # makes that exactly pi/2, so its pair goes (a, b) -> (-b, a) -> (-a, -b) -> ...
    x = np.zeros((1, 5, 1, 4))
    x[0, :, 0] = [0.3, -0.7, 1.25, -2.5]
    y = o.rope(x, base=(2.0 / math.pi) ** 2)
    a, b = 1.25, -2.5
    want = [(a, b), (-b, a), (-a, -b), (b, -a), (a, b)]
    for s in range(5):
        assert np.allclose(y[0, s, 0, 2:], want[s], atol=1e-12, rtol=0), (s, y[0, s, 0, 2:])
    # the first pair turns by one radian per position: at least its norm is kept
    assert np.allclose(np.hypot(y[0, :, 0, 0], y[0, :, 0, 1]), math.hypot(0.3, -0.7), atol=1e-12)


def check_relative_position(o):
    # <R_m q, R_n k> depends on m - n only: put the same q at every position
    # and the same k at every position
    S, D = 12, 16
    q = np.broadcast_to(RNG.standard_normal(D), (1, S, 1, D)).copy()
    k = np.broadcast_to(RNG.standard_normal(D), (1, S, 1, D)).copy()
    rq, rk = o.rope(q)[0, :, 0], o.rope(k)[0, :, 0]
    dots = rq @ rk.T
    for delta in range(-S + 1, S):
        d = np.diagonal(dots, offset=-delta)
        assert np.allclose(d, d[0], atol=1e-10, rtol=0), delta


def check_numpy_complex_pairs(o):
    # second formulation: adjacent pairs as numpy complex numbers times unit phasors
    B, S, H, D, base = 2, 6, 3, 8, 10000.0
    x = _x(B, S, H, D)
    z = x.reshape(B, S, H, D // 2, 2)
    zc = z[..., 0] + 1j * z[..., 1]
    ang = np.arange(S)[:, None] * base ** (-np.arange(0, D, 2) / D)[None, :]   # [S, D/2]
    rc = zc * np.exp(1j * ang)[None, :, None, :]
    want = np.stack([rc.real, rc.imag], axis=-1).reshape(B, S, H, D)
    assert np.allclose(o.rope(x, base=base), want, atol=1e-12, rtol=0)


def check_attention_gradient_through_rope(o):
    # f(q, k, v) = sum(W * O(rope(q), rope(k), v)): dq = rope^T(dq of the rotated q), same for k
    B, S, Hq, Hkv, D, sc = 1, 4, 2, 1, 4, 0.6
    q, k, v = _x(B, S, Hq, D), _x(B, S, Hkv, D), _x(B, S, Hkv, D)
    W = RNG.standard_normal((B, S, Hq, D))

    def f(q_, k_):
        out, _ = o.attn_fwd(o.rope(q_), o.rope(k_), v, sc, True)
        return float(np.sum(W * out))

    dqr, dkr, _, _ = o.attn_bwd(o.rope(q), o.rope(k), v, W, sc, True)
    dq, dk = o.rope(dqr, inverse=True), o.rope(dkr, inverse=True)
    h = 1e-6
    for arr, grad, which in ((q, dq, "q"), (k, dk, "k")):
        for idx in [(0, 1, 0, 1), (0, 3, arr.shape[2] - 1, 2), (0, 2, 0, 3)]:
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            fd = (f(p, k) - f(m, k)) / (2 * h) if which == "q" else (f(q, p) - f(q, m)) / (2 * h)
            assert abs(fd - grad[idx]) < 1e-6, (which, idx, fd, grad[idx])


CHECKS = [check_position_zero_is_identity, check_inverse_undoes, check_pair_norms_preserved,
          check_quarter_turn, check_relative_position, check_numpy_complex_pairs,
          check_attention_gradient_through_rope]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_rope_pin(oracle_mod, check):
    check(oracle_mod.oracle.default())


def test_rope_rejects_bad_sizes(oracle_mod):
    with pytest.raises(ValueError):
        oracle_mod.rope(np.zeros((1, 2, 1, 3)))            # odd D
    with pytest.raises(ValueError):
        oracle_mod.rope(np.zeros((1, 2, 1, 4)), base=0.0)  # no frequencies


# ------------------------------------------------------------------ mutants
SRC = os.path.join(os.path.dirname(orc.__file__), "attn_oracle.c")

MUTANTS = {
    "half_split_pairs": ("const double x0 = row[2 * p], x1 = row[2 * p + 1];\n"
                         "                    row[2 * p] = x0 * c - x1 * sn;\n"
                         "                    row[2 * p + 1] = x0 * sn + x1 * c;",
                         "const double x0 = row[p], x1 = row[p + D / 2];\n"
                         "                    row[p] = x0 * c - x1 * sn;\n"
                         "                    row[p + D / 2] = x0 * sn + x1 * c;"),
    "exponent_without_two": ("pow(base, -2.0 * p / D)", "pow(base, -1.0 * p / D)"),
    "inverse_ignored": ("const double sgn = inverse ? -1.0 : 1.0;", "const double sgn = 1.0;"),
    "position_off_by_one": ("sgn * (double)s * pow(", "sgn * (double)(s + 1) * pow("),
    "sine_sign": ("row[2 * p] = x0 * c - x1 * sn;", "row[2 * p] = x0 * c + x1 * sn;"),
}


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(c),
                           "-lm"])
    return orc.Oracle(str(so))


def _failures(o):
    failed = []
    for check in CHECKS:
        try:
            check(o)
        except AssertionError:
            failed.append(check.__name__)
    return failed


def test_unmodified_rope_passes(tmp_path):
    assert _failures(_build(tmp_path, "clean", open(SRC).read())) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_rope_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found"
    assert _failures(_build(tmp_path, name, src.replace(old, new))), f"mutant {name} passed every pin"
