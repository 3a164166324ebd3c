"""The oracle's pins catch plausible mistakes (CPU only).

Each case copies ``oracle/attn_oracle.c``, plants one mistake by a textual
replacement (a dropped term, a wrong sign, a wrong index, a transposed operand,
an off-by-one mask), compiles the copy into a temporary library and runs the
pin checks of ``test_oracle_pins.py`` against it.  At least one pin must fail
for every mutant; the unmodified source must pass them all.
"""
import os
import subprocess

import pytest

import oracle.oracle as orc
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(orc.__file__), "attn_oracle.c")

MUTANTS = {
    "score_without_scale": ("p[j] = z->scale * dot(", "p[j] = dot("),
    "gqa_head_modulo": ("const int kv = h / (z->Hq / z->Hkv);\n    const double* qi",
                        "const int kv = h % z->Hkv;\n    const double* qi"),
    "mask_hides_diagonal": ("if (z->causal && j > i) {", "if (z->causal && j >= i) {"),
    "mask_always_on": ("if (z->causal && j > i) {", "if (j > i) {"),
    "lse_in_log2": ("*lse = m + log(l);", "*lse = m + log2(l);"),
    "softmax_unnormalised": ("for (int j = 0; j < z->S; ++j) p[j] /= l;", "(void)0;"),
    "ds_sign_flipped": ("ds[j] = p[j] * (dp - dr);", "ds[j] = p[j] * (dr - dp);"),
    "dk_wrong_operand": ("dkj[d] += ds[j] * qi[d];", "dkj[d] += ds[j] * doi[d];"),
    "dv_uses_ds": ("dvj[d] += p[j] * doi[d];", "dvj[d] += ds[j] * doi[d];"),
    "dq_without_scale": ("for (int d = 0; d < D; ++d) dqi[d] *= scale;", "(void)0;"),
    "dk_without_scale": ("dk[at(&z, b, j, kv, Hkv, d)] *= scale;", "(void)0;"),
    "rowsum_wrong_operand": ("const double dr = dot(doi, o_row, z->D);",
                             "const double dr = dot(doi, doi, z->D);"),
    "dq_rows_wrong_index": ("for (int d = 0; d < D; ++d) out[d] += ds[j] * kj[d];",
                      "for (int d = 0; d < D; ++d) out[d] += ds[j] * kj[0];"),
    "dkdv_rows_no_scale": ("exp(scale * dot(qi, kj, D) - lse_u[i])", "exp(dot(qi, kj, D) - lse_u[i])"),
    "dkdv_rows_sign": ("pij * (dot(doi, vj, D) - dr_u[i])", "pij * (dr_u[i] - dot(doi, vj, D))"),
    "dkdv_rows_mask": ("if (causal && j > i) continue;", "if (causal && j >= i) continue;"),
}

CHECKS = [
    (pins.test_hand_worked_example, dict(mode="causal")),
    (pins.test_hand_worked_example, dict(mode="noncausal")),
    (pins.test_central_differences, dict(Hq=2, Hkv=1, S=3, D=4, causal=True)),
    (pins.test_central_differences, dict(Hq=2, Hkv=1, S=3, D=4, causal=False)),
    (pins.test_rows_sum_to_one_and_causal_zeros, {}),
    (pins.test_first_row_is_v0, {}),
    (pins.test_identical_keys_prefix_mean, {}),
    (pins.test_key_shift_invariance, {}),
    (pins.test_gqa_equals_expanded_mha, {}),
    (pins.test_rowsum_identity_and_zero_sum, {}),
    (pins.test_torch_float64_sdpa, dict(B=1, S=64, Hq=2, Hkv=1, D=16, causal=True)),
    (pins.test_row_samplers_match_full, {}),
]


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o",
                           str(so), str(c), "-lm"])
    return orc.Oracle(str(so))


def _failures(o):
    failed = []
    for fn, kw in CHECKS:
        try:
            fn(o, **kw)
        except AssertionError:
            failed.append(fn.__name__)
    return failed


def test_unmodified_source_passes(tmp_path):
    assert _failures(_build(tmp_path, "clean", open(SRC).read())) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    failed = _failures(_build(tmp_path, name, src.replace(old, new)))
    assert failed, f"mutant {name} passed every pin"
