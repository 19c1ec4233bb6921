"""Plant a mistake in a copy of the oracle and check that a pin catches it.

Each mutant is a one-line textual change to oracle.c (a dropped term, a wrong
index or sign, a swapped operand), compiled to a temporary library on the CPU.
"""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "visibility_off_by_one": ("j * p->s_c1 + p->l_c1 - 1 <= i; ++j", "j * p->s_c1 + p->l_c1 <= i; ++j"),
    "head_group_mapping": ("int h = g * G + hh;\n        double lse = lse_over(", "int h = hh * p->h_kv + g;\n        double lse = lse_over("),
    "lse_drops_max": ("return m + log(s);", "return log(s);"),
    "coarse_correction_dropped": ("lse_over(p, q, kc2, nv2, i, g * G + hh, g, z) + log(4.0);", "lse_over(p, q, kc2, nv2, i, g * G + hh, g, z);"),
    "coarse_stride": ("c.s_c1 = 4 * p->s_c1;", "c.s_c1 = 2 * p->s_c1;"),
    "coarse_length": ("c.l_c1 = 4 * p->l_c1;", "c.l_c1 = 2 * p->l_c1;"),
    "score_scale_dropped": ("z[j] = p->scale * dot;", "z[j] = dot;"),
    "pool_window_literal_start": ("return k_first <= b_last && k_last >= b_first;", "return k_first >= b_first && k_first <= b_last;"),
    "ties_to_higher_block": ("return (a->b > c->b) - (a->b < c->b);", "return (a->b < c->b) - (a->b > c->b);"),
    "local_set_too_wide": ("b > bi - p->n_local", "b >= bi - p->n_local"),
    "k_excludes_forced": ("r < nr && count < p->k; ++r", "r < nr && r < p->k; ++r"),
    "attention_not_inclusive": ("t < (idx[r] + 1) * p->B && t <= i; ++t", "t < (idx[r] + 1) * p->B && t < i; ++t"),
    "values_from_keys": ("const uint16_t* vr = v +", "const uint16_t* vr = k +"),
    "mean_divides_by_stride": ("orc_bf16_round(s / p->l_c1)", "orc_bf16_round(s / p->s_c1)"),
    "ties_away_from_zero": ("else if (rem == 0.5 && fmod(lo, 2.0) != 0.0) r = lo + 1.0;", "else if (rem == 0.5) r = lo + 1.0;"),
    "bwd_drops_D": ("double ds = P[a] * (dp - D);", "double ds = P[a] * dp;"),
    "bwd_dk_unscaled": ("dk_acc[kv + c] += p->scale * ds * bf16_value(qr[c]);", "dk_acc[kv + c] += ds * bf16_value(qr[c]);"),
    "bwd_dv_from_ds": ("dv_acc[kv + c] += P[a] * bf16_value(dor[c]);", "dv_acc[kv + c] += ds * bf16_value(dor[c]);"),
    "kernel_window_short": ("t < j * p->s_c1 + p->l_c1; ++t", "t < j * p->s_c1 + p->l_c1 - 1; ++t"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    c = tmp_path / "oracle_mut.c"
    c.write_text(mutated)
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c), "-o", str(so), "-lm"])
    handle = oracle.load(str(so))
    caught = []
    with oracle.use(handle):
        for pin in pins.ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
