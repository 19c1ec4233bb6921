"""Plant a mistake in a copy of the oracle and check that a pin catches it.

Each mutant is a one-line textual change to oracle.c (a dropped term, a wrong
index or sign, a swapped operand), compiled to a temporary library on the CPU.
The pins run against each mutant in a child process: a mutant that writes out
of bounds (k_excludes_forced fills more than k slots) may corrupt memory, and
that must not take the test session down with it.
"""
import os
import subprocess
import sys

import pytest

import oracle

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")
TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)

# Runs every pin against the library in argv[1] until one fails; prints the
# name of each pin that failed its assertions.
CHILD = """
import sys
sys.path[:0] = [%r, %r]
import oracle, pins
with oracle.use(oracle.load(sys.argv[1])):
    for pin in pins.ALL_PINS:
        try:
            pin()
        except AssertionError:
            print("CAUGHT", pin.__name__, flush=True)
            break
"""

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
    "bf16_overflow_edge": ("if (y > 3.3895313892515355e38) f = INFINITY;", "if (y >= 3.3895313892515355e38) f = INFINITY;"),
    "empty_list_divides_by_zero": ("orow[c] = ntok ? orow[c] / L : 0.0;", "orow[c] = orow[c] / L;"),
    "shared_padding_not_zero": ("so[j] = j < nv ? shared[j] : 0.0;", "so[j] = j < nv ? shared[j] : 1.0;"),
    "cmp_drops_own_block": ("co[b] = b <= bi ? cmp[b] : -INFINITY;", "co[b] = b < bi ? cmp[b] : -INFINITY;"),
    "blocks_floor_not_ceil": ("int n_blk = (n + p->B - 1) / p->B;\n    int G = p->h_q / p->h_kv;", "int n_blk = n / p->B + 1;\n    int G = p->h_q / p->h_kv;"),
    "batch_row_stride_dropped": ("orc_select_row(p, cmp, i, idx_out + ((size_t)r * p->h_kv + g) * p->k);", "orc_select_row(p, cmp, i, idx_out + ((size_t)r + g) * p->k);"),
}


def _mutant_source(name):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    return src.replace(old, new, 1)


@pytest.fixture(scope="module")
def outcomes(tmp_path_factory):
    """Compile every mutant and run the pins against each in its own child
    process, a few at a time.  name -> (caught pin names, return code, stderr)."""
    d = tmp_path_factory.mktemp("mutants")
    jobs = []
    for name in sorted(MUTANTS):
        try:
            src = _mutant_source(name)
        except AssertionError as e:
            jobs.append((name, None, str(e)))
            continue
        c = d / (name + ".c")
        c.write_text(src)
        so = d / ("lib" + name + ".so")
        subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(c),
                               "-o", str(so), "-lm"])
        jobs.append((name, so, None))
    env = dict(os.environ, OMP_NUM_THREADS="2")
    width = max(1, min(8, (os.cpu_count() or 2) // 2))
    out, running = {}, []
    pending = list(jobs)
    while pending or running:
        while pending and len(running) < width:
            name, so, err = pending.pop(0)
            if so is None:
                out[name] = ([], None, err)
                continue
            proc = subprocess.Popen([sys.executable, "-c", CHILD % (ROOT, TESTS), str(so)],
                                    stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True,
                                    env=env)
            running.append((name, proc))
        if running:
            name, proc = running.pop(0)
            stdout, stderr = proc.communicate(timeout=600)
            caught = [ln.split()[1] for ln in stdout.splitlines() if ln.startswith("CAUGHT ")]
            out[name] = (caught, proc.returncode, stderr)
    return out


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, outcomes):
    caught, rc, stderr = outcomes[name]
    assert rc is not None, stderr                 # the mutation site exists
    # a pin's failed assertion, or else the mutant crashing the oracle under a pin
    assert caught or rc < 0, f"no pin caught mutant {name}: {stderr[-2000:]}"
