"""The synthetic needles as a sanity figure (not parity): the benchmark's
needle_recall counting rule on a hand example, and the oracle's selection
finding every planted needle on a small needle workload; the closed form of
the score kernel's exponential count."""
import numpy as np

import bench
import oracle
from trainable_block_sparse_mean_b200 import synth


def test_needle_recall_counting_rule():
    # two kv heads, three needles; a span starting at 48 crosses into block 1
    needles = [(500, 64), (900, 48), (700, 128)]
    sel = np.full((2, 3, 4), -1, np.int32)
    sel[0, 0, :2] = [0, 1]          # needle 0 sits in block 1: found on head 0
    sel[1, 0, :2] = [0, 2]          # not on head 1
    sel[0, 1, :1] = [1]             # span 48..79 touches blocks 0 and 1: found
    sel[1, 1, :1] = [0]             # found through block 0
    sel[0, 2, :2] = [0, 3]          # span 128..159 is block 2: missed on both heads
    out = bench.needle_recall(sel, needles)
    assert out == {"found": 3, "total": 6, "recall": 0.5}
    assert bench.needle_recall(sel[:, :0], [])["recall"] is None


def test_oracle_finds_every_planted_needle():
    sh = synth.Shape(n=8192, h_q=32, h_kv=2, k=16, n_needles=24)
    data = synth.make_prefill(sh, seed=1)
    assert len(data["needles"]) == 24
    rows = np.array([t for t, _ in data["needles"]], np.int32)
    out = oracle.prefill_rows(oracle.params(sh), data["q"], data["k"], data["v"], rows)
    rec = bench.needle_recall(out["idx"].transpose(1, 0, 2), data["needles"])
    assert rec["recall"] == 1.0, rec


def test_score_exp_figures_closed_form():
    # one exponential per (head, visible kernel) in each pass; kernel j is
    # visible to query i when 16j + 31 <= i
    n, h_q = 4100, 8
    vis = sum((i - 31) // 16 + 1 for i in range(31, n))
    f = bench.score_exp_figures(n, h_q, 2.0, 148, 1965.0)
    assert f["exp_per_step"] == 2 * h_q * vis
    assert abs(f["exp_per_s"] - 2 * h_q * vis / 2e-3) < 1.0
    assert f["mufu_peak_per_s"] == 16 * 148 * 1965e6
    assert abs(f["mufu_frac"] - 0.75 * f["exp_per_s"] / f["mufu_peak_per_s"]) < 1e-4
    big = bench.score_exp_figures(131072, 32, 1.0, 148, 1965.0)["exp_per_step"]
    assert abs(big - 3.43e10) / 3.43e10 < 0.01
