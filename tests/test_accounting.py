"""The benchmark's accounting against brute force (CPU only).

The roofline figures divide algorithmic work by measured time, so the work
formulas in bench.py are pinned here against the method itself: the attention
FLOPs against the visible keys of the oracle's own block lists, and the score
chunking that bench.py mirrors against the library's workspace layout."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle  # noqa: E402
from trainable_block_sparse_mean_b200 import build as build_mod  # noqa: E402
from trainable_block_sparse_mean_b200 import infv2, synth  # noqa: E402


def test_attention_flops_match_the_oracle_lists():
    # every row of a 3000-token sequence: 4*d FLOP per (head, selected visible key)
    sh = synth.Shape(n=3000, h_q=4, h_kv=1, d=128, k=8)
    data = synth.make_prefill(sh, seed=2)
    rows = np.arange(sh.n, dtype=np.int32)
    ref = oracle.prefill_rows(oracle.params(sh), data["q"], data["k"], data["v"], rows)
    keys = 0
    for r, i in enumerate(rows):
        for b in (int(x) for x in ref["idx"][r, 0]):
            if b >= 0:
                keys += max(0, min(64 * b + 63, int(i)) - 64 * b + 1)
    assert bench.prefill_work(sh, sh.n)["attn"] == 4 * sh.d * sh.h_q * keys


def test_chunk_rows_mirror_the_library():
    # the S^shared piece of the prefill workspace is one chunk of chunk_rows rows
    build_mod.build()
    for name in ("prefill_32k", "prefill_128k"):
        sh = synth.CONFIGS[name]["shape"]
        p = infv2.params_of(sh)
        n = sh.n
        ws = infv2.infv2_prefill_workspace_size(p, [0, n])
        r256 = lambda x: (x + 255) // 256 * 256
        nc = infv2.num_kernels(p, n)
        rest = ws - r256(nc * p.h_kv * 256) - r256(p.h_kv * n * p.k * 4)
        rows = bench._chunk_rows(p, n)
        assert rest == r256(rows * p.h_kv * infv2.shared_ld(n) * 4), name
        assert rows % 128 == 0 or rows == n


def test_decode_bytes_match_the_oracle_lists():
    # one decode step at query position L per sequence: the visible K^C1 rows,
    # the K and V rows of the selected visible keys, and q, o, the new K and V
    sh = synth.Shape(n=0, h_q=4, h_kv=2, d=128, k=8)
    p = oracle.params(sh)
    lens = np.array([700, 1500, 3000], np.int32)
    kc1_rows = keys = 0
    for s, L in enumerate(int(x) for x in lens):
        sq = synth.make_decode_sequence(sh, L, 1, 4, s)
        q = np.zeros((L + 1, sh.h_q, sh.d), np.uint16)
        q[L] = sq["q_new"][0]
        ref = oracle.prefill_rows(p, q, sq["k"][:L + 1], sq["v"][:L + 1], np.array([L], np.int32))
        kc1_rows += sh.h_kv * oracle.visible_kernels(p, L)
        for g in range(sh.h_kv):
            for b in (int(x) for x in ref["idx"][0, g]):
                if b >= 0:
                    keys += min(64 * b + 63, L) - 64 * b + 1
    row = sh.d * 2
    want = kc1_rows * row + keys * 2 * row + len(lens) * (2 * sh.h_q * row + 2 * 2 * sh.h_kv * row)
    assert bench.decode_bytes(sh, lens) == want
