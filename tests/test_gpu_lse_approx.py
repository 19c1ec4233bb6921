"""The LSE approximation (pass 1 over the coarse kernels K^C2) against the
fp64 oracle in the same mode: coarse compression bit for bit, the scores and
their log-sum-exp, and whole prefills."""
import numpy as np
import pytest
import torch

import oracle
from test_gpu_prefill import _rows, check_sequence, run_prefill
from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2, synth
from trainable_block_sparse_mean_b200.workloads import to_dev, to_host_bits

pytestmark = pytest.mark.gpu

SCORE_REL = 2e-5   # fp32 tensor-core dot products + fp32 softmax vs fp64


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    infv2.lib()


@pytest.mark.parametrize("n,h_kv", [(127, 2), (128, 1), (300, 2), (2048, 1), (4177, 2)])
def test_compress_k2_bit_exact(n, h_kv):
    sh = synth.Shape(n=n, h_q=2 * h_kv, h_kv=h_kv)
    d = synth.make_prefill(sh, seed=n)
    p = infv2.params_of(sh)
    kc2 = infv2.infv2_compress_k2(p, to_dev(d["k"]))
    torch.cuda.synchronize()
    want = oracle.compress_k2(oracle.params(sh), d["k"])
    got = to_host_bits(kc2) if kc2.numel() else np.zeros((0, h_kv, 128), np.uint16)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


@pytest.mark.parametrize("n,h_q,h_kv,q_begin,q_len", [
    (2048, 4, 1, 0, 2048),        # G=4
    (3000, 32, 2, 0, 3000),       # G=16, ragged tail
    (3000, 32, 2, 100, 1333),     # a chunk that straddles the first coarse row (127)
    (3000, 32, 2, 1000, 1000),    # a chunk past it
    (700, 8, 1, 0, 700),          # G=8
    (600, 2, 2, 0, 600),          # G=1
    (900, 4, 2, 0, 900),          # G=2
    (20000, 16, 2, 19000, 1000),  # several coarse tiles
    (100, 4, 1, 0, 100),          # shorter than one coarse kernel: every row exact
])
def test_block_scores_approx_match_oracle(n, h_q, h_kv, q_begin, q_len):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=8)
    d = synth.make_prefill(sh, seed=n + h_q + 1)
    p = infv2.params_of(sh)
    op = oracle.params(sh, lse_approx=1)
    kd = to_dev(d["k"])
    kc1 = infv2.infv2_compress_k(p, kd)
    kc2 = infv2.infv2_compress_k2(p, kd)
    ld = infv2.shared_ld(n)
    slse = torch.full((h_q, q_len), 7.0, device="cuda")
    s = infv2.infv2_block_scores_approx(p, to_dev(d["q"]), kc1, kc2, n, q_begin, q_len, ld=ld,
                                        score_lse=slse)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    s, slse = s.cpu().numpy(), slse.cpu().numpy()
    rng = np.random.default_rng(n)
    rows = np.unique(np.concatenate([np.array([q_begin, 126, 127, 128, 190, 191, q_begin + q_len - 1]),
                                     rng.integers(q_begin, q_begin + q_len, 40)]))
    rows = rows[(rows >= q_begin) & (rows < q_begin + q_len)].astype(np.int32)
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows, want_shared=True, want_score_lse=True)
    for r, i in enumerate(rows):
        nv = oracle.visible_kernels(op, i)
        for g in range(h_kv):
            want = ref["shared"][r, g, :nv]
            got = s[g, i - q_begin, :nv]
            err = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
            assert err.max(initial=0) <= SCORE_REL, (i, g, err.max(), int(err.argmax()))
        lw, lg = ref["score_lse"][r], slse[:, i - q_begin]
        if nv == 0:
            assert np.all(np.isneginf(lg))
        else:
            assert np.allclose(lg, lw, rtol=0, atol=2e-5), (i, lg - lw)


@pytest.mark.parametrize("n,h_q,h_kv,k", [(5000, 32, 2, 16), (9000, 16, 2, 64), (3000, 8, 1, 8)])
def test_prefill_approx_matches_oracle(n, h_q, h_kv, k):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k, n_needles=8)
    data = synth.make_prefill(sh, seed=9)
    dev = run_prefill(sh, data, [0, n], lse_approx=1)
    check_sequence(sh, data, dev, 0, n, _rows(n, 300, 2), dense=False, lse_approx=1)


def test_decode_rejects_the_approximation():
    p = infv2.params(32, 2, lse_approx=1)
    import ctypes
    size = ctypes.c_size_t()
    assert infv2.lib().infv2_decode_workspace_size(ctypes.byref(p), 4, 4096, ctypes.byref(size)) == infv2.ERR_UNSUPPORTED


@pytest.mark.slow
def test_prefill_approx_128k_sampled():
    """The 128k workload with the approximation: sampled rows against the
    oracle in the same mode."""
    sh = synth.CONFIGS["prefill_128k"]["shape"]
    data = synth.make_prefill(sh, seed=0)
    dev = run_prefill(sh, data, [0, sh.n], lse_approx=1)
    check_sequence(sh, data, dev, 0, sh.n, _rows(sh.n, 200, 3), dense=False, lse_approx=1)
