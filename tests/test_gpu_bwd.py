"""Backward of the block-sparse (and dense) attention against the fp64 oracle:
dq on every row, dk and dv summed over every query, on the oracle's own block
lists (and on lists with holes), with D taken from the GPU forward output as
the method's backward defines it."""
import numpy as np
import pytest
import torch

import oracle
import parity
from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2, synth
from trainable_block_sparse_mean_b200.workloads import to_dev, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    infv2.lib()


def _run(sh, d, idx_np, seed):
    """GPU forward + backward on the given lists (None: dense); oracle backward
    on the same lists with the GPU's forward output."""
    p = infv2.params_of(sh)
    op = oracle.params(sh)
    n = sh.n
    q, k, v = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    lse = torch.empty((sh.h_q, n), device="cuda")
    if idx_np is None:
        o = infv2.infv2_dense_attn(p, q, k, v, lse=lse)
        idx_dev = None
    else:
        idx_dev = torch.from_numpy(idx_np).cuda()
        o = infv2.infv2_sparse_attn(p, q, k, v, idx_dev, lse=lse)
    rng = np.random.default_rng(seed)
    d_o = synth.bf16_bits(rng.standard_normal((n, sh.h_q, sh.d)).astype(np.float32))
    dq, dk, dv = infv2.infv2_sparse_attn_bwd(p, q, k, v, idx_dev, o, lse, to_dev(d_o))
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    o_host = synth.bf16_to_f32(to_host_bits(o)).astype(np.float64)
    rows = np.arange(n, dtype=np.int32)
    if idx_np is None:
        idx_rows = np.full((n, sh.h_kv, sh.k), -1, np.int32)
        for i in range(n):
            nb = i // 64 + 1
            assert nb <= sh.k
            idx_rows[i, :, :nb] = np.arange(nb)
    else:
        idx_rows = idx_np.transpose(1, 0, 2).copy()
    rq, rk, rv = oracle.attend_bwd_rows(op, d["q"], d["k"], d["v"], d_o, rows, idx_rows, o_host)
    return (dq.cpu().numpy(), dk.cpu().numpy(), dv.cpu().numpy()), (rq, rk, rv)


@pytest.mark.parametrize("n,h_q,h_kv,k", [(2048, 4, 1, 8), (3001, 32, 2, 16), (1500, 16, 2, 4),
                                         (1300, 2, 2, 6), (1100, 4, 2, 5)])
def test_bwd_on_oracle_indices(n, h_q, h_kv, k):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k)
    d = synth.make_prefill(sh, seed=n)
    ref = oracle.prefill_rows(oracle.params(sh), d["q"], d["k"], d["v"], np.arange(n, dtype=np.int32))
    idx = ref["idx"].transpose(1, 0, 2).copy()        # [h_kv, n, k]
    got, want = _run(sh, d, idx, seed=1)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got, want):
        parity.assert_grads_close(g_, w_, name)


@pytest.mark.parametrize("n,h_q,h_kv", [(777, 4, 1), (1000, 32, 2), (64, 16, 2), (1, 2, 1), (130, 8, 2)])
def test_bwd_dense(n, h_q, h_kv):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=64)
    d = synth.make_prefill(sh, seed=n + 3)
    got, want = _run(sh, d, None, seed=2)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got, want):
        parity.assert_grads_close(g_, w_, name)


def test_bwd_lists_with_holes():
    n, h_q, h_kv, k = 1999, 32, 2, 16
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k)
    d = synth.make_prefill(sh, seed=23)
    rng = np.random.default_rng(4)
    idx = np.full((h_kv, n, k), -1, np.int32)
    for g in range(h_kv):
        for i in range(n):
            nb = i // 64 + 1
            cnt = min(nb, int(rng.integers(1, k + 1)))
            chosen = np.sort(rng.choice(nb, size=cnt, replace=False))
            slots = np.sort(rng.choice(k, size=cnt, replace=False))
            idx[g, i, slots] = chosen
    got, want = _run(sh, d, idx, seed=3)
    for name, g_, w_ in zip(("dq", "dk", "dv"), got, want):
        parity.assert_grads_close(g_, w_, name)


def test_bwd_workspace_too_small_is_rejected():
    p = infv2.params(4, 1, k=8)
    n = 300
    q = torch.zeros((n, 4, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.zeros((n, 1, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((4, n), device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(infv2.Infv2Error) as e:
        infv2.infv2_sparse_attn_bwd(p, q, k, k, None, q, lse, q, workspace=ws)
    assert e.value.status == infv2.ERR_WORKSPACE


@pytest.mark.slow
def test_bwd_32k_sampled():
    """The 32k workload through the prefill's own block lists: dq on sampled rows
    against the oracle; dk, dv through invariants that hold at any size
    (sum_t dv_t = sum of dO over the group's heads; sum_t dk_t = scale * sum_i
    (sum_t dS_t) q_i, which is 0 up to D's use of the bf16 forward output)."""
    sh = synth.CONFIGS["prefill_32k"]["shape"]
    d = synth.make_prefill(sh, seed=0)
    p, op = infv2.params_of(sh), oracle.params(sh)
    n = sh.n
    q, k, v = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    idx = torch.empty((sh.h_kv, n, sh.k), dtype=torch.int32, device="cuda")
    lse = torch.empty((sh.h_q, n), device="cuda")
    o = infv2.infv2_prefill(p, q, k, v, [0, n], idx_out=idx, lse=lse)
    d_o = synth.bf16_bits(np.random.default_rng(8).standard_normal((n, sh.h_q, sh.d)).astype(np.float32))
    dq, dk, dv = infv2.infv2_sparse_attn_bwd(p, q, k, v, idx, o, lse, to_dev(d_o))
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    rows = np.unique(np.concatenate([[0, 63, 64, 4095, 4096, n - 1],
                                     np.random.default_rng(1).integers(0, n, 60)])).astype(np.int32)
    o_host = synth.bf16_to_f32(to_host_bits(o))[rows].astype(np.float64)
    idx_rows = idx.cpu().numpy()[:, rows].transpose(1, 0, 2).copy()
    rq, _, _ = oracle.attend_bwd_rows(op, d["q"], d["k"], d["v"], d_o, rows, idx_rows, o_host)
    parity.assert_grads_close(dq.cpu().numpy()[rows], rq, "dq sampled")
    go = synth.bf16_to_f32(d_o).astype(np.float64).reshape(n, sh.h_kv, sh.G, sh.d).sum(axis=2)
    dvs = dv.cpu().numpy().astype(np.float64).sum(axis=0)
    want = go.sum(axis=0)
    # the GPU rounds P to bf16 for P^T dO: per (row, head) the weights sum to 1
    # within ~2^-9 sqrt(sum P^2), a random error that grows as sqrt(rows * heads)
    assert np.abs(dvs - want).max() <= 5e-3 * np.abs(want).max() + 0.5, np.abs(dvs - want).max()
    dks = np.abs(dk.cpu().numpy().astype(np.float64).sum(axis=0)).max()
    assert dks <= 2e-2 * np.abs(dk.cpu().numpy()).sum(axis=0).max(), dks
