"""End-to-end prefill parity (infv2_prefill through the C ABI) against the
fp64 oracle: every row at the oracle sanity size, sampled rows at the full
32k / 128k sizes and on the varlen switch sweep, plus edge cases."""
import numpy as np
import pytest
import torch

import bench
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


def run_prefill(shape, data, cu, lse_approx=0):
    p = infv2.params_of(shape)
    p.lse_approx = lse_approx
    q, k, v = to_dev(data["q"]), to_dev(data["k"]), to_dev(data["v"])
    T = q.shape[0]
    idx = torch.full((shape.h_kv, T, shape.k), -3, dtype=torch.int32, device="cuda")
    lse = torch.empty((shape.h_q, T), device="cuda")
    o = infv2.infv2_prefill(p, q, k, v, cu, idx_out=idx, lse=lse)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    return dict(p=p, q=q, k=k, v=v, o=o, idx=idx, lse=lse)


def check_sequence(shape, data, dev, off, n, rows, dense, max_bad=0, lse_approx=0):
    """Compare rows (sequence-local) of one sequence starting at token `off`."""
    op = oracle.params(shape, lse_approx=lse_approx)
    sl = slice(off, off + n)
    ref = oracle.prefill_rows(op, data["q"][sl], data["k"][sl], data["v"][sl], rows, want_cmp=True)
    o_gpu = synth.bf16_to_f32(to_host_bits(dev["o"][sl]))[rows]
    lse_gpu = dev["lse"][:, off:off + n].cpu().numpy()[:, rows].T
    if dense:
        parity.assert_outputs_close(o_gpu, ref["o"], "dense prefill")
        assert np.allclose(lse_gpu, ref["lse"], atol=2e-3, rtol=0)
        return dict(rows=len(rows))
    gi = dev["idx"][:, off:off + n].cpu().numpy()[:, rows].transpose(1, 0, 2)
    n_eq, n_sw, bad = parity.compare_indices(gi, ref["idx"], ref["cmp"])
    assert len(bad) <= max_bad, bad[:5]
    same = np.array([all(np.array_equal(gi[r, g], ref["idx"][r, g]) for g in range(shape.h_kv))
                     for r in range(len(rows))])
    # outputs on rows whose block sets agree
    parity.assert_outputs_close(o_gpu[same], ref["o"][same], "prefill (same sets)")
    assert np.allclose(lse_gpu[same], ref["lse"][same], atol=2e-3, rtol=0)
    # outputs on the oracle's own indices for every sampled row
    p = dev["p"]
    idx_fix = dev["idx"][:, sl].clone()
    idx_fix[:, torch.from_numpy(rows).long().cuda()] = torch.from_numpy(
        ref["idx"].transpose(1, 0, 2).copy()).cuda()
    o2 = infv2.infv2_sparse_attn(p, dev["q"][sl], dev["k"][sl], dev["v"][sl], idx_fix.contiguous())
    torch.cuda.synchronize()
    o2 = synth.bf16_to_f32(to_host_bits(o2))[rows]
    parity.assert_outputs_close(o2, ref["o"], "sparse attention on oracle indices")
    return dict(rows=len(rows), equal=n_eq, swapped=n_sw)


def _rows(n, count, seed):
    rng = np.random.default_rng(seed)
    fixed = [0, 31, 63, 64, 4095, 4096, 4097, n // 2, n - 65, n - 64, n - 2, n - 1]
    r = np.concatenate([np.array([x for x in fixed if 0 <= x < n]), rng.integers(0, n, count)])
    return np.unique(r).astype(np.int32)


def test_prefill_2k_every_row():
    sh = synth.CONFIGS["prefill_2k"]["shape"]
    data = synth.make_prefill(sh, seed=0)
    dev = run_prefill(sh, data, [0, sh.n])
    st = check_sequence(sh, data, dev, 0, sh.n, np.arange(sh.n, dtype=np.int32), dense=False)
    assert st["equal"] + st["swapped"] == sh.n


@pytest.mark.parametrize("n,h_q,h_kv,k", [(12345, 32, 2, 64), (5000, 16, 2, 16), (3000, 8, 1, 8),
                                         # k = 256, the largest supported: at G = 16 a tile's
                                         # lists (8 tokens x 256) exactly fill the tensor-core
                                         # kernel's staging buffer
                                         (20000, 16, 1, 256),
                                         # G = 4 with k = 128: 32 tokens x 128 entries overflow
                                         # that buffer, so the per-token kernel runs instead
                                         (10000, 4, 1, 128)])
def test_medium_sizes(n, h_q, h_kv, k):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k, n_needles=8)
    data = synth.make_prefill(sh, seed=7)
    dev = run_prefill(sh, data, [0, n])
    check_sequence(sh, data, dev, 0, n, _rows(n, 300, 1), dense=False)


@pytest.mark.slow
def test_prefill_32k_sampled():
    sh = synth.CONFIGS["prefill_32k"]["shape"]
    data = synth.make_prefill(sh, seed=0)
    dev = run_prefill(sh, data, [0, sh.n])
    rows = _rows(sh.n, 120, 2)
    rows = np.unique(np.concatenate([rows, [t for t, _ in data["needles"]]])).astype(np.int32)
    check_sequence(sh, data, dev, 0, sh.n, rows, dense=False)
    # sanity figure: every planted needle's block is selected by its target query
    targets = torch.tensor([t for t, _ in data["needles"]], dtype=torch.long, device="cuda")
    sel = dev["idx"].index_select(1, targets).cpu().numpy()
    assert bench.needle_recall(sel, data["needles"])["recall"] == 1.0


@pytest.mark.slow
def test_prefill_128k_sampled():
    sh = synth.CONFIGS["prefill_128k"]["shape"]
    data = synth.make_prefill(sh, seed=0)
    dev = run_prefill(sh, data, [0, sh.n])
    rows = _rows(sh.n, 48, 3)
    check_sequence(sh, data, dev, 0, sh.n, rows, dense=False)
    # invariants on every row: own/local/init blocks present, count = min(k, b_i+1)
    idx = dev["idx"].cpu().numpy()
    i = np.arange(sh.n)
    bi = i // 64
    for g in range(sh.h_kv):
        cnt = (idx[g] >= 0).sum(1)
        assert np.array_equal(cnt, np.minimum(sh.k, bi + 1))
        assert np.all(idx[g, :, 0] == 0)
        valid = idx[g] >= 0
        assert np.all(np.where(valid, idx[g], 0) <= bi[:, None])
        last = np.take_along_axis(idx[g], (cnt - 1)[:, None], 1)[:, 0]
        assert np.array_equal(last, bi)


@pytest.mark.slow
def test_varlen_switch_sweep():
    cfg = synth.CONFIGS["varlen_sweep"]
    sh = cfg["shape"]
    lengths = cfg["lengths"]
    data = synth.make_varlen(sh, lengths, seed=0)
    cu = data["cu_seqlens"]
    dev = run_prefill(sh, data, cu)
    for s, n in enumerate(lengths):
        dense = n <= sh.k * sh.B
        check_sequence(sh, data, dev, int(cu[s]), n, _rows(n, 24 if n > 8192 else 40, 10 + s), dense)
        if dense:   # dense sequences leave idx_out untouched
            assert np.all(dev["idx"][:, cu[s]:cu[s + 1]].cpu().numpy() == -3)


def test_varlen_edge_cases():
    # empty sequences, shorter than one kernel, exactly one kernel / block,
    # ragged tails, and both dense (n <= k*B = 256) and sparse sequences
    sh = synth.Shape(n=0, h_q=16, h_kv=2, k=4)
    lengths = [0, 5, 31, 32, 64, 65, 256, 257, 0, 600, 1100]
    data = synth.make_varlen(sh, lengths, seed=4)
    cu = data["cu_seqlens"]
    dev = run_prefill(sh, data, cu)
    for s, n in enumerate(lengths):
        if n == 0:
            continue
        rows = np.arange(n, dtype=np.int32)
        check_sequence(sh, data, dev, int(cu[s]), n, rows, dense=n <= sh.k * sh.B)


def test_workspace_too_small_is_rejected():
    sh = synth.Shape(n=2000, h_q=4, h_kv=1, k=8)
    data = synth.make_prefill(sh, seed=1)
    p = infv2.params_of(sh)
    need = infv2.infv2_prefill_workspace_size(p, [0, 2000])
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(infv2.Infv2Error) as e:
        infv2.infv2_prefill(p, to_dev(data["q"]), to_dev(data["k"]), to_dev(data["v"]), [0, 2000],
                            workspace=ws)
    assert e.value.status == infv2.ERR_WORKSPACE
