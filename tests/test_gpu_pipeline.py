"""Prefill over host buffers (infv2_pipeline_* through the C ABI): every
queued batch's host output equals, bit for bit, infv2_prefill of the same
inputs on the device, and sampled rows of every batch match the fp64 oracle
directly.  Four submits over two slots exercise slot reuse (the third and
fourth batches overwrite the slots of the first and second)."""
import numpy as np
import pytest
import torch

import oracle
import parity
from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2, synth
from trainable_block_sparse_mean_b200.workloads import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    infv2.lib()


def _pinned(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).pin_memory()


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("lengths,h_q,h_kv", [
    ([700, 300, 5000, 1300], 16, 2),
    ([2048], 16, 2),
    # 40000 tokens at h_kv = 8: four score chunks, so the attention runs as four
    # row ranges between them (the single-launch device prefill is the reference)
    ([40000, 300], 16, 8),
])
def test_pipeline_matches_device_prefill_and_oracle(lengths, h_q, h_kv):
    # k*B = 512: 300-token sequences are dense, the others sparse
    sh = synth.Shape(n=0, h_q=h_q, h_kv=h_kv, k=8)
    sets = [synth.make_varlen(sh, lengths, seed=s, n_needles=2) for s in range(3)]
    cu = [int(x) for x in sets[0]["cu_seqlens"]]
    T = cu[-1]
    p = infv2.params_of(sh)
    compute = torch.cuda.Stream()
    pl = infv2.infv2_pipeline_create(p, cu, stream=compute)
    inputs = [(_pinned(d["q"]), _pinned(d["k"]), _pinned(d["v"])) for d in sets]
    order = [0, 1, 2, 0]
    outs = [torch.full((T, sh.h_q, sh.d), -1, dtype=torch.int16).pin_memory() for _ in order]
    lses = [torch.full((sh.h_q, T), float("nan")).pin_memory() for _ in order]
    for j, s in enumerate(order):
        infv2.infv2_pipeline_submit(pl, *inputs[s], outs[j], None if j == 1 else lses[j])
    infv2.infv2_pipeline_sync(pl)
    infv2.infv2_pipeline_destroy(pl)
    assert infv2.infv2_device_status() == 0
    assert torch.isnan(lses[1]).all()          # no lse requested for the second batch
    op = oracle.params(sh)
    rng = np.random.default_rng(5)
    for j, s in enumerate(order):
        d = sets[s]
        lse = torch.empty((sh.h_q, T), device="cuda")
        idx = torch.full((sh.h_kv, T, sh.k), -3, dtype=torch.int32, device="cuda")
        o = infv2.infv2_prefill(p, to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]), cu,
                                idx_out=idx, lse=lse)
        torch.cuda.synchronize()
        assert np.array_equal(outs[j].numpy().view(np.uint16), _bits(o)), (j, s)
        if j != 1:
            assert torch.equal(lses[j], lse.cpu()), (j, s)
        if j == 3:
            continue                           # same inputs as batch 0
        got = synth.bf16_to_f32(outs[j].numpy().view(np.uint16))
        gi = idx.cpu().numpy()
        for si in range(len(lengths)):
            off, n = cu[si], cu[si + 1] - cu[si]
            rows = np.unique(np.concatenate([[0, n - 1], rng.integers(0, n, 12)])).astype(np.int32)
            sl = slice(off, off + n)
            ref = oracle.prefill_rows(op, d["q"][sl], d["k"][sl], d["v"][sl], rows, want_cmp=True)
            same = np.ones(len(rows), bool)
            if n > sh.k * sh.B:                # sparse: outputs where the block sets agree
                g_idx = gi[:, off + rows].transpose(1, 0, 2)
                _, _, bad = parity.compare_indices(g_idx, ref["idx"], ref["cmp"])
                assert not bad, bad[:3]
                same = np.array([np.array_equal(g_idx[r], ref["idx"][r]) for r in range(len(rows))])
                assert same.sum() >= len(rows) // 2
            parity.assert_outputs_close(got[sl][rows][same], ref["o"][same],
                                        "pipeline batch %d seq %d" % (j, si))


def test_pipeline_join_orders_a_stream_after_the_copies():
    sh = synth.Shape(n=0, h_q=4, h_kv=1, k=8)
    d = synth.make_varlen(sh, [1500], seed=9)
    cu = [int(x) for x in d["cu_seqlens"]]
    T = cu[-1]
    p = infv2.params_of(sh)
    pl = infv2.infv2_pipeline_create(p, cu)
    q, k, v = _pinned(d["q"]), _pinned(d["k"]), _pinned(d["v"])
    o = torch.zeros((T, sh.h_q, sh.d), dtype=torch.int16).pin_memory()
    side = torch.cuda.Stream()
    infv2.infv2_pipeline_wait(pl, side)
    infv2.infv2_pipeline_submit(pl, q, k, v, o)
    infv2.infv2_pipeline_join(pl, side)
    side.synchronize()                         # the join alone orders the host read
    want = infv2.infv2_prefill(p, to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]), cu)
    torch.cuda.synchronize()
    assert np.array_equal(o.numpy().view(np.uint16), _bits(want))
    infv2.infv2_pipeline_destroy(pl)


@pytest.mark.parametrize("lengths", [[0, 300, 0, 1000], [300, 400]])
def test_pipeline_empty_and_dense_only_batches(lengths):
    # empty sequences between the others; an all-dense batch (no prefill workspace)
    sh = synth.Shape(n=0, h_q=8, h_kv=2, k=8)
    d = synth.make_varlen(sh, lengths, seed=4)
    cu = [int(x) for x in d["cu_seqlens"]]
    T = cu[-1]
    p = infv2.params_of(sh)
    pl = infv2.infv2_pipeline_create(p, cu)
    o = torch.zeros((T, sh.h_q, sh.d), dtype=torch.int16).pin_memory()
    lse = torch.zeros((sh.h_q, T)).pin_memory()
    infv2.infv2_pipeline_submit(pl, _pinned(d["q"]), _pinned(d["k"]), _pinned(d["v"]), o, lse)
    infv2.infv2_pipeline_sync(pl)
    infv2.infv2_pipeline_destroy(pl)
    want_lse = torch.empty((sh.h_q, T), device="cuda")
    want = infv2.infv2_prefill(p, to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]), cu, lse=want_lse)
    torch.cuda.synchronize()
    assert np.array_equal(o.numpy().view(np.uint16), _bits(want))
    assert torch.equal(lse, want_lse.cpu())
