"""Per-stage parity of the CUDA library against the fp64 oracle (small sizes
that still span several tiles and a ragged tail)."""
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


def _problem(n, h_q, h_kv, k=8, seed=0, n_needles=0):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k, n_needles=n_needles)
    return sh, synth.make_prefill(sh, seed=seed)


def _sample_rows(n, count, seed=0):
    rng = np.random.default_rng(seed)
    fixed = [r for r in (0, 1, 30, 31, 32, 46, 47, 63, 64, 127, 128, 511, 512, n - 2, n - 1) if 0 <= r < n]
    extra = rng.integers(0, n, size=count) if n > 0 else []
    return np.unique(np.array(fixed + list(extra), dtype=np.int64)).astype(np.int32)


# ---------------------------------------------------------------- stage 1

@pytest.mark.parametrize("n,h_kv", [(2048, 1), (1000, 2), (31, 2), (32, 1), (47, 2), (4177, 2)])
def test_compress_bit_exact(n, h_kv):
    sh, d = _problem(n, 2 * h_kv, h_kv)
    p = infv2.params_of(sh)
    kc1 = infv2.infv2_compress_k(p, to_dev(d["k"]))
    torch.cuda.synchronize()
    want = oracle.compress_k(oracle.params(sh), d["k"])
    got = to_host_bits(kc1) if kc1.numel() else np.zeros((0, h_kv, 128), np.uint16)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


def test_compress_extreme_values_bit_exact():
    # wide magnitude spread, ties and signed zeros inside kernels
    sh = synth.Shape(n=256, h_q=2, h_kv=2)
    rng = np.random.default_rng(5)
    k = (rng.standard_normal((256, 2, 128)) * np.exp(rng.uniform(-20, 20, (256, 2, 128)))).astype(np.float32)
    k[:40, 0, :8] = 1.0
    k[7, 0, :8] = np.array([1.125, 1.375, 1.25, 1.75, 2.0, 1.0625, 1.1875, -0.0], np.float32)
    kb = synth.bf16_bits(k)
    p = infv2.params_of(sh)
    got = to_host_bits(infv2.infv2_compress_k(p, to_dev(kb)))
    want = oracle.compress_k(oracle.params(sh), kb)
    assert np.array_equal(got, want)


def test_compress_every_bf16_value_bit_exact():
    # 32 equal rows per value: every finite bf16 bit pattern (subnormals, the
    # largest finite value) is its own mean; a zero mean is +0 on both sides
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = np.where((bits & 0x7F80) != 0x7F80, bits, 0).astype(np.uint16)
    sh = synth.Shape(n=32, h_q=512, h_kv=512)
    kb = np.broadcast_to(vals.reshape(1, 512, 128), (32, 512, 128)).copy()
    p = infv2.params_of(sh)
    got = to_host_bits(infv2.infv2_compress_k(p, to_dev(kb)))
    want = oracle.compress_k(oracle.params(sh), kb)
    assert np.array_equal(got, want)
    vals[vals == 0x8000] = 0
    assert np.array_equal(got[0].reshape(-1), vals)


# ---------------------------------------------------------------- stage 2

SCORE_REL = 2e-5   # fp32 tensor-core dot products + fp32 softmax vs fp64


@pytest.mark.parametrize("n,h_q,h_kv,q_begin,q_len", [
    (2048, 4, 1, 0, 2048),        # the 2k workload's shape, G=4 (32 tokens per tile)
    (3000, 32, 2, 0, 3000),       # G=16, ragged tail, 188 kernels (2 tiles)
    (3000, 32, 2, 1000, 1333),    # a chunk in the middle of the sequence
    (700, 8, 1, 0, 700),          # G=8
    (600, 2, 2, 0, 600),          # G=1 (128 tokens per tile)
    (900, 4, 2, 0, 900),          # G=2
])
def test_block_scores_match_oracle(n, h_q, h_kv, q_begin, q_len):
    sh, d = _problem(n, h_q, h_kv, seed=n + h_q)
    p = infv2.params_of(sh)
    op = oracle.params(sh)
    kc1 = infv2.infv2_compress_k(p, to_dev(d["k"]))
    ld = infv2.shared_ld(n)
    slse = torch.full((h_q, q_len), 7.0, device="cuda")
    s = infv2.infv2_block_scores(p, to_dev(d["q"]), kc1, n, q_begin, q_len, ld=ld, score_lse=slse)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    s = s.cpu().numpy()
    slse = slse.cpu().numpy()
    rows = _sample_rows(n, 40, seed=n)
    rows = rows[(rows >= q_begin) & (rows < q_begin + q_len)]
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows, want_shared=True, want_score_lse=True)
    for r, i in enumerate(rows):
        nv = oracle.visible_kernels(op, i)
        for g in range(h_kv):
            want = ref["shared"][r, g, :nv]
            got = s[g, i - q_begin, :nv]
            err = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
            assert err.max(initial=0) <= SCORE_REL, (i, g, err.max(), int(err.argmax()))
        lw = ref["score_lse"][r]
        lg = slse[:, i - q_begin]
        if nv == 0:
            assert np.all(np.isneginf(lg))
        else:
            assert np.allclose(lg, lw, rtol=0, atol=2e-5), (i, lg - lw)


@pytest.mark.parametrize("n,h_q,h_kv,q_begin,q_len", [
    (2048, 4, 1, 0, 2048),        # G=4, one kernel tile: carries between warp quarters
    (3000, 32, 2, 0, 3000),       # G=16, ragged tail
    (3000, 32, 2, 1000, 1333),    # a chunk in the middle of the sequence
    (700, 8, 1, 0, 700),          # G=8
    (600, 2, 2, 0, 600),          # G=1
    (900, 4, 2, 0, 900),          # G=2
    (17000, 32, 2, 16000, 1000),  # 9 kernel tiles: windows across tile boundaries
])
def test_pooled_block_scores_match_oracle(n, h_q, h_kv, q_begin, q_len):
    """Scores with max pooling fused into the score kernel: S^cmp[b] for b < i/B."""
    sh, d = _problem(n, h_q, h_kv, seed=n + 3 * h_q)
    p = infv2.params_of(sh)
    op = oracle.params(sh)
    kc1 = infv2.infv2_compress_k(p, to_dev(d["k"]))
    ldc = infv2.cmp_ld(n)
    sentinel = 7.25
    s = torch.full((h_kv, q_len, ldc), sentinel, device="cuda")
    infv2.infv2_block_scores_pooled(p, to_dev(d["q"]), kc1, n, q_begin, q_len, s, ldc)
    # the unfused scores of the same kernel, pooled on the host in fp32
    ld = infv2.shared_ld(n)
    full = infv2.infv2_block_scores(p, to_dev(d["q"]), kc1, n, q_begin, q_len, ld=ld)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    s = s.cpu().numpy()
    full = full.cpu().numpy()
    rows = _sample_rows(n, 40, seed=n + 1)
    rows = rows[(rows >= q_begin) & (rows < q_begin + q_len)]
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows, want_cmp=True)
    for r, i in enumerate(rows):
        nb = int(i) // 64
        nv = oracle.visible_kernels(op, i)
        for g in range(h_kv):
            got = s[g, i - q_begin, :nb]
            want = ref["cmp"][r, g, :nb]
            err = np.abs(got - want) / np.maximum(np.abs(want), 1e-30)
            assert err.max(initial=0) <= SCORE_REL, (i, g, err.max(), int(err.argmax()))
            assert np.all(s[g, i - q_begin, nb:] == sentinel)   # own block onwards untouched
            row = full[g, i - q_begin, :nv]
            pooled = np.array([row[max(4 * b - 1, 0):min(4 * b + 4, nv)].max() for b in range(nb)],
                              np.float32)
            assert np.array_equal(got, pooled), (i, g)


@pytest.mark.parametrize("n,h_q,h_kv,k", [(2048, 4, 1, 8), (5000, 32, 2, 16), (9000, 16, 2, 64),
                                         (3000, 4, 1, 3), (3000, 4, 1, 4)])
def test_select_pooled_exact_on_oracle_scores(n, h_q, h_kv, k):
    """Top-k from S^cmp, decided on the same fp32 values as the oracle."""
    sh, d = _problem(n, h_q, h_kv, k=k, seed=4)
    op = oracle.params(sh)
    p = infv2.params_of(sh)
    rows = _sample_rows(n, 200, seed=2)
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows, want_cmp=True)
    c32 = ref["cmp"].astype(np.float32)               # [rows, h_kv, n_blk]
    ties = np.round(c32 * 32) / 32
    const = np.full_like(c32, 0.5)
    n_blk = c32.shape[2]
    ldc = infv2.cmp_ld(n)
    for vals in (c32, ties, const):
        buf = np.full((h_kv, len(rows), ldc), np.nan, np.float32)
        for r, i in enumerate(rows):   # only b < i/B is defined; the rest stays NaN
            buf[:, r, :int(i) // 64] = vals[r, :, :int(i) // 64]
        dev = torch.from_numpy(buf).cuda()
        idx = torch.full((h_kv, n, k), -2, dtype=torch.int32, device="cuda")
        for r, i in enumerate(rows):
            infv2.infv2_select_topk_pooled(p, dev[:, r:r + 1, :].contiguous(), ldc, n, int(i), 1, idx)
        torch.cuda.synchronize()
        idx = idx.cpu().numpy()
        for r, i in enumerate(rows):
            for g in range(h_kv):
                want = oracle.select_row(op, vals[r, g, :int(i) // 64 + 1].astype(np.float64), int(i))
                assert np.array_equal(idx[g, i, :], want), (i, g)
        assert n_blk == (n + 63) // 64


# ---------------------------------------------------------------- stages 3-4

@pytest.mark.parametrize("n,h_q,h_kv,k", [(2048, 4, 1, 8), (5000, 32, 2, 16), (9000, 16, 2, 64),
                                         (3000, 4, 1, 3), (3000, 4, 1, 4)])
def test_select_exact_on_oracle_scores(n, h_q, h_kv, k):
    """The selection decision is taken on the same fp32 values on both sides:
    the scores as computed, a copy quantised to create many exact ties, and a
    constant copy (every block tied); k = 3 leaves only the forced blocks."""
    sh, d = _problem(n, h_q, h_kv, k=k, seed=3)
    op = oracle.params(sh)
    p = infv2.params_of(sh)
    rows = _sample_rows(n, 200, seed=1)
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows, want_shared=True)
    sh32 = ref["shared"].astype(np.float32)          # [rows, h_kv, nc]
    nc = sh32.shape[2]
    # quantise a copy to create exact ties in the block scores
    ties = np.round(sh32 * 64) / 64
    const = np.full_like(sh32, 0.25)
    for vals in (sh32, ties, const):
        ld = infv2.shared_ld(n)
        buf = np.zeros((h_kv, len(rows), ld), np.float32)
        buf[:, :, :nc] = vals.transpose(1, 0, 2)
        # the GPU select reads the row of query i at position (i - q_begin); give
        # each sampled row its own one-row call
        got = np.zeros((len(rows), h_kv, k), np.int32)
        dev = torch.from_numpy(buf).cuda()
        idx = torch.full((h_kv, n, k), -2, dtype=torch.int32, device="cuda")
        for r, i in enumerate(rows):
            row = dev[:, r:r + 1, :].contiguous()
            infv2.infv2_select_topk(p, row, ld, n, int(i), 1, idx)
        torch.cuda.synchronize()
        idx = idx.cpu().numpy()
        for r, i in enumerate(rows):
            got[r] = idx[:, i, :]
        want, _ = oracle.select_rows(op, vals.astype(np.float64), rows, (n + 63) // 64)
        assert np.array_equal(got, want)


# ---------------------------------------------------------------- stage 5

@pytest.mark.parametrize("n,h_q,h_kv,k", [(2048, 4, 1, 8), (2048, 16, 1, 8), (3001, 32, 2, 16),
                                         (1500, 16, 2, 4)])
def test_sparse_attn_on_oracle_indices(n, h_q, h_kv, k):
    sh, d = _problem(n, h_q, h_kv, k=k, seed=11)
    op = oracle.params(sh)
    p = infv2.params_of(sh)
    rows = np.arange(n, dtype=np.int32) if n <= 2048 else _sample_rows(n, 150)
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows)
    idx = np.full((h_kv, n, k), -1, np.int32)
    idx[:, :, 0] = (np.arange(n) // 64)[None, :]   # rows not sampled: own block only
    idx[:, rows, :] = ref["idx"].transpose(1, 0, 2)
    q, kk, vv, ii = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]), torch.from_numpy(idx).cuda()
    first = None
    for rep in range(3):   # repeated launches: a pipeline race shows up as run-to-run change
        lse = torch.empty((h_q, n), device="cuda")
        o = infv2.infv2_sparse_attn(p, q, kk, vv, ii, lse=lse)
        torch.cuda.synchronize()
        assert infv2.infv2_device_status() == 0
        og = synth.bf16_to_f32(to_host_bits(o))[rows]
        parity.assert_outputs_close(og, ref["o"], "sparse_attn")
        lg = lse.cpu().numpy()[:, rows].T
        assert np.allclose(lg, ref["lse"], rtol=0, atol=2e-3)
        if first is None:
            first = og
        else:
            assert np.array_equal(og, first), "sparse_attn is not deterministic"


def test_sparse_attn_lists_with_holes():
    """Entries < 0 anywhere in a list are ignored; neighbouring tokens with
    overlapping and disjoint lists share the fetched blocks."""
    n, h_q, h_kv, k = 1999, 32, 2, 16
    sh, d = _problem(n, h_q, h_kv, k=k, seed=23)
    op = oracle.params(sh)
    p = infv2.params_of(sh)
    rng = np.random.default_rng(4)
    idx = np.full((h_kv, n, k), -1, np.int32)
    for g in range(h_kv):
        for i in range(n):
            nb = i // 64 + 1
            cnt = min(nb, int(rng.integers(1, k + 1)))
            chosen = np.sort(rng.choice(nb, size=cnt, replace=False))
            slots = np.sort(rng.choice(k, size=cnt, replace=False))   # -1 holes between them
            idx[g, i, slots] = chosen
    rows = _sample_rows(n, 120, seed=6)
    want_o, want_lse = oracle.attend_rows(op, d["q"], d["k"], d["v"], rows,
                                          idx[:, rows, :].transpose(1, 0, 2).copy())
    lse = torch.empty((h_q, n), device="cuda")
    o = infv2.infv2_sparse_attn(p, to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]),
                                torch.from_numpy(idx).cuda(), lse=lse)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    og = synth.bf16_to_f32(to_host_bits(o))[rows]
    parity.assert_outputs_close(og, want_o, "sparse_attn holes")
    assert np.allclose(lse.cpu().numpy()[:, rows].T, want_lse, rtol=0, atol=2e-3)


@pytest.mark.parametrize("n,h_q,h_kv", [(1024, 32, 2), (777, 4, 1), (64, 16, 2), (1, 2, 1), (130, 8, 2)])
def test_dense_attn_matches_oracle(n, h_q, h_kv):
    sh, d = _problem(n, h_q, h_kv, k=64, seed=17)
    op = oracle.params(sh)
    p = infv2.params_of(sh)
    rows = _sample_rows(n, 100)
    ref = oracle.prefill_rows(op, d["q"], d["k"], d["v"], rows)
    lse = torch.empty((h_q, n), device="cuda")
    o = infv2.infv2_dense_attn(p, to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"]), lse=lse)
    torch.cuda.synchronize()
    og = synth.bf16_to_f32(to_host_bits(o))[rows]
    parity.assert_outputs_close(og, ref["o"], "dense_attn")
    assert np.allclose(lse.cpu().numpy()[:, rows].T, ref["lse"], rtol=0, atol=2e-3)


@pytest.mark.parametrize("dense", [False, True])
def test_attn_rows_split_equals_whole(dense):
    """Chunked prefill: attention over row ranges (the oracle's block lists, or
    dense) leaves rows outside a range alone; ranges that end on tile
    boundaries (multiples of 128/G tokens) give the whole-sequence call's bits,
    and ranges that cut a tile agree with it to within rounding (a row's
    probabilities are rounded against a reference maximum that the other
    tokens of its tile can move)."""
    n, h_q, h_kv, k = 3000, 16, 2, 8
    tq = 128 // (h_q // h_kv)
    sh, d = _problem(n, h_q, h_kv, k=k, seed=29)
    p = infv2.params_of(sh)
    q, kk, vv = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    ii = None
    if not dense:
        ref = oracle.prefill_rows(oracle.params(sh), d["q"], d["k"], d["v"], np.arange(n, dtype=np.int32))
        ii = torch.from_numpy(ref["idx"].transpose(1, 0, 2).copy()).cuda()
    lse = torch.empty((h_q, n), device="cuda")
    whole = (infv2.infv2_dense_attn(p, q, kk, vv, lse=lse) if dense
             else infv2.infv2_sparse_attn(p, q, kk, vv, ii, lse=lse))
    for cuts, exact in (([0, tq, 64, 44 * tq, 2048, n - n % tq, n], True),
                        ([0, 1, 64, 700, 701, 2048, 2999, n], False)):
        o = torch.full_like(q, 7.0)
        lse2 = torch.full((h_q, n), 7.0, device="cuda")
        for r0, r1 in zip(cuts[:-1], cuts[1:]):
            infv2.infv2_sparse_attn_rows(p, q, kk, vv, ii, r0, r1, o=o, lse=lse2)
            torch.cuda.synchronize()
            assert torch.all(o[r1:].view(torch.int16) == torch.full_like(q, 7.0)[r1:].view(torch.int16))
        infv2.infv2_sparse_attn_rows(p, q, kk, vv, ii, 5, 5, o=o, lse=lse2)   # empty: no-op
        torch.cuda.synchronize()
        assert infv2.infv2_device_status() == 0
        if exact:
            assert torch.equal(o.view(torch.int16), whole.view(torch.int16))
            assert torch.equal(lse2, lse)
        else:
            parity.assert_outputs_close(o.float().cpu().numpy(), whole.double().cpu().numpy(),
                                        "row ranges cutting tiles")
            assert float((lse2 - lse).abs().max()) <= 1e-3


def test_timeout_path_reports_and_recovers():
    assert infv2.infv2_device_status() == 0
    infv2.infv2_selftest_timeout(2000)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == infv2.ERR_TIMEOUT
    assert infv2.infv2_device_status() == 0     # cleared
    x = torch.ones(4, device="cuda") * 2        # the context is still usable
    assert float(x.sum()) == 8.0


# ---------------------------------------------------------------- varlen stage forms

def test_varlen_stage_calls_equal_the_single_sequence_calls():
    """Each varlen stage call issues, per sequence, the single-sequence call's
    launches on the packed tensors: a sequence's K^C1, S^shared block, block
    lists, O and lse equal the single-sequence results bit for bit (an empty
    sequence, one without a complete kernel, a dense-sized and two sparse
    ones; two kv heads, so the packed head strides differ from the
    per-sequence ones)."""
    sh = synth.Shape(n=0, h_q=16, h_kv=2, k=8)
    lengths = [300, 2000, 0, 5000, 31]
    d = synth.make_varlen(sh, lengths, seed=9)
    p = infv2.params_of(sh)
    q, k, v = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    cu = [int(x) for x in synth.cu_seqlens_of(lengths)]
    T = cu[-1]
    ck = infv2.infv2_varlen_kernel_offsets(p, cu)
    kc1 = infv2.infv2_compress_k_varlen(p, k, cu)
    s_sh, ld = infv2.infv2_block_scores_varlen(p, q, kc1, cu)
    idx = infv2.infv2_select_topk_varlen(p, s_sh, ld, cu)
    lse = torch.full((sh.h_q, T), 7.0, device="cuda")
    o = infv2.infv2_sparse_attn_varlen(p, q, k, v, idx, cu, lse=lse)
    lse_d = torch.full((sh.h_q, T), 7.0, device="cuda")
    od = infv2.infv2_dense_attn_varlen(p, q, k, v, cu, lse=lse_d)
    torch.cuda.synchronize()
    assert infv2.infv2_device_status() == 0
    for s, n in enumerate(lengths):
        if n == 0:
            continue
        a, b = cu[s], cu[s + 1]
        qs, ks, vs = q[a:b].contiguous(), k[a:b].contiguous(), v[a:b].contiguous()
        kc1_s = infv2.infv2_compress_k(p, ks)
        assert ck[s + 1] - ck[s] == kc1_s.shape[0]
        assert torch.equal(kc1[ck[s]:ck[s + 1]], kc1_s), s
        s_s = infv2.infv2_block_scores(p, qs, kc1_s, n, 0, n, ld=ld)
        blk = s_sh[sh.h_kv * ld * a: sh.h_kv * ld * b].view(sh.h_kv, n, ld)
        assert torch.equal(blk, s_s), s
        idx_s = infv2.infv2_select_topk(p, s_s, ld, n, 0, n)
        assert torch.equal(idx[:, a:b], idx_s), s
        lse_s = torch.empty((sh.h_q, n), device="cuda")
        o_s = infv2.infv2_sparse_attn(p, qs, ks, vs, idx_s, lse=lse_s)
        assert torch.equal(o[a:b], o_s) and torch.equal(lse[:, a:b], lse_s), s
        lse_ds = torch.empty((sh.h_q, n), device="cuda")
        od_s = infv2.infv2_dense_attn(p, qs, ks, vs, lse=lse_ds)
        assert torch.equal(od[a:b], od_s) and torch.equal(lse_d[:, a:b], lse_ds), s
