"""Decode-step parity (infv2_decode through the C ABI): the appended cache
rows, the incremental K^C1 (bit-exact against the oracle's compression of the
same tokens), the selected blocks and the output of the query at position L,
which must equal the oracle's prefill row L of the (L+1)-token sequence.  The
decode attention is also re-run on the oracle's own block lists
(infv2_decode_attn) for every checked row, so a row whose selection differs by
a legal swap still has its output checked."""
import numpy as np
import pytest
import torch

import oracle
import parity
from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2, synth
from trainable_block_sparse_mean_b200.workloads import DecodeState, to_host_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    infv2.lib()


def _sequence_tokens(data, s, upto):
    """Tokens 0..upto-1 of sequence s in [n, h_kv, d] layout."""
    L0 = int(data["lens"][s])
    k = data["k_cache"][s, :, :L0].transpose(1, 0, 2)
    v = data["v_cache"][s, :, :L0].transpose(1, 0, 2)
    steps = upto - L0
    if steps > 0:
        k = np.concatenate([k, data["k_new"][:steps, s]], 0)
        v = np.concatenate([v, data["v_new"][:steps, s]], 0)
    return k[:upto], v[:upto]


def run_and_check(shape, data, steps, check_seqs, check_steps):
    st = DecodeState(shape, data)
    op = oracle.params(shape)
    B = st.batch
    stats = dict(equal=0, swapped=0, attn_checked=0)
    for t in range(steps):
        idx = torch.full((B, shape.h_kv, shape.k), -3, dtype=torch.int32, device="cuda")
        lse = torch.empty((B, shape.h_q), device="cuda")
        o = st.step(t, idx_out=idx, lse=lse)
        torch.cuda.synchronize()
        assert infv2.infv2_device_status() == 0
        lens = st.seqlens.cpu().numpy()
        assert np.array_equal(lens, data["lens"] + t + 1)
        if t not in check_steps:
            continue
        og = synth.bf16_to_f32(to_host_bits(o))
        gi = idx.cpu().numpy()
        refs = {}
        for s in check_seqs:
            L = int(data["lens"][s]) + t          # query position of this step
            k, v = _sequence_tokens(data, s, L + 1)
            qfull = np.zeros((L + 1, shape.h_q, shape.d), np.uint16)
            qfull[L] = data["q"][t, s]
            ref = oracle.prefill_rows(op, qfull, k, v, np.array([L], np.int32), want_cmp=True)
            n_eq, n_sw, bad = parity.compare_indices(gi[s:s + 1], ref["idx"], ref["cmp"])
            assert not bad, (s, t, bad)
            stats["equal"] += n_eq
            stats["swapped"] += n_sw
            if n_sw == 0:
                parity.assert_outputs_close(og[s:s + 1], ref["o"], f"decode seq {s} step {t}")
                assert np.allclose(lse.cpu().numpy()[s], ref["lse"][0], atol=2e-3, rtol=0)
            refs[s] = ref
        # the decode attention on the oracle's block lists, for every checked row
        idx_ref = idx.clone()
        for s in check_seqs:
            idx_ref[s] = torch.from_numpy(refs[s]["idx"][0]).cuda()
        pos = torch.from_numpy((data["lens"] + t).astype(np.int32)).cuda()
        lse2 = torch.empty((B, shape.h_q), device="cuda")
        o2 = infv2.infv2_decode_attn(st.p, st.q[t], st.k_cache, st.v_cache, pos, idx_ref,
                                     st.workspace, lse=lse2)
        torch.cuda.synchronize()
        assert infv2.infv2_device_status() == 0
        assert torch.equal(pos.cpu(), torch.from_numpy((data["lens"] + t).astype(np.int32)))
        og2 = synth.bf16_to_f32(to_host_bits(o2))
        for s in check_seqs:
            parity.assert_outputs_close(og2[s:s + 1], refs[s]["o"], f"decode attention seq {s} step {t}")
            assert np.allclose(lse2.cpu().numpy()[s], refs[s]["lse"][0], atol=2e-3, rtol=0)
            stats["attn_checked"] += 1
    # caches: appended rows and K^C1 of every complete kernel
    kc = to_host_bits(st.k_cache)
    vc = to_host_bits(st.v_cache)
    kc1 = to_host_bits(st.kc1_cache)
    for s in check_seqs:
        n_now = int(data["lens"][s]) + steps
        k, v = _sequence_tokens(data, s, n_now)
        assert np.array_equal(kc[s, :, :n_now], k.transpose(1, 0, 2))
        assert np.array_equal(vc[s, :, :n_now], v.transpose(1, 0, 2))
        want = oracle.compress_k(op, k)
        nc = want.shape[0]
        assert np.array_equal(kc1[s, :, :nc], want.transpose(1, 0, 2))
    return stats


@pytest.mark.parametrize("h_q,h_kv,steps", [(16, 2, 40), (2, 2, 12), (4, 2, 12), (4, 1, 12)])
def test_decode_small_mixed_lengths(h_q, h_kv, steps):
    # dense (L+1 <= k*B) and sparse sequences, kernels completing during the run;
    # group sizes 8, 1, 2 and 4
    sh = synth.Shape(n=0, h_q=h_q, h_kv=h_kv, k=8)
    lens = np.array([0, 20, 31, 100, 511, 700, 3000, 5000], np.int32)
    data = _with_lengths(sh, lens, steps=steps, cap=5100, seed=3)
    run_and_check(sh, data, steps, range(len(lens)), check_steps=set(range(steps)))


def _with_lengths(sh, lens, steps, cap, seed):
    batch = len(lens)
    h_q, h_kv, d = sh.h_q, sh.h_kv, sh.d
    out = dict(k_cache=np.zeros((batch, h_kv, cap, d), np.uint16),
               v_cache=np.zeros((batch, h_kv, cap, d), np.uint16),
               k_new=np.zeros((steps, batch, h_kv, d), np.uint16),
               v_new=np.zeros((steps, batch, h_kv, d), np.uint16),
               q=np.zeros((steps, batch, h_q, d), np.uint16), lens=np.asarray(lens, np.int32), cap=cap)
    for s, L in enumerate(lens):
        sq = synth.make_decode_sequence(sh, int(L), steps, seed, s)
        out["k_cache"][s, :, :L] = sq["k"][:L].transpose(1, 0, 2)
        out["v_cache"][s, :, :L] = sq["v"][:L].transpose(1, 0, 2)
        out["k_new"][:, s] = sq["k"][L:L + steps]
        out["v_new"][:, s] = sq["v"][L:L + steps]
        out["q"][:, s] = sq["q_new"]
    return out


@pytest.mark.slow
def test_decode_batch32_sampled():
    """The batch-32 decode workload as configured: every sequence holds its own
    seeded data (cache lengths U[16k, 128k]); eight sequences, the shortest and
    the longest cache among them, are checked against the oracle on three
    consecutive steps."""
    cfg = synth.CONFIGS["decode_batch32"]
    sh = cfg["shape"]
    data = synth.make_decode(sh, cfg["batch"], cfg["len_lo"], cfg["len_hi"], 3, seed=0)
    order = np.argsort(data["lens"])
    sample = sorted({int(order[0]), int(order[-1]), 0, 7, 12, 19, 25, 31})
    assert len(sample) >= 8
    stats = run_and_check(sh, data, 3, sample, check_steps={0, 1, 2})
    assert stats["equal"] + stats["swapped"] == 3 * len(sample) * sh.h_kv
    assert stats["attn_checked"] == 3 * len(sample)


def test_decode_rejects_small_workspace():
    sh = synth.Shape(n=0, h_q=4, h_kv=1, k=8)
    data = _with_lengths(sh, [100, 200], steps=1, cap=256, seed=1)
    st = DecodeState(sh, data)
    st.workspace = st.workspace[:128]
    with pytest.raises(infv2.Infv2Error) as e:
        st.step(0)
    assert e.value.status == infv2.ERR_WORKSPACE
