"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Each pin is a plain function that raises AssertionError on a mismatch.  The
pins use hand-worked fixtures (tests/golden), closed forms, invariants,
brute force by set enumeration, and library routines (torch fp64 softmax /
scaled_dot_product_attention) for the special cases that reduce to them.
test_oracle_pins.py runs them on the oracle; test_oracle_mutants.py runs them
on builds of the oracle with planted mistakes and expects each to be caught.
"""
from __future__ import annotations

import os
from fractions import Fraction

import numpy as np
import torch

import oracle
from trainable_block_sparse_mean_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                yield line.split()


def _bf16(x) -> np.ndarray:
    return synth.bf16_bits(np.asarray(x, np.float32))


def _f64(b) -> np.ndarray:
    return synth.bf16_to_f32(b).astype(np.float64)


def _shape(**kw) -> synth.Shape:
    return synth.Shape(**kw)


# --------------------------------------------------------------------------
# stage 1: mean pooling of K
# --------------------------------------------------------------------------

def pin_compress_hand():
    sh = _shape(n=64, h_q=1, h_kv=1, d=2)
    p = oracle.params(sh)
    t = np.arange(64, dtype=np.float32)
    k = _bf16(np.stack([t, -t / 2], axis=1)[:, None, :])
    kc1 = _f64(oracle.compress_k(p, k))
    assert kc1.shape == (3, 1, 2), kc1.shape
    for j, c, val in _lines("compress_hand.txt"):
        assert kc1[int(j), 0, int(c)] == float(val), (j, c, kc1[int(j), 0, int(c)], val)


def pin_compress_ties():
    sh = _shape(n=32, h_q=1, h_kv=1, d=1)
    p = oracle.params(sh)
    for odd, exact, want in _lines("compress_ties.txt"):
        col = np.ones(32, np.float32)
        col[7] = float(odd)
        k = _bf16(col[:, None, None])
        got = _f64(oracle.compress_k(p, k))[0, 0, 0]
        assert float(Fraction(float(odd)) + 31) / 32 == float(exact)
        assert got == float(want), (odd, got, want)


def pin_compress_constant_and_ramp():
    sh = _shape(n=200, h_q=2, h_kv=2, d=4)
    p = oracle.params(sh)
    c = np.array([0.375, -2.5, 7.0, 1e-3], np.float32)
    k = np.zeros((200, 2, 4), np.float32)
    k[:, 0, :] = c
    k[:, 1, :] = (np.arange(200, dtype=np.float32) * 0.25)[:, None]
    kb = _bf16(k)
    kc1 = _f64(oracle.compress_k(p, kb))
    nc = (200 - 32) // 16 + 1
    assert kc1.shape[0] == nc
    cb = _f64(_bf16(c))
    for j in range(nc):
        assert np.array_equal(kc1[j, 0], cb), (j, kc1[j, 0])
        # ramp 0.25*t over tokens 16j..16j+31 -> 0.25*(16j + 15.5), exact in bf16 here
        mid = 0.25 * (16 * j + 15.5)
        assert np.all(kc1[j, 1] == _f64(_bf16(np.float32(mid)))), (j, kc1[j, 1], mid)


def _rne_bf16_fraction(x: Fraction) -> float:
    """Nearest bf16 value to the exact rational x, ties to even (brute force)."""
    if x == 0:
        return 0.0
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    q = max(e - 7, -133)
    scaled = abs(x) / Fraction(2) ** q
    lo = scaled.numerator // scaled.denominator
    rem = scaled - lo
    r = lo + 1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1) else lo
    return sign * float(Fraction(r) * Fraction(2) ** q)


def pin_compress_bruteforce():
    sh = _shape(n=96, h_q=2, h_kv=2, d=8)
    p = oracle.params(sh)
    rng = np.random.default_rng(11)
    k = _bf16(rng.standard_normal((96, 2, 8)).astype(np.float32) * 3)
    kv = _f64(k)
    kc1 = _f64(oracle.compress_k(p, k))
    nc = (96 - 32) // 16 + 1
    assert kc1.shape == (nc, 2, 8)
    for j in range(nc):
        for g in range(2):
            for c in range(8):
                s = sum(Fraction(float(kv[t, g, c])) for t in range(16 * j, 16 * j + 32))
                want = _rne_bf16_fraction(s / 32)
                assert kc1[j, g, c] == want, (j, g, c, kc1[j, g, c], want)


def pin_visibility():
    p = oracle.params(_shape())
    for n in range(0, 140):
        want = sum(1 for j in range(n) if 16 * j + 32 <= n)
        assert oracle.num_kernels(p, n) == want, (n,)
    for i in range(0, 200):
        # kernel j covers tokens 16j..16j+31; visible to query i if all <= i
        want = sum(1 for j in range(i + 1) if set(range(16 * j, 16 * j + 32)) <= set(range(i + 1)))
        assert oracle.visible_kernels(p, i) == want, (i,)


def pin_coarse_kernels_bruteforce():
    """LSE approximation: K^C2 is the bf16 mean over l_C2 = 4 l_C1 = 128 tokens at
    stride s_C2 = 4 s_C1 = 64, visible to query i when its last token is <= i."""
    sh = _shape(n=300, h_q=2, h_kv=2, d=8)
    p = oracle.params(sh)
    for n in range(0, 400, 7):
        assert oracle.num_coarse_kernels(p, n) == sum(1 for c in range(n) if 64 * c + 128 <= n), (n,)
    for i in range(0, 400, 3):
        assert oracle.visible_coarse_kernels(p, i) == sum(1 for c in range(i + 1) if 64 * c + 127 <= i), (i,)
    rng = np.random.default_rng(12)
    k = _bf16(rng.standard_normal((300, 2, 8)).astype(np.float32) * 3)
    kv = _f64(k)
    kc2 = _f64(oracle.compress_k2(p, k))
    assert kc2.shape == ((300 - 128) // 64 + 1, 2, 8), kc2.shape
    for c in range(kc2.shape[0]):
        for g in range(2):
            for e in range(8):
                s_ = sum(Fraction(float(kv[t, g, e])) for t in range(64 * c, 64 * c + 128))
                want = _rne_bf16_fraction(s_ / 128)
                assert kc2[c, g, e] == want, (c, g, e, kc2[c, g, e], want)


def pin_coarse_lse_closed_forms():
    """Constant keys: every logit is z0, so the estimate is z0 + log(nv2) + log 4 and
    each normalised score is exp(z0 - estimate) = 1 / (4 nv2).  Two visible coarse
    kernels: the estimate is max + log(1 + exp(-|D|)) + log 4."""
    sh = _shape(n=512, h_q=4, h_kv=2, d=8)
    p = oracle.params(sh)
    rng = np.random.default_rng(21)
    q = _bf16(rng.standard_normal((512, 4, 8)))
    k = _bf16(np.broadcast_to(rng.standard_normal((1, 2, 8)), (512, 2, 8)))
    kc1, kc2 = oracle.compress_k(p, k), oracle.compress_k2(p, k)
    qf, kf = _f64(q), _f64(k)
    for i in (127, 191, 300, 511):
        nv2 = (i - 127) // 64 + 1
        nv1 = (i - 31) // 16 + 1
        for g in range(2):
            lse = oracle.coarse_lse_row(p, q, kc2, i, g)
            assert lse is not None, (i, g)
            for hh in range(2):
                z0 = float(qf[i, g * 2 + hh] @ kf[0, g]) / np.sqrt(8)
                assert abs(lse[hh] - (z0 + np.log(nv2) + np.log(4.0))) < 1e-12, (i, g, hh)
            s_, used = oracle.shared_scores_row_lse(p, q, kc1, i, g, lse)
            assert np.allclose(used, lse, rtol=0, atol=0)
            assert np.allclose(s_, 2.0 / (4 * nv2), rtol=1e-12, atol=0), (i, s_[:3])
            assert len(s_) == nv1
    sh, data = _small_problem(n=256, h_q=4, h_kv=2, d=16, seed=13)
    p = oracle.params(sh)
    kc2 = oracle.compress_k2(p, data["k"])
    qf, K2 = _f64(data["q"]), _f64(kc2)
    for g in range(2):
        lse = oracle.coarse_lse_row(p, data["q"], kc2, 191, g)   # coarse kernels 0 and 1
        assert lse is not None
        for hh in range(2):
            z = [float(qf[191, g * 2 + hh] @ K2[c, g]) / 4.0 for c in (0, 1)]
            want = max(z) + np.log1p(np.exp(-abs(z[0] - z[1]))) + np.log(4.0)
            assert abs(lse[hh] - want) < 1e-12, (g, hh, lse[hh], want)
        assert oracle.coarse_lse_row(p, data["q"], kc2, 126, g) is None


def pin_coarse_lse_only_where_a_coarse_kernel_is_visible():
    """With the approximation on, rows that see no coarse kernel keep the exact
    log-sum-exp and scores; later rows use the estimate."""
    sh, data = _small_problem(n=400, h_q=4, h_kv=2, d=16, seed=17)
    pe, pa = oracle.params(sh), oracle.params(sh, lse_approx=1)
    rows = np.array([31, 64, 126, 127, 250, 399], np.int32)
    ex = oracle.prefill_rows(pe, data["q"], data["k"], data["v"], rows, want_shared=True, want_score_lse=True)
    ap = oracle.prefill_rows(pa, data["q"], data["k"], data["v"], rows, want_shared=True, want_score_lse=True)
    kc2 = oracle.compress_k2(pa, data["k"])
    for r, i in enumerate(rows):
        if i < 127:
            assert np.array_equal(ex["shared"][r], ap["shared"][r]) and np.array_equal(ex["score_lse"][r], ap["score_lse"][r])
        else:
            for g in range(2):
                want = oracle.coarse_lse_row(pa, data["q"], kc2, int(i), g)
                assert want is not None and np.array_equal(ap["score_lse"][r, g * 2:g * 2 + 2], want)
            assert not np.array_equal(ex["score_lse"][r], ap["score_lse"][r])


# --------------------------------------------------------------------------
# stage 2: S^C1 softmax and the group sum S^shared
# --------------------------------------------------------------------------

def _small_problem(n=300, h_q=4, h_kv=2, d=16, seed=5, **kw):
    sh = _shape(n=n, h_q=h_q, h_kv=h_kv, d=d, **kw)
    data = synth.make_prefill(sh, seed=seed)
    return sh, data


def pin_scores_sum_to_G():
    sh, data = _small_problem()
    p = oracle.params(sh)
    kc1 = oracle.compress_k(p, data["k"])
    for i in (31, 47, 120, 299):
        for g in range(sh.h_kv):
            s, _ = oracle.shared_scores_row(p, data["q"], kc1, i, g)
            assert abs(s.sum() - sh.G) < 1e-12, (i, g, s.sum())
            assert np.all(s > 0)


def pin_scores_uniform_when_kernels_equal():
    sh = _shape(n=256, h_q=4, h_kv=1, d=8)
    p = oracle.params(sh)
    rng = np.random.default_rng(3)
    q = _bf16(rng.standard_normal((256, 4, 8)))
    k = _bf16(np.broadcast_to(rng.standard_normal((1, 1, 8)), (256, 1, 8)))
    kc1 = oracle.compress_k(p, k)
    for i in (31, 63, 200, 255):
        s, _ = oracle.shared_scores_row(p, q, kc1, i, 0)
        nv = (i - 31) // 16 + 1
        assert len(s) == nv
        assert np.allclose(s, 4.0 / nv, rtol=0, atol=1e-14), (i, s)


def pin_scores_two_kernels_closed_form():
    # query 47 sees exactly kernels 0 and 1: S^C1(h) = (sigmoid(-D), sigmoid(D))
    sh, data = _small_problem(n=64, h_q=4, h_kv=2, d=16, seed=9)
    p = oracle.params(sh)
    kc1 = oracle.compress_k(p, data["k"])
    q, K = _f64(data["q"]), _f64(kc1)
    for g in range(2):
        s, _ = oracle.shared_scores_row(p, data["q"], kc1, 47, g)
        want = np.zeros(2)
        for hh in range(2):
            h = g * 2 + hh
            D = (q[47, h] @ K[1, g] - q[47, h] @ K[0, g]) / np.sqrt(16)
            want += [1 / (1 + np.exp(D)), 1 / (1 + np.exp(-D))]
        assert np.allclose(s, want, rtol=1e-13, atol=0), (g, s, want)


def pin_scores_torch_softmax():
    sh, data = _small_problem(n=333, h_q=8, h_kv=2, d=32, seed=21)
    p = oracle.params(sh)
    kc1 = oracle.compress_k(p, data["k"])
    q = torch.from_numpy(_f64(data["q"]))
    K = torch.from_numpy(_f64(kc1))
    for i in (40, 100, 332):
        nv = (i - 31) // 16 + 1
        for g in range(2):
            s, lse = oracle.shared_scores_row(p, data["q"], kc1, i, g)
            z = (q[i, g * 4:(g + 1) * 4] @ K[:nv, g].T) / np.sqrt(32)     # [G, nv]
            want = torch.softmax(z, dim=-1).sum(0).numpy()
            assert np.allclose(s, want, rtol=1e-12, atol=1e-15), (i, g)
            assert np.allclose(lse, torch.logsumexp(z, dim=-1).numpy(), rtol=1e-13, atol=1e-13)


def pin_scores_group_mapping():
    # heads 0,1 form group 0 and heads 2,3 group 1 (consecutive query heads share
    # a kv head).  Group 0's queries are zero -> uniform scores; group 1's queries
    # point at kernel 0 of kv head 1 -> concentrated there.
    sh = _shape(n=128, h_q=4, h_kv=2, d=8)
    p = oracle.params(sh)
    k = np.zeros((128, 2, 8), np.float32)
    k[:32, 1, 0] = 4.0                      # kernel 0 of kv head 1 only
    q = np.zeros((128, 4, 8), np.float32)
    q[:, 2:4, 0] = 8.0
    kb, qb = _bf16(k), _bf16(q)
    kc1 = oracle.compress_k(p, kb)
    i = 127
    nv = (i - 31) // 16 + 1
    s0, _ = oracle.shared_scores_row(p, qb, kc1, i, 0)
    s1, _ = oracle.shared_scores_row(p, qb, kc1, i, 1)
    assert np.allclose(s0, 2.0 / nv, atol=1e-14)
    # kernel 0 of kv head 1 has mean 4 in dim 0 (tokens 0..31); kernel 1 covers
    # tokens 16..47 -> mean 2; later kernels 0.  Logits 32/sqrt(8), 16/sqrt(8), 0.
    z = np.array([32.0, 16.0] + [0.0] * (nv - 2)) / np.sqrt(8)
    want = 2 * np.exp(z - z.max()) / np.exp(z - z.max()).sum()
    assert np.allclose(s1, want, rtol=1e-12, atol=1e-15), (s1[:3], want[:3])


# --------------------------------------------------------------------------
# stage 3: max pooling into block scores
# --------------------------------------------------------------------------

def pin_maxpool_hand():
    p = oracle.params(_shape())
    fx = {ln[0]: ln[1:] for ln in _lines("maxpool_hand.txt")}
    i = int(fx["query"][0])
    shared = np.array([float(x) for x in fx["shared"]])
    assert len(shared) == oracle.visible_kernels(p, i)
    got = oracle.block_scores_row(p, shared, i)
    assert np.array_equal(got, [float(x) for x in fx["expected"]]), got


def pin_maxpool_bruteforce():
    p = oracle.params(_shape())
    rng = np.random.default_rng(4)
    for i in (31, 63, 64, 95, 130, 511, 700):
        nv = oracle.visible_kernels(p, i)
        shared = rng.random(nv)
        got = oracle.block_scores_row(p, shared, i)
        for b in range(i // 64 + 1):
            blk = set(range(64 * b, 64 * b + 64))
            win = [shared[j] for j in range(nv) if blk & set(range(16 * j, 16 * j + 32))]
            want = max(win) if win else -np.inf
            assert got[b] == want, (i, b, got[b], want)


# --------------------------------------------------------------------------
# stage 4: selection
# --------------------------------------------------------------------------

def pin_select_hand():
    fx = list(_lines("select_hand.txt"))
    i = int(fx[0][1])
    cmp_ = np.array([float(x) for x in fx[1][1:]])
    for ln in fx[2:]:
        k = int(ln[1])
        want = [int(x) for x in ln[3:]]
        p = oracle.params(_shape(k=k, n_init=1, n_local=2))
        got = oracle.select_row(p, cmp_, i)
        assert list(got) == want + [-1] * (k - len(want)), (k, got, want)


def _select_bruteforce(cmp_, i, k, n_init, n_local, B=64):
    bi = i // B
    cand = list(range(bi + 1))
    if len(cand) <= k:
        return sorted(cand)
    forced = [b for b in cand if b < n_init or b > bi - n_local]
    rest = sorted((b for b in cand if b not in forced), key=lambda b: (-cmp_[b], b))
    return sorted(forced + rest[:k - len(forced)])


def pin_select_bruteforce():
    rng = np.random.default_rng(8)
    for trial in range(60):
        n_init = int(rng.integers(0, 3))
        n_local = int(rng.integers(1, 3))
        k = int(rng.integers(n_init + n_local, 20))
        i = int(rng.integers(0, 64 * 40))
        # coarse values so that ties are common
        cmp_ = rng.integers(0, 6, size=i // 64 + 1).astype(np.float64) / 4
        p = oracle.params(_shape(k=k, n_init=n_init, n_local=n_local))
        got = [b for b in oracle.select_row(p, cmp_, i) if b >= 0]
        assert got == _select_bruteforce(cmp_, i, k, n_init, n_local), (trial, got)


def pin_select_invariants():
    sh = synth.CONFIGS["prefill_2k"]["shape"]
    data = synth.make_prefill(sh, seed=0)
    p = oracle.params(sh)
    rows = np.array([0, 30, 31, 63, 64, 200, 511, 512, 513, 777, 1500, 2047])
    out = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows)
    for r, i in enumerate(rows):
        bi = i // sh.B
        sel = out["idx"][r, 0]
        got = [b for b in sel if b >= 0]
        assert len(got) == min(sh.k, bi + 1)
        assert all(x < y for x, y in zip(got, got[1:]))
        assert all(0 <= b <= bi for b in got)
        assert all(b == -1 for b in sel[len(got):])
        forced = {b for b in range(bi + 1) if b < sh.n_init or b > bi - sh.n_local}
        assert forced <= set(got), (i, got)


# --------------------------------------------------------------------------
# stage 5: attention
# --------------------------------------------------------------------------

def _sdpa(q, k, v, mask):
    """torch fp64 attention of q [h_q, d] over keys [T, h_kv, d] with a bool mask [T]."""
    h_q, d = q.shape
    G = h_q // k.shape[1]
    kk = k.repeat_interleave(G, dim=1).permute(1, 0, 2)         # [h_q, T, d]
    vv = v.repeat_interleave(G, dim=1).permute(1, 0, 2)
    out = torch.nn.functional.scaled_dot_product_attention(
        q[:, None, :], kk, vv, attn_mask=mask[None, None, :].expand(h_q, 1, -1),
        scale=1.0 / np.sqrt(d))[:, 0, :]
    z = (q[:, None, :] * kk).sum(-1) / np.sqrt(d)
    lse = torch.logsumexp(z.masked_fill(~mask[None, :], -np.inf), dim=-1)
    return out.numpy(), lse.numpy()


def pin_attend_dense_matches_sdpa():
    # n <= k*B: dense causal attention for every row
    sh, data = _small_problem(n=150, h_q=4, h_kv=2, d=16, seed=2, k=8)
    p = oracle.params(sh)
    rows = np.array([0, 1, 17, 63, 64, 100, 149])
    out = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows)
    q, k, v = (torch.from_numpy(_f64(data[x])) for x in ("q", "k", "v"))
    for r, i in enumerate(rows):
        mask = torch.arange(150) <= i
        o, lse = _sdpa(q[i], k, v, mask)
        assert np.allclose(out["o"][r], o, rtol=1e-12, atol=1e-12), i
        assert np.allclose(out["lse"][r], lse, rtol=1e-12, atol=1e-12), i


def pin_attend_block_mask_matches_sdpa():
    sh, data = _small_problem(n=700, h_q=4, h_kv=2, d=16, seed=6, k=3)
    p = oracle.params(sh)
    rows = np.array([5, 64, 130, 300, 450, 699])
    out = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows)
    q, k, v = (torch.from_numpy(_f64(data[x])) for x in ("q", "k", "v"))
    t = torch.arange(700)
    for r, i in enumerate(rows):
        for g in range(2):
            blocks = [b for b in out["idx"][r, g] if b >= 0]
            mask = (t <= i) & torch.isin(t // 64, torch.tensor(blocks))
            o, lse = _sdpa(q[i, 2 * g:2 * g + 2], k[:, g:g + 1], v[:, g:g + 1], mask)
            assert np.allclose(out["o"][r, 2 * g:2 * g + 2], o, rtol=1e-12, atol=1e-12), (i, g)
            assert np.allclose(out["lse"][r, 2 * g:2 * g + 2], lse, rtol=1e-12, atol=1e-12)


def pin_attend_closed_forms():
    # equal keys -> uniform weights -> O is the mean of the visible values and
    # lse = z + log(count)
    sh = _shape(n=130, h_q=2, h_kv=1, d=8, k=8)
    p = oracle.params(sh)
    rng = np.random.default_rng(1)
    q = _bf16(rng.standard_normal((130, 2, 8)))
    krow = _bf16(rng.standard_normal(8))
    k = np.broadcast_to(krow, (130, 1, 8)).copy()
    v = _bf16(rng.standard_normal((130, 1, 8)))
    vv = _f64(v)
    for i in (0, 5, 64, 129):
        blocks = list(range(i // 64 + 1))
        o, lse = oracle.attend_row(p, q, k, v, i, 0, blocks)
        want = vv[:i + 1, 0].mean(0)
        assert np.allclose(o, want[None], rtol=1e-12, atol=1e-13), i
        z = _f64(q)[i] @ _f64(krow) / np.sqrt(8)
        assert np.allclose(lse, z + np.log(i + 1), rtol=1e-12, atol=1e-12)


def pin_early_rows_are_dense():
    # in a sparse sequence, a query with at most k visible blocks attends densely
    sh, data = _small_problem(n=1000, h_q=2, h_kv=1, d=16, seed=12, k=4)
    p = oracle.params(sh)
    rows = np.array([10, 100, 200, 255])
    out = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows)
    q, k, v = (torch.from_numpy(_f64(data[x])) for x in ("q", "k", "v"))
    for r, i in enumerate(rows):
        o, lse = _sdpa(q[i], k, v, torch.arange(1000) <= i)
        assert np.allclose(out["o"][r], o, rtol=1e-12, atol=1e-12), i


# --------------------------------------------------------------------------
# backward of the attention (block lists fixed)
# --------------------------------------------------------------------------

def _bwd_problem(n=300, h_q=4, h_kv=2, d=16, seed=31, k=3):
    sh, data = _small_problem(n=n, h_q=h_q, h_kv=h_kv, d=d, seed=seed, k=k)
    p = oracle.params(sh)
    rows = np.arange(n, dtype=np.int32)
    fwd = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows)
    rng = np.random.default_rng(seed + 1)
    d_o = _bf16(rng.standard_normal((n, h_q, d)))
    return sh, p, data, rows, fwd, d_o


def pin_attend_bwd_matches_autograd():
    """Every row's block-sparse causal attention written as one masked softmax
    in torch fp64; autograd of sum(O * dO) gives dq, dk, dv."""
    sh, p, data, rows, fwd, d_o = _bwd_problem()
    n, G = sh.n, sh.G
    dq, dk, dv = oracle.attend_bwd_rows(p, data["q"], data["k"], data["v"], d_o, rows, fwd["idx"], fwd["o"])
    q, k, v, go = (torch.from_numpy(_f64(x)).requires_grad_(True) for x in (data["q"], data["k"], data["v"], d_o))
    t = torch.arange(n)
    mask = torch.zeros((sh.h_kv, n, n), dtype=torch.bool)
    for i in range(n):
        for g in range(sh.h_kv):
            blocks = torch.tensor([b for b in fwd["idx"][i, g] if b >= 0])
            mask[g, i] = (t <= i) & torch.isin(t // 64, blocks)
    kk = k.repeat_interleave(G, dim=1).permute(1, 0, 2)      # [h_q, n, d]
    vv = v.repeat_interleave(G, dim=1).permute(1, 0, 2)
    qq = q.permute(1, 0, 2)
    z = qq @ kk.transpose(1, 2) / np.sqrt(sh.d)
    z = z.masked_fill(~mask.repeat_interleave(G, dim=0), -np.inf)
    o = torch.softmax(z, dim=-1) @ vv                        # [h_q, n, d]
    (o * go.detach().permute(1, 0, 2)).sum().backward()
    assert np.allclose(o.detach().permute(1, 0, 2).numpy(), fwd["o"], rtol=0, atol=1e-12)
    assert np.allclose(dq, q.grad.numpy(), rtol=0, atol=1e-11), np.abs(dq - q.grad.numpy()).max()
    assert np.allclose(dk, k.grad.numpy(), rtol=0, atol=1e-11), np.abs(dk - k.grad.numpy()).max()
    assert np.allclose(dv, v.grad.numpy(), rtol=0, atol=1e-11), np.abs(dv - v.grad.numpy()).max()


def pin_attend_bwd_closed_forms():
    """Row 0 sees token 0 only: P = 1, so dq_0 = 0 and token 0 receives dv = dO_0
    (plus the later rows' shares).  Over all rows, sum_t dv_t = sum of dO over
    the rows and the group's heads, and sum_t dk_t = 0 (sum_t dS_t = 0)."""
    sh, p, data, rows, fwd, d_o = _bwd_problem(n=260, seed=41)
    dq, dk, dv = oracle.attend_bwd_rows(p, data["q"], data["k"], data["v"], d_o, rows[:1],
                                        fwd["idx"][:1], fwd["o"][:1])
    assert np.all(dq[0] == 0.0)
    assert np.allclose(dv[0], _f64(d_o)[0].reshape(sh.h_kv, sh.G, sh.d).sum(axis=1), rtol=0, atol=1e-14)
    assert np.all(dk == 0.0) and np.all(dv[1:] == 0.0)
    dq, dk, dv = oracle.attend_bwd_rows(p, data["q"], data["k"], data["v"], d_o, rows, fwd["idx"], fwd["o"])
    go = _f64(d_o).reshape(sh.n, sh.h_kv, sh.G, sh.d).sum(axis=2)      # [n, h_kv, d]
    assert np.allclose(dv.sum(axis=0), go.sum(axis=0), rtol=0, atol=1e-10)
    assert np.allclose(dk.sum(axis=0), 0.0, rtol=0, atol=1e-10), np.abs(dk.sum(axis=0)).max()


# --------------------------------------------------------------------------
# rounding, padding and the batch entry points
# --------------------------------------------------------------------------

_BF16_MAX = float(Fraction(2) ** 127 * (2 - Fraction(1, 128)))   # largest finite bf16


def pin_compress_keeps_every_bf16_value():
    """The mean of 32 copies of a bf16 value is that value, so compression must
    return every finite bf16 bit pattern unchanged: every subnormal, 1.0, the
    largest finite value.  A zero mean is +0 (the sum starts from +0, so 32
    copies of -0 give +0: the sign of a zero is a convention, not a value)."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = np.where((bits & 0x7F80) != 0x7F80, bits, 0).astype(np.uint16)
    vals[vals == 0x8000] = 0
    h_kv = 512
    p = oracle.params(_shape(n=32, h_q=h_kv, h_kv=h_kv, d=128))
    k = np.broadcast_to(vals.reshape(1, h_kv, 128), (32, h_kv, 128)).copy()
    kc1 = oracle.compress_k(p, k)
    assert kc1.shape == (1, h_kv, 128), kc1.shape
    got = kc1[0].reshape(-1)
    bad = np.nonzero(got != vals)[0]
    assert bad.size == 0, [(hex(int(vals[x])), hex(int(got[x]))) for x in bad[:5]]


def pin_bf16_round_nearest_even():
    """Rounding of arbitrary doubles to bf16 against exact rational arithmetic:
    normal and subnormal magnitudes, exact halfway points, and the overflow
    edge (at or beyond the largest finite value plus half an ulp: infinity)."""
    rng = np.random.default_rng(31)
    xs = list(rng.standard_normal(300) * np.exp2(rng.integers(-140, 128, 300)))
    for b in rng.integers(0, 0x7F7F, 200):             # midpoints between neighbours
        lo = float(_f64(np.array([b], np.uint16))[0])
        hi = float(_f64(np.array([b + 1], np.uint16))[0])
        xs += [(lo + hi) / 2, -(lo + hi) / 2]
    half_ulp = float(Fraction(2) ** (127 - 8))
    xs += [_BF16_MAX, _BF16_MAX + half_ulp / 2, _BF16_MAX + half_ulp, 1.0, -1.0, 2.0 ** -133,
           2.0 ** -134, 3 * 2.0 ** -135, 0.0, -0.0]
    for x in xs:
        got = float(_f64(np.array([oracle.bf16_round(x)], np.uint16))[0])
        want = _rne_bf16_fraction(Fraction(x))
        if abs(want) > _BF16_MAX:
            want = np.copysign(np.inf, x)
        assert got == want and np.signbit(got) == np.signbit(x if x != 0 else x), (x, got, want)


def pin_batch_rows_match_single_rows():
    """The batch entry points (several rows, two kv heads) put every row and
    head where the single-row stages put it: S^shared (zero beyond the visible
    kernels), the score log-sum-exp, S^cmp (minus infinity beyond the query's
    block), the selection and the attention."""
    for n in (700, 640):                               # 640: a whole number of blocks
        _batch_rows_case(n, np.array([0, 40, 64, 300, 511, n - 60, n - 1], np.int32))


def _batch_rows_case(n, rows):
    sh, data = _small_problem(n=n, h_q=8, h_kv=2, d=16, seed=21, k=4)
    p = oracle.params(sh)
    G = sh.h_q // sh.h_kv
    out = oracle.prefill_rows(p, data["q"], data["k"], data["v"], rows, want_cmp=True,
                              want_shared=True, want_score_lse=True)
    kc1 = oracle.compress_k(p, data["k"])
    nc = oracle.num_kernels(p, sh.n)
    for r, i in enumerate(rows):
        nv = oracle.visible_kernels(p, int(i))
        bi = int(i) // 64
        for g in range(sh.h_kv):
            s_row, lse = oracle.shared_scores_row(p, data["q"], kc1, int(i), g)
            assert np.array_equal(out["shared"][r, g, :nv], s_row), (i, g)
            assert np.all(out["shared"][r, g, nv:nc] == 0.0), (i, g)
            assert np.array_equal(out["score_lse"][r, g * G:(g + 1) * G], lse), (i, g)
            cmp_row = oracle.block_scores_row(p, s_row, int(i))
            assert np.array_equal(out["cmp"][r, g, :bi + 1], cmp_row), (i, g)
            assert np.all(out["cmp"][r, g, bi + 1:] == -np.inf), (i, g)
            idx = oracle.select_row(p, cmp_row, int(i))
            assert np.array_equal(out["idx"][r, g], idx), (i, g)
            o, l = oracle.attend_row(p, data["q"], data["k"], data["v"], int(i), g, idx)
            assert np.array_equal(out["o"][r, g * G:(g + 1) * G], o), (i, g)
            assert np.array_equal(out["lse"][r, g * G:(g + 1) * G], l), (i, g)
    # the selection and attention batch entries over the same rows
    ld = nc + 5
    shared = np.full((len(rows), sh.h_kv, ld), 7.0)    # padding beyond nv must not be read
    for r, i in enumerate(rows):
        nv = oracle.visible_kernels(p, int(i))
        shared[r, :, :nv] = out["shared"][r, :, :nv]
    n_blk = (sh.n + 63) // 64
    idx, cmp_ = oracle.select_rows(p, shared, rows, n_blk)
    assert np.array_equal(idx, out["idx"])
    assert np.array_equal(cmp_, out["cmp"])
    o, lse = oracle.attend_rows(p, data["q"], data["k"], data["v"], rows, out["idx"])
    assert np.array_equal(o, out["o"]) and np.array_equal(lse, out["lse"])


def pin_attend_empty_block_list():
    """A query that selected no block attends to nothing: O = 0, lse = -inf."""
    sh, data = _small_problem(n=200, h_q=4, h_kv=2, d=16, seed=3, k=4)
    p = oracle.params(sh)
    o, lse = oracle.attend_row(p, data["q"], data["k"], data["v"], 150, 1, [-1, -1, -1, -1])
    assert np.all(o == 0.0) and np.all(lse == -np.inf), (o, lse)


def pin_attend_blocks_past_the_query_add_nothing():
    """T(i) holds only tokens t <= i (arXiv summary, Appendix A; the causal
    visible-token set): list entries past the query's own block, in range or
    beyond the sequence, leave O and lse bit for bit as the list without them,
    and a list of only such entries is the empty set (O = 0, lse = -inf)."""
    sh, data = _small_problem(n=300, h_q=4, h_kv=2, d=16, seed=5, k=6)
    p = oracle.params(sh)
    i, g = 150, 0                    # own block 2; blocks 3, 4 are in range but later
    base = [0, 1, 2, -1, -1, -1]
    more = [0, 1, 2, 3, 4, 10 ** 6]
    o0, l0 = oracle.attend_row(p, data["q"], data["k"], data["v"], i, g, base)
    o1, l1 = oracle.attend_row(p, data["q"], data["k"], data["v"], i, g, more)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
    assert np.all(np.isfinite(l0))
    o2, l2 = oracle.attend_row(p, data["q"], data["k"], data["v"], i, g, [3, 4, 10 ** 6, -1, -1, -1])
    assert np.all(o2 == 0.0) and np.all(l2 == -np.inf), (o2, l2)


def pin_maxpool_literal_window():
    """The literal reading of the max-pool window (kernels 4b .. 4b+4 of the
    visible ones; pool_rule = 1), by brute force, and that it differs from
    the intersection rule exactly where kernel 4b-1 or 4b+4 decides the max."""
    p1 = oracle.params(_shape(), pool_rule=1)
    p0 = oracle.params(_shape())
    rng = np.random.default_rng(8)
    differs = 0
    for i in (31, 63, 64, 95, 130, 511, 700):
        nv = oracle.visible_kernels(p1, i)
        shared = rng.random(nv)
        got = oracle.block_scores_row(p1, shared, i)
        inter = oracle.block_scores_row(p0, shared, i)
        for b in range(i // 64 + 1):
            win = [shared[j] for j in range(4 * b, 4 * b + 5) if j < nv]
            assert got[b] == (max(win) if win else -np.inf), (i, b)
            differs += got[b] != inter[b]
    assert differs > 0


ALL_PINS = [v for k_, v in sorted(globals().items()) if k_.startswith("pin_")]
