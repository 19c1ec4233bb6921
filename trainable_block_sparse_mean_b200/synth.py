"""Seeded synthetic inputs for InfLLM-V2 block-sparse attention.

This module only draws random numbers and rounds them to bf16.  It holds none of
the method's arithmetic (no pooling, scoring, selection or attention), so both
the CUDA path and the fp64 oracle can consume its arrays without sharing any of
the computation.

Recipe (the pages measure on RULER/LongBench with a trained 8B model; these
seeded arrays stand in for those workloads with the model's attention shapes,
h_q=32, h_kv=2, d=128, from "InfLLM-V2" page 1, Experiments):

* Q and V: i.i.d. N(0, 1).
* K: i.i.d. N(0, 1) plus one offset vector per (kv head, 64-token block) drawn
  from N(0, 0.5**2) per dimension, so that blocks differ in how relevant they
  are to a query.
* Needles (configs with n_needles > 0): needle m picks a target query
  t_m ~ U[k*B, n) and a kernel-aligned span start p_m = 16*u in block >= 1 with
  p_m + 31 < t_m - n_local*B.  For every kv head g it adds gamma=8 times the
  unit vector of sum_{h in g} Q[t_m, h] to K[p_m : p_m+32, g].
* Everything is drawn in float32 and rounded once to bf16 (round to nearest,
  ties to even).  Arrays of bf16 are returned as uint16 bit patterns.
"""
from __future__ import annotations

import dataclasses

import numpy as np

__all__ = [
    "Shape", "CONFIGS", "bf16_bits", "bf16_to_f32", "make_prefill",
    "make_varlen", "make_decode", "cu_seqlens_of",
]


@dataclasses.dataclass(frozen=True)
class Shape:
    """Method parameters and sizes of one workload."""
    n: int = 2048
    h_q: int = 4
    h_kv: int = 1
    d: int = 128
    B: int = 64
    l_c1: int = 32
    s_c1: int = 16
    pool_l: int = 5
    pool_s: int = 4
    n_init: int = 1
    n_local: int = 2
    k: int = 8
    n_needles: int = 0

    @property
    def G(self) -> int:
        return self.h_q // self.h_kv


# The five workloads (sizes from the method's 8B GQA backbone and selection
# hyper-parameters: block 64, kernel 32, stride 16, pooling 5/4).
CONFIGS = {
    # single 2k sequence, G=4, 8 blocks total: small enough for the oracle
    "prefill_2k": dict(shape=Shape(n=2048, h_q=4, h_kv=1, k=8)),
    # single 32k sequence, G=16, 64 blocks (4096 keys), 32 needles
    "prefill_32k": dict(shape=Shape(n=32768, h_q=32, h_kv=2, k=64, n_needles=32)),
    # single 128k sequence, G=16, 64 blocks, 128 needles
    "prefill_128k": dict(shape=Shape(n=131072, h_q=32, h_kv=2, k=64, n_needles=128)),
    # batched decode: 32 sequences with cache lengths U[16384, 131072]
    "decode_batch32": dict(shape=Shape(n=0, h_q=32, h_kv=2, k=64), batch=32,
               len_lo=16384, len_hi=131072, steps=64),
    # dense/sparse switch sweep: eight sequences of 1k..96k tokens
    "varlen_sweep": dict(shape=Shape(n=0, h_q=32, h_kv=2, k=64),
               lengths=(1024, 2048, 4096, 8192, 16384, 32768, 65536, 98304)),
}


def bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen uint16 bf16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _normal(rng: np.random.Generator, shape, dtype=np.float32) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=dtype)


def make_prefill(shape: Shape, seed: int = 0, n: int | None = None,
                 n_needles: int | None = None) -> dict:
    """One sequence of n tokens: q [n,h_q,d], k/v [n,h_kv,d] as bf16 bits.

    The draw order is fixed (Q, K noise, K block offsets, V, needles) so that a
    seed names one array set.
    """
    n = shape.n if n is None else n
    n_needles = shape.n_needles if n_needles is None else n_needles
    rng = np.random.default_rng(seed)
    h_q, h_kv, d, B = shape.h_q, shape.h_kv, shape.d, shape.B
    n_blk = (n + B - 1) // B
    q = bf16_bits(_normal(rng, (n, h_q, d)))
    kf = _normal(rng, (n, h_kv, d))
    off = _normal(rng, (h_kv, max(n_blk, 1), d)) * np.float32(0.5)
    for g in range(h_kv):
        # token t gets the offset of its block t // B
        kf[:, g, :] += np.repeat(off[g], B, axis=0)[:n]
    v = bf16_bits(_normal(rng, (n, h_kv, d)))
    needles = []
    lo_t = shape.k * shape.B
    G = shape.G
    for _ in range(n_needles):
        if n <= lo_t:
            break
        t = int(rng.integers(lo_t, n))
        hi_u = (t - shape.n_local * B - shape.l_c1) // shape.s_c1
        lo_u = B // shape.s_c1
        if hi_u < lo_u:
            continue
        p = shape.s_c1 * int(rng.integers(lo_u, hi_u + 1))
        qf = bf16_to_f32(q[t])
        for g in range(h_kv):
            dirv = qf[g * G:(g + 1) * G].sum(axis=0, dtype=np.float64)
            dirv = dirv / max(np.linalg.norm(dirv), 1e-30)
            kf[p:p + shape.l_c1, g, :] += np.float32(8.0) * dirv.astype(np.float32)
        needles.append((t, p))
    k = bf16_bits(kf)
    return dict(q=q, k=k, v=v, n=n, needles=needles)


def cu_seqlens_of(lengths) -> np.ndarray:
    out = np.zeros(len(lengths) + 1, dtype=np.int32)
    out[1:] = np.cumsum(np.asarray(lengths, dtype=np.int64)).astype(np.int32)
    return out


def make_varlen(shape: Shape, lengths, seed: int = 0, n_needles: int = 0) -> dict:
    """Packed varlen batch ("thd" layout); sequence s is drawn from seed [seed, s]."""
    parts = [make_prefill(shape, seed=[seed, s], n=int(L), n_needles=n_needles)
             for s, L in enumerate(lengths)]
    cat = lambda key: np.concatenate([p[key] for p in parts], axis=0)
    return dict(q=cat("q"), k=cat("k"), v=cat("v"),
                cu_seqlens=cu_seqlens_of(lengths), lengths=list(map(int, lengths)))


def decode_lengths(batch: int, lo: int, hi: int, seed: int = 0) -> np.ndarray:
    """Cache length per sequence, uniform on [lo, hi]."""
    rng = np.random.default_rng(seed)
    return rng.integers(lo, hi + 1, size=batch).astype(np.int32)


def make_decode_sequence(shape: Shape, L: int, steps: int, seed: int, s: int) -> dict:
    """History of sequence s (L cached tokens) plus `steps` new tokens.

    Returns k/v [L+steps, h_kv, d] (the first L rows are the cache, row L+t is
    the token appended at decode step t) and q_new [steps, h_q, d].  The same
    value distributions as make_prefill (no needles), but only the queries of
    the new tokens are drawn: a decode step never reads the history's queries.
    Draw order: q_new, K noise, K block offsets, V, from seed [seed, 1000 + s].
    """
    rng = np.random.default_rng([seed, 1000 + s])
    n = L + steps
    h_kv, d, B = shape.h_kv, shape.d, shape.B
    n_blk = (n + B - 1) // B
    q_new = bf16_bits(_normal(rng, (steps, shape.h_q, d)))
    kf = _normal(rng, (n, h_kv, d))
    off = _normal(rng, (h_kv, max(n_blk, 1), d)) * np.float32(0.5)
    for g in range(h_kv):
        kf[:, g, :] += np.repeat(off[g], B, axis=0)[:n]
    v = bf16_bits(_normal(rng, (n, h_kv, d)))
    return dict(k=bf16_bits(kf), v=v, q_new=q_new, L=L)


def make_decode(shape: Shape, batch: int, len_lo: int, len_hi: int, steps: int,
                seed: int = 0, cap: int | None = None, only=None) -> dict:
    """Batched decode workload in cache layout.

    k_cache/v_cache [batch, h_kv, cap, d] hold each sequence's first L_s tokens;
    k_new/v_new [steps, batch, h_kv, d] and q [steps, batch, h_q, d] are the
    tokens of each decode step.  `only` restricts generation to a subset of
    sequences (others stay zero) for tests that check a sample.
    """
    lens = decode_lengths(batch, len_lo, len_hi, seed)
    cap = int(cap if cap is not None else int(lens.max()) + steps)
    h_q, h_kv, d = shape.h_q, shape.h_kv, shape.d
    k_cache = np.zeros((batch, h_kv, cap, d), np.uint16)
    v_cache = np.zeros((batch, h_kv, cap, d), np.uint16)
    k_new = np.zeros((steps, batch, h_kv, d), np.uint16)
    v_new = np.zeros((steps, batch, h_kv, d), np.uint16)
    q = np.zeros((steps, batch, h_q, d), np.uint16)
    sel = range(batch) if only is None else only
    for s in sel:
        L = int(lens[s])
        sq = make_decode_sequence(shape, L, steps, seed, s)
        k_cache[s, :, :L] = sq["k"][:L].transpose(1, 0, 2)
        v_cache[s, :, :L] = sq["v"][:L].transpose(1, 0, 2)
        k_new[:, s] = sq["k"][L:L + steps]
        v_new[:, s] = sq["v"][L:L + steps]
        q[:, s] = sq["q_new"]
    return dict(k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                q=q, lens=lens, cap=cap)
