"""ctypes front end of the fp64 CPU oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg use it.  The CUDA library never imports it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("l_c1", ctypes.c_int), ("s_c1", ctypes.c_int),
                ("pool_l", ctypes.c_int), ("pool_s", ctypes.c_int),
                ("n_init", ctypes.c_int), ("n_local", ctypes.c_int), ("k", ctypes.c_int),
                ("h_q", ctypes.c_int), ("h_kv", ctypes.c_int), ("d", ctypes.c_int),
                ("scale", ctypes.c_double), ("pool_rule", ctypes.c_int),
                ("lse_approx", ctypes.c_int)]


def params(shape, scale=None, pool_rule=0, lse_approx=0) -> Params:
    """Oracle parameters from a synth.Shape (scale defaults to 1/sqrt(d))."""
    sc = 1.0 / np.sqrt(shape.d) if scale is None else float(scale)
    return Params(shape.B, shape.l_c1, shape.s_c1, shape.pool_l, shape.pool_s,
                  shape.n_init, shape.n_local, shape.k, shape.h_q, shape.h_kv, shape.d,
                  sc, pool_rule, lse_approx)


def _declare(L):
    P = ctypes.POINTER(Params)
    vp = ctypes.c_void_p
    i = ctypes.c_int
    L.orc_num_threads.restype = i
    L.orc_bf16_round.restype = ctypes.c_uint16
    L.orc_bf16_round.argtypes = [ctypes.c_double]
    L.orc_num_kernels.argtypes = [P, i]
    L.orc_visible_kernels.argtypes = [P, i]
    L.orc_compress_k.argtypes = [P, vp, i, vp]
    L.orc_num_coarse_kernels.argtypes = [P, i]
    L.orc_visible_coarse_kernels.argtypes = [P, i]
    L.orc_compress_k2.argtypes = [P, vp, i, vp]
    L.orc_coarse_lse_row.argtypes = [P, vp, vp, i, i, vp]
    L.orc_shared_scores_row_lse.argtypes = [P, vp, vp, i, i, vp, vp, vp]
    L.orc_shared_scores_row.argtypes = [P, vp, vp, i, i, vp, vp]
    L.orc_block_scores_row.argtypes = [P, vp, i, i, vp]
    L.orc_select_row.argtypes = [P, vp, i, vp]
    L.orc_attend_row.argtypes = [P, vp, vp, vp, i, i, vp, i, vp, vp]
    L.orc_prefill_rows.argtypes = [P, vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp, vp]
    L.orc_select_rows.argtypes = [P, vp, i, vp, i, vp, vp, i]
    L.orc_attend_rows.argtypes = [P, vp, vp, vp, vp, i, vp, vp, vp]
    L.orc_attend_bwd_rows.argtypes = [P, vp, vp, vp, vp, i, vp, i, vp, vp, vp, vp, vp]
    return L


def load(path: str):
    """Load an oracle build from `path` (tests load planted-mistake builds this way)."""
    return _declare(ctypes.CDLL(path))


def lib():
    global _lib
    if _lib is None:
        _lib = load(build())
    return _lib


_active = None


class use:
    """Context manager: route this module's functions to another oracle build."""

    def __init__(self, handle):
        self.handle = handle

    def __enter__(self):
        global _active
        self.prev, _active = _active, self.handle
        return self

    def __exit__(self, *exc):
        global _active
        _active = self.prev


def _L():
    return _active if _active is not None else lib()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return _L().orc_num_threads()


def bf16_round(x: float) -> int:
    return int(_L().orc_bf16_round(float(x)))


def num_kernels(p: Params, n: int) -> int:
    return _L().orc_num_kernels(ctypes.byref(p), n)


def visible_kernels(p: Params, i: int) -> int:
    return _L().orc_visible_kernels(ctypes.byref(p), i)


def compress_k(p: Params, k: np.ndarray) -> np.ndarray:
    k = _c(k, np.uint16)
    n = k.shape[0]
    out = np.zeros((max(num_kernels(p, n), 0), p.h_kv, p.d), np.uint16)
    _L().orc_compress_k(ctypes.byref(p), _ptr(k), n, _ptr(out))
    return out


def num_coarse_kernels(p: Params, n: int) -> int:
    return _L().orc_num_coarse_kernels(ctypes.byref(p), n)


def visible_coarse_kernels(p: Params, i: int) -> int:
    return _L().orc_visible_coarse_kernels(ctypes.byref(p), i)


def compress_k2(p: Params, k: np.ndarray) -> np.ndarray:
    """Coarse kernels K^C2 of the LSE approximation (l_C2 = 4 l_C1, s_C2 = 4 s_C1)."""
    k = _c(k, np.uint16)
    n = k.shape[0]
    out = np.zeros((max(num_coarse_kernels(p, n), 0), p.h_kv, p.d), np.uint16)
    _L().orc_compress_k2(ctypes.byref(p), _ptr(k), n, _ptr(out))
    return out


def coarse_lse_row(p: Params, q, kc2, i: int, g: int):
    """Approximate per-head LSE of row i (None when no coarse kernel is visible)."""
    q = _c(q, np.uint16)
    kc2 = _c(kc2, np.uint16)
    out = np.zeros(p.h_q // p.h_kv, np.float64)
    ok = _L().orc_coarse_lse_row(ctypes.byref(p), _ptr(q), _ptr(kc2), i, g, _ptr(out))
    return out if ok else None


def shared_scores_row_lse(p: Params, q, kc1, i: int, g: int, lse_in=None):
    """S^shared of row i normalised by the given per-head LSE (exact when None)."""
    q = _c(q, np.uint16)
    kc1 = _c(kc1, np.uint16)
    nv = visible_kernels(p, i)
    out = np.zeros(max(nv, 1), np.float64)
    lse = np.zeros(p.h_q // p.h_kv, np.float64)
    li = None if lse_in is None else _c(np.asarray(lse_in, np.float64), np.float64)
    _L().orc_shared_scores_row_lse(ctypes.byref(p), _ptr(q), _ptr(kc1), i, g,
                                   None if li is None else _ptr(li), _ptr(out), _ptr(lse))
    return out[:nv], lse


def shared_scores_row(p: Params, q, kc1, i: int, g: int):
    """(S^shared[j] for visible j, per-head natural LSE of the S^C1 softmax)."""
    q = _c(q, np.uint16)
    kc1 = _c(kc1, np.uint16)
    nv = visible_kernels(p, i)
    out = np.zeros(max(nv, 1), np.float64)
    lse = np.zeros(p.h_q // p.h_kv, np.float64)
    _L().orc_shared_scores_row(ctypes.byref(p), _ptr(q), _ptr(kc1), i, g, _ptr(out), _ptr(lse))
    return out[:nv], lse


def block_scores_row(p: Params, shared, i: int) -> np.ndarray:
    shared = _c(shared, np.float64)
    out = np.zeros(i // p.B + 1, np.float64)
    _L().orc_block_scores_row(ctypes.byref(p), _ptr(shared), len(shared), i, _ptr(out))
    return out


def select_row(p: Params, s_cmp, i: int) -> np.ndarray:
    s_cmp = _c(s_cmp, np.float64)
    idx = np.zeros(p.k, np.int32)
    _L().orc_select_row(ctypes.byref(p), _ptr(s_cmp), i, _ptr(idx))
    return idx


def attend_row(p: Params, q, k, v, i: int, g: int, idx):
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    idx = _c(idx, np.int32)
    G = p.h_q // p.h_kv
    o = np.zeros((G, p.d), np.float64)
    lse = np.zeros(G, np.float64)
    _L().orc_attend_row(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), i, g, _ptr(idx),
                         len(idx), _ptr(o), _ptr(lse))
    return o, lse


def prefill_rows(p: Params, q, k, v, rows, want_cmp=False, want_shared=False,
                 want_score_lse=False) -> dict:
    """The whole layer at the given query rows of one sequence (see oracle.c)."""
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    rows = _c(rows, np.int32)
    n = k.shape[0]
    nr = len(rows)
    n_blk = (n + p.B - 1) // p.B
    nc = num_kernels(p, n)
    idx = np.zeros((nr, p.h_kv, p.k), np.int32)
    o = np.zeros((nr, p.h_q, p.d), np.float64)
    lse = np.zeros((nr, p.h_q), np.float64)
    cmp_ = np.zeros((nr, p.h_kv, n_blk), np.float64) if want_cmp else None
    sh = np.zeros((nr, p.h_kv, max(nc, 1)), np.float64) if want_shared else None
    sl = np.zeros((nr, p.h_q), np.float64) if want_score_lse else None
    _L().orc_prefill_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), n, _ptr(rows), nr,
                           _ptr(idx), _ptr(o), _ptr(lse), _ptr(cmp_), _ptr(sh), _ptr(sl))
    out = dict(idx=idx, o=o, lse=lse)
    if want_cmp:
        out["cmp"] = cmp_
    if want_shared:
        out["shared"] = sh[:, :, :nc]
    if want_score_lse:
        out["score_lse"] = sl
    return out


def select_rows(p: Params, shared, rows, n_blk: int):
    """Selection from given S^shared rows [nrows][h_kv][ld] (float64 values)."""
    shared = _c(shared, np.float64)
    rows = _c(rows, np.int32)
    nr = len(rows)
    idx = np.zeros((nr, p.h_kv, p.k), np.int32)
    cmp_ = np.zeros((nr, p.h_kv, n_blk), np.float64)
    _L().orc_select_rows(ctypes.byref(p), _ptr(shared), shared.shape[-1], _ptr(rows), nr,
                          _ptr(idx), _ptr(cmp_), n_blk)
    return idx, cmp_


def attend_rows(p: Params, q, k, v, rows, idx):
    q, k, v = _c(q, np.uint16), _c(k, np.uint16), _c(v, np.uint16)
    rows = _c(rows, np.int32)
    idx = _c(idx, np.int32)
    nr = len(rows)
    o = np.zeros((nr, p.h_q, p.d), np.float64)
    lse = np.zeros((nr, p.h_q), np.float64)
    _L().orc_attend_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(rows), nr,
                          _ptr(idx), _ptr(o), _ptr(lse))
    return o, lse


def attend_bwd_rows(p: Params, q, k, v, d_o, rows, idx, o):
    """Backward of the attention at the given rows (see oracle.c).
    o: [nrows, h_q, d] forward output (float); idx: [nrows, h_kv, k].
    Returns dq [nrows, h_q, d] and dk, dv [n, h_kv, d] summed over those rows."""
    q, k, v, d_o = (_c(x, np.uint16) for x in (q, k, v, d_o))
    rows = _c(rows, np.int32)
    idx = _c(idx, np.int32)
    o = _c(np.asarray(o, np.float64), np.float64)
    n = k.shape[0]
    nr = len(rows)
    dq = np.zeros((nr, p.h_q, p.d), np.float64)
    dk = np.zeros((n, p.h_kv, p.d), np.float64)
    dv = np.zeros((n, p.h_kv, p.d), np.float64)
    _L().orc_attend_bwd_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(d_o), n, _ptr(rows),
                             nr, _ptr(idx), _ptr(o), _ptr(dq), _ptr(dk), _ptr(dv))
    return dq, dk, dv
