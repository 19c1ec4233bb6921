"""Thin Python binding of libinfv2.so (argument marshalling only).

Every function has the name of the C entry point it calls and takes torch
CUDA tensors; all computation happens in the library's kernels.  A missing
library or a non-zero status raises.  Nothing here falls back to the CPU.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# INFV2_BUILD=checks loads the INFV2_CHECKS debug build (device-side index and
# invariant checks) instead of the default one.
LIB_PATH = os.path.join(_HERE, "libinfv2_checks.so" if os.environ.get("INFV2_BUILD") == "checks"
                        else "libinfv2.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_CHECK = range(7)

SYMBOLS = [
    "infv2_default_params", "infv2_check_params", "infv2_status_string", "infv2_num_kernels",
    "infv2_device_status", "infv2_compress_k", "infv2_block_scores", "infv2_select_topk",
    "infv2_sparse_attn", "infv2_dense_attn", "infv2_prefill_workspace_size", "infv2_prefill",
    "infv2_decode_workspace_size", "infv2_decode", "infv2_select_blocks_noalloc",
    "infv2_selftest_timeout", "infv2_block_scores_pooled", "infv2_select_topk_pooled",
    "infv2_compress_k2", "infv2_block_scores_approx", "infv2_sparse_attn_bwd_workspace_size",
    "infv2_sparse_attn_bwd", "infv2_pipeline_workspace_size", "infv2_pipeline_create",
    "infv2_pipeline_submit", "infv2_pipeline_wait", "infv2_pipeline_join", "infv2_pipeline_sync",
    "infv2_pipeline_destroy", "infv2_sparse_attn_rows", "infv2_decode_attn",
    "infv2_selftest_exp2", "infv2_varlen_kernel_offsets", "infv2_compress_k_varlen",
    "infv2_block_scores_varlen", "infv2_select_topk_varlen", "infv2_sparse_attn_varlen",
    "infv2_dense_attn_varlen", "infv2_get_device_status",
]


class Params(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("l_c1", ctypes.c_int), ("s_c1", ctypes.c_int),
                ("pool_l", ctypes.c_int), ("pool_s", ctypes.c_int), ("n_init", ctypes.c_int),
                ("n_local", ctypes.c_int), ("k", ctypes.c_int), ("h_q", ctypes.c_int),
                ("h_kv", ctypes.c_int), ("d", ctypes.c_int), ("scale", ctypes.c_float),
                ("window", ctypes.c_int), ("lse_approx", ctypes.c_int)]


class Infv2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s failed: %s (status %d)" % (where, status_string(status), status))
        self.status = status


_lib = None


def lib():
    """Load libinfv2.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("%s not built: run python -m trainable_block_sparse_mean_b200.build"
                              % os.path.basename(LIB_PATH))
        L = ctypes.CDLL(LIB_PATH)
        P = ctypes.POINTER(Params)
        vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        L.infv2_default_params.argtypes = [P, i, i]
        L.infv2_default_params.restype = None
        L.infv2_check_params.argtypes = [P]
        L.infv2_status_string.argtypes = [i]
        L.infv2_status_string.restype = ctypes.c_char_p
        L.infv2_num_kernels.argtypes = [P, i]
        L.infv2_device_status.argtypes = [vp]
        L.infv2_get_device_status.argtypes = [vp]
        L.infv2_compress_k.argtypes = [P, vp, i, vp, vp]
        L.infv2_block_scores.argtypes = [P, vp, vp, i, i, i, vp, i, vp, vp]
        L.infv2_select_topk.argtypes = [P, vp, i, i, i, i, vp, vp]
        L.infv2_block_scores_pooled.argtypes = [P, vp, vp, i, i, i, vp, i, vp]
        L.infv2_compress_k2.argtypes = [P, vp, i, vp, vp]
        L.infv2_sparse_attn_bwd_workspace_size.argtypes = [P, i, ctypes.POINTER(sz)]
        L.infv2_sparse_attn_bwd.argtypes = [P, vp, vp, vp, vp, i, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.infv2_block_scores_approx.argtypes = [P, vp, vp, vp, i, i, i, vp, i, vp, vp]
        L.infv2_select_topk_pooled.argtypes = [P, vp, i, i, i, i, vp, vp]
        L.infv2_sparse_attn.argtypes = [P, vp, vp, vp, vp, i, vp, vp, vp]
        L.infv2_sparse_attn_rows.argtypes = [P, vp, vp, vp, vp, i, i, i, vp, vp, vp]
        L.infv2_dense_attn.argtypes = [P, vp, vp, vp, i, vp, vp, vp]
        L.infv2_prefill_workspace_size.argtypes = [P, vp, i, ctypes.POINTER(sz)]
        L.infv2_prefill.argtypes = [P, vp, vp, vp, vp, i, vp, sz, vp, vp, vp, vp]
        L.infv2_decode_workspace_size.argtypes = [P, i, i, ctypes.POINTER(sz)]
        L.infv2_decode.argtypes = [P, vp, vp, vp, vp, vp, vp, vp, i, i, vp, sz, vp, vp, vp, vp]
        L.infv2_decode_attn.argtypes = [P, vp, vp, vp, vp, i, i, vp, vp, sz, vp, vp, vp]
        L.infv2_select_blocks_noalloc.argtypes = [P, vp, vp, i, i, i, vp, vp]
        L.infv2_selftest_timeout.argtypes = [i, vp]
        L.infv2_selftest_exp2.argtypes = [i, vp, vp, i, vp]
        L.infv2_varlen_kernel_offsets.argtypes = [P, vp, i, vp]
        L.infv2_compress_k_varlen.argtypes = [P, vp, vp, i, vp, vp]
        L.infv2_block_scores_varlen.argtypes = [P, vp, vp, vp, i, vp, i, vp]
        L.infv2_select_topk_varlen.argtypes = [P, vp, i, vp, i, vp, vp]
        L.infv2_sparse_attn_varlen.argtypes = [P, vp, vp, vp, vp, vp, i, vp, vp, vp]
        L.infv2_dense_attn_varlen.argtypes = [P, vp, vp, vp, vp, i, vp, vp, vp]
        L.infv2_pipeline_workspace_size.argtypes = [P, vp, i, ctypes.POINTER(sz)]
        L.infv2_pipeline_create.argtypes = [P, vp, i, vp, sz, vp, ctypes.POINTER(vp)]
        L.infv2_pipeline_submit.argtypes = [vp, vp, vp, vp, vp, vp]
        L.infv2_pipeline_wait.argtypes = [vp, vp]
        L.infv2_pipeline_join.argtypes = [vp, vp]
        L.infv2_pipeline_sync.argtypes = [vp]
        L.infv2_pipeline_destroy.argtypes = [vp]
        _lib = L
    return _lib


def status_string(st: int) -> str:
    return lib().infv2_status_string(st).decode()


def _check(st: int, where: str):
    if st != OK:
        raise Infv2Error(st, where)


def params(h_q: int, h_kv: int, k: int = 64, n_init: int = 1, n_local: int = 2,
           scale: float | None = None, window: int = 0, lse_approx: int = 0) -> Params:
    p = Params()
    lib().infv2_default_params(ctypes.byref(p), h_q, h_kv)
    p.k, p.n_init, p.n_local, p.window, p.lse_approx = k, n_init, n_local, window, lse_approx
    if scale is not None:
        p.scale = scale
    return p


def params_of(shape) -> Params:
    """Library parameters from a synth.Shape."""
    p = params(shape.h_q, shape.h_kv, k=shape.k, n_init=shape.n_init, n_local=shape.n_local)
    p.B, p.l_c1, p.s_c1, p.pool_l, p.pool_s, p.d = (shape.B, shape.l_c1, shape.s_c1,
                                                   shape.pool_l, shape.pool_s, shape.d)
    p.scale = 1.0 / math.sqrt(shape.d)
    return p


def _ptr(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def num_kernels(p: Params, n: int) -> int:
    return lib().infv2_num_kernels(ctypes.byref(p), n)


def shared_ld(n: int) -> int:
    """Row pitch of S^shared: >= kernel count and 4 kernels per block, x32."""
    nc = (n - 32) // 16 + 1 if n >= 32 else 0
    nb = (n + 63) // 64
    return ((max(nc, 4 * nb) + 31) // 32) * 32


def infv2_check_params(p: Params) -> int:
    return lib().infv2_check_params(ctypes.byref(p))


def infv2_device_status(stream=None) -> int:
    return lib().infv2_device_status(_stream(stream))


def infv2_get_device_status(stream=None) -> int:
    """infv2_device_status under its second name."""
    return lib().infv2_get_device_status(_stream(stream))


def infv2_compress_k(p: Params, k: torch.Tensor, kc1: torch.Tensor | None = None, stream=None):
    n = k.shape[0]
    if kc1 is None:
        kc1 = torch.empty((max(num_kernels(p, n), 0), p.h_kv, p.d), dtype=torch.bfloat16,
                          device=k.device)
    _check(lib().infv2_compress_k(ctypes.byref(p), _ptr(k), n, _ptr(kc1) if kc1.numel() else None,
                                  _stream(stream)), "infv2_compress_k")
    return kc1


def num_coarse_kernels(p: Params, n: int) -> int:
    """Coarse kernels of the LSE approximation (length 4*l_c1, stride 4*s_c1)."""
    return (n - 4 * p.l_c1) // (4 * p.s_c1) + 1 if n >= 4 * p.l_c1 else 0


def infv2_compress_k2(p: Params, k: torch.Tensor, kc2: torch.Tensor | None = None, stream=None):
    n = k.shape[0]
    if kc2 is None:
        kc2 = torch.empty((num_coarse_kernels(p, n), p.h_kv, p.d), dtype=torch.bfloat16,
                          device=k.device)
    _check(lib().infv2_compress_k2(ctypes.byref(p), _ptr(k), n, _ptr(kc2) if kc2.numel() else None,
                                   _stream(stream)), "infv2_compress_k2")
    return kc2


def infv2_block_scores_approx(p: Params, q, kc1, kc2, n: int, q_begin: int, q_len: int,
                              s_shared=None, ld: int | None = None, score_lse=None, stream=None):
    ld = shared_ld(n) if ld is None else ld
    if s_shared is None:
        s_shared = torch.zeros((p.h_kv, q_len, ld), dtype=torch.float32, device=q.device)
    _check(lib().infv2_block_scores_approx(
        ctypes.byref(p), _ptr(q), _ptr(kc1) if kc1.numel() else None,
        _ptr(kc2) if kc2.numel() else None, n, q_begin, q_len, _ptr(s_shared), ld,
        _ptr(score_lse), _stream(stream)), "infv2_block_scores_approx")
    return s_shared


def infv2_block_scores(p: Params, q, kc1, n: int, q_begin: int, q_len: int, s_shared=None,
                       ld: int | None = None, score_lse=None, stream=None):
    ld = shared_ld(n) if ld is None else ld
    if s_shared is None:
        s_shared = torch.zeros((p.h_kv, q_len, ld), dtype=torch.float32, device=q.device)
    _check(lib().infv2_block_scores(ctypes.byref(p), _ptr(q), _ptr(kc1) if kc1.numel() else None,
                                    n, q_begin, q_len, _ptr(s_shared), ld, _ptr(score_lse),
                                    _stream(stream)), "infv2_block_scores")
    return s_shared


def infv2_select_topk(p: Params, s_shared, ld: int, n: int, q_begin: int, q_len: int, idx=None,
                      stream=None):
    if idx is None:
        idx = torch.full((p.h_kv, n, p.k), -2, dtype=torch.int32, device=s_shared.device)
    _check(lib().infv2_select_topk(ctypes.byref(p), _ptr(s_shared), ld, n, q_begin, q_len,
                                   _ptr(idx), _stream(stream)), "infv2_select_topk")
    return idx


def cmp_ld(n: int) -> int:
    """Row pitch (floats) of S^cmp for an n-token sequence: blocks rounded to 32."""
    return ((n + 63) // 64 + 31) // 32 * 32


def infv2_block_scores_pooled(p: Params, q, kc1, n: int, q_begin: int, q_len: int, s_cmp=None,
                              ld_cmp: int | None = None, stream=None):
    ld_cmp = cmp_ld(n) if ld_cmp is None else ld_cmp
    if s_cmp is None:
        s_cmp = torch.zeros((p.h_kv, q_len, ld_cmp), dtype=torch.float32, device=q.device)
    _check(lib().infv2_block_scores_pooled(ctypes.byref(p), _ptr(q),
                                           _ptr(kc1) if kc1.numel() else None, n, q_begin,
                                           q_len, _ptr(s_cmp), ld_cmp, _stream(stream)),
           "infv2_block_scores_pooled")
    return s_cmp


def infv2_select_topk_pooled(p: Params, s_cmp, ld_cmp: int, n: int, q_begin: int, q_len: int,
                             idx=None, stream=None):
    if idx is None:
        idx = torch.full((p.h_kv, n, p.k), -2, dtype=torch.int32, device=s_cmp.device)
    _check(lib().infv2_select_topk_pooled(ctypes.byref(p), _ptr(s_cmp), ld_cmp, n, q_begin, q_len,
                                          _ptr(idx), _stream(stream)),
           "infv2_select_topk_pooled")
    return idx


def infv2_sparse_attn(p: Params, q, k, v, idx, o=None, lse=None, stream=None):
    n = q.shape[0]
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_sparse_attn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), n,
                                   _ptr(o), _ptr(lse), _stream(stream)), "infv2_sparse_attn")
    return o


def infv2_sparse_attn_rows(p: Params, q, k, v, idx, r0: int, r1: int, o=None, lse=None,
                           stream=None):
    """Attention over query rows r0..r1-1 of the sequence (idx None: dense)."""
    n = q.shape[0]
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_sparse_attn_rows(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), n,
                                        r0, r1, _ptr(o), _ptr(lse), _stream(stream)),
           "infv2_sparse_attn_rows")
    return o


def infv2_sparse_attn_bwd_workspace_size(p: Params, n: int) -> int:
    out = ctypes.c_size_t()
    _check(lib().infv2_sparse_attn_bwd_workspace_size(ctypes.byref(p), n, ctypes.byref(out)),
           "infv2_sparse_attn_bwd_workspace_size")
    return out.value


def infv2_sparse_attn_bwd(p: Params, q, k, v, idx, o, lse, d_o, workspace=None, stream=None):
    """Gradients (dq, dk, dv) in fp32 of the attention over idx (None: dense)."""
    n = q.shape[0]
    dq = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    dk = torch.empty(k.shape, dtype=torch.float32, device=q.device)
    dv = torch.empty(v.shape, dtype=torch.float32, device=q.device)
    need = infv2_sparse_attn_bwd_workspace_size(p, n)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().infv2_sparse_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx), n,
                                       _ptr(o), _ptr(lse), _ptr(d_o), _ptr(dq), _ptr(dk), _ptr(dv),
                                       _ptr(workspace), workspace.numel(), _stream(stream)),
           "infv2_sparse_attn_bwd")
    return dq, dk, dv


def infv2_dense_attn(p: Params, q, k, v, o=None, lse=None, stream=None):
    n = q.shape[0]
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_dense_attn(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), n, _ptr(o),
                                  _ptr(lse), _stream(stream)), "infv2_dense_attn")
    return o


def infv2_prefill_workspace_size(p: Params, cu_seqlens) -> int:
    cu = (ctypes.c_int * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    out = ctypes.c_size_t(0)
    _check(lib().infv2_prefill_workspace_size(ctypes.byref(p), ctypes.cast(cu, ctypes.c_void_p),
                                              len(cu_seqlens) - 1, ctypes.byref(out)),
           "infv2_prefill_workspace_size")
    return out.value


def infv2_prefill(p: Params, q, k, v, cu_seqlens, workspace=None, idx_out=None, o=None, lse=None,
                  stream=None):
    """Whole layer over a packed varlen batch; cu_seqlens is a host sequence."""
    cu = (ctypes.c_int * len(cu_seqlens))(*[int(x) for x in cu_seqlens])
    need = infv2_prefill_workspace_size(p, cu_seqlens)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_prefill(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                               ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1,
                               _ptr(workspace), workspace.numel(), _ptr(idx_out), _ptr(o),
                               _ptr(lse), _stream(stream)), "infv2_prefill")
    return o


def _cu_array(cu_seqlens):
    return (ctypes.c_int * len(cu_seqlens))(*[int(x) for x in cu_seqlens])


def _host_ptr(t, nbytes: int, what: str):
    """Address of a contiguous host tensor of exactly nbytes (None passes)."""
    if t is None:
        return None
    if t.is_cuda or not t.is_contiguous():
        raise ValueError("%s: expected a contiguous host tensor" % what)
    if t.numel() * t.element_size() != nbytes:
        raise ValueError("%s: %d bytes, the pipeline's shape needs %d"
                         % (what, t.numel() * t.element_size(), nbytes))
    return ctypes.c_void_p(t.data_ptr())


class Pipeline:
    """Handle of an infv2_pipeline (the device workspace it keeps alive, and
    the varlen shape it was created for)."""

    def __init__(self, handle, workspace, p: Params, cu_seqlens, stream):
        self.handle, self.workspace, self.stream = handle, workspace, stream
        T = int(cu_seqlens[-1])
        self.q_bytes = T * p.h_q * p.d * 2
        self.kv_bytes = T * p.h_kv * p.d * 2
        self.lse_bytes = T * p.h_q * 4


def infv2_pipeline_workspace_size(p: Params, cu_seqlens) -> int:
    cu = _cu_array(cu_seqlens)
    out = ctypes.c_size_t(0)
    _check(lib().infv2_pipeline_workspace_size(ctypes.byref(p), ctypes.cast(cu, ctypes.c_void_p),
                                               len(cu_seqlens) - 1, ctypes.byref(out)),
           "infv2_pipeline_workspace_size")
    return out.value


def infv2_pipeline_create(p: Params, cu_seqlens, workspace=None, stream=None,
                          device=None) -> Pipeline:
    """Pipeline for prefill over host buffers; `stream` is the compute stream.

    The pipeline binds to the current CUDA device; `device` (where the
    workspace is allocated when none is given) must be that device."""
    need = infv2_pipeline_workspace_size(p, cu_seqlens)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device or "cuda")
    cu = _cu_array(cu_seqlens)
    h = ctypes.c_void_p()
    s = torch.cuda.current_stream() if stream is None else stream
    _check(lib().infv2_pipeline_create(ctypes.byref(p), ctypes.cast(cu, ctypes.c_void_p),
                                       len(cu_seqlens) - 1, _ptr(workspace), workspace.numel(),
                                       _stream(s), ctypes.byref(h)), "infv2_pipeline_create")
    return Pipeline(h, workspace, p, cu_seqlens, s)


def infv2_pipeline_submit(pl: Pipeline, q_host, k_host, v_host, o_host, lse_host=None):
    """Queue one batch: host bf16 q/k/v in, host bf16 o (and fp32 lse) out."""
    _check(lib().infv2_pipeline_submit(pl.handle, _host_ptr(q_host, pl.q_bytes, "q_host"),
                                       _host_ptr(k_host, pl.kv_bytes, "k_host"),
                                       _host_ptr(v_host, pl.kv_bytes, "v_host"),
                                       _host_ptr(o_host, pl.q_bytes, "o_host"),
                                       _host_ptr(lse_host, pl.lse_bytes, "lse_host")),
           "infv2_pipeline_submit")


def infv2_pipeline_wait(pl: Pipeline, stream=None):
    _check(lib().infv2_pipeline_wait(pl.handle, _stream(stream)), "infv2_pipeline_wait")


def infv2_pipeline_join(pl: Pipeline, stream=None):
    _check(lib().infv2_pipeline_join(pl.handle, _stream(stream)), "infv2_pipeline_join")


def infv2_pipeline_sync(pl: Pipeline):
    _check(lib().infv2_pipeline_sync(pl.handle), "infv2_pipeline_sync")


def infv2_pipeline_destroy(pl: Pipeline):
    if pl.handle is not None and pl.handle.value:
        h, pl.handle = pl.handle, None
        _check(lib().infv2_pipeline_destroy(h), "infv2_pipeline_destroy")


def infv2_decode_workspace_size(p: Params, batch: int, cap: int) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().infv2_decode_workspace_size(ctypes.byref(p), batch, cap, ctypes.byref(out)),
           "infv2_decode_workspace_size")
    return out.value


def infv2_decode(p: Params, q, k_new, v_new, k_cache, v_cache, kc1_cache, seqlens, workspace,
                 idx_out=None, o=None, lse=None, stream=None):
    batch, cap = k_cache.shape[0], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_decode(ctypes.byref(p), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                              _ptr(v_cache), _ptr(kc1_cache), _ptr(seqlens), batch, cap,
                              _ptr(workspace), workspace.numel(), _ptr(idx_out), _ptr(o),
                              _ptr(lse), _stream(stream)), "infv2_decode")
    return o


def infv2_decode_attn(p: Params, q, k_cache, v_cache, pos, idx, workspace, o=None, lse=None,
                      stream=None):
    """Decode attention alone over given block lists idx [batch, h_kv, k] at
    query positions pos (int32 [batch], device); caches and pos are not written."""
    batch, cap = k_cache.shape[0], k_cache.shape[2]
    if o is None:
        o = torch.empty_like(q)
    _check(lib().infv2_decode_attn(ctypes.byref(p), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                                   _ptr(pos), batch, cap, _ptr(idx), _ptr(workspace),
                                   workspace.numel(), _ptr(o), _ptr(lse), _stream(stream)),
           "infv2_decode_attn")
    return o


def infv2_select_blocks_noalloc(p: Params, q, kc1, n: int, q_begin: int, q_len: int, idx,
                                stream=None):
    """Block selection with the library's fixed device scratch (no allocation)."""
    _check(lib().infv2_select_blocks_noalloc(ctypes.byref(p), _ptr(q),
                                             _ptr(kc1) if kc1.numel() else None, n, q_begin,
                                             q_len, _ptr(idx), _stream(stream)),
           "infv2_select_blocks_noalloc")
    return idx


def infv2_selftest_exp2(which: int, x, stream=None):
    """2^x through one of the kernels' exponential forms (0: MUFU, 1: the
    score kernel's degree-5 polynomial, 2: the attention's cubic)."""
    y = torch.empty_like(x)
    _check(lib().infv2_selftest_exp2(which, _ptr(x), _ptr(y), x.numel(), _stream(stream)),
           "infv2_selftest_exp2")
    return y


def infv2_selftest_timeout(limit_us: int, stream=None):
    _check(lib().infv2_selftest_timeout(limit_us, _stream(stream)), "infv2_selftest_timeout")


# ------------------------------------------------------------ varlen stage forms
# cu_seqlens: a host sequence of batch + 1 offsets (packed "thd" tensors).

def infv2_varlen_kernel_offsets(p: Params, cu_seqlens):
    cu = _cu_array(cu_seqlens)
    out = (ctypes.c_int * len(cu_seqlens))()
    _check(lib().infv2_varlen_kernel_offsets(ctypes.byref(p), ctypes.cast(cu, ctypes.c_void_p),
                                             len(cu_seqlens) - 1, ctypes.cast(out, ctypes.c_void_p)),
           "infv2_varlen_kernel_offsets")
    return list(out)


def infv2_compress_k_varlen(p: Params, k, cu_seqlens, kc1=None, stream=None):
    """K^C1 of every sequence, packed: sequence s's kernels from row cu_kernels[s]."""
    ck = infv2_varlen_kernel_offsets(p, cu_seqlens)
    if kc1 is None:
        kc1 = torch.empty((max(ck[-1], 1), p.h_kv, 128), dtype=torch.bfloat16, device=k.device)
    cu = _cu_array(cu_seqlens)
    _check(lib().infv2_compress_k_varlen(ctypes.byref(p), _ptr(k), ctypes.cast(cu, ctypes.c_void_p),
                                         len(cu_seqlens) - 1, _ptr(kc1), _stream(stream)),
           "infv2_compress_k_varlen")
    return kc1


def infv2_block_scores_varlen(p: Params, q, kc1, cu_seqlens, s_shared=None, ld=None, stream=None):
    """S^shared of every row; sequence s's [h_kv, n_s, ld] block at float
    offset h_kv*ld*cu_seqlens[s] of a flat buffer.  Returns (s_shared, ld)."""
    n_max = max((b - a for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:])), default=0)
    if ld is None:
        ld = shared_ld(n_max)
    T = int(cu_seqlens[-1])
    if s_shared is None:
        s_shared = torch.zeros(max(p.h_kv * T * ld, 4), dtype=torch.float32, device=q.device)
    cu = _cu_array(cu_seqlens)
    _check(lib().infv2_block_scores_varlen(ctypes.byref(p), _ptr(q), _ptr(kc1),
                                           ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1,
                                           _ptr(s_shared), ld, _stream(stream)),
           "infv2_block_scores_varlen")
    return s_shared, ld


def infv2_select_topk_varlen(p: Params, s_shared, ld: int, cu_seqlens, idx=None, stream=None):
    T = int(cu_seqlens[-1])
    if idx is None:
        idx = torch.empty((p.h_kv, T, p.k), dtype=torch.int32, device=s_shared.device)
    cu = _cu_array(cu_seqlens)
    _check(lib().infv2_select_topk_varlen(ctypes.byref(p), _ptr(s_shared), ld,
                                          ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1,
                                          _ptr(idx), _stream(stream)), "infv2_select_topk_varlen")
    return idx


def infv2_sparse_attn_varlen(p: Params, q, k, v, idx, cu_seqlens, o=None, lse=None, stream=None):
    if o is None:
        o = torch.empty_like(q)
    cu = _cu_array(cu_seqlens)
    _check(lib().infv2_sparse_attn_varlen(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(idx),
                                          ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1,
                                          _ptr(o), _ptr(lse), _stream(stream)),
           "infv2_sparse_attn_varlen")
    return o


def infv2_dense_attn_varlen(p: Params, q, k, v, cu_seqlens, o=None, lse=None, stream=None):
    if o is None:
        o = torch.empty_like(q)
    cu = _cu_array(cu_seqlens)
    _check(lib().infv2_dense_attn_varlen(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                         ctypes.cast(cu, ctypes.c_void_p), len(cu_seqlens) - 1,
                                         _ptr(o), _ptr(lse), _stream(stream)),
           "infv2_dense_attn_varlen")
    return o
