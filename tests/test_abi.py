"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function declared in include/infv2.h, and its host-only logic
(parameter validation, sizes, argument errors) behaves as documented."""
import ctypes
import os
import re

import numpy as np
import pytest

from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "infv2.h")


@pytest.fixture(scope="module", autouse=True)
def _built():
    build_mod.build()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(infv2_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_binding_symbols():
    assert set(declared_functions()) == set(infv2.SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(infv2.LIB_PATH)
    missing = [s for s in declared_functions() if not hasattr(lib, s)]
    assert not missing, missing


def test_checks_build_exports_the_same_symbols():
    # the INFV2_CHECKS debug variant is the same ABI with device-side checks
    path = build_mod.build(checks=True)
    lib = ctypes.CDLL(path)
    missing = [s for s in declared_functions() if not hasattr(lib, s)]
    assert not missing, missing
    lib.infv2_status_string.restype = ctypes.c_char_p
    assert b"INFV2_CHECKS" in lib.infv2_status_string(infv2.ERR_CHECK)


def test_default_params_and_checks():
    p = infv2.params(32, 2)
    assert (p.B, p.l_c1, p.s_c1, p.pool_l, p.pool_s, p.d, p.k) == (64, 32, 16, 5, 4, 128, 64)
    assert abs(p.scale - 128 ** -0.5) < 1e-7
    assert infv2.infv2_check_params(p) == infv2.OK
    bad = infv2.params(32, 2)
    bad.h_q = 30  # not a multiple of h_kv... 30 % 2 == 0 but G = 15 unsupported
    assert infv2.infv2_check_params(bad) == infv2.ERR_UNSUPPORTED
    bad = infv2.params(32, 3)
    assert infv2.infv2_check_params(bad) == infv2.ERR_INVALID_ARG
    bad = infv2.params(32, 2, k=2, n_init=1, n_local=2)   # k < n_init + n_local
    assert infv2.infv2_check_params(bad) == infv2.ERR_INVALID_ARG
    bad = infv2.params(32, 2, window=200, n_local=2)      # needs n_local >= ceil(200/64)+1 = 5
    assert infv2.infv2_check_params(bad) == infv2.ERR_INVALID_ARG
    ok = infv2.params(32, 2, window=200, n_local=5)
    assert infv2.infv2_check_params(ok) == infv2.OK
    bad = infv2.params(32, 2)
    bad.d = 64
    assert infv2.infv2_check_params(bad) == infv2.ERR_UNSUPPORTED
    bad = infv2.params(32, 2)
    bad.n_local = 0
    assert infv2.infv2_check_params(bad) == infv2.ERR_INVALID_ARG
    assert infv2.infv2_check_params(infv2.params(64, 2)) == infv2.ERR_UNSUPPORTED  # G = 32


def test_num_kernels_matches_definition():
    p = infv2.params(4, 1)
    for n in range(0, 300):
        want = (n - 32) // 16 + 1 if n >= 32 else 0
        assert infv2.num_kernels(p, n) == want


def test_status_strings():
    for st in range(6):
        assert infv2.status_string(st)
    assert infv2.status_string(99) == "unknown status"


def test_workspace_sizes_are_host_only():
    p = infv2.params(32, 2)
    # all-dense batch needs no workspace
    assert infv2.infv2_prefill_workspace_size(p, [0, 1024, 3072]) == 0
    n = 131072
    ws = infv2.infv2_prefill_workspace_size(p, [0, n])
    nc = (n - 32) // 16 + 1
    assert ws >= nc * 2 * 128 * 2 + 2 * n * 64 * 4
    assert infv2.infv2_decode_workspace_size(p, 32, 131136) > 0
    with pytest.raises(infv2.Infv2Error):
        infv2.infv2_prefill_workspace_size(p, [5, 100])   # cu_seqlens[0] must be 0
    with pytest.raises(infv2.Infv2Error):
        infv2.infv2_prefill_workspace_size(p, [0, 100, 50])  # negative length


def test_argument_errors_before_any_launch():
    L = infv2.lib()
    p = infv2.params(32, 2)
    P = ctypes.byref(p)
    assert L.infv2_compress_k(P, None, 100, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_compress_k(P, None, -1, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_compress_k(P, None, 0, None, None) == infv2.OK       # nothing to do
    assert L.infv2_block_scores(P, None, None, 100, 50, 60, None, 128, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_select_topk(P, None, 128, 100, 0, 0, None, None) == infv2.OK
    assert L.infv2_select_topk(P, None, 6, 100, 0, 10, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_block_scores_pooled(P, None, None, 100, 50, 60, None, 4, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_block_scores_pooled(P, None, None, 100, 0, 0, None, 4, None) == infv2.OK
    # ld_cmp below ceil(n/B) or not a multiple of 4 is rejected before any pointer is used
    assert L.infv2_block_scores_pooled(P, 16, 16, 1000, 0, 10, 16, 12, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_block_scores_pooled(P, 16, 16, 1000, 0, 10, 16, 18, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_select_topk_pooled(P, None, 4, 100, 0, 0, None, None) == infv2.OK
    assert L.infv2_select_topk_pooled(P, 16, 2, 100, 0, 10, 16, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_select_topk_pooled(P, 8, 4, 100, 0, 10, 16, None) == infv2.ERR_INVALID_ARG  # misaligned
    assert L.infv2_sparse_attn(P, None, None, None, None, 10, None, None, None) == infv2.ERR_INVALID_ARG
    # row ranges: bounds checked first; an empty range does nothing
    assert L.infv2_sparse_attn_rows(P, None, None, None, None, 100, 5, 5, None, None, None) == infv2.OK
    assert L.infv2_sparse_attn_rows(P, None, None, None, None, 100, 0, 10, None, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_sparse_attn_rows(P, 16, 16, 16, None, 100, -1, 10, 16, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_sparse_attn_rows(P, 16, 16, 16, None, 100, 20, 10, 16, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_sparse_attn_rows(P, 16, 16, 16, None, 100, 0, 101, 16, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_dense_attn(P, None, None, None, 0, None, None, None) == infv2.OK
    assert L.infv2_decode(P, None, None, None, None, None, None, None, 0, 16, None, 0, None, None,
                          None, None) == infv2.OK
    assert L.infv2_selftest_timeout(0, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_selftest_exp2(3, None, None, 4, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_selftest_exp2(1, None, None, 0, None) == infv2.OK
    assert L.infv2_selftest_exp2(1, None, None, 4, None) == infv2.ERR_INVALID_ARG
    # decode attention alone: an empty batch does nothing; bad shapes, missing
    # pointers and a small or misaligned workspace are refused before any launch
    assert L.infv2_decode_attn(P, None, None, None, None, 0, 16, None, None, 0, None, None, None) == infv2.OK
    assert L.infv2_decode_attn(P, None, None, None, None, -1, 16, None, None, 0, None, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_decode_attn(P, 16, 16, 16, 16, 2, 0, 16, 256, 1 << 20, 16, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_decode_attn(P, 16, 16, 16, None, 2, 256, 16, 256, 1 << 20, 16, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_decode_attn(P, 16, 16, 16, 16, 2, 256, 16, 256, 64, 16, None, None) == infv2.ERR_WORKSPACE
    assert L.infv2_decode_attn(P, 16, 16, 16, 16, 2, 256, 16, 16, 1 << 30, 16, None, None) == infv2.ERR_INVALID_ARG
    # the LSE approximation flag: 0 or 1; decode does not take it
    assert p.lse_approx == 0
    pa = infv2.params(32, 2, lse_approx=1)
    assert L.infv2_check_params(ctypes.byref(pa)) == infv2.OK
    pa.lse_approx = 2
    assert L.infv2_check_params(ctypes.byref(pa)) == infv2.ERR_INVALID_ARG
    pa.lse_approx = 1
    sz = ctypes.c_size_t()
    assert L.infv2_decode_workspace_size(ctypes.byref(pa), 4, 4096, ctypes.byref(sz)) == infv2.ERR_UNSUPPORTED
    assert L.infv2_compress_k2(P, None, 0, None, None) == infv2.OK
    assert L.infv2_compress_k2(P, None, 200, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_block_scores_approx(P, None, None, None, 100, 50, 60, None, 128, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_prefill_workspace_size(ctypes.byref(pa), (ctypes.c_int * 2)(0, 10000), 1, ctypes.byref(sz)) == infv2.OK
    assert L.infv2_check_params(None) == infv2.ERR_INVALID_ARG


def _r256(x):
    return (x + 255) // 256 * 256


def test_pipeline_workspace_and_argument_errors():
    L = infv2.lib()
    p = infv2.params(32, 2)
    P = ctypes.byref(p)
    for cu in ([0, 131072], [0, 300, 5000, 5001]):
        T = cu[-1]
        q, kv, lse = T * 32 * 128 * 2, T * 2 * 128 * 2, T * 32 * 4
        slot = 2 * _r256(q) + 2 * _r256(kv) + _r256(lse)
        want = _r256(infv2.infv2_prefill_workspace_size(p, cu)) + 2 * slot
        assert infv2.infv2_pipeline_workspace_size(p, cu) == want
    sz = ctypes.c_size_t()
    cu = (ctypes.c_int * 3)(0, 100, 300)
    assert L.infv2_pipeline_workspace_size(P, cu, 0, ctypes.byref(sz)) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_workspace_size(P, (ctypes.c_int * 2)(0, 0), 1, ctypes.byref(sz)) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_workspace_size(P, (ctypes.c_int * 2)(4, 9), 1, ctypes.byref(sz)) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_workspace_size(P, cu, 2, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_workspace_size(P, cu, 2, ctypes.byref(sz)) == infv2.OK
    h = ctypes.c_void_p()
    # every argument error is caught before the workspace is touched or CUDA is called
    assert L.infv2_pipeline_create(P, cu, 2, 4096, sz.value, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_create(P, cu, 2, None, sz.value, None, ctypes.byref(h)) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_create(P, cu, 2, 4096 + 16, sz.value, None, ctypes.byref(h)) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_create(P, cu, 2, 4096, sz.value - 1, None, ctypes.byref(h)) == infv2.ERR_WORKSPACE
    assert not h.value
    assert L.infv2_pipeline_submit(None, 16, 16, 16, 16, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_wait(None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_join(None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_sync(None) == infv2.ERR_INVALID_ARG
    assert L.infv2_pipeline_destroy(None) == infv2.OK


def test_pipeline_binding_checks_host_buffer_sizes():
    import torch
    p = infv2.params(4, 1)
    pl = infv2.Pipeline(ctypes.c_void_p(), None, p, [0, 100], None)   # no handle: nothing is called
    q = torch.zeros((100, 4, 128), dtype=torch.bfloat16)
    kv = torch.zeros((100, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        infv2.infv2_pipeline_submit(pl, q[:99], kv, kv, q)
    with pytest.raises(ValueError):
        infv2.infv2_pipeline_submit(pl, q, kv, kv, q, torch.zeros((4, 99)))
    with pytest.raises(ValueError):
        infv2.infv2_pipeline_submit(pl, q, torch.zeros((100, 2, 128), dtype=torch.bfloat16)[:, :1], kv, q)
    infv2.infv2_pipeline_destroy(pl)   # a handle that was never created: no-op


def test_binding_refuses_host_tensors():
    # device-pointer entry points take CUDA tensors only: a CPU tensor never
    # reaches the library, so there is no silent host path
    import torch
    p = infv2.params(4, 1)
    q = torch.zeros((64, 4, 128), dtype=torch.bfloat16)
    kv = torch.zeros((64, 1, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        infv2.infv2_dense_attn(p, q, kv, kv, o=q)


def test_varlen_kernel_offsets_and_argument_errors():
    p = infv2.params(16, 2, k=8)
    cu = [0, 10, 100, 100, 5000]
    ck = infv2.infv2_varlen_kernel_offsets(p, cu)
    nc = [infv2.num_kernels(p, b - a) for a, b in zip(cu[:-1], cu[1:])]
    assert ck == [0] + list(np.cumsum(nc))
    assert nc[0] == 0 and nc[2] == 0
    L = infv2.lib()
    pp = ctypes.byref(p)
    arr = lambda xs: (ctypes.c_int * len(xs))(*xs)
    bad = [arr([5, 10]), arr([0, 10, 4])]          # must start at 0; must not decrease
    for c in bad:
        assert L.infv2_varlen_kernel_offsets(pp, c, 2 if len(c) == 3 else 1, arr([0, 0, 0])) == infv2.ERR_INVALID_ARG
        nb = len(c) - 1
        assert L.infv2_compress_k_varlen(pp, None, c, nb, None, None) == infv2.ERR_INVALID_ARG
        assert L.infv2_block_scores_varlen(pp, None, None, c, nb, None, 32, None) == infv2.ERR_INVALID_ARG
        assert L.infv2_select_topk_varlen(pp, None, 32, c, nb, None, None) == infv2.ERR_INVALID_ARG
        assert L.infv2_sparse_attn_varlen(pp, None, None, None, None, c, nb, None, None, None) == infv2.ERR_INVALID_ARG
        assert L.infv2_dense_attn_varlen(pp, None, None, None, c, nb, None, None, None) == infv2.ERR_INVALID_ARG
    good = arr([0, 100, 3000])
    # missing tensors, and an S^shared pitch below the longest sequence's kernel count
    assert L.infv2_compress_k_varlen(pp, None, good, 2, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_block_scores_varlen(pp, None, None, good, 2, None, 64, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_select_topk_varlen(pp, None, 32, good, 2, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_sparse_attn_varlen(pp, None, None, None, None, good, 2, None, None, None) == infv2.ERR_INVALID_ARG
    assert L.infv2_dense_attn_varlen(pp, None, None, None, good, 2, None, None, None) == infv2.ERR_INVALID_ARG
    # an empty batch (or only empty sequences) does nothing and succeeds
    assert L.infv2_sparse_attn_varlen(pp, None, None, None, None, arr([0, 0]), 1, None, None, None) == infv2.OK
    assert L.infv2_compress_k_varlen(pp, None, arr([0]), 0, None, None) == infv2.OK


def test_device_status_second_name():
    # both names are the same call (no GPU here: both report the failed read)
    L = infv2.lib()
    a, b = L.infv2_device_status(None), L.infv2_get_device_status(None)
    assert a == b
