"""The allocation-free selection entry point against the workspace path.

infv2_select_blocks_noalloc exists for callers that cannot allocate device
memory (an arena or pool they do not own, a frozen allocator, a plugin that
only sees input and output pointers); it keeps its S^shared scratch in a
fixed array inside the library.  Its block lists must equal those of
infv2_block_scores + infv2_select_topk run on caller scratch (the same
kernels on the same fp32 values, so the tolerance is exact equality), on two
calls in a row.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

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


def _reference(p, q, kc1, n):
    ld = infv2.shared_ld(n)
    s = infv2.infv2_block_scores(p, q, kc1, n, 0, n, ld=ld)
    return infv2.infv2_select_topk(p, s, ld, n, 0, n)


def _noalloc(p, q, kc1, n, q_begin, q_len, idx):
    """Call the C entry point directly through the C ABI."""
    st = infv2.lib().infv2_select_blocks_noalloc(
        ctypes.byref(p), ctypes.c_void_p(q.data_ptr()),
        ctypes.c_void_p(kc1.data_ptr()) if kc1.numel() else None, n, q_begin, q_len,
        ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("n,h_q,h_kv,k", [(20000, 32, 2, 64), (2048, 4, 1, 8)])
def test_noalloc_matches_workspace_path_twice(n, h_q, h_kv, k):
    sh = synth.Shape(n=n, h_q=h_q, h_kv=h_kv, k=k, n_needles=4)
    d = synth.make_prefill(sh, seed=21)
    p = infv2.params_of(sh)
    q, kk = to_dev(d["q"]), to_dev(d["k"])
    kc1 = infv2.infv2_compress_k(p, kk)
    ref = _reference(p, q, kc1, n)
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row share (and reuse) the fixed scratch
        idx = torch.full((h_kv, n, k), -7, dtype=torch.int32, device="cuda")
        assert _noalloc(p, q, kc1, n, 0, n, idx) == infv2.OK
        torch.cuda.synchronize()
        assert infv2.infv2_device_status() == 0
        assert torch.equal(idx, ref)


def test_noalloc_row_range_and_limits():
    sh = synth.Shape(n=9000, h_q=16, h_kv=2, k=16)
    d = synth.make_prefill(sh, seed=5)
    p = infv2.params_of(sh)
    q, kk = to_dev(d["q"]), to_dev(d["k"])
    kc1 = infv2.infv2_compress_k(p, kk)
    ref = _reference(p, q, kc1, sh.n)
    idx = torch.full((2, sh.n, 16), -7, dtype=torch.int32, device="cuda")
    assert _noalloc(p, q, kc1, sh.n, 3000, 5000, idx) == infv2.OK
    torch.cuda.synchronize()
    assert torch.equal(idx[:, 3000:8000], ref[:, 3000:8000])
    assert bool((idx[:, :3000] == -7).all()) and bool((idx[:, 8000:] == -7).all())
    # beyond the fixed scratch (one 128-token tile of S^shared must fit in 16
    # MiB): refused before any launch; the buffers have the sizes the call
    # names, so even a launch could not read or write past them
    big = 300000
    pb = infv2.params_of(synth.Shape(n=big, h_q=2, h_kv=2, k=16))
    q_big = torch.zeros((big, 2, 128), dtype=torch.bfloat16, device="cuda")
    kc1_big = torch.zeros((infv2.num_kernels(pb, big), 2, 128), dtype=torch.bfloat16, device="cuda")
    idx_big = torch.full((2, big, 16), -7, dtype=torch.int32, device="cuda")
    assert _noalloc(pb, q_big, kc1_big, big, 0, 1, idx_big) == infv2.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert bool((idx_big == -7).all())
