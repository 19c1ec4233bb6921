"""Child process of test_gpu_checks.py.

Runs a set of small cases on the library that the INFV2_BUILD environment
variable selects (the default build, or "checks" for the INFV2_CHECKS debug
build) and saves every output and every device status word to an .npz file:

    python tests/checks_child.py OUT.npz

Keys "v_*" are outputs of valid input, which must not depend on the build;
"st_*" are device statuses read after each case; "f_*", "m_*" and "e_*" are
the block-list edge cases (entries past a query's own block, the same lists
with those entries as -1, and a row left with no block).
"""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from trainable_block_sparse_mean_b200 import infv2, synth  # noqa: E402
from trainable_block_sparse_mean_b200.workloads import DecodeState, to_dev, to_host_bits  # noqa: E402


def _status():
    torch.cuda.synchronize()
    return np.int32(infv2.infv2_device_status())


def _attn(p, q, k, v, idx, n, h_q):
    lse = torch.empty((h_q, n), device="cuda")
    o = infv2.infv2_sparse_attn(p, q, k, v, idx, lse=lse)
    torch.cuda.synchronize()
    return to_host_bits(o), lse.cpu().numpy()


def prefill_cases(res, name, sh, seed):
    d = synth.make_prefill(sh, seed=seed)
    p = infv2.params_of(sh)
    q, k, v = to_dev(d["q"]), to_dev(d["k"]), to_dev(d["v"])
    n = sh.n
    idx = torch.full((sh.h_kv, n, sh.k), -3, dtype=torch.int32, device="cuda")
    lse = torch.empty((sh.h_q, n), device="cuda")
    o = infv2.infv2_prefill(p, q, k, v, [0, n], idx_out=idx, lse=lse)
    res["st_%s_prefill" % name] = _status()
    res["v_%s_o" % name] = to_host_bits(o)
    res["v_%s_lse" % name] = lse.cpu().numpy()
    res["v_%s_idx" % name] = idx.cpu().numpy()

    # entries past a query's own block: ascending, at the end of the list
    full_rows = [n - 1, n - 200, 1500]
    pad_row = 100  # 2 candidate blocks <= k: the list is padded with -1
    idx_f, idx_m = idx.clone(), idx.clone()
    for g in range(sh.h_kv):
        for r in full_rows:
            own = r // 64
            idx_f[g, r, sh.k - 3:] = torch.tensor([own + 1, own + 2, 10 ** 6], dtype=torch.int32)
            idx_m[g, r, sh.k - 3:] = -1
        own = pad_row // 64
        idx_f[g, pad_row, 2:5] = torch.tensor([own + 1, own + 5, 99999], dtype=torch.int32)
    res["f_%s_o" % name], res["f_%s_lse" % name] = _attn(p, q, k, v, idx_f, n, sh.h_q)
    res["st_%s_future" % name] = _status()
    res["m_%s_o" % name], res["m_%s_lse" % name] = _attn(p, q, k, v, idx_m, n, sh.h_q)
    res["st_%s_masked" % name] = _status()

    # a row whose every entry lies past its own block: nothing to attend to
    r_e = 2000
    idx_e = idx.clone()
    idx_e[:, r_e] = torch.arange(r_e // 64 + 1, r_e // 64 + 1 + sh.k, dtype=torch.int32)
    o_e, lse_e = _attn(p, q, k, v, idx_e, n, sh.h_q)
    res["st_%s_empty" % name] = _status()
    res["e_%s_o" % name] = o_e[r_e]
    res["e_%s_lse" % name] = lse_e[:, r_e]

    # invalid lists: a repeated block, and two entries out of order
    idx_d = idx.clone()
    idx_d[0, n - 1, 5] = idx_d[0, n - 1, 4]
    _attn(p, q, k, v, idx_d, n, sh.h_q)
    res["st_%s_repeat" % name] = _status()
    idx_s = idx.clone()
    idx_s[0, n - 7, 3], idx_s[0, n - 7, 4] = idx[0, n - 7, 4], idx[0, n - 7, 3]
    _attn(p, q, k, v, idx_s, n, sh.h_q)
    res["st_%s_order" % name] = _status()

    # backward on the valid lists (dq is written per row, so it is deterministic),
    # then on the list with a repeated block
    d_o = to_dev(synth.bf16_bits(np.random.default_rng(seed + 1)
                                 .standard_normal((n, sh.h_q, sh.d)).astype(np.float32)))
    dq, _, _ = infv2.infv2_sparse_attn_bwd(p, q, k, v, idx, o, lse, d_o)
    res["st_%s_bwd" % name] = _status()
    res["v_%s_dq" % name] = dq.cpu().numpy()
    infv2.infv2_sparse_attn_bwd(p, q, k, v, idx_d, o, lse, d_o)
    res["st_%s_bwd_repeat" % name] = _status()


def decode_case(res):
    sh = synth.Shape(n=0, h_q=16, h_kv=1, k=16)
    lens = np.array([1500, 4000], np.int32)
    steps, cap = 2, 4096
    dd = dict(k_cache=np.zeros((2, 1, cap, 128), np.uint16), v_cache=np.zeros((2, 1, cap, 128), np.uint16),
              k_new=np.zeros((steps, 2, 1, 128), np.uint16), v_new=np.zeros((steps, 2, 1, 128), np.uint16),
              q=np.zeros((steps, 2, 16, 128), np.uint16), lens=lens, cap=cap)
    for s, L in enumerate(lens):
        sq = synth.make_decode_sequence(sh, int(L), steps, 21, s)
        dd["k_cache"][s, 0, :L] = sq["k"][:L, 0]
        dd["v_cache"][s, 0, :L] = sq["v"][:L, 0]
        dd["k_new"][:, s] = sq["k"][L:L + steps]
        dd["v_new"][:, s] = sq["v"][L:L + steps]
        dd["q"][:, s] = sq["q_new"]
    st = DecodeState(sh, dd)
    for t in range(steps):
        idx = torch.full((2, 1, sh.k), -3, dtype=torch.int32, device="cuda")
        o = st.step(t, idx_out=idx)
        res["st_decode_%d" % t] = _status()
        res["v_decode_o_%d" % t] = to_host_bits(o)
        res["v_decode_idx_%d" % t] = idx.cpu().numpy()


def main(out):
    torch.cuda.set_device(0)
    infv2.lib()
    res = {"lib": np.array(os.path.basename(infv2.LIB_PATH))}
    # G = 16 runs the tensor-core attention, G = 2 the per-token kernel
    prefill_cases(res, "g16", synth.Shape(n=3000, h_q=16, h_kv=1, k=16), seed=11)
    prefill_cases(res, "g2", synth.Shape(n=2500, h_q=4, h_kv=2, k=8), seed=12)
    decode_case(res)
    np.savez(out, **res)


if __name__ == "__main__":
    main(sys.argv[1])
