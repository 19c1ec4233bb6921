"""Comparison rules of the CUDA path against the fp64 oracle.

* Selected blocks: per (query, kv head) the sets must be equal, except swaps
  of a GPU-chosen block a (not in the oracle's set) with a missing block b
  whose oracle block scores differ by at most 1e-5 relative.
* Attention outputs: on the same block sets, bf16 O within max-abs 2e-2 and
  mean-abs 2e-3 of the fp64 O.
"""
from __future__ import annotations

import numpy as np

SWAP_REL = 1e-5
O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3


def compare_indices(gpu_idx: np.ndarray, orc_idx: np.ndarray, orc_cmp: np.ndarray | None,
                    rel: float = SWAP_REL):
    """gpu_idx/orc_idx [rows, h_kv, k]; orc_cmp [rows, h_kv, n_blk] (oracle S^cmp).

    Returns (n_equal, n_swapped, bad) where bad lists (row, g, extra, missing)."""
    n_eq = n_sw = 0
    bad = []
    R, H, _ = orc_idx.shape
    for r in range(R):
        for g in range(H):
            a = [int(x) for x in gpu_idx[r, g] if x >= 0]
            b = [int(x) for x in orc_idx[r, g] if x >= 0]
            if a == b:
                n_eq += 1
                continue
            sa, sb = set(a), set(b)
            extra, missing = sorted(sa - sb), sorted(sb - sa)
            ok = (len(a) == len(b) and len(extra) == len(missing) and len(set(a)) == len(a)
                  and a == sorted(a) and orc_cmp is not None)
            if ok:
                ce = sorted(orc_cmp[r, g, extra])
                cm = sorted(orc_cmp[r, g, missing])
                for x, y in zip(ce, cm):
                    if not (np.isfinite(x) and np.isfinite(y)
                            and abs(x - y) <= rel * max(abs(x), abs(y))):
                        ok = False
                        break
            if ok:
                n_sw += 1
            else:
                bad.append((r, g, extra, missing))
    return n_eq, n_sw, bad


def compare_outputs(o_gpu: np.ndarray, o_orc: np.ndarray):
    """(max_abs, mean_abs) of bf16/float GPU output against fp64 oracle output."""
    d = np.abs(o_gpu.astype(np.float64) - o_orc)
    return float(d.max()) if d.size else 0.0, float(d.mean()) if d.size else 0.0


def assert_outputs_close(o_gpu, o_orc, what=""):
    mx, mean = compare_outputs(o_gpu, o_orc)
    assert mx <= O_MAX_ABS and mean <= O_MEAN_ABS, f"{what}: max-abs {mx:.3e} mean-abs {mean:.3e}"
    return mx, mean


def assert_grads_close(got, want, name, rel_fro=5e-3, rel_max=1e-2):
    """fp32 gradients against the fp64 oracle: relative Frobenius error of the
    whole tensor and the largest element error relative to the largest
    reference magnitude.  The GPU rounds P and dS to bf16 for its MMAs
    (relative 2^-9 per element, averaging out over the sums)."""
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    assert np.all(np.isfinite(got)), name
    if np.abs(want).max() < 1e-9:
        # an exactly-zero gradient (e.g. a query that sees one token): fp32
        # rounding of dO.v - D leaves residues far below the data's scale
        assert np.abs(got).max() < 1e-4, (name, np.abs(got).max())
        return
    scale = np.abs(want).max()
    fro = np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30)
    mx = np.abs(got - want).max() / scale
    assert fro <= rel_fro and mx <= rel_max, (name, fro, mx)
