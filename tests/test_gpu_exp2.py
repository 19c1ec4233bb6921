"""The kernels' exponential forms against fp64 2^x, each held to the bound its
comment states: the MUFU instruction, the score kernel's degree-5 FMA-pipe
polynomial and the attention's FMA-pipe cubic (whose clamped bottom must be an
exact zero, so that masked keys add nothing)."""
import numpy as np
import pytest
import torch

from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    infv2.lib()


def _eval(which, x):
    y = infv2.infv2_selftest_exp2(which, torch.from_numpy(x.astype(np.float32)).cuda())
    torch.cuda.synchronize()
    return y.cpu().numpy().astype(np.float64)


def _grid(lo, hi):
    # a dense grid, every integer and half-integer (the split's edges), and
    # the neighbours of each half-integer
    g = np.linspace(lo, hi, 2_000_001, dtype=np.float32)
    half = np.arange(2 * lo, 2 * hi + 1, dtype=np.float32) / 2
    edges = np.concatenate([half, np.nextafter(half, np.float32(-np.inf)),
                            np.nextafter(half, np.float32(np.inf))])
    x = np.concatenate([g, edges])
    return x[(x >= lo) & (x <= hi)]


@pytest.mark.parametrize("which,lo,hi,bound", [(0, -126.0, 127.0, 1e-6),
                                               (1, -126.0, 127.0, 2.5e-7),
                                               (2, -126.0, 64.0, 1.1e-4)])
def test_relative_error_within_stated_bound(which, lo, hi, bound):
    x = _grid(lo, hi)
    y = _eval(which, x)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y / want - 1.0)
    assert np.all(np.isfinite(y))
    assert rel.max() <= bound, (which, float(rel.max()), float(x[np.argmax(rel)]))


def test_bottom_and_special_values():
    x = np.array([-np.inf, -1000.0, -200.0, -127.0, -127.0 + 1e-5], np.float32)
    for which in (0, 1, 2):
        y = _eval(which, x)
        assert np.all(np.isfinite(y)) and np.all(y >= 0.0), (which, y)
        assert np.all(y < 1e-37), (which, y)          # nothing a sum would notice
    y = _eval(2, np.array([-np.inf, -1000.0, -127.0], np.float32))
    assert np.array_equal(y, np.zeros(3)), y          # the cubic's bottom is exactly zero
    y = _eval(2, np.array([64.0, 80.0, np.inf], np.float32))
    assert np.array_equal(y, np.full(3, 2.0 ** 64)), y  # clamped at 2^64
    assert _eval(0, np.array([np.inf], np.float32))[0] == np.inf
