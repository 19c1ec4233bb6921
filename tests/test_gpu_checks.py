"""The INFV2_CHECKS debug build (libinfv2_checks.so) against the default build.

Each build runs the cases of checks_child.py in its own process (the
INFV2_BUILD variable selects the library).  The debug build's device-side
checks must leave every result of valid input unchanged and silent, and must
turn a block list with a repeated or out-of-order entry into INFV2_ERR_CHECK in
the device error word (attention on both kernels and the backward), where the
default build, which does not look, reports nothing.  Both builds must skip
list entries past a query's own block: the same bits as the list with those
entries set to -1, and a row left with no block gets O = 0 and lse = -inf.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

from trainable_block_sparse_mean_b200 import build as build_mod
from trainable_block_sparse_mean_b200 import infv2

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
NAMES = ("g16", "g2")


def _run(tmp_path, which):
    out = str(tmp_path / ("%s.npz" % which))
    env = dict(os.environ)
    env["INFV2_BUILD"] = which
    r = subprocess.run([sys.executable, os.path.join(HERE, "checks_child.py"), out], env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-4000:]
    return dict(np.load(out))


@pytest.fixture(scope="module")
def results(tmp_path_factory):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build_mod.build()
    build_mod.build(checks=True)
    tmp = tmp_path_factory.mktemp("checks")
    return _run(tmp, "default"), _run(tmp, "checks")


def test_children_loaded_each_build(results):
    plain, checked = results
    assert str(plain["lib"]) == "libinfv2.so"
    assert str(checked["lib"]) == "libinfv2_checks.so"


def test_valid_input_same_bits_and_no_error(results):
    plain, checked = results
    keys = sorted(x for x in plain if x.startswith("v_"))
    assert len(keys) >= 12
    for key in keys:
        assert np.array_equal(plain[key], checked[key], equal_nan=True), key
    for res in results:
        for name in NAMES:
            for case in ("prefill", "future", "masked", "empty", "bwd"):
                assert int(res["st_%s_%s" % (name, case)]) == infv2.OK, (str(res["lib"]), name, case)
        assert int(res["st_decode_0"]) == infv2.OK and int(res["st_decode_1"]) == infv2.OK


def test_invalid_lists_reported_by_checks_build_only(results):
    plain, checked = results
    for name in NAMES:
        for case in ("repeat", "order", "bwd_repeat"):
            assert int(checked["st_%s_%s" % (name, case)]) == infv2.ERR_CHECK, (name, case)
            assert int(plain["st_%s_%s" % (name, case)]) == infv2.OK, (name, case)


def test_entries_past_own_block_are_skipped(results):
    for res in results:
        for name in NAMES:
            assert np.array_equal(res["f_%s_o" % name], res["m_%s_o" % name]), (str(res["lib"]), name)
            assert np.array_equal(res["f_%s_lse" % name], res["m_%s_lse" % name]), (str(res["lib"]), name)
            assert not (res["e_%s_o" % name] & 0x7FFF).any(), name  # O = 0 (either sign)
            assert np.all(np.isneginf(res["e_%s_lse" % name])), name
