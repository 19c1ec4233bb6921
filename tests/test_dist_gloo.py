"""Multi-rank plumbing of bench.py on CPU with the gloo backend (world size 2),
and the benchmark's algorithmic-work accounting against closed forms."""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402
from trainable_block_sparse_mean_b200 import synth  # noqa: E402


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # each rank measured its own replica; the job step is the slowest rank's
        ms = bench.max_over_ranks(dist, 10.0 + 5.0 * rank, "cpu")
        dist.barrier()
        q.put((rank, ms, bench.job_throughput(world, 131072, ms)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world, port = 2, 29611
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p_ in procs:
        p_.start()
    for p_ in procs:
        p_.join(120)
        assert p_.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, ms, tps in res:
        assert ms == 15.0                      # max over ranks, seen by every rank
        assert tps == pytest.approx(2 * 131072 / 0.015)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(None, 3.5, "cpu") == 3.5
    assert bench.job_throughput(1, 1000, 10.0) == pytest.approx(1e5)


def test_reference_arm_non_zero_rank_exits_quietly():
    env = dict(os.environ, WORLD_SIZE="2", RANK="1", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_prefill_work_matches_closed_form():
    sh = synth.CONFIGS["prefill_128k"]["shape"]
    w = bench.prefill_work(sh, sh.n)
    # two passes x 2*d FLOP per (head, query, visible kernel):
    # sum_i nv(i) with nv(i) = (i-31)//16 + 1 for i >= 31
    n = sh.n
    m = (n - 31 + 15) // 16          # number of distinct nv values reached
    i = np.arange(31, n)
    assert w["score"] == 4 * 128 * 32 * ((i - 31) // 16 + 1).sum()
    assert abs(w["score"] / 1e12 - 8.79) < 0.01
    assert abs(w["attn"] / 1e12 - 8.59) < 0.01
    assert m > 0
    dense = bench.prefill_work(synth.Shape(n=1000, h_q=4, h_kv=1, k=64), 1000)
    assert dense["dense"] and dense["attn"] == 4 * 128 * 4 * (1000 * 1001 // 2)


def test_decode_bytes_at_seed0_lengths():
    cfg = synth.CONFIGS["decode_batch32"]
    lens = synth.decode_lengths(cfg["batch"], cfg["len_lo"], cfg["len_hi"], 0)
    b = bench.decode_bytes(cfg["shape"], lens)
    assert 2.0e8 < b < 2.3e8          # ~213 MB: K^C1 rows + 4096 selected keys of K and V
    assert abs(lens.mean() - 76825) < 1
