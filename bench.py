"""Benchmark of the InfLLM-V2 block-sparse attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one whole prefill of a 131072-token sequence (h_q=32, h_kv=2,
d=128, top-k 64 blocks of 64): stage-1 compression, the two-pass scores,
max-pool + top-k selection and block-sparse attention, through the C ABI
(infv2_prefill).  Inputs are seeded synthetic bf16 arrays already resident in
HBM (Q alone is 1.07 GB, larger than L2, so no L2 flush is needed).  Rank 0
prints one JSON line.  With torchrun, every rank runs its own replica of the
workload (independent sequences, no collective on the data path) and the
reported time is the maximum over ranks.

Also reported: a per-stage breakdown timed with CUDA events on the launching
stream, the roofline of the dominant kernel, an end-to-end figure through host
buffers, the batched decode step (32 sequences, 16k-128k cached tokens), SM
clocks sampled during the timed region, and the fp64 CPU oracle timed on a
bounded sample of query rows.  --impl reference times that oracle as the
reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from trainable_block_sparse_mean_b200 import synth  # noqa: E402

METRIC = "sparse prefill tokens/s + TFLOP/s at 128k (% of peak); decode µs/token"
WORKLOAD = "prefill_128k: prefill, single sequence n=131072, h_q=32, h_kv=2, d=128, bf16, top-k 64 blocks of 64, 128 needles"
B, D = 64, 128


# ------------------------------------------------------------------ accounting

def visible_kernels(i):
    i = np.asarray(i, dtype=np.int64)
    return np.where(i >= 31, (i - 31) // 16 + 1, 0)


def prefill_work(shape: synth.Shape, n: int):
    """Algorithmic FLOPs of one prefill: two score passes over the visible
    kernels (2*d each per head), attention over the selected visible tokens
    (4*d per head and key); dense attention over all visible tokens when
    n <= k*B."""
    i = np.arange(n, dtype=np.int64)
    bi = i // B
    h = shape.h_q
    if n <= shape.k * B:
        att_keys = (i + 1).sum()
        return dict(score=0.0, attn=float(4 * D * h * att_keys), dense=True)
    score = float(2 * 2 * D * h * visible_kernels(i).sum())
    sel = np.minimum(shape.k, bi + 1)
    keys = B * (sel - 1) + (i % B) + 1
    return dict(score=score, attn=float(4 * D * h * keys.sum()), dense=False)


def decode_bytes(shape: synth.Shape, lens):
    """Algorithmic HBM bytes of one decode step at query positions `lens`:
    the visible K^C1 rows, the selected K and V rows, q, o and the new K/V."""
    L = np.asarray(lens, np.int64)
    bi = L // B
    sel = np.minimum(shape.k, bi + 1)
    keys = B * (sel - 1) + (L % B) + 1
    row = D * 2
    kc1 = shape.h_kv * visible_kernels(L).sum() * row
    kv = shape.h_kv * keys.sum() * 2 * row
    small = len(L) * (2 * shape.h_q * row + 2 * 2 * shape.h_kv * row)
    return float(kc1 + kv + small)


# ------------------------------------------------------------------ ranks

def max_over_ranks(dist, x: float, device) -> float:
    """Maximum of a per-rank float over all ranks (identity without a group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


MUFU_PER_SM_CLK = 16   # ex2 per SM per clock (CUDA programming guide, arithmetic throughput)
FMA_EXP_SHARE = 0.25   # share of the score kernel's exponentials on the FMA-pipe polynomial


def score_exp_figures(n: int, h_q: int, ms_score: float, sms: int, sm_mhz: float):
    """The score kernel's secondary bound: one exponential per (head, visible
    kernel) in each of its two passes, against the MUFU rate at the clock the
    run saw.  mufu_frac counts the share that the MUFU executes."""
    exps = 2.0 * h_q * float(visible_kernels(np.arange(n)).sum())
    rate = exps / (ms_score / 1e3)
    peak = MUFU_PER_SM_CLK * sms * sm_mhz * 1e6
    return {"exp_per_step": exps, "exp_per_s": round(rate, 1), "mufu_peak_per_s": round(peak, 1),
            "sm_count": sms, "sm_mhz": sm_mhz, "fma_share": FMA_EXP_SHARE,
            "mufu_frac": round(rate * (1.0 - FMA_EXP_SHARE) / peak, 4)}


def _score_exp_of(n, h_q, stage, dev, clk):
    try:
        import torch
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        mhz = float(clk["sm_mhz"]) if clk and clk.get("sm_mhz") else 1965.0
        ms = stage["per_kernel"]["score_kernel"]["ms_per_step"]
        return score_exp_figures(n, h_q, ms, sms, mhz)
    except Exception as e:   # a secondary figure never ends the benchmark
        return {"error": str(e)[:200]}


def needle_recall(sel, needles, B: int = 64, span: int = 32):
    """Sanity figure of the synthetic needles (not parity): the share of
    (needle, kv head) pairs whose target query selected a block that the
    needle's span of `span` keys intersects.  sel: [h_kv, len(needles), k]
    block lists at the needles' target rows; needles: (target, span start)."""
    found = total = 0
    for r, (_, p0) in enumerate(needles):
        blocks = {p0 // B, (p0 + span - 1) // B}
        for g in range(sel.shape[0]):
            total += 1
            found += bool(blocks & {int(x) for x in sel[g, r]})
    return {"found": found, "total": total, "recall": round(found / total, 4) if total else None}


def _needle_recall_of(idx, needles):
    """needle_recall on the benchmark's own block lists [h_kv, n, k] (device)."""
    try:
        if idx is None or not needles:
            return None
        import torch
        rows = torch.tensor([t for t, _ in needles], dtype=torch.long, device=idx.device)
        return needle_recall(idx.index_select(1, rows).cpu().numpy(), needles)
    except Exception as e:   # a sanity figure never ends the benchmark
        return {"error": str(e)[:200]}


def job_throughput(world: int, units_per_rank: int, ms_per_step: float) -> float:
    """Whole-job units/s: every rank processes its own replica; the step time
    is the slowest rank's."""
    return world * units_per_rank / (ms_per_step / 1e3)


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "100"], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ------------------------------------------------------------------ peaks / profiles

def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def workload_config(shape, world):
    """The `config` object of both arms' JSON lines (the same workload)."""
    return {"workload": WORKLOAD, "n": shape.n, "h_q": shape.h_q, "h_kv": shape.h_kv,
            "d": shape.d, "block": shape.B, "top_k_blocks": shape.k,
            "n_init": shape.n_init, "n_local": shape.n_local, "l_c1": shape.l_c1,
            "s_c1": shape.s_c1, "pool_l": shape.pool_l, "pool_s": shape.pool_s,
            "parallelism": "replicas" if world > 1 else "single GPU",
            "l2": "no flush: Q (1.07 GB) alone exceeds the 126 MB L2"}


def recorded_traffic(kernel: str):
    """DRAM bytes per unit from the committed ncu summary, if the kernel's
    source has not changed since the capture (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    # one source file or a list of them (a kernel and the header that holds its body)
    srcs = rec["source"] if isinstance(rec["source"], list) else [rec["source"]]
    shas = rec["sha256"] if isinstance(rec["sha256"], list) else [rec["sha256"]]
    for name, sha in zip(srcs, shas):
        src = os.path.join(ROOT, name)
        if not os.path.exists(src) or hashlib.sha256(open(src, "rb").read()).hexdigest() != sha:
            return None
    return rec


# ------------------------------------------------------------------ our arm

def run_ours(args, rank, world, local_rank, dist):
    import torch
    from trainable_block_sparse_mean_b200 import infv2
    from trainable_block_sparse_mean_b200.workloads import DecodeState, to_dev

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.only == "decode":   # profiling runs: the decode steps only
        dec = _decode(args, infv2, torch, None, rank, dev, torch.cuda.current_stream(),
                      lambda x: x, DecodeState)
        return {"metric": METRIC, "decode": dec}
    if args.only == "dense":    # profiling runs: the dense 4096-token attention only
        return {"metric": METRIC, "dense": _dense_timing(args, infv2, torch, dev,
                                                         torch.cuda.current_stream())}
    shape = synth.CONFIGS[args.workload]["shape"]
    n = shape.n
    p = infv2.params_of(shape)
    data = synth.make_prefill(shape, seed=rank)
    q, k, v = to_dev(data["q"], dev), to_dev(data["k"], dev), to_dev(data["v"], dev)
    cu = [0, n]
    ws = torch.empty(infv2.infv2_prefill_workspace_size(p, cu), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((shape.h_q, n), device=dev)
    stream = torch.cuda.current_stream()

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_ranks(x):
        return max_over_ranks(dist, x, dev)

    def step():
        infv2.infv2_prefill(p, q, k, v, cu, workspace=ws, o=o, lse=lse)

    if args.only == "backward":  # profiling runs: the attention backward only
        return {"metric": METRIC, "workload": args.workload,
                "backward": _backward_timing(args, infv2, torch, p, shape, q, k, v, ws,
                                             torch.cuda.current_stream())}
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if infv2.infv2_device_status() != 0:
        raise RuntimeError("kernel error word set during warm-up")

    clocks = ClockSampler(local_rank).start() if rank == 0 else None
    time.sleep(0.3 if clocks else 0)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms = e0.elapsed_time(e1) / args.steps
    clk = clocks.stop() if clocks else None
    ms = max_ranks(ms)
    chunk_rows = _chunk_rows(p, n)
    n_chunks = (n + chunk_rows - 1) // chunk_rows
    launches_per_step = 1 + 2 * n_chunks + 1

    if args.only == "prefill":   # profiling runs: the timed prefill steps only
        return {"metric": METRIC, "ms_per_step": round(ms, 4), "workload": args.workload,
                "launches_per_step": launches_per_step}
    # ---- per-stage breakdown on the same stream (CUDA events between launches)
    stage = _stage_breakdown(args, infv2, torch, p, shape, q, k, v, o, lse, ws, stream, chunk_rows)
    fused = _fused_pool_timing(args, infv2, torch, p, shape, q, k, ws, stream, chunk_rows, stage)
    approx = _lse_approx_timing(args, infv2, torch, shape, q, k, v, o, lse, stream, ms)
    bwd = _backward_timing(args, infv2, torch, p, shape, q, k, v, ws, stream)
    # ---- end to end through host buffers
    e2e = _end_to_end(args, infv2, torch, p, shape, data, cu, stream, dev, max_ranks)
    # ---- decode
    dec = _decode(args, infv2, torch, shape, rank, dev, stream, max_ranks, DecodeState)
    # ---- the other configurations and dense attention (reported beside the headline)
    cfgs = _other_configs(args, infv2, torch, dev, stream, rank)
    dense = _dense_timing(args, infv2, torch, dev, stream)
    if infv2.infv2_device_status() != 0:
        raise RuntimeError("kernel error word set during the benchmark")

    work = prefill_work(shape, n)
    flops = work["score"] + work["attn"]
    peaks = measured_peaks()
    tps = job_throughput(world, n, ms)
    tflops = world * flops / (ms / 1e3) / 1e12
    # dominant kernel and its roofline
    dom = max(stage["per_kernel"], key=lambda kk: stage["per_kernel"][kk]["ms_per_step"])
    dk = stage["per_kernel"][dom]
    unit_flops = {"score_kernel": work["score"], "attn_tc_kernel": work["attn"],
                  "select_kernel": None, "compress_k_kernel": None}[dom]
    if unit_flops is not None:
        per_launch = unit_flops / dk["launches_per_step"]
        achieved = per_launch / (dk["ms_per_launch"] / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"kernel": dom, "bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                "peak_source": peaks["source"] + " burst bf16 (cuBLAS)"}
    else:
        byts = dk.get("bytes_per_step", 0.0) / dk["launches_per_step"]
        achieved = byts / (dk["ms_per_launch"] / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"kernel": dom, "bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": peaks["source"]}
    tr = recorded_traffic(dom)
    roof["traffic"] = (tr["dram_bytes_per_launch_per_token"] * n / dk["launches_per_step"]
                       if tr and "dram_bytes_per_launch_per_token" in tr else
                       (tr["dram_bytes_per_launch"] if tr and "dram_bytes_per_launch" in tr else None))
    sel_ms = sum(stage["per_kernel"][x]["ms_per_step"] for x in
                 ("compress_k_kernel", "score_kernel", "select_kernel"))
    out = {
        "metric": METRIC, "value": round(tps, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) Q/V, K with per-block offsets and 128 planted needles)",
        "config": workload_config(shape, world),
        "tflops": round(tflops, 2),
        "tflops_frac_of_peak": round(tflops / world / peaks["bf16_tflops"], 4),
        "algorithmic_tflop_per_step": {"score": round(work["score"] / 1e12, 3),
                                       "attention": round(work["attn"] / 1e12, 3)},
        "selection_share": round(sel_ms / stage["ms_per_step"], 4),
        "stages": stage["per_kernel"],
        "fused_pool": fused,
        "lse_approx": approx,
        "backward": bwd,
        "roofline": roof,
        "needle_recall": _needle_recall_of(stage.get("idx"), data.get("needles")),
        "score_exp": _score_exp_of(n, p.h_q, stage, dev, clk),
        "e2e": e2e,
        "decode": dec,
        "configs": cfgs,
        "dense": dense,
        "gpu_launches": launches_per_step * args.steps,
        "peaks": peaks,
    }
    if clk:
        out["clocks"] = clk
    return out


def _chunk_rows(p, n):
    # mirrors the library's chunking of S^shared (1 GiB budget, multiples of 128 rows)
    ld = ((max((n - 32) // 16 + 1, 4 * ((n + 63) // 64)) + 31) // 32) * 32
    rows = (1 << 30) // (p.h_kv * ld * 4)
    rows = max(128, (rows // 128) * 128)
    return min(rows, n)


def _stage_breakdown(args, infv2, torch, p, shape, q, k, v, o, lse, ws, stream, chunk_rows):
    """Run the prefill stage by stage through the C ABI, with CUDA events
    around every launch, and average each kernel's duration."""
    n = shape.n
    nc = infv2.num_kernels(p, n)
    ld = infv2.shared_ld(n)
    kc1 = ws[: nc * p.h_kv * 128 * 2].view(torch.bfloat16).view(nc, p.h_kv, 128)
    off_sh = ((nc * p.h_kv * 256) + 255) // 256 * 256
    s_sh = ws[off_sh: off_sh + p.h_kv * chunk_rows * ld * 4].view(torch.float32).view(p.h_kv, chunk_rows, ld)
    idx = torch.empty((p.h_kv, n, p.k), dtype=torch.int32, device=q.device)
    names = ["compress_k_kernel", "score_kernel", "select_kernel", "attn_tc_kernel"]

    def one(record):
        evs = []
        def ev():
            e = torch.cuda.Event(enable_timing=True)
            e.record(stream)
            return e
        a = ev()
        infv2.infv2_compress_k(p, k, kc1)
        evs.append(("compress_k_kernel", a, ev()))
        for q0 in range(0, n, chunk_rows):
            ql = min(chunk_rows, n - q0)
            a = ev()
            infv2.infv2_block_scores(p, q, kc1, n, q0, ql, s_sh[:, :ql] if ql == chunk_rows else
                                     s_sh.view(-1)[: p.h_kv * ql * ld].view(p.h_kv, ql, ld), ld)
            b = ev()
            infv2.infv2_select_topk(p, s_sh.view(-1)[: p.h_kv * ql * ld].view(p.h_kv, ql, ld), ld, n,
                                    q0, ql, idx)
            evs.append(("score_kernel", a, b))
            evs.append(("select_kernel", b, ev()))
        a = ev()
        infv2.infv2_sparse_attn(p, q, k, v, idx, o, lse)
        evs.append(("attn_tc_kernel", a, ev()))
        return evs

    for _ in range(max(1, args.warmup)):
        one(False)
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    all_evs = []
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        all_evs.append(one(True))
    e1.record(stream)
    torch.cuda.synchronize()
    per = {nm: {"ms_per_step": 0.0, "launches_per_step": 0} for nm in names}
    for evs in all_evs:
        for nm, a, b in evs:
            per[nm]["ms_per_step"] += a.elapsed_time(b)
            per[nm]["launches_per_step"] += 1
    for nm in names:
        per[nm]["ms_per_step"] /= steps
        per[nm]["launches_per_step"] //= steps
        per[nm]["ms_per_launch"] = per[nm]["ms_per_step"] / max(1, per[nm]["launches_per_step"])
    # algorithmic bytes of the memory-bound stages
    per["compress_k_kernel"]["bytes_per_step"] = float(n * p.h_kv * 256 + nc * p.h_kv * 256)
    vis = visible_kernels(np.arange(n)).sum()
    per["select_kernel"]["bytes_per_step"] = float(p.h_kv * vis * 4 + p.h_kv * n * p.k * 4)
    for nm in names:
        per[nm] = {kk: (round(vv, 4) if isinstance(vv, float) else vv) for kk, vv in per[nm].items()}
    return dict(per_kernel=per, ms_per_step=e0.elapsed_time(e1) / steps, idx=idx)


def _timed(torch, stream, fn, warm, steps):
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def _prefill_figures(args, infv2, torch, dev, stream, shape, data, cu, flops, stages=True):
    """Tokens/s and algorithmic TFLOP/s of infv2_prefill over one (varlen)
    batch; with `stages`, the stage breakdown of a single sequence: selection
    share and the attention kernel's TFLOP/s against the measured peak."""
    from trainable_block_sparse_mean_b200.workloads import to_dev
    p = infv2.params_of(shape)
    q, k, v = to_dev(data["q"], dev), to_dev(data["k"], dev), to_dev(data["v"], dev)
    ws = torch.empty(max(infv2.infv2_prefill_workspace_size(p, cu), 256), dtype=torch.uint8, device=dev)
    o = torch.empty_like(q)
    lse = torch.empty((shape.h_q, q.shape[0]), device=dev)
    steps = max(3, min(args.steps, 10))
    ms = _timed(torch, stream, lambda: infv2.infv2_prefill(p, q, k, v, cu, workspace=ws, o=o, lse=lse),
                max(1, args.warmup), steps)
    peaks = measured_peaks()
    T = int(cu[-1])
    out = {"tokens": T, "ms_per_step": round(ms, 4), "tokens_per_s": round(T / (ms / 1e3), 1),
           "algorithmic_tflop": round(flops["total"] / 1e12, 4),
           "tflops": round(flops["total"] / (ms / 1e3) / 1e12, 2),
           "tflops_frac_of_peak": round(flops["total"] / (ms / 1e3) / 1e12 / peaks["bf16_tflops"], 4)}
    if stages:
        st = _stage_breakdown(args, infv2, torch, p, shape, q, k, v, o, lse, ws, stream,
                              _chunk_rows(p, shape.n))
        per = st["per_kernel"]
        sel = sum(per[x]["ms_per_step"] for x in ("compress_k_kernel", "score_kernel", "select_kernel"))
        at = per["attn_tc_kernel"]["ms_per_step"]
        out["selection_share"] = round(sel / st["ms_per_step"], 4)
        out["stages_ms"] = {kk: per[kk]["ms_per_step"] for kk in per}
        out["attention"] = {"kernel": "attn_tc_kernel", "ms": at,
                            "tflops": round(flops["attn"] / (at / 1e3) / 1e12, 2),
                            "frac": round(flops["attn"] / (at / 1e3) / 1e12 / peaks["bf16_tflops"], 4)}
    return out


def _other_configs(args, infv2, torch, dev, stream, rank):
    """The configurations besides the headline: the 2k and 32k single
    sequences and the varlen dense/sparse switch sweep (its dense sequences,
    n <= k*B, and its sparse ones timed apart as well as together)."""
    out = {}
    for name in ("prefill_2k", "prefill_32k"):
        sh = synth.CONFIGS[name]["shape"]
        data = synth.make_prefill(sh, seed=rank)
        w = prefill_work(sh, sh.n)
        out[name] = _prefill_figures(args, infv2, torch, dev, stream, sh, data, [0, sh.n],
                                     dict(total=w["score"] + w["attn"], attn=w["attn"]))
    cfg = synth.CONFIGS["varlen_sweep"]
    sh = cfg["shape"]
    lengths = list(cfg["lengths"])
    sweep = {}
    for part, lens in (("all", lengths), ("dense", [x for x in lengths if x <= sh.k * sh.B]),
                       ("sparse", [x for x in lengths if x > sh.k * sh.B])):
        data = synth.make_varlen(sh, lens, seed=rank)
        tot = 0.0
        for L in lens:
            w = prefill_work(sh, L)
            tot += w["score"] + w["attn"]
        fig = _prefill_figures(args, infv2, torch, dev, stream, sh, data, list(data["cu_seqlens"]),
                               dict(total=tot, attn=0.0), stages=False)
        fig["lengths"] = lens
        sweep[part] = fig
    out["varlen_sweep"] = sweep
    return out


def _dense_timing(args, infv2, torch, dev, stream):
    """Dense causal attention (infv2_dense_attn) over a 4096-token sequence at
    h_q=32, h_kv=2: the kernel a sequence of at most k*B tokens takes."""
    from trainable_block_sparse_mean_b200.workloads import to_dev
    sh = synth.Shape(n=4096, h_q=32, h_kv=2, k=64)
    data = synth.make_prefill(sh, seed=0)
    p = infv2.params_of(sh)
    q, k, v = to_dev(data["q"], dev), to_dev(data["k"], dev), to_dev(data["v"], dev)
    o = torch.empty_like(q)
    ms = _timed(torch, stream, lambda: infv2.infv2_dense_attn(p, q, k, v, o=o), max(3, args.warmup),
                max(10, min(args.steps, 50)))
    flops = prefill_work(sh, sh.n)["attn"]
    peaks = measured_peaks()
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": "dense causal attention, n=4096, h_q=32, h_kv=2, d=128, bf16",
            "kernel": "attn_tc_kernel", "us": round(ms * 1e3, 2),
            "algorithmic_tflop": round(flops / 1e12, 4),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peaks["bf16_tflops"],
                         "unit": "TFLOP/s", "frac": round(tf / peaks["bf16_tflops"], 4)}}


def _fused_pool_timing(args, infv2, torch, p, shape, q, k, ws, stream, chunk_rows, stage):
    """The alternative stage 2-4 path with max pooling fused into the score
    kernel (block scores S^cmp out, top-k-only selection), timed over the same
    row chunks as the unfused stages; reported beside them, not in the step."""
    n = shape.n
    nc = infv2.num_kernels(p, n)
    ldc = infv2.cmp_ld(n)
    kc1 = ws[: nc * p.h_kv * 128 * 2].view(torch.bfloat16).view(nc, p.h_kv, 128)
    off = ((nc * p.h_kv * 256) + 255) // 256 * 256
    s_cmp = ws[off: off + p.h_kv * chunk_rows * ldc * 4].view(torch.float32)
    idx = torch.empty((p.h_kv, n, p.k), dtype=torch.int32, device=q.device)
    infv2.infv2_compress_k(p, k, kc1)

    def one():
        evs = []
        for q0 in range(0, n, chunk_rows):
            ql = min(chunk_rows, n - q0)
            buf = s_cmp[: p.h_kv * ql * ldc].view(p.h_kv, ql, ldc)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            c = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            infv2.infv2_block_scores_pooled(p, q, kc1, n, q0, ql, buf, ldc)
            b.record(stream)
            infv2.infv2_select_topk_pooled(p, buf, ldc, n, q0, ql, idx)
            c.record(stream)
            evs.append((a, b, c))
        return evs

    one()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    runs = [one() for _ in range(steps)]
    torch.cuda.synchronize()
    sc = sum(a.elapsed_time(b) for r in runs for a, b, _ in r) / steps
    se = sum(b.elapsed_time(c) for r in runs for _, b, c in r) / steps
    unfused = stage["per_kernel"]["score_kernel"]["ms_per_step"] + stage["per_kernel"]["select_kernel"]["ms_per_step"]
    return {"score_kernel_pooled_ms_per_step": round(sc, 4), "select_pooled_kernel_ms_per_step": round(se, 4),
            "total_ms_per_step": round(sc + se, 4), "unfused_total_ms_per_step": round(unfused, 4),
            "chunk_rows": chunk_rows, "used_in_step": False}


def _lse_approx_timing(args, infv2, torch, shape, q, k, v, o, lse, stream, exact_ms):
    """The whole prefill with the LSE approximation (pass 1 over the coarse
    kernels), timed like the headline step; reported beside it, not instead."""
    n = shape.n
    pa = infv2.params_of(shape)
    pa.lse_approx = 1
    cu = [0, n]
    ws = torch.empty(infv2.infv2_prefill_workspace_size(pa, cu), dtype=torch.uint8, device=q.device)
    nc2 = infv2.num_coarse_kernels(pa, n)

    def step():
        infv2.infv2_prefill(pa, q, k, v, cu, workspace=ws, o=o, lse=lse)

    for _ in range(max(1, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 10))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    return {"ms_per_step": round(ms, 4), "tokens_per_s": round(n / (ms / 1e3), 1),
            "exact_ms_per_step": round(exact_ms, 4), "coarse_kernels": nc2,
            "used_in_step": False,
            "note": "pass-1 log-sum-exp from the coarse kernels K^C2 (l=128, s=64); selection "
                    "differs from the exact path where the estimate reorders near-equal blocks"}


def _backward_timing(args, infv2, torch, p, shape, q, k, v, ws, stream):
    """The attention backward (dq, dk, dv) on the prefill's own block lists,
    timed on the device; reported beside the forward step."""
    n = shape.n
    cu = [0, n]
    idx = torch.empty((p.h_kv, n, p.k), dtype=torch.int32, device=q.device)
    o = torch.empty_like(q)
    lse = torch.empty((p.h_q, n), device=q.device)
    infv2.infv2_prefill(p, q, k, v, cu, workspace=ws, idx_out=idx, o=o, lse=lse)
    gen = torch.Generator(device=q.device)
    gen.manual_seed(1)
    d_o = torch.randn(q.shape, generator=gen, device=q.device).to(torch.bfloat16)
    bws = torch.empty(infv2.infv2_sparse_attn_bwd_workspace_size(p, n), dtype=torch.uint8,
                      device=q.device)

    def step():
        return infv2.infv2_sparse_attn_bwd(p, q, k, v, idx, o, lse, d_o, workspace=bws)

    step()
    torch.cuda.synchronize()
    steps = max(3, min(args.steps, 5))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    attn = prefill_work(shape, n)["attn"]          # 4*d FLOP per (head, selected visible key)
    executed = attn * 14.0 / 4.0                   # S, dP, dS.K (dq) + S, dP, P^T.dO, dS^T.Q (dk, dv)
    return {"ms_per_step": round(ms, 3), "tflop_executed": round(executed / 1e12, 3),
            "tflops_executed": round(executed / (ms / 1e3) / 1e12, 1),
            "note": "dq, dk, dv in fp32 over the prefill's block lists (selection fixed)"}


def _end_to_end(args, infv2, torch, p, shape, data, cu, stream, dev, max_over_ranks):
    """Same metric through the C ABI with host buffers (infv2_pipeline_*):
    every step copies its inputs from pinned host memory and reads its output
    back.  The library's pipeline copies on its own two streams into two
    device slots, so that step j+1's inputs travel and step j-1's output
    returns while step j computes (as a serving loop would pipeline them), and
    within a step the score chunks wait only for the Q rows they read and each
    finished attention row range of O leaves while the next computes; every
    copy of every timed step is inside the timed region."""
    qh = torch.from_numpy(data["q"].view(np.int16)).pin_memory()
    kh = torch.from_numpy(data["k"].view(np.int16)).pin_memory()
    vh = torch.from_numpy(data["v"].view(np.int16)).pin_memory()
    ohs = [torch.empty_like(qh).pin_memory() for _ in range(2)]
    pl = infv2.infv2_pipeline_create(p, cu, stream=stream, device=dev)
    try:
        for j in range(2):
            infv2.infv2_pipeline_submit(pl, qh, kh, vh, ohs[j % 2])
        infv2.infv2_pipeline_sync(pl)
        steps = max(3, min(args.steps, 10))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        infv2.infv2_pipeline_wait(pl, stream)
        for j in range(steps):
            infv2.infv2_pipeline_submit(pl, qh, kh, vh, ohs[j % 2])
        infv2.infv2_pipeline_join(pl, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        infv2.infv2_pipeline_sync(pl)
    finally:
        infv2.infv2_pipeline_destroy(pl)
    ms = max_over_ranks(e0.elapsed_time(e1) / steps)
    h2d = qh.numel() * 2 + kh.numel() * 2 + vh.numel() * 2
    d2h = ohs[0].numel() * 2
    world = int(os.environ.get("WORLD_SIZE", "1"))
    return {"value": round(job_throughput(world, shape.n, ms), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "api": "infv2_pipeline_submit (host buffers)",
            "overlap": "Q copied in 8192-token parts and O returned per attention row range "
                       "(8 per sequence) on the pipeline's own streams; step j+1's inputs and "
                       "step j-1's output travel while step j computes (two device slots)"}


def _decode(args, infv2, torch, shape3, rank, dev, stream, max_over_ranks, DecodeState):
    """Batched decode: each step (3 launches: logits with the cache append and
    K^C1 update; selection; split-KV attention whose last piece per row merges
    and advances seqlens) is captured once into a CUDA graph,
    as a serving loop would run it, and the graphs are replayed in order (each
    replay appends its own token and advances seqlens on the device)."""
    cfg = dict(synth.CONFIGS["decode_batch32"])
    if args.decode_small:   # profiler runs: 8 sequences of at most 32k tokens
        cfg.update(batch=8, len_lo=16384, len_hi=32768)
    sh = cfg["shape"]
    steps_avail = cfg["steps"]
    data = synth.make_decode(sh, cfg["batch"], cfg["len_lo"], cfg["len_hi"], steps_avail,
                             seed=rank)
    st = DecodeState(sh, data, device=dev)
    o = torch.empty((cfg["batch"], sh.h_q, sh.d), dtype=torch.bfloat16, device=dev)
    warm = min(args.warmup, 8)
    for t in range(warm):
        st.step(t, o=o)
    torch.cuda.synchronize()
    timed = min(steps_avail - warm, 48)
    graphs = []
    cap_stream = torch.cuda.Stream(device=dev)
    for t in range(warm, warm + timed):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap_stream, capture_error_mode="relaxed"):
            st.step(t, o=o)
        graphs.append(g)
    torch.cuda.synchronize()
    evs = []
    for g in graphs:
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    times = [a.elapsed_time(b) for a, b in evs]
    lens_now = st.seqlens.cpu().numpy()
    assert np.array_equal(lens_now, data["lens"] + warm + timed), "decode graphs did not advance"
    us = max_over_ranks(float(np.median(times)) * 1e3)
    lens_mid = data["lens"] + warm + timed // 2
    byts = decode_bytes(sh, lens_mid)
    peaks = measured_peaks()
    gbs = byts / (us / 1e6) / 1e9
    del graphs
    return {"workload": "decode_batch32: batch 32, one query token each, cache lengths U[16384, 131072] "
                        "(seed-0 mean %.0f), h_q=32, h_kv=2, top-k 64" % data["lens"].mean(),
            "us_per_step": round(us, 2), "us_per_token_per_sequence": round(us, 2),
            "us_per_token_aggregate": round(us / cfg["batch"], 3),
            "launches_per_step": 3, "timing": "CUDA graph per step, median of %d replays" % timed,
            "algorithmic_bytes_per_step": int(byts),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4)}}


# ------------------------------------------------------------------ CPU oracle

def oracle_sample(target_s=12.0, seed=0):
    """Time the fp64 oracle on a bounded random sample of query rows of the
    128k workload (rows drawn uniformly; cost grows with the row index)."""
    import oracle
    shape = synth.CONFIGS["prefill_128k"]["shape"]
    data = synth.make_prefill(shape, seed=0)
    op = oracle.params(shape)
    rng = np.random.default_rng(seed)
    threads = oracle.num_threads()
    # calibrate on one batch of `threads` rows, then size the sample
    rows = rng.integers(0, shape.n, size=threads).astype(np.int32)
    t0 = time.perf_counter()
    oracle.prefill_rows(op, data["q"], data["k"], data["v"], rows)
    t_cal = time.perf_counter() - t0
    n_rows = max(threads, int(threads * target_s / max(t_cal, 1e-3)))
    rows = rng.integers(0, shape.n, size=n_rows).astype(np.int32)
    t0 = time.perf_counter()
    oracle.prefill_rows(op, data["q"], data["k"], data["v"], rows)
    dt = time.perf_counter() - t0
    return {"value": round(n_rows / dt, 3), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": "%d query rows drawn uniformly from the 131072-token sequence (all stages, "
                      "fp64, OpenMP over rows), %.1f s" % (n_rows, dt)}, data, shape


def run_reference(args):
    import oracle
    oracle.build()
    shape = synth.CONFIGS["prefill_128k"]["shape"]
    data = synth.make_prefill(shape, seed=0)
    op = oracle.params(shape)
    threads = oracle.num_threads()
    rng = np.random.default_rng(1)
    rows = rng.integers(0, shape.n, size=threads).astype(np.int32)
    t0 = time.perf_counter()
    oracle.prefill_rows(op, data["q"], data["k"], data["v"], rows)
    per_batch = time.perf_counter() - t0
    # size each step to about 6 s of CPU work
    rows_per_step = max(threads, int(threads * 6.0 / max(per_batch, 1e-3)))
    for _ in range(args.warmup):
        r = rng.integers(0, shape.n, size=threads).astype(np.int32)
        oracle.prefill_rows(op, data["q"], data["k"], data["v"], r)
    t_total, n_total = 0.0, 0
    for _ in range(args.steps):
        r = rng.integers(0, shape.n, size=rows_per_step).astype(np.int32)
        t0 = time.perf_counter()
        oracle.prefill_rows(op, data["q"], data["k"], data["v"], r)
        t_total += time.perf_counter() - t0
        n_total += rows_per_step
    v = n_total / t_total
    sample = ("%d query rows per step drawn uniformly from the 131072-token sequence "
              "(all stages, fp64, OpenMP over rows)" % rows_per_step)
    return {"impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": "tokens/s",
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t_total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(shape, int(os.environ.get("WORLD_SIZE", "1"))),
            "cpu_baseline": {"value": round(v, 3), "unit": "tokens/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(v, 3), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workload", choices=["prefill_128k", "prefill_32k"], default="prefill_128k",
                    help="prefill workload: prefill_128k (131072 tokens, the reported one) or prefill_32k (32768)")
    ap.add_argument("--decode-small", action="store_true",
                    help="with --only decode: 8 sequences of 16k-32k tokens (profiler runs)")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "backward", "dense"], default="all",
                    help="prefill / decode / backward / dense: time only that part (for profiler runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)))
        return 0

    from trainable_block_sparse_mean_b200 import build as lib_build
    if rank == 0 or world == 1:
        lib_build.build()
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
        dist.barrier()
    try:
        out = run_ours(args, rank, world, local_rank, dist)
        if rank == 0 and not args.no_cpu_baseline and args.only == "all":
            cpu, _, _ = oracle_sample()
            out["cpu_baseline"] = cpu
        if rank == 0:
            print(json.dumps(out))
    finally:
        if dist is not None:
            dist.barrier()
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
