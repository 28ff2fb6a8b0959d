#!/usr/bin/env python
"""Benchmark: XAttention block-sparse prefill attention, one layer per step.

One step = one pass of the whole path (score -> select -> block-sparse attention)
over one layer of seeded synthetic input (all heads), on the stream the kernels are
launched on. Default workload: Llama-3.1-8B-shaped GQA prefill at 128K tokens
(32 query / 8 KV heads, head dim 128, stride 8, tau 0.9, causal).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torchrun, one rank per GPU): by default one layer is split
by KV-head group (each rank holds its groups' Q/K/V, runs the unchanged kernels
on them, and O is all-gathered with NCCL: strong scaling); with --split replicas
every rank runs a layer of its own with no collective (weak scaling). The
reported time is the max over ranks.

After the main workload, a second leg times the video-DiT-shaped layer (the
non-causal workload where the selection keeps ~3% of the blocks) with its own
dense attention, reported under "video".

`--impl reference` times the CPU fp64 oracle (the only reference this method has)
on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synthetic as sy  # noqa: E402

METRIC = "128K-token prefill attention ms/layer and kept-block TFLOPS (% of BF16 peak)"
# scale of the scoring softmax (name -> (description, value for stride S and head dim C))
SCORE_SCALES = {
    "sqrt_sc": ("1/sqrt(stride*C)", lambda S, C: 1.0 / math.sqrt(S * C)),
    "sqrt_c": ("1/sqrt(C)", lambda S, C: 1.0 / math.sqrt(C)),
    "s_sqrt_c": ("1/(stride*sqrt(C))", lambda S, C: 1.0 / (S * math.sqrt(C))),
}
UNIT = "ms/layer"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="llama8b_gqa_128k", choices=sorted(sy.WORKLOADS))
    ap.add_argument("--stride", type=int, default=None)
    ap.add_argument("--seed", type=int, default=sy.DEFAULT_SEED)
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="CPU work budget of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--fused-select", action="store_true",
                    help="score and select in the one fused call instead of two calls")
    ap.add_argument("--score-scale", default="sqrt_sc", choices=sorted(SCORE_SCALES),
                    help="scale of the scoring softmax: 1/sqrt(stride*C) (default), "
                         "1/sqrt(C) or 1/(stride*sqrt(C)); the method leaves it open")
    ap.add_argument("--split", default="heads", choices=["heads", "replicas"],
                    help="with several GPUs: split one layer by KV-head group (default) or run "
                         "one independent layer per GPU")
    ap.add_argument("--no-video", action="store_true",
                    help="skip the second leg (the video-DiT-shaped non-causal layer)")
    ap.add_argument("--group-select", action="store_true",
                    help="GQA-shared kept lists (union over each KV group; a variant the "
                         "method does not define) instead of per-head lists")
    return ap.parse_args()


def workload_of(a):
    w = sy.workload(a.workload)
    return w.with_(stride=a.stride) if a.stride else w


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "dram_traffic_llama8b_gqa_128k.json")
KERNEL_SOURCES = {"attn_tc": ["attn_tc.cuh", "common.cuh", "sm100.cuh"],
                  "score_tc": ["score_tc.cuh", "select.cuh", "common.cuh", "sm100.cuh"]}


def kernel_source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "block_sparse_long_04_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(kernel: str, workload: str, stride: int):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None
    when there is none for this workload or the kernel's sources changed since."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    d = json.load(open(TRAFFIC_FILE))
    k = d.get("kernels", {}).get(kernel)
    if (k is None or d.get("workload") != workload or d.get("stride") != stride
            or k.get("source_sha256") != kernel_source_hash(kernel)):
        return None
    return k["dram_bytes_read"] + k["dram_bytes_write"]


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"],
                    bf16_sustained=d["bf16_tflops_sustained"], source="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# ------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled while the timed region runs.

    nvidia-smi takes a few hundred ms to start, so the sampler is started before
    the warm-up and every sample carries its arrival time; summary() keeps the
    samples that arrived between mark_start() and mark_end() (plus one sampling
    period of slack at the end)."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    PERIOD_MS = 50

    def __init__(self, index):
        self.index, self.rows, self.proc = index, [], None
        self.t_start, self.t_end = None, None

    def mark_start(self):
        self.t_start = time.monotonic()

    def mark_end(self):
        self.t_end = time.monotonic()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-i", str(self.index), "-lms", str(self.PERIOD_MS)], stdout=subprocess.PIPE,
                stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.monotonic(), [x.strip() for x in line.split(",")]))

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = self.rows
        if self.t_start is not None and self.t_end is not None:
            slack = self.PERIOD_MS / 1000.0
            rows = [r for t, r in rows if self.t_start <= t <= self.t_end + slack]
        else:
            rows = [r for _, r in rows]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# --------------------------------------------------------- CPU oracle sample
def score_scale_of(a, w) -> float:
    return SCORE_SCALES[a.score_scale][1](w.stride, w.C)


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity set)."""
    return len(os.sched_getaffinity(0))


def blas_threads() -> int:
    from threadpoolctl import threadpool_info
    return max(1, sum(i.get("num_threads", 0) for i in threadpool_info()
                      if i.get("user_api") == "blas"))


def oracle_sample(w, Qb, Kb, Vb, tau, seconds, sig, seed=0):
    """Time the oracle on uniformly drawn (head, query block) units until `seconds`
    of work are done; returns (ms per layer extrapolated by unit count, units, desc)."""
    import oracle as orc
    rng = np.random.default_rng(seed)
    nb, grp = w.nb, w.Hq // w.Hkv
    sa = 1 / math.sqrt(w.C)
    done, t_work = 0, 0.0
    cache = {}
    while t_work < seconds or done < 4:
        h, r = int(rng.integers(w.Hq)), int(rng.integers(nb))
        if h not in cache:   # input widening is data movement, not timed
            cache.clear()
            cache[h] = tuple(orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // grp], Vb[0, h // grp]))
        q, k, v = cache[h]
        t0 = time.perf_counter()
        s = orc.block_scores(q, k, w.stride, w.block, sig, w.causal, rows=[r])
        kept = {r: orc.select_row(s[r], r, float(tau[h]), w.causal)}
        orc.block_sparse_attention(q, k, v, kept, w.block, w.causal, sa, rows=[r])
        t_work += time.perf_counter() - t0
        done += 1
    units = w.B * w.Hq * nb
    desc = (f"{done} (head, query-block) units of the {w.name} layer drawn uniformly at random "
            f"(score row + select + sparse attention each), {t_work:.1f} s; full-layer time "
            f"extrapolated by unit count (x{units / done:.3g})")
    return t_work / done * units * 1e3, done, desc


def reference_arm(a, w, rank, world):
    """--impl reference: the CPU oracle as the timed arm, rank 0 only."""
    if rank != 0:
        return 0
    Qb, Kb, Vb = sy.layer_inputs(w, a.seed)
    tau = sy.tau_vector(w, a.seed)
    per_step = max(2.0, min(a.cpu_seconds, 60.0 / max(1, a.steps + a.warmup)))
    for i in range(a.warmup):
        oracle_sample(w, Qb, Kb, Vb, tau, per_step, score_scale_of(a, w), seed=100 + i)
    vals, units, desc = [], 0, ""
    for i in range(a.steps):
        v, u, desc = oracle_sample(w, Qb, Kb, Vb, tau, per_step, score_scale_of(a, w), seed=i)
        vals.append(v)
        units += u
    val = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": a.gpus,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": val, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, a),
        "cpu_baseline": {"value": val, "unit": UNIT, "cores": host_cores(),
                         "blas_threads": blas_threads(), "kind": "oracle",
                         "sample": f"per step: {desc}"},
        "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_of(w, a, world=1):
    split = getattr(a, "split", "heads")
    if world > 1 and split == "heads":
        par = (f"one layer split by KV-head group over {world} GPUs "
               f"({w.Hkv // world} KV groups, {w.Hq // world} query heads each); "
               "NCCL all-gather of O")
    elif world > 1:
        par = "one independent layer per GPU (no collective)"
    else:
        par = "one GPU"
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.M, "C": w.C,
            "block": w.block, "stride": w.stride, "causal": w.causal,
            "tau": list(w.tau_range) if w.tau_range else w.tau,
            "score_scale": SCORE_SCALES[a.score_scale][0], "softmax_scale": "1/sqrt(C)",
            "l2": "no flush; inputs larger than L2 (126 MB): Q %.2f GB, K and V %.2f GB each" % (
                w.B * w.Hq * w.M * w.C * 2 / 1e9, w.B * w.Hkv * w.M * w.C * 2 / 1e9)
            if w.B * w.Hkv * w.M * w.C * 2 > 126e6 else "inputs fit in L2 (not a bench workload)",
            "parallelism": par}


# ------------------------------------------------------- multi-rank helpers
def dist_max(x: float, dist=None, device=None) -> float:
    """Max of a per-rank float over all ranks (the job time is the slowest rank)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_ms_per_layer(total_ms_max: float, steps: int, world: int, batch: int) -> float:
    """Whole-job ms per layer: every rank processed `steps` layers of `batch`
    sequences in `total_ms_max` (max over ranks) milliseconds."""
    return total_ms_max / (steps * world * batch)


def head_shard(Hq: int, Hkv: int, world: int, rank: int):
    """KV heads [kv_lo, kv_hi) and query heads [h_lo, h_hi) of `rank` when one
    layer is split by KV-head group over `world` ranks. Every unit of the method
    (a query head's scoring, selection and attention) reads only its own KV head,
    so whole groups are the shards and no step exchanges data."""
    if Hkv % world != 0:
        raise ValueError(f"{Hkv} KV heads do not split evenly over {world} ranks")
    per = Hkv // world
    g = Hq // Hkv
    kv_lo, kv_hi = rank * per, (rank + 1) * per
    return kv_lo, kv_hi, kv_lo * g, kv_hi * g


def gather_heads(O_local, dist, world: int, out=None):
    """All-gather of every rank's O [B, Hq/world, M, C] into the layer's O.

    Returns a tensor of shape [world, B, Hq/world, M, C] (rank-major); for B = 1
    its memory is exactly O [1, Hq, M, C] with the heads in order, and for B > 1
    `.permute(1, 0, 2, 3, 4)` gives [B, world, Hq/world, M, C]."""
    import torch
    if out is None:
        out = torch.empty((world,) + tuple(O_local.shape), dtype=O_local.dtype,
                          device=O_local.device)
    dist.all_gather_into_tensor(out.view(-1), O_local.contiguous().view(-1))
    return out


# ------------------------------------------------------------ our arm
class Layer:
    """One (local) layer's inputs in pinned host memory and on the device, its
    thresholds and its buffers. With heads=(kv_lo, kv_hi) only those KV groups of
    the workload (the same bits as in the whole layer)."""

    def __init__(self, w, seed, dev, heads=None):
        import torch
        import block_sparse_long_04_b200 as xa
        kv_lo, kv_hi = (0, w.Hkv) if heads is None else heads
        g = w.group
        hq, hkv = (kv_hi - kv_lo) * g, kv_hi - kv_lo
        self.w, self.hq, self.hkv = w, hq, hkv
        self.Qh = torch.empty((w.B, hq, w.M, w.C), dtype=torch.bfloat16).pin_memory()
        self.Kh = torch.empty((w.B, hkv, w.M, w.C), dtype=torch.bfloat16).pin_memory()
        self.Vh = torch.empty((w.B, hkv, w.M, w.C), dtype=torch.bfloat16).pin_memory()
        self.views = tuple(t.view(torch.int16).numpy().view(np.uint16)
                           for t in (self.Qh, self.Kh, self.Vh))
        sy.layer_inputs(w, seed, out=self.views, heads=(kv_lo, kv_hi))
        self.tau_np = np.ascontiguousarray(sy.tau_vector(w, seed)[kv_lo * g:kv_hi * g])
        self.Q, self.K, self.V = (t.to(dev) for t in (self.Qh, self.Kh, self.Vh))
        self.tau = torch.from_numpy(self.tau_np).to(dev)
        self.bufs = xa.Buffers.allocate(w.B, hq, w.M, w.C, w.stride, w.causal, device=dev)


def time_layer(xa, L, ss, sa, stream, steps, warmup, gather=None, fused=False, group=None):
    """Runs `warmup` untimed passes of score -> select -> attention (-> gather) over
    layer L and returns (step, per-step events, start event, end event): step(ev)
    issues one pass recording ev[0..4] around its stages."""
    import torch
    w, bufs = L.w, L.bufs

    def step(ev=None):
        rec = (lambda i: ev[i].record(stream)) if ev is not None else (lambda i: None)
        rec(0)
        if group is not None:
            g_rp, g_col, g_ws = group
            xa.xattn_score(L.Q, L.K, w.stride, w.causal, ss, bufs.scores, bufs.score_ws,
                           stream=stream)
            rec(1)
            xa.xattn_select_group(bufs.scores, L.tau, xa.XATTN_SELECT_THRESHOLD, L.hkv, w.causal,
                                  g_rp, g_col, bufs.nnz, g_ws, stream=stream)
            rec(2)
            xa.xattn_sparse_attn_group(L.Q, L.K, L.V, g_rp, g_col, w.causal, sa, bufs.O,
                                       stream=stream)
        else:
            if not fused:
                xa.xattn_score(L.Q, L.K, w.stride, w.causal, ss, bufs.scores, bufs.score_ws,
                               stream=stream)
                rec(1)
                xa.xattn_select(bufs.scores, L.tau, w.causal, bufs.row_ptr, bufs.col_idx,
                                bufs.nnz, bufs.select_ws, stream=stream)
            else:
                # the scoring kernel ranks and cuts each row; then the scan and fill passes
                xa.xattn_score_select(L.Q, L.K, L.tau, xa.XATTN_SELECT_THRESHOLD, w.stride,
                                      w.causal, ss, bufs.scores, bufs.row_ptr, bufs.col_idx,
                                      bufs.nnz, bufs.score_ws, stream=stream)
                rec(1)
            rec(2)
            xa.xattn_sparse_attn(L.Q, L.K, L.V, bufs.row_ptr, bufs.col_idx, w.causal, sa, bufs.O,
                                 stream=stream)
        rec(3)
        if gather is not None:
            gather(bufs.O)
        rec(4)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(stream.device)
    if xa.xattn_get_device_error() != xa.XATTN_OK:
        raise RuntimeError("device error during warm-up")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    return step, evs, t0, t1


def stage_means(evs):
    st = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)  # noqa: E731
    return {"score": st(0, 1), "select": st(1, 2), "sparse_attn": st(2, 3), "gather": st(3, 4)}


def video_leg(xa, a, dev, stream):
    """The video-DiT-shaped layer (non-causal, frame x position structure) on the
    same GPU after the main workload: score + select + attend, and the build's own
    dense attention, with its own clock samples."""
    import torch
    w = sy.workload("video_dit_118k")
    # the sampler starts before the inputs are built: nvidia-smi needs a few hundred
    # ms before its first sample, longer than this leg's timed region
    clk = ClockSampler(dev.index or 0).__enter__()
    try:
        L = Layer(w, a.seed, dev)
    except BaseException:
        clk.__exit__(None, None, None)
        raise
    ss, sa = SCORE_SCALES[a.score_scale][1](w.stride, w.C), 1 / math.sqrt(w.C)
    steps, warmup = max(3, min(a.steps, 10)), max(3, min(a.warmup, 3))
    try:
        step, evs, t0, t1 = time_layer(xa, L, ss, sa, stream, steps, warmup)
        torch.cuda.synchronize(dev)
        clk.mark_start()
        t0.record(stream)
        for i in range(steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
        ms = t0.elapsed_time(t1) / steps
        stages = stage_means(evs)
        Od = torch.empty_like(L.Q)
        for _ in range(warmup):
            xa.xattn_dense_attn(L.Q, L.K, L.V, w.causal, sa, Od, stream=stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        d0.record(stream)
        for _ in range(steps):
            xa.xattn_dense_attn(L.Q, L.K, L.V, w.causal, sa, Od, stream=stream)
        d1.record(stream)
        torch.cuda.synchronize(dev)
    finally:
        clk.__exit__(None, None, None)
    if xa.xattn_get_device_error() != xa.XATTN_OK:
        raise RuntimeError("device error in the video leg")
    dense_ms = d0.elapsed_time(d1) / steps
    nnz = int(L.bufs.nnz.item())
    cand = w.B * w.Hq * w.nb * w.nb
    pk = peaks()
    kept_tflops = 4.0 * w.block ** 2 * w.C * nnz / (stages["sparse_attn"] * 1e-3) / 1e12
    score_tflops = 2.0 * w.M * w.M * w.C * w.Hq * w.B / w.stride / (stages["score"] * 1e-3) / 1e12
    out = {"workload": w.name, "config": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "seq_len": w.M,
                                          "C": w.C, "stride": w.stride, "causal": w.causal,
                                          "tau": w.tau},
           "steps": steps, "warmup": warmup, "ms_per_layer": ms, "density": nnz / cand,
           "nnz": nnz, "stages_ms": {k: v for k, v in stages.items() if k != "gather"},
           "dense_attn_ms": dense_ms, "speedup_vs_dense": dense_ms / ms,
           "kept_block_tflops": kept_tflops,
           "kept_block_frac_of_bf16_peak": kept_tflops / pk["bf16_sustained"],
           "score_tflops": score_tflops, "score_frac_of_bf16_peak": score_tflops / pk["bf16_sustained"],
           "clocks": clk.summary()}
    del L
    torch.cuda.empty_cache()
    return out


def main():
    a = parse()
    w = workload_of(a)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if a.impl == "reference":
        return reference_arm(a, w, rank, world)

    import torch
    import block_sparse_long_04_b200 as xa
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    split = world > 1 and a.split == "heads"
    if split and a.group_select:
        raise SystemExit("--group-select runs on one GPU or as replicas")

    def barrier():
        if dist is not None:
            dist.barrier()

    def max_over_ranks(x):
        return dist_max(x, dist, dev)

    # inputs: generated on the host (pinned), copied once; resident in HBM when timed.
    # Split: this rank's KV groups of the one layer; replicas: a layer of its own.
    if split:
        kv_lo, kv_hi, h_lo, h_hi = head_shard(w.Hq, w.Hkv, world, rank)
        L = Layer(w, a.seed, dev, heads=(kv_lo, kv_hi))
    else:
        L = Layer(w, a.seed + rank, dev)
    bufs = L.bufs
    stream = torch.cuda.current_stream(dev)
    ss = score_scale_of(a, w)
    sa = 1 / math.sqrt(w.C)
    G = w.Hq // w.Hkv
    O_full = None
    gather = None
    if split:
        O_full = torch.empty((world,) + tuple(bufs.O.shape), dtype=bufs.O.dtype, device=dev)
        gather = lambda O: gather_heads(O, dist, world, O_full)  # noqa: E731
    group = None
    if a.group_select:
        group = (torch.empty(w.B * w.Hkv * w.nb + 1, dtype=torch.int32, device=dev),
                 torch.empty(xa.max_kept(w.B, w.Hkv, w.nb, w.causal), dtype=torch.int32,
                             device=dev),
                 torch.empty(xa.xattn_select_group_workspace_size(w.B, w.Hq, w.Hkv, w.nb),
                             dtype=torch.uint8, device=dev))

    # unfused: score 2 (the sweep, then the block scores from its partials),
    # select 3 (count, scan, fill), attention 1;
    # fused: score with row cuts 1, scan 1, fill 1, attention 1
    # grouped: score 2, select 4 (count, group count, scan, group fill), attention 1
    launches_per_step = 7 if a.group_select else (4 if a.fused_select else 6)
    clk = ClockSampler(local).__enter__()      # started early: nvidia-smi is slow to start
    try:
        step, evs, t0, t1 = time_layer(xa, L, ss, sa, stream, a.steps, a.warmup,
                                       gather=gather, fused=a.fused_select, group=group)
        barrier()
        torch.cuda.synchronize(dev)
        clk.mark_start()
        t0.record(stream)
        for i in range(a.steps):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        clk.mark_end()
    finally:
        clk.__exit__(None, None, None)
    barrier()
    total_ms = max_over_ranks(t0.elapsed_time(t1))
    ms_step = total_ms / a.steps
    # ms per layer for the whole job: a split layer is one layer per step; replicas
    # process `world` layers per step
    value = total_ms / (a.steps * w.B) if split else job_ms_per_layer(total_ms, a.steps, world, w.B)
    stages = stage_means(evs)
    st_score, st_select, st_attn = stages["score"], stages["select"], stages["sparse_attn"]

    nnz_local = int(bufs.nnz.item()) * (G if a.group_select else 1)   # attended (head, block) pairs
    nnz = nnz_local
    if dist is not None and split:
        t = torch.tensor([nnz_local], dtype=torch.int64, device=dev)
        dist.all_reduce(t)
        nnz = int(t.item())
    if xa.xattn_get_device_error() != xa.XATTN_OK:
        raise RuntimeError("device error during the timed steps")
    b2, C = w.block ** 2, w.C
    kept_flops_local = 4.0 * b2 * C * nnz_local
    hq_layer = w.Hq
    cand = w.B * hq_layer * (w.nb * (w.nb + 1) // 2 if w.causal else w.nb * w.nb)
    cand_local = w.B * L.hq * (w.nb * (w.nb + 1) // 2 if w.causal else w.nb * w.nb)
    density = nnz / cand if split else nnz_local / cand_local
    dense_eq_flops = (2.0 if w.causal else 4.0) * w.M * w.M * C * w.Hq * w.B
    pk = peaks()
    attn_tflops = kept_flops_local / (st_attn * 1e-3) / 1e12
    roofline = {"kernel": "sparse_attn", "bound": "tensor", "achieved": attn_tflops,
                "peak": pk["bf16_sustained"], "unit": "TFLOP/s",
                "frac": attn_tflops / pk["bf16_sustained"],
                "peak_source": f"{pk['source']} bf16 sustained (kernel runs inside a long step)",
                "traffic": (None if (a.group_select or split)
                            else measured_traffic("attn_tc", w.name, w.stride)),
                "algorithmic": "4*b^2*C FLOP per kept (head, query block, key block), "
                               "diagonal blocks counted in full"}
    score_flops = (1.0 if w.causal else 2.0) * w.M * w.M * C * L.hq * w.B / w.stride
    extra = {
        "stages_ms": ({"score": st_score, "select": st_select, "sparse_attn": st_attn}
                      if not a.fused_select else
                      {"score_select": st_score + st_select, "sparse_attn": st_attn}),
        "density": density, "nnz": nnz,
        "kept_block_tflops": attn_tflops,
        "kept_block_frac_of_bf16_peak": attn_tflops / pk["bf16_sustained"],
        "dense_equivalent_tflops": dense_eq_flops / (value * 1e-3) / 1e12,
        # fused: the score stage also holds the row ranking, scan and fill
        "score_tflops": score_flops / (st_score * 1e-3) / 1e12,
        "score_frac_of_bf16_peak": score_flops / (st_score * 1e-3) / 1e12 / pk["bf16_sustained"],
        # selection (count + scan + fill): reads the candidate scores, writes
        # row_ptr and the kept lists; HBM-bound by design
        "select_gbs": (4.0 * (cand_local + nnz_local + w.B * L.hq * w.nb) / (st_select * 1e-3) / 1e9
                       if st_select > 0 else None),
        # secondary ceiling of the attention: b^2 exponentials per kept block
        "attn_exp2_per_s": w.block ** 2 * nnz_local / (st_attn * 1e-3),
    }
    if split:   # the all-gather is NCCL's kernel, not counted among ours
        extra["stages_ms"]["gather_o"] = stages["gather"]

    # dense baseline (the build's own dense attention), same (local) inputs
    if not a.no_dense:
        Od = torch.empty_like(L.Q)
        for _ in range(max(1, a.warmup)):
            xa.xattn_dense_attn(L.Q, L.K, L.V, w.causal, sa, Od, stream=stream)
        d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        d0.record(stream)
        for _ in range(a.steps):
            xa.xattn_dense_attn(L.Q, L.K, L.V, w.causal, sa, Od, stream=stream)
        d1.record(stream)
        torch.cuda.synchronize(dev)
        dense_ms = max_over_ranks(d0.elapsed_time(d1)) / a.steps
        extra["dense_attn_ms"] = dense_ms
        extra["dense_attn_tflops"] = (dense_eq_flops * L.hq / w.Hq) / (dense_ms * 1e-3) / 1e12
        extra["dense_attn_frac_of_bf16_peak"] = extra["dense_attn_tflops"] / pk["bf16_sustained"]
        extra["speedup_vs_dense"] = dense_ms / ms_step
        del Od

    # End to end through the public API with host buffers: every step copies its
    # Q/K/V (and tau) in from pinned host memory and its O back out. Two device
    # buffer sets and separate H2D / D2H streams let step i+1's input copy and
    # step i-1's output copy overlap step i's compute, as a serving pipeline does.
    # Split: each rank copies in its own heads; rank 0 copies the gathered O out.
    e2e = None
    if not a.no_e2e:
        O_out = O_full if split else None
        Oh = torch.empty(tuple(O_out.shape) if split else tuple(bufs.O.shape),
                         dtype=torch.bfloat16).pin_memory() if (not split or rank == 0) else None
        tau_h = torch.from_numpy(L.tau_np).pin_memory()
        sets = [(L.Q, L.K, L.V, L.tau, bufs)]
        sets.append((torch.empty_like(L.Q), torch.empty_like(L.K), torch.empty_like(L.V),
                     torch.empty_like(L.tau),
                     xa.Buffers.allocate(w.B, L.hq, w.M, w.C, w.stride, w.causal, device=dev)))
        h2d, d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev = lambda: torch.cuda.Event()  # noqa: E731
        h2d_done, comp_done, d2h_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
        outs = [O_full, torch.empty_like(O_full)] if split else None

        def e2e_steps(n):
            for i in range(n):
                sb = i % 2
                q, k, v, t, bb = sets[sb]
                if i >= 2:                       # compute of step i-2 no longer reads set sb
                    h2d.wait_event(comp_done[sb])
                with torch.cuda.stream(h2d):
                    q.copy_(L.Qh, non_blocking=True)
                    k.copy_(L.Kh, non_blocking=True)
                    v.copy_(L.Vh, non_blocking=True)
                    t.copy_(tau_h, non_blocking=True)
                h2d_done[sb].record(h2d)
                stream.wait_event(h2d_done[sb])
                if i >= 2:                       # O of step i-2 has been copied out
                    stream.wait_event(d2h_done[sb])
                xa.xattn_prefill(q, k, v, t, w.stride, w.causal, bb, score_scale=ss,
                                 stream=stream)
                src = bb.O
                if split:
                    src = gather_heads(bb.O, dist, world, outs[sb])
                comp_done[sb].record(stream)
                d2h.wait_event(comp_done[sb])
                if Oh is not None:
                    with torch.cuda.stream(d2h):
                        Oh.copy_(src, non_blocking=True)
                d2h_done[sb].record(d2h)

        e2e_steps(max(1, a.warmup))
        torch.cuda.synchronize(dev)
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        h2d.wait_event(e0)
        e2e_steps(a.steps)
        stream.wait_stream(d2h)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_total = max_over_ranks(e0.elapsed_time(e1))
        h2d_b = sum(t.numel() * t.element_size() for t in (L.Qh, L.Kh, L.Vh)) + L.tau_np.nbytes
        d2h_b = Oh.numel() * Oh.element_size() if Oh is not None else 0
        if split:   # whole job: every rank's inputs in, the gathered O out once
            h2d_b *= world
            d2h_b = w.B * w.Hq * w.M * w.C * 2
        e2e = {"value": (e2e_total / (a.steps * w.B) if split
                         else job_ms_per_layer(e2e_total, a.steps, world, w.B)),
               "unit": UNIT, "h2d_bytes_per_step": h2d_b, "d2h_bytes_per_step": d2h_b,
               "pipelined": "double-buffered device sets; H2D of step i+1 and D2H of step "
                            "i-1 overlap step i's compute"}
        del Oh, sets

    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        v, units, desc = oracle_sample(w, *L.views, L.tau_np, a.cpu_seconds, ss)
        cpu = {"value": v, "unit": UNIT, "cores": host_cores(), "blas_threads": blas_threads(),
               "kind": "oracle", "sample": desc}

    video = None
    if world == 1 and not a.no_video and w.name != "video_dit_118k":
        del L, bufs
        torch.cuda.empty_cache()
        video = video_leg(xa, a, dev, stream)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": False,
        "scaling": "strong" if split else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": dict(config_of(w, a, world), selection=(
            "GQA-shared union over each KV group (variant)" if a.group_select else
            "per head, fused with scoring" if a.fused_select else "per head")),
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches_per_step * a.steps, "clocks": clk.summary(), **extra,
    }
    if video is not None:
        line["video"] = video
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
