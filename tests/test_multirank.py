"""The multi-rank host logic of bench.py on CPU (gloo, world size 2): the job time
is the max over ranks, the whole-job metric divides by every rank's layers, and
the reference arm runs on rank 0 only."""
import json
import math
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import synthetic as sy


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = 100.0 + 10.0 * rank          # rank 1 is the slow one
        total = bench.dist_max(local_ms, dist, torch.device("cpu"))
        out[rank] = (total, bench.job_ms_per_layer(total, steps=5, world=world, batch=1))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_max_over_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 110.0
    assert res[0][1] == pytest.approx(110.0 / (5 * 2))


def test_single_rank_helpers():
    assert bench.dist_max(3.5) == 3.5
    assert bench.job_ms_per_layer(50.0, steps=5, world=1, batch=2) == 5.0


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        seed, steps, warmup, cpu_seconds, gpus = 1, 1, 0, 0.1, 2
    w = sy.workload("tiny_1h_2k")
    assert bench.reference_arm(A, w, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("name,desc", [("sqrt_sc", "1/sqrt(stride*C)"), ("sqrt_c", "1/sqrt(C)"),
                                       ("s_sqrt_c", "1/(stride*sqrt(C))")])
def test_reference_arm_reports_the_score_scale(capsys, name, desc):
    """The scoring-softmax scale the method leaves open is a bench option; the
    reference line names the one it timed the oracle with."""
    class A:
        seed, steps, warmup, cpu_seconds, gpus, score_scale = 1, 1, 0, 0.05, 1, name
    w = sy.workload("tiny_1h_2k")
    assert bench.reference_arm(A, w, rank=0, world=1) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["config"]["score_scale"] == desc
    S, C = w.stride, w.C
    want = {"sqrt_sc": 1 / math.sqrt(S * C), "sqrt_c": 1 / math.sqrt(C),
            "s_sqrt_c": 1 / (S * math.sqrt(C))}[name]
    assert math.isclose(bench.score_scale_of(A, w), want)


def test_clock_sampler_keeps_only_the_timed_window():
    import bench
    clk = bench.ClockSampler(0)
    row = lambda mhz, cap: ["0", str(mhz), "1965", "700", "x", "Not Active", "Not Active",
                            "Not Active", cap]
    clk.rows = [(1.0, row(1965, "Not Active")),    # warm-up, before the window
                (2.0, row(1500, "Active")),
                (2.5, row(1520, "Active")),
                (9.0, row(1965, "Not Active"))]    # after the window
    clk.t_start, clk.t_end = 1.5, 2.6
    s = clk.summary()
    assert s["samples"] == 2 and s["sm_mhz"] == 1510.0 and s["reasons"] == ["sw_power_cap"]
    clk.t_start, clk.t_end = 3.0, 3.1
    assert clk.summary()["reasons"] == ["unsampled"]


# ------------------------------------------------ one layer split by KV-head group
@pytest.mark.parametrize("Hq,Hkv,world", [(32, 8, 1), (32, 8, 2), (32, 8, 4), (32, 8, 8),
                                          (24, 24, 3), (24, 24, 8), (4, 2, 2)])
def test_head_shard_covers_every_head_once(Hq, Hkv, world):
    seen = []
    for rank in range(world):
        kv_lo, kv_hi, h_lo, h_hi = bench.head_shard(Hq, Hkv, world, rank)
        assert kv_hi - kv_lo == Hkv // world and h_hi - h_lo == Hq // world
        # every query head of the shard reads a KV head of the same shard
        assert all(kv_lo <= h // (Hq // Hkv) < kv_hi for h in range(h_lo, h_hi))
        seen += list(range(h_lo, h_hi))
    assert seen == list(range(Hq))


def test_head_shard_rejects_uneven_groups():
    with pytest.raises(ValueError):
        bench.head_shard(32, 8, 3, 0)


def _split_worker(rank, world, port, out):
    """One rank of a layer split by KV-head group: generate only its own heads,
    compute their O with a CPU stand-in (the oracle, per head), all-gather O with
    bench.gather_heads; rank 0 returns the gathered layer."""
    import datetime
    import numpy as np
    import oracle as orc
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = sy.workload("llama8b_gqa_32k", M=256, C=16, Hq=4, Hkv=2, n_heavy=8)
        kv_lo, kv_hi, h_lo, h_hi = bench.head_shard(w.Hq, w.Hkv, world, rank)
        Qb, Kb, Vb = sy.layer_inputs(w, heads=(kv_lo, kv_hi))
        g = w.group
        o = np.zeros((w.B, h_hi - h_lo, w.M, w.C))
        for i in range(h_hi - h_lo):
            q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, i], Kb[0, i // g], Vb[0, i // g]))
            o[0, i] = orc.dense_attention(q, k, v, True, 0.25, block=128)[0]
        full = bench.gather_heads(torch.from_numpy(o), dist, world)
        if rank == 0:
            out["O"] = full.numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_head_split_gathers_the_single_rank_layer():
    """The gathered O of a two-rank split equals the one-rank layer, head by head,
    in layer order ([world, B, Hq/world, M, C] is O [B, Hq, M, C] for B = 1)."""
    import numpy as np
    import oracle as orc
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_split_worker, args=(2, port, out), nprocs=2, join=True)
        got = out["O"]
    w = sy.workload("llama8b_gqa_32k", M=256, C=16, Hq=4, Hkv=2, n_heavy=8)
    Qb, Kb, Vb = sy.layer_inputs(w)
    assert got.shape == (2, 1, 2, w.M, w.C)
    layer = got.reshape(1, 4, w.M, w.C)
    for h in range(4):
        q, k, v = (orc.bf16_to_f64(x) for x in (Qb[0, h], Kb[0, h // 2], Vb[0, h // 2]))
        np.testing.assert_array_equal(layer[0, h], orc.dense_attention(q, k, v, True, 0.25,
                                                                        block=128)[0])
