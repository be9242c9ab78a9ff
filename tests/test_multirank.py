"""Host logic of the multi-GPU bench path on CPU: two gloo ranks.

The path shards into independent layers (weak scaling, no data-path
collective): each rank draws its own seeded layer, runs the whole path on it
and only the timings meet, as a max over ranks.  Here the per-rank work is the
fp64 oracle on the small 2:4 workload, so the test needs no GPU.
"""
import json
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch.distributed as dist

    import bench
    import datagen
    import oracle

    os.environ.update(WORLD_SIZE=str(world), RANK=str(rank), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        w, r, local = bench.rank_env()
        layer = datagen.WORKLOADS["small_2of4"]
        X, W = bench.rank_inputs(layer, r)
        res = oracle.run_layer(X, W, layer.n, layer.m, eps=layer.eps)
        # a stand-in per-rank timing: rank r is slower by r ms
        ms = bench.max_over_ranks([1.0 + r, 10.0 - r], w)
        flops = 2.0 * layer.T * layer.R * layer.K
        rec = {"world": w, "rank": r, "local": local, "ms": ms,
               "value": bench.job_tflops(w, flops, ms[0]),
               "x_sum": int(X.astype(np.int64).sum()), "mask_sum": int(res["mask"].astype(np.int64).sum())}
        with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
            json.dump(rec, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    recs = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for r, rec in enumerate(recs):
        assert (rec["world"], rec["rank"], rec["local"]) == (world, r, r)
        assert rec["ms"] == [2.0, 10.0]              # max over ranks, element by element
    flops = 2.0 * 128 * 256 * 512
    assert recs[0]["value"] == pytest.approx(world * flops / 2e-3 / 1e12)
    # every rank works on its own seeded layer
    assert recs[0]["x_sum"] != recs[1]["x_sum"]


def test_single_rank_helpers():
    import bench
    import datagen
    assert bench.max_over_ranks([3.0, 1.5], 1) == [3.0, 1.5]
    assert bench.job_tflops(4, 2e12, 1000.0) == pytest.approx(8.0)
    layer = datagen.WORKLOADS["small_2of4"]
    X0, W0 = bench.rank_inputs(layer, 0)
    X0b, _ = datagen.layer_inputs(layer)
    assert np.array_equal(X0, X0b)                   # rank 0 = the workload's own seed


def _bench_lines(args, timeout=600):
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), *args], cwd=root,
                       capture_output=True, text=True, timeout=timeout)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return [json.loads(ln) for ln in lines]


def test_bench_launches_two_ranks_itself():
    # `bench.py --gpus 2` outside torchrun starts two ranks (torch.distributed.run,
    # rendezvous on 127.0.0.1); with the CPU stand-in for the per-rank work they
    # meet over gloo and rank 0 alone prints one line for the whole job
    lines = _bench_lines(["--gpus", "2", "--cpu-standin", "--workload", "small_2of4",
                          "--steps", "2", "--warmup", "3"])
    assert len(lines) == 1
    assert lines[0]["n_gpus"] == 2 and lines[0]["scaling"] == "weak"
    assert lines[0]["value"] > 0 and lines[0]["ms_per_step"] > 0


def test_reference_arm_under_two_ranks_prints_once():
    # the reference arm under two ranks: rank 0 runs the oracle, rank 1 exits
    lines = _bench_lines(["--impl", "reference", "--gpus", "2", "--workload", "small_2of4",
                          "--steps", "2", "--warmup", "3", "--cpu-seconds", "1"])
    assert len(lines) == 1
    assert lines[0]["impl"] == "reference" and lines[0]["n_gpus"] == 2
    assert lines[0]["cpu_baseline"]["kind"] == "oracle"
