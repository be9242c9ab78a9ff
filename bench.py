#!/usr/bin/env python
"""Benchmark of the N:M-pruned linear layer hot path on B200.

One step = one pass of the whole path over one layer of synthetic input:
  a1 H = mean_t x^2            (nm_hessian_diag; for the ternary layer the
                                absmean quantisation, nm_ternary_quantize)
  a2 S = (H + eps) W^2 and
  a3 top-n per group + compress, in one pass (nm_score_prune_compress: the
                                scores stay in registers)
  a4 + a6 sliding-window pack and operand preparation in one pass
                               (nm_sparse_prepare_from_mask: window index
                                pairs formed from the mask as the operand's
                                metadata is written)
  a5+a7 sparse GEMM Y = X W_sparse^T on the lifted activations (nm_sparse_gemm:
               6:8 middle windows gathered, 4:6 / 8:10 X' lifted, before the GEMM)
  a8 own dense GEMM on the masked W (nm_dense_gemm), the speedup reference.

Prints ONE JSON line.  `value` is the sparse GEMM's effective TFLOP/s,
2*T*R*K / t_gemm summed over all ranks' layers; the other stages are timed in
the same steps and reported in `stages_ms`.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...   (the fp64 CPU oracle on a sample)

The default workload is the Llama-7B gate/up projection (11008 x 4096, 2:4)
at 8192 tokens.  With --gpus N > 1 outside torchrun, the script starts N ranks
itself (torch.distributed.run, one process per GPU); each rank prunes and
multiplies its own seeded layer and only the timings meet (max over ranks).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import datagen  # noqa: E402

DEFAULT_WORKLOAD = "llama7b_gate_T8192"
METRIC = "N:M sparse GEMM effective TFLOP/s, % of 2:4 TC peak, speedup vs own dense"
L2_FLUSH_BYTES = 256 << 20
CHECK_TOL = 1e-2   # max|Y - Yref| / max|Yref| of the GEMM outputs


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), "measured"
    except Exception:
        return 6650.0, 1590.0, "fallback"


def sustained_bf16():
    """Dense bf16 TFLOP/s held for seconds under the power cap (the
    denominator for a kernel timed inside a long loop), and its source."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1400.0, "fallback"


PAIR_MODE = {4: "PMODE_SP24", 6: "PMODE_SP24 on K'", 8: "PMODE_SP68T", 10: "PMODE_SP24 on K'"}


def recorded_traffic(workload: str):
    """DRAM bytes per launch of the sparse GEMM from the committed ncu summary
    profiles/gemm_wide_<workload>.md, if the kernel source is unchanged since."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"gemm_wide_{workload}.md")
    src = os.path.join(ROOT, "semi_structured_sparse_diag_b200", "csrc", "nm_gemm.cu")
    try:
        text = open(path).read()
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    fields = dict(ln.split(":", 1) for ln in text.splitlines()
                  if ln.startswith(("traffic_bytes_per_launch:", "source_sha256_16:")))
    if fields.get("source_sha256_16", "").strip() != sha:
        return None
    try:
        return int(fields["traffic_bytes_per_launch"].strip())
    except (KeyError, ValueError):
        return None


def workload_config(layer: datagen.Layer, l2_note: str):
    G = (layer.K + layer.m - 1) // layer.m
    KL = G * (layer.m // 2 - 1) * 4
    return {
        "workload": layer.name, "R": layer.R, "K": layer.K, "T": layer.T,
        "pattern": f"{layer.n}:{layer.m}", "lifted_K": KL, "score": layer.score,
        "ternary": layer.ternary, "eps": layer.eps, "x_outlier_channels": layer.x_outliers,
        "w_sigma": layer.w_sigma, "seed": layer.seed, "l2": l2_note,
    }


# --------------------------------------------------------------------------
# clocks sampled with nvidia-smi during the timed region
# --------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            return None
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm_, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(nm_)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------------------
# multi-rank host logic (one process per GPU; weak scaling, no data-path
# collective: each rank prunes and multiplies its own seeded layer)
# --------------------------------------------------------------------------
def rank_env():
    """(world size, rank, local rank) from the torchrun environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_inputs(layer: datagen.Layer, rank: int):
    """The seeded (X, W) bf16 bit patterns of this rank's layer."""
    return datagen.layer_inputs(layer, seed=layer.seed + rank)


def max_over_ranks(values, world: int, device=None):
    """Each rank's timings -> the slowest rank's, element by element."""
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput: all ranks' work over the slowest rank's time."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def _free_port() -> int:
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch_ranks(nranks: int, argv, timeout_s: float = 1800.0) -> int:
    """Start `nranks` copies of this script under torch.distributed.run (one
    process per GPU, rendezvous on 127.0.0.1) with the same arguments; rank 0
    prints the JSON line.  Returns the launcher's exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nranks}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.abspath(__file__), *argv]
    env = dict(os.environ)
    env.setdefault("OMP_NUM_THREADS", "1")
    try:
        return subprocess.run(cmd, env=env, timeout=timeout_s).returncode
    except subprocess.TimeoutExpired:
        print(json.dumps({"error": f"ranks did not finish within {timeout_s:.0f} s"}), file=sys.stderr)
        return 124


def run_cpu_standin(args):
    """Host logic of the multi-rank run without a GPU: every rank runs the
    oracle's whole path on its own seeded layer (gloo process group), the
    step times meet as a max over ranks, rank 0 prints one line.  It exercises
    the launcher, the rank environment and the aggregation; its numbers are CPU
    numbers and say nothing about the GPU path."""
    import datetime

    import torch.distributed as dist

    import oracle
    world, rank, _local = rank_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = rank_inputs(layer, rank)
    secs = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        res = oracle.run_layer(X_h, W_h, layer.n, layer.m, eps=layer.eps, score=layer.score,
                               ternary_values=layer.ternary)
        oracle.gemm_masked(X_h, res["mask"], res["V"], layer.m, rows=np.arange(min(8, layer.T)))
        if i >= args.warmup:
            secs.append(time.perf_counter() - t0)
    if world > 1:
        dist.barrier()
    ms = max_over_ranks([1e3 * sum(secs) / len(secs)], world)[0]
    flops = 2.0 * min(8, layer.T) * layer.R * layer.K
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps({"metric": "cpu stand-in of the multi-rank step (host logic only)",
                          "value": round(job_tflops(world, flops, ms), 9), "unit": "TFLOP/s",
                          "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
                          "standin": "cpu", "config": {"workload": layer.name}}), flush=True)


# --------------------------------------------------------------------------
# our arm
# --------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    import semi_structured_sparse_diag_b200 as nm

    world, rank, local = rank_env()
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but {world} ranks were started")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = rank_inputs(layer, rank)
    R, K, T, n, m = layer.R, layer.K, layer.T, layer.n, layer.m
    lib = nm.load()
    stream = torch.cuda.current_stream()

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)

    X = dev_bf16(X_h)
    W = dev_bf16(W_h)
    G = (K + m - 1) // m
    KL = G * (m // 2 - 1) * 4
    KLpad = (KL + 127) // 128 * 128
    # persistent buffers (allocated once, outside the timed region)
    H = torch.empty(K, dtype=torch.float64, device=dev)
    ws_needed = lib.nm_hessian_workspace_bytes(T, K)
    ws = torch.empty(max(16, ws_needed), dtype=torch.uint8, device=dev)
    mask = torch.empty((R, (G * m + 31) // 32), dtype=torch.int32, device=dev)
    vals = torch.empty((R, G * n), dtype=torch.bfloat16, device=dev)
    meta = torch.empty((R, (G + 1) // 2), dtype=torch.uint8, device=dev) if m == 4 else None
    packed = torch.empty(lib.nm_sparse_prepare_bytes(R, K, m), dtype=torch.uint8, device=dev)
    gws_bytes = lib.nm_sparse_gemm_workspace_bytes(T, K, m)
    gws = torch.empty(max(1, gws_bytes), dtype=torch.uint8, device=dev)
    dws_bytes = lib.nm_dense_gemm_workspace_bytes(T, K, R)
    dws = torch.empty(max(1, dws_bytes), dtype=torch.uint8, device=dev)
    ldy = (R + 7) // 8 * 8
    Y = torch.empty((T, ldy), dtype=torch.bfloat16, device=dev)
    Yd = torch.empty((T, ldy), dtype=torch.bfloat16, device=dev)
    V = W
    Wq = gamma = tws = None
    if layer.ternary:
        Wq = torch.empty((R, K), dtype=torch.bfloat16, device=dev)
        gamma = torch.empty(1, dtype=torch.float64, device=dev)
        tws = torch.empty(lib.nm_ternary_workspace_bytes(R), dtype=torch.uint8, device=dev)
        V = Wq
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    s = stream.cuda_stream

    def chk(st, what):
        if st != 0:
            raise nm.NMError(f"{what}: {lib.nm_status_string(st).decode()}")

    # a1 (or the ternary quantisation of C4-style layers), a2+a3 fused, a4, a6,
    # a5+a7, a8
    stage_names = ["hessian_or_ternary", "score_prune", "pack_prepare", "sparse_gemm", "dense_gemm"]
    launches_per_step = 0

    def step(ev=None, Xs=X, Ws=W):
        nonlocal launches_per_step
        cnt = 0
        Vs = Wq if layer.ternary else Ws
        if ev is not None:
            ev[0].record(stream)
        if layer.ternary:
            chk(lib.nm_ternary_quantize(Ws.data_ptr(), R, K, K, Wq.data_ptr(), gamma.data_ptr(),
                                        tws.data_ptr(), tws.numel(), s), "ternary")
            cnt += 3
        if layer.score == "hessian":
            chk(lib.nm_hessian_diag(Xs.data_ptr(), T, K, K, H.data_ptr(), ws.data_ptr(), ws.numel(), s),
                "hessian")
            cnt += lib.nm_hessian_launch_count(T, K)  # H (+ a finish kernel where clusters do not fit)
        if ev is not None:
            ev[1].record(stream)
        # a2 + a3 in one pass: scores formed in registers, never written
        chk(lib.nm_score_prune_compress(H.data_ptr() if layer.score == "hessian" else None, layer.eps,
                                        Ws.data_ptr(), K, Vs.data_ptr(), K, R, K, n, m, mask.data_ptr(),
                                        vals.data_ptr(), meta.data_ptr() if meta is not None else None, s),
            "score_prune")
        cnt += 1
        if ev is not None:
            ev[2].record(stream)
        # a4 + a6: for (2N-2):2N the window index pairs are formed from the mask
        # as the operand's metadata is written (the window metadata is never
        # stored); 2:4 has no window pack and copies the prune's meta24
        if m == 4:
            chk(lib.nm_sparse_prepare(vals.data_ptr(), meta.data_ptr(), R, K, m, packed.data_ptr(),
                                      packed.numel(), s), "pack_prepare")
        else:
            chk(lib.nm_sparse_prepare_from_mask(vals.data_ptr(), mask.data_ptr(), R, K, m, packed.data_ptr(),
                                                packed.numel(), s), "pack_prepare")
        cnt += 2
        if ev is not None:
            ev[3].record(stream)
        chk(lib.nm_sparse_gemm(Xs.data_ptr(), T, K, K, packed.data_ptr(), R, m, Y.data_ptr(), ldy,
                               gws.data_ptr(), gws_bytes, s), "sparse_gemm")
        cnt += 1 if m == 4 else 2  # + the middle-window gather (6:8) or the lift (4:6, 8:10)
        if ev is not None:
            ev[4].record(stream)
        chk(lib.nm_dense_gemm(Xs.data_ptr(), T, K, K, Wdense.data_ptr(), R, K, Yd.data_ptr(), ldy,
                              dws.data_ptr(), dws_bytes, s), "dense_gemm")
        cnt += 1
        if ev is not None:
            ev[5].record(stream)
        launches_per_step = cnt

    # comparator input: the masked weights as a dense matrix (set-up, not timed)
    Wdense = torch.empty_like(W)
    step_pre = True
    if step_pre:
        # one untimed pass produces the mask; densify it for the dense GEMM
        Wdense.copy_(W)
        step()
        torch.cuda.synchronize()
        nm.check_device_error()
        bits = ((mask.view(torch.int32).unsqueeze(-1) >> torch.arange(32, device=dev, dtype=torch.int32)) & 1)
        bits = bits.reshape(R, -1)[:, :K].bool()
        Wdense = torch.where(bits, V, torch.zeros_like(V)).contiguous()

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    nm.check_device_error()

    def barrier():
        if world > 1:
            dist.barrier()

    clocks = ClockSampler(local) if rank == 0 else None
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stage_names) + 1)]
           for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()  # L2 flush between timed steps (outside the events)
        step(evs[i])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop() if clocks else None
    nm.check_device_error()

    stage_ms = {k: 0.0 for k in stage_names}
    step_ms = 0.0
    for e in evs:
        for j, k in enumerate(stage_names):
            stage_ms[k] += e[j].elapsed_time(e[j + 1])
        step_ms += e[0].elapsed_time(e[-1])
    stage_ms = {k: v / args.steps for k, v in stage_ms.items()}
    step_ms /= args.steps
    gemm_ms = stage_ms["sparse_gemm"]
    dense_ms = stage_ms["dense_gemm"]
    step_ms, gemm_ms, dense_ms = max_over_ranks([step_ms, gemm_ms, dense_ms], world, dev)

    # ------------------------------------------------ end-to-end through the C ABI
    Xh = torch.from_numpy(X_h.view(np.int16)).pin_memory()
    Wh = torch.from_numpy(W_h.view(np.int16)).pin_memory()
    Yh = torch.empty((T, ldy), dtype=torch.int16).pin_memory()
    Xe = torch.empty_like(X)
    We = torch.empty_like(W)
    e2e_steps = max(1, min(args.steps, 5))
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_ms = 0.0
    for _ in range(e2e_steps):
        flush.zero_()
        e0.record(stream)
        Xe.view(torch.int16).copy_(Xh, non_blocking=True)
        We.view(torch.int16).copy_(Wh, non_blocking=True)
        step(None, Xe, We)
        Yh.copy_(Y.view(torch.int16), non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms += e0.elapsed_time(e1)
    e2e_ms /= e2e_steps
    e2e_ms = max_over_ranks([e2e_ms], world, dev)[0]
    nm.check_device_error()

    # output check: the sparse product against the own dense GEMM of the same
    # masked weights (both fp32 accumulations rounded to bf16)
    Ys, Yr = Y[:, :R].float(), Yd[:, :R].float()
    dense_err = ((Ys - Yr).abs().max() / Yr.abs().max().clamp_min(1e-30)).item()
    check = {"y_vs_own_dense": dense_err, "tol": CHECK_TOL}
    # a failure on any rank fails the job (same collective on every rank)
    ok = max_over_ranks([0.0 if dense_err <= CHECK_TOL else 1.0], world, dev)[0] == 0.0

    hbm, bf16_tf, peak_src = peaks()
    # the timed region is a second or more of back-to-back steps: the sustained
    # dense rate is the denominator; 2:4 sparse bf16 = 2 x dense (nominal 4.5 / 2.25)
    bf16_sus, sus_src = sustained_bf16()
    sparse_peak = 2.0 * bf16_sus
    burst_peak = 2.0 * bf16_tf
    flops_eff = 2.0 * T * R * K                 # dense-equivalent of the original layer
    flops_lift = 2.0 * T * R * KLpad            # dense-equivalent of the lifted 2:4 problem
    value = job_tflops(world, flops_eff, gemm_ms)
    achieved = flops_lift / (gemm_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(step_ms, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": workload_config(layer, "flushed between steps (256 MiB write)"),
        "pct_of_2to4_peak": round(100.0 * achieved / sparse_peak, 2),
        "pct_of_2to4_burst_peak": round(100.0 * achieved / burst_peak, 2),
        "speedup_vs_own_dense": round(dense_ms / gemm_ms, 4),
        "speedup_bound": round(K / (KL / 2), 4),
        "stages_ms": {k: round(v, 4) for k, v in stage_ms.items()},
        "roofline": {
            "kernel": f"k_gemm_wide<{PAIR_MODE[m]}>",
            "bound": "tensor",
            "achieved": round(achieved, 2),
            "peak": round(sparse_peak, 1),
            "peak_source": (f"2 x {sus_src} dense bf16 sustained ({bf16_sus} TFLOP/s; the timed region is "
                            f"{args.steps} back-to-back steps)"),
            "unit": "TFLOP/s",
            "frac": round(achieved / sparse_peak, 4),
            "frac_of_burst": round(achieved / burst_peak, 4),
            "burst_peak": round(burst_peak, 1),
            "traffic": recorded_traffic(layer.name),
            "traffic_source": f"profiles/gemm_wide_{layer.name}.md (ncu dram read+write per launch)",
            "per_unit": "2*R*K'pad flops per token; units per launch = T tokens",
        },
        "e2e": {
            "value": round(job_tflops(world, flops_eff, e2e_ms), 3),
            "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 4),
            "h2d_bytes_per_step": int(X_h.nbytes + W_h.nbytes),
            "d2h_bytes_per_step": int(T * ldy * 2),
            "note": "whole step (all stages) with pinned H2D of X, W and D2H of Y in the timed region",
        },
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    if clk:
        # SM cycles of the sparse GEMM stage at the median clock seen under load
        clk["sparse_gemm_kcycles_at_median_clock"] = round(gemm_ms * clk["sm_mhz"], 1)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb, Y64, (tok, rows_w) = cpu_baseline(layer, X_h, W_h, budget_s=args.cpu_seconds)
        line["cpu_baseline"] = cb
        # the same sampled outputs from the GPU against the oracle's fp64 product
        Yg = Y[:tok, :rows_w].float().double().cpu().numpy()
        den = float(np.max(np.abs(Y64))) or 1.0
        check["y_vs_oracle_sample"] = float(np.max(np.abs(Yg - Y64)) / den)
        check["oracle_sample"] = f"tokens 0..{tok - 1} x weight rows 0..{rows_w - 1}"
        ok = ok and check["y_vs_oracle_sample"] <= CHECK_TOL
    check["ok"] = bool(ok)
    line["check"] = check
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if not ok:
        raise SystemExit("bench.py: the sparse GEMM output failed its check (see the line's \"check\")")


# --------------------------------------------------------------------------
# the oracle on a bounded sample (CPU baseline and the reference arm)
# --------------------------------------------------------------------------
def oracle_sample_step(layer, X_h, W_h, rows_w: int, tok: int):
    """One oracle step on a sample: H on all of X (for a ternary layer, gamma
    over all of W); S/prune/pack on `rows_w` weight rows; fp64 GEMM of `tok`
    tokens against those rows.  Returns (seconds, sample flops
    (dense-equivalent), stage seconds, the sampled fp64 outputs [tok x rows_w])."""
    import oracle
    t0 = time.perf_counter()
    Wsub = np.ascontiguousarray(W_h[:rows_w])
    V = Wsub
    if layer.ternary:
        _, Vall = oracle.ternary(W_h)    # gamma is a mean over the whole tensor
        V = np.ascontiguousarray(Vall[:rows_w])
    if layer.score == "hessian":
        H = oracle.hessian_diag(X_h)
        S = oracle.score_hessian(H, Wsub, layer.eps)
    else:
        S = oracle.score_magnitude(Wsub)
    t1 = time.perf_counter()
    mask, vals, meta = oracle.prune(S, V, layer.n, layer.m)
    if layer.m > 4:
        oracle.slide_pack(mask, layer.K, layer.m)
    t2 = time.perf_counter()
    rows = np.arange(tok, dtype=np.int64)
    Y64 = oracle.gemm_masked(X_h, mask, V, layer.m, rows=rows)
    t3 = time.perf_counter()
    return t3 - t0, 2.0 * tok * rows_w * layer.K, {"score": t1 - t0, "prune_pack": t2 - t1,
                                                   "gemm": t3 - t2}, Y64


def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def _sample_size(layer, budget_s):
    # ~1 GFLOP/s-per-core class fp64 loops: size the GEMM sample to the budget
    rate = 0.25e9 * _cores()   # fp64 multiply-adds per second, roughly
    rows_w = max(8, min(layer.R, 1024, int(budget_s * rate / (2.0 * layer.K))))
    tok = max(1, min(layer.T, int(budget_s * rate / (2.0 * rows_w * layer.K))))
    return rows_w, tok


def cpu_baseline(layer, X_h, W_h, budget_s=10.0):
    rows_w, tok = _sample_size(layer, budget_s)
    sec, flops, stages, Y64 = oracle_sample_step(layer, X_h, W_h, rows_w, tok)
    return {
        "value": round(flops / stages["gemm"] / 1e12, 6),
        "unit": "TFLOP/s",
        "cores": _cores(),
        "kind": "oracle",
        "sample": (f"{layer.name}: H over all {layer.T} tokens, score+prune+pack on {rows_w} of "
                   f"{layer.R} weight rows, fp64 GEMM of {tok} tokens x {rows_w} rows x K={layer.K}; "
                   f"value = sample GEMM flops / oracle GEMM seconds; step {sec:.2f} s"),
        "stage_seconds": {k: round(v, 3) for k, v in stages.items()},
    }, Y64, (tok, rows_w)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = datagen.layer_inputs(layer)
    # per-step sample sized so that the whole run stays within a few minutes
    rows_w, tok = _sample_size(layer, min(args.cpu_seconds / 2, 90.0 / (args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample_step(layer, X_h, W_h, min(rows_w, 128), 1)
    secs, gsecs, flops = [], [], 0.0
    for _ in range(args.steps):
        s, f, st, _ = oracle_sample_step(layer, X_h, W_h, rows_w, tok)
        secs.append(s)
        gsecs.append(st["gemm"])
        flops = f
    value = flops / (sum(gsecs) / len(gsecs)) / 1e12
    sample = (f"{layer.name}: per step H over all {layer.T} tokens, score+prune+pack on {rows_w} of "
              f"{layer.R} weight rows, fp64 GEMM of {tok} tokens x {rows_w} rows x K={layer.K}")
    line = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * sum(secs) / len(secs), 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(layer, "host memory (CPU oracle)"),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": _cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_prep(args):
    """The HBM-bound prep kernels of one workload's W, each launched alone and
    timed with CUDA events (L2 flushed): score, prune and fused score + prune
    (2:4, 6:8 and the workload's pattern), ternary quantisation.  One JSON
    line.  With --reps 0 every kernel is launched once (the ncu driver)."""
    import torch

    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    dev = torch.device("cuda", 0)
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = datagen.layer_inputs(layer)
    R, K = layer.R, layer.K
    W = torch.from_numpy(W_h.view(np.int16)).to(dev).view(torch.bfloat16)
    X = torch.from_numpy(X_h.view(np.int16)).to(dev).view(torch.bfloat16)
    H = nm.hessian_diag(X)
    S = torch.empty((R, K), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream().cuda_stream

    def chk(st, what):
        if st != 0:
            raise nm.NMError(f"{what}: {lib.nm_status_string(st).decode()}")

    def timed(fn):
        ts = []
        for i in range(args.reps + 1):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i:
                ts.append(e0.elapsed_time(e1) * 1000)
        return sorted(ts)[len(ts) // 2] if ts else float("nan")

    out = {"prep": layer.name, "R": R, "K": K, "us": {}, "GBs": {}}

    def rec(name, us, nbytes):
        if us == us:  # not NaN (--reps 0: launches only, for ncu)
            out["us"][name] = round(us, 1)
            out["GBs"][name] = round(nbytes / us / 1e3, 0)

    E = R * K
    T = X.shape[0]
    Hb = torch.empty(K, dtype=torch.float64, device=dev)
    hws = torch.empty(max(lib.nm_hessian_workspace_bytes(T, K), 16), dtype=torch.uint8, device=dev)
    rec("hessian_diag", timed(lambda: chk(lib.nm_hessian_diag(X.data_ptr(), T, K, K, Hb.data_ptr(), hws.data_ptr(),
                                                             hws.numel(), s), "hessian")), 2 * T * K + 8 * K)
    # the same reduction on the first 2048 tokens (the 6:8 layer's calibration size)
    T2 = min(T, 2048)
    rec(f"hessian_diag_T{T2}", timed(lambda: chk(lib.nm_hessian_diag(X.data_ptr(), T2, K, K, Hb.data_ptr(),
                                                                     hws.data_ptr(), hws.numel(), s), "hessian")),
        2 * T2 * K + 8 * K)
    # Hutchinson with 16 sign vectors: X is read twice (u = X z, then x * p)
    zb = torch.from_numpy(datagen.rademacher_bits(16, K, seed=0).view(np.int32)).to(dev)
    uws = torch.empty(lib.nm_hutchinson_workspace_bytes(T, K, 16), dtype=torch.uint8, device=dev)
    rec("hutchinson_S16", timed(lambda: chk(lib.nm_hutchinson_diag(
        X.data_ptr(), T, K, K, zb.data_ptr(), 16, Hb.data_ptr(), uws.data_ptr(), uws.numel(), s), "hutchinson")),
        4 * T * K + 8 * K)
    rec("score", timed(lambda: chk(lib.nm_score_from_hessian(H.data_ptr(), layer.eps, W.data_ptr(), R, K, K,
                                                             S.data_ptr(), s), "score")), 6 * E)
    for m in sorted({4, 8, layer.m}):
        n = m - 2
        G = (K + m - 1) // m
        mask = torch.empty((R, (G * m + 31) // 32), dtype=torch.int32, device=dev)
        vals = torch.empty((R, G * n), dtype=torch.bfloat16, device=dev)
        meta = torch.empty((R, (G + 1) // 2), dtype=torch.uint8, device=dev)
        mp = meta.data_ptr() if m == 4 else None
        wr = R * G * n * 2 + mask.numel() * 4 + (meta.numel() if m == 4 else 0)
        rec(f"prune_{n}of{m}", timed(lambda: chk(lib.nm_prune_compress(
            S.data_ptr(), K, W.data_ptr(), K, R, K, n, m, mask.data_ptr(), vals.data_ptr(), mp, s), "prune")),
            6 * E + wr)
        rec(f"score_prune_{n}of{m}", timed(lambda: chk(lib.nm_score_prune_compress(
            H.data_ptr(), layer.eps, W.data_ptr(), K, W.data_ptr(), K, R, K, n, m, mask.data_ptr(),
            vals.data_ptr(), mp, s), "score_prune")), 2 * E + wr)
        # a4 and a6 (the window pack, the operand preparation from the window
        # metadata) and the two in one pass from the mask
        pbytes = lib.nm_sparse_prepare_bytes(R, K, m)
        packed = torch.empty(pbytes, dtype=torch.uint8, device=dev)
        chk(lib.nm_score_prune_compress(H.data_ptr(), layer.eps, W.data_ptr(), K, W.data_ptr(), K, R, K, n, m,
                                        mask.data_ptr(), vals.data_ptr(), mp, s), "score_prune")
        nwb = (G * (m // 2 - 1) + 1) // 2
        wmeta = meta if m == 4 else torch.empty((R, nwb), dtype=torch.uint8, device=dev)
        if m > 4:
            rec(f"slide_pack_{n}of{m}", timed(lambda: chk(lib.slide_pack(mask.data_ptr(), R, K, m, wmeta.data_ptr(),
                                                                         s), "slide_pack")),
                mask.numel() * 4 + wmeta.numel())
        rec(f"prepare_{n}of{m}", timed(lambda: chk(lib.nm_sparse_prepare(vals.data_ptr(), wmeta.data_ptr(), R, K, m,
                                                                          packed.data_ptr(), pbytes, s), "prepare")),
            vals.numel() * 2 + wmeta.numel() + pbytes)
        rec(f"prepare_from_mask_{n}of{m}", timed(lambda: chk(lib.nm_sparse_prepare_from_mask(
            vals.data_ptr(), mask.data_ptr(), R, K, m, packed.data_ptr(), pbytes, s), "prepare_from_mask")),
            vals.numel() * 2 + mask.numel() * 4 + pbytes)
    Wq = torch.empty((R, K), dtype=torch.bfloat16, device=dev)
    gamma = torch.empty(1, dtype=torch.float64, device=dev)
    tws = torch.empty(lib.nm_ternary_workspace_bytes(R), dtype=torch.uint8, device=dev)
    rec("ternary_quantize", timed(lambda: chk(lib.nm_ternary_quantize(
        W.data_ptr(), R, K, K, Wq.data_ptr(), gamma.data_ptr(), tws.data_ptr(), tws.numel(), s), "ternary")),
        6 * E)
    nm.check_device_error()
    print(json.dumps(out), flush=True)


def run_f8(args):
    """The FP8 form of the layer (SlideSparse sec. 2B/2C): the fused per-token
    quantise + lift kernel and the kind::f8f6f4 sparse GEMM, each launched
    alone and timed with CUDA events (L2 flushed), next to the bf16 sparse
    GEMM on the same layer.  One JSON line."""
    import torch

    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    dev = torch.device("cuda", 0)
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = datagen.layer_inputs(layer)
    R, K, m = layer.R, layer.K, layer.m
    T = X_h.shape[0]
    W = torch.from_numpy(W_h.view(np.int16)).to(dev).view(torch.bfloat16)
    X = torch.from_numpy(X_h.view(np.int16)).to(dev).view(torch.bfloat16)
    H = nm.hessian_diag(X)
    mask, vals, meta24 = nm.score_prune_compress(H, W, m - 2, m, eps=layer.eps)
    wmeta = meta24 if m == 4 else nm.slide_pack(mask, K, m)
    packed8 = nm.sparse_prepare_f8(vals, wmeta, R, K, m)
    packed16 = nm.sparse_prepare(vals, wmeta, R, K, m)
    Xq, xs = nm.quant_lift_f8(X, m)
    Y8 = nm.sparse_gemm_f8(Xq, xs, packed8, R, K, m)
    Y16 = nm.sparse_gemm(X, packed16, R, m)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    KLf = lib.nm_lifted_cols_f8(K, m)

    def timed(fn):
        ts = []
        for i in range(args.reps + 1):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            if i:
                ts.append(e0.elapsed_time(e1) * 1000)
        return sorted(ts)[len(ts) // 2] if ts else float("nan")

    def chk(st, what):
        if st != 0:
            raise nm.NMError(f"{what}: {lib.nm_status_string(st).decode()}")

    q_us = timed(lambda: chk(lib.nm_quant_lift_f8(X.data_ptr(), T, K, K, m, Xq.data_ptr(), Xq.shape[1],
                                                  xs.data_ptr(), s), "quant_lift_f8"))
    g8_us = timed(lambda: chk(lib.nm_sparse_gemm_f8(Xq.data_ptr(), T, K, Xq.shape[1], xs.data_ptr(),
                                                    packed8.data_ptr(), R, m, Y8.data_ptr(), Y8.stride(0), s),
                              "sparse_gemm_f8"))
    g16_us = timed(lambda: nm.sparse_gemm(X, packed16, R, m, Y=Y16))
    nm.check_device_error()
    hbm, bf16_peak, _src = peaks()
    f8_sparse_peak = 2 * 2 * bf16_peak   # fp8 dense = 2 x bf16 dense (nominal ratio); 2:4 doubles it
    flops8 = 2.0 * T * R * KLf            # dense-equivalent on the lifted K'
    out = {"f8": layer.name, "R": R, "K": K, "T": T, "pattern": f"{m - 2}:{m}", "lifted_K_f8": KLf,
           "us": {"quant_lift_f8": round(q_us, 1), "sparse_gemm_f8": round(g8_us, 1),
                  "sparse_gemm_bf16": round(g16_us, 1)},
           "quant_lift_f8_GBs": round((2 * T * K + T * KLf + 4 * T) / q_us / 1e3, 0),
           "quant_lift_f8_pct_hbm": round(100 * (2 * T * K + T * KLf + 4 * T) / q_us / 1e3 / hbm, 1),
           "gemm_f8_TFLOPs_on_lifted": round(flops8 / g8_us / 1e6, 1),
           "gemm_f8_pct_of_f8_2to4_peak": round(100 * flops8 / g8_us / 1e6 / f8_sparse_peak, 1),
           "f8_2to4_peak_TFLOPs": f8_sparse_peak, "peak_source": "2 x 2 x measured dense bf16 burst",
           "effective_TFLOPs_on_K": {"f8": round(2.0 * T * R * K / g8_us / 1e6, 1),
                                     "bf16": round(2.0 * T * R * K / g16_us / 1e6, 1)}}
    print(json.dumps(out), flush=True)


def run_probe(args):
    """Tensor-pipe and HBM probes (calibration, not the bench line)."""
    import torch

    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    dev = torch.device("cuda", 0)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {"probe": "tcgen05 MMA-only loop and HBM copy", "sms": sms, "mma": [], "copy": None}
    cyc = torch.zeros(sms, dtype=torch.int64, device=dev)
    ns = torch.zeros(sms, dtype=torch.int64, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    iters = 4096
    clocks = ClockSampler(0)
    for sparse in (0, 1):
        for n in (128, 192, 256):
            for rep in range(2):
                st = lib.nm_probe_mma(sparse, n, sms, iters, cyc.data_ptr(), ns.data_ptr(), s)
                if st != 0:
                    raise nm.NMError(lib.nm_status_string(st).decode())
                torch.cuda.synchronize()
            nm.check_device_error()
            kk = 32 if sparse else 16
            flops_cta = 4.0 * iters * 2 * 128 * n * kk  # dense-equivalent (logical K)
            t = ns.double().max().item() * 1e-9
            c = cyc.double().median().item()
            out["mma"].append({"sparse": sparse, "N": n, "tflops_dense_equiv": round(sms * flops_cta / t / 1e12, 1),
                               "flop_per_clk_per_sm": round(flops_cta / c, 1),
                               "clk_per_instr": round(c / (4 * iters), 2)})
    nbytes = 2 << 30
    a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    b = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    best = 0.0
    for _ in range(5):
        e0.record()
        st = lib.nm_probe_copy(a.data_ptr(), b.data_ptr(), nbytes, sms * 8, s)
        e1.record()
        torch.cuda.synchronize()
        best = max(best, 2 * nbytes / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    out["copy"] = {"GB_per_s_read_plus_write": round(best, 1), "bytes": nbytes}
    out["clocks"] = clocks.stop()
    print(json.dumps(out), flush=True)


def run_ablation(args):
    """Design-choice evidence: the sparse GEMM variants on one workload, each timed
    alone (median of 10 after 3 warm-ups, L2 flushed before each run)."""
    import torch

    import semi_structured_sparse_diag_b200 as nm
    lib = nm.load()
    dev = torch.device("cuda", 0)
    layer = datagen.WORKLOADS[args.workload]
    X_h, W_h = datagen.layer_inputs(layer)
    R, K, T, n, m = layer.R, layer.K, layer.T, layer.n, layer.m
    X = torch.from_numpy(X_h.view(np.int16)).to(dev).view(torch.bfloat16)
    W = torch.from_numpy(W_h.view(np.int16)).to(dev).view(torch.bfloat16)
    _, S = nm.score(X, W, eps=layer.eps)
    mask, vals, meta = nm.prune_compress(S, W, n, m)
    wm = meta if m == 4 else nm.slide_pack(mask, K, m)
    packed = nm.sparse_prepare(vals, wm, R, K, m)
    bits = ((mask.unsqueeze(-1) >> torch.arange(32, device=dev, dtype=torch.int32)) & 1)
    Wd = torch.where(bits.reshape(R, -1)[:, :K].bool(), W, torch.zeros_like(W)).contiguous()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream().cuda_stream
    Y = torch.empty((T, (R + 7) // 8 * 8), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(1, lib.nm_sparse_gemm_workspace_bytes(T, K, m)), dtype=torch.uint8, device=dev)

    def timed(fn):
        ts = []
        for i in range(13):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            st = fn()
            e1.record()
            torch.cuda.synchronize()
            if st != 0:
                raise nm.NMError(lib.nm_status_string(st).decode())
            if i >= 3:
                ts.append(e0.elapsed_time(e1))
        nm.check_device_error()
        return sorted(ts)[len(ts) // 2]

    ldy = Y.stride(0)
    dws = torch.empty(lib.nm_dense_gemm_workspace_bytes(T, K, R), dtype=torch.uint8, device=dev)
    sparse_call = lambda: lib.nm_sparse_gemm(X.data_ptr(), T, K, K, packed.data_ptr(), R, m, Y.data_ptr(),
                                             ldy, ws.data_ptr(), ws.numel(), s)
    dense_call = lambda: lib.nm_dense_gemm(X.data_ptr(), T, K, K, Wd.data_ptr(), R, K, Y.data_ptr(), ldy,
                                           dws.data_ptr(), dws.numel(), s)
    res = {}
    res["library (TMA operands; 6:8 gather / 4:6, 8:10 lift before the GEMM)"] = timed(sparse_call)
    for pol, nm_pol in ((1, "whole tiles"), (2, "stream-K")):
        nm.set_gemm_schedule(pol)
        try:
            res[f"library, {nm_pol} forced"] = timed(sparse_call)
            res[f"own dense GEMM, CTA pair, {nm_pol} forced"] = timed(dense_call)
        finally:
            nm.set_gemm_schedule(0)
    res["256 x 256 pair tile (nm_sparse_gemm_tile256)"] = timed(
        lambda: lib.nm_sparse_gemm_tile256(X.data_ptr(), T, K, K, packed.data_ptr(), R, m, Y.data_ptr(),
                                           ldy, ws.data_ptr(), ws.numel(), s))
    res["in-kernel lift (nm_sparse_gemm_fused)"] = timed(
        lambda: lib.nm_sparse_gemm_fused(X.data_ptr(), T, K, K, packed.data_ptr(), R, m, Y.data_ptr(),
                                         ldy, s))
    res["own dense GEMM, CTA pair (nm_dense_gemm)"] = timed(dense_call)
    res["own dense GEMM, single CTA (nm_gemm_1cta)"] = timed(
        lambda: lib.nm_gemm_1cta(0, X.data_ptr(), T, K, K, Wd.data_ptr(), R, K, Y.data_ptr(), ldy, s))
    if m == 4:
        res["2:4 sparse, single CTA (nm_gemm_1cta)"] = timed(
            lambda: lib.nm_gemm_1cta(1, X.data_ptr(), T, K, K, packed.data_ptr(), R, 0, Y.data_ptr(),
                                     ldy, s))
    Yt = torch.empty((T, R), dtype=torch.bfloat16, device=dev)
    res["torch.matmul bf16 (cuBLAS), context"] = timed(lambda: (torch.matmul(X, Wd.t(), out=Yt), 0)[1])
    G = (K + m - 1) // m
    KL = G * (m // 2 - 1) * 4
    nkb = 3 * ((G + 31) // 32) if m == 8 else (KL + 127) // 128
    flops_lift = 2.0 * T * R * nkb * 128
    out = {"ablation": layer.name, "pattern": f"{n}:{m}", "R": R, "K": K, "T": T, "ms": {}, "pct_of_peak": {}}
    _, bf16_tf, _ = peaks()
    for k, v in res.items():
        out["ms"][k] = round(v, 4)
        sparse = "dense" not in k and "torch" not in k
        f = flops_lift if sparse else 2.0 * T * R * K
        pk = 2 * bf16_tf if sparse else bf16_tf
        out["pct_of_peak"][k] = round(100 * f / (v * 1e-3) / 1e12 / pk, 1)
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    # default: ~1 s of timed GPU work on the default workload, so the clock
    # sampler sees the kernels under load
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(datagen.WORKLOADS))
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--probe", action="store_true", help="run the tensor-pipe / HBM probes instead")
    ap.add_argument("--ablation", action="store_true", help="time the GEMM variants instead")
    ap.add_argument("--prep", action="store_true", help="time the HBM-bound prep kernels instead")
    ap.add_argument("--reps", type=int, default=5, help="--prep / --f8: timed launches per kernel")
    ap.add_argument("--f8", action="store_true", help="time the FP8 quantise+lift and FP8 sparse GEMM instead")
    ap.add_argument("--cpu-standin", action="store_true",
                    help="host logic of the multi-rank run on CPU (gloo, the oracle as per-rank work)")
    args = ap.parse_args()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(launch_ranks(args.gpus, sys.argv[1:]))
    if args.cpu_standin:
        return run_cpu_standin(args)
    if args.prep:
        return run_prep(args)
    if args.f8:
        return run_f8(args)
    if args.probe:
        run_probe(args)
        return
    if args.ablation:
        run_ablation(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
