#!/usr/bin/env python3
"""Benchmark of the fused chunked KL loss, forward + backward, on B200.

One step = one fckl_fwd_bwd call over the whole workload (every chunk: teacher
prep, fused projection + log-sum-exp, recompute + dlogits, dH and dW GEMMs).
Default workload: the largest single-GPU one, 256K tokens (N=262144, H=4096,
V=128256, K=100, T=2, 10% rows masked, chunk 2048; "Knowledge Distillation 비용
줄이기", section "chunked KL loss가 하는 일").  Other workloads: --config
(0 tiny, 1 the 8K Llama-3.1-8B -> ~3B student shape, 2 the 32K toy output
projection, 3 the gpt-oss-20b student shape); --rows shrinks a workload's row
count (small cases for profiler captures).

Under torchrun with N ranks (--mode dp, the default there) the ranks run
row-sharded data parallelism: every rank holds one shard of N_rows rows of a
global batch of N * N_rows rows ("scaling": "weak"), the ranks all-reduce the
valid-row count, and the dW all-reduce overlaps the last dW GEMM
(chunked_kl_loss_tcgen05_b200.dp).  --mode replicas runs independent replicas
with no data-path collective.  Timing is the max over ranks.
`--impl reference` times the fp64 CPU oracle instead, on a bounded sample of
rows of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import dataclasses

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "fused KL fwd+bwd tokens/s & TFLOP/s (frac of BF16 peak); peak GiB vs seq len"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "source": "fallback"}

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum, mean over the
# launches of one call) from the ncu capture of the current kernels on this workload,
# summarised under profiles/.  Reset an entry to None when its kernel changes.
MEASURED_TRAFFIC = {
    # 256K workload: captured on a 4096-row cut of it, whose first chunk (2048
    # rows) has the full-size launch shape; dW = mean over a full call's launches
    # (one storing launch, the rest reduce-adding)
    "scale_256k_N262144_H4096_V128256_K100_T2": {
        "fwd_logits_lse": 1.31e9, "bwd_dlogits": 2.02e9, "dH_gemm": 3.66e9, "dW_gemm": 4.73e9},
}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        d["source"] = "measured"
        return d
    except Exception:
        return dict(FALLBACK_PEAKS)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", type=int, default=4)
    ap.add_argument("--rows", type=int, default=0,
                    help="use only this many rows of the workload (0 = all; same H, V, K, T, "
                         "chunk and mask fraction)")
    ap.add_argument("--dw-rows", type=int, default=0,
                    help="group chunks so that each dW GEMM covers at least this many rows "
                         "(fckl_problem.dw_rows; 0 = one dW GEMM per chunk)")
    ap.add_argument("--mode", default="", choices=["", "dp", "replicas"],
                    help="multi-GPU mode under torchrun (default dp)")
    ap.add_argument("--dp-slices", type=int, default=8,
                    help="dp mode: vocabulary slices of the last dW GEMM whose all-reduce "
                         "overlaps the rest")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="also time the step replayed from a captured CUDA graph")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-grouped", action="store_true",
                    help="skip the extra timing with chunks grouped per dW GEMM (dw_grouped)")
    ap.add_argument("--cpu-rows", type=int, default=0, help="rows in the oracle sample (0 = auto)")
    ap.add_argument("--profile-json", default="")
    ap.add_argument("--mem-sweep", action="store_true",
                    help="print peak device memory vs sequence length instead of timing")
    ap.add_argument("--sweep-chunk", type=int, default=2048,
                    help="--mem-sweep: rows per chunk")
    ap.add_argument("--sweep-s", default="8192,16384,32768,65536,131072,262144",
                    help="--mem-sweep: comma-separated sequence lengths")
    ap.add_argument("--vs-cublas", type=float, default=0.0, metavar="SECONDS",
                    help="instead of the contract line: run the fused step and the four plain "
                         "cuBLAS GEMMs of the same shapes back to back for SECONDS each, clocks "
                         "sampled, and print both")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def workload(args) -> synth.Config:
    """The selected workload, optionally cut to its first --rows rows."""
    cfg = synth.CONFIGS[args.config]
    if args.rows and args.rows != cfg.N:
        cfg = dataclasses.replace(cfg, N=int(args.rows), name=f"{cfg.name}_rows{int(args.rows)}")
    return cfg


def workload_config(cfg: synth.Config, C: int, dw_rows: int = 0) -> dict:
    return {"workload": cfg.name, "N_rows": cfg.N, "H": cfg.H, "V": cfg.V, "K": cfg.K, "T": cfg.T,
            "chunk": C, "dw_rows": dw_rows, "mask_frac": cfg.mask_frac,
            "l2": "inputs larger than L2 (W alone is %.0f MB > 126 MB)" % (cfg.V * cfg.H * 2 / 1e6),
            "data": "synthetic seeded (synth recipe)"}


def library_chunk(cfg: synth.Config) -> int:
    """The chunk the library resolves for this workload, restated here so that
    the oracle arm never loads the library: an explicit chunk capped at N, or
    (chunk = 0) the largest multiple of 128 rows whose bf16 dlogits block
    [chunk, V rounded up to 64] fits in 1 GiB, at least 128, capped at N rounded
    up to 64, then at N (tests/test_boundary.py checks that both agree)."""
    C = cfg.chunk
    if C == 0:
        Vp = (cfg.V + 63) // 64 * 64
        C = (1 << 30) // (Vp * 2) // 128 * 128
        C = max(C, 128)
        C = min(C, (cfg.N + 63) // 64 * 64)
    return min(C, cfg.N)


# ------------------------------------------------------------------ oracle arm
def oracle_rows_per_sec(inp, n_rows, reps=1):
    import oracle
    rows = synth.sample_rows(inp, n_rows)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.oracle_from_inputs(inp, rows=rows, row_block=256)
    dt = time.perf_counter() - t0
    return rows.size * reps / dt, rows.size, dt


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def auto_cpu_rows(cfg):
    """Rows of the oracle sample: ~6*H*V fp64 flops per row (logits, dH, dW
    contribution), ~1 TFLOP per sample (a few seconds on a many-core host).
    The CUDA arm's cpu_baseline and the reference arm use the same sample."""
    per_row = 6.0 * cfg.H * cfg.V
    return int(max(16, min(1024, 1e12 / per_row)))


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    cfg = workload(args)
    inp = synth.make_inputs(cfg)
    n_rows = args.cpu_rows or auto_cpu_rows(cfg)
    times = []
    for i in range(args.warmup + args.steps):
        rps, n, dt = oracle_rows_per_sec(inp, n_rows)
        if i >= args.warmup:
            times.append(dt)
    ms = 1e3 * statistics.mean(times)
    value = n_rows / (ms / 1e3)
    sample = f"{n_rows} seeded valid rows of the workload per step (fwd + bwd incl. dW contribution)"
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": dict(workload_config(cfg, library_chunk(cfg), args.dw_rows),
                           parallelism=f"oracle on rank 0 of {world}",
                           flush="inputs larger than L2"),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cpu_cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ clocks
class ClockSampler:
    def __init__(self, index):
        self.proc = None
        self.path = None
        self.index = index

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                 "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                 "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for ln in fh:
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------------------ GPU arm
def run_cuda(args):
    import torch
    import torch.distributed as dist
    from chunked_kl_loss_tcgen05_b200 import (FcklProblem, fckl_check, fckl_resolved_chunk,
                                              fckl_profile_begin, fckl_profile_end)
    from chunked_kl_loss_tcgen05_b200.torch_api import (alloc_workspace, arrays_to_device,
                                                        fused_kl_fwd_bwd)

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    # one GPU: the plain fused call, unless --mode dp asks for the data-parallel
    # path on a one-rank process group (its collectives then run on one rank)
    mode = (args.mode if args.mode == "dp" else "single") if world == 1 else (args.mode or "dp")
    use_pg = world > 1 or mode == "dp"
    if use_pg:
        import datetime
        if "MASTER_ADDR" not in os.environ:
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("MASTER_PORT", "29511")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if use_pg:
            dist.barrier()

    cfg = workload(args)
    # Every rank's shard (dp) or replica is the same seeded workload: the work
    # and its cost do not depend on the values.
    inp = synth.make_inputs(cfg)
    prob = FcklProblem(cfg.N, cfg.H, cfg.V, cfg.K, cfg.T, cfg.chunk, dw_rows=args.dw_rows)
    C = fckl_resolved_chunk(prob)
    n_valid = int(inp.row_mask.sum())
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask, dev)
    ws = alloc_workspace(prob, dev)
    torch.cuda.synchronize()
    torch.cuda.reset_peak_memory_stats(dev)

    outs = (torch.empty(1, device=dev), torch.empty(cfg.N, cfg.H, device=dev),
            torch.empty(cfg.V, cfg.H, device=dev))

    if mode == "dp":
        from chunked_kl_loss_tcgen05_b200.dp import fused_kl_fwd_bwd_dp

        def step():
            return fused_kl_fwd_bwd_dp(*d, T=cfg.T, chunk=cfg.chunk, workspace=ws,
                                       n_slices=args.dp_slices, out=outs, dw_rows=args.dw_rows)
    else:
        def step():
            return fused_kl_fwd_bwd(*d, T=cfg.T, chunk=cfg.chunk, workspace=ws, check=False,
                                    out=outs, dw_rows=args.dw_rows)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = fckl_check(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    if st != 0:
        raise SystemExit(f"device error after warm-up: status {st}")

    # Untimed breakdown pass: events around every kernel (they add gaps, so this
    # pass only apportions time between kernel kinds and picks the dominant one).
    fckl_profile_begin(None)
    for _ in range(2):
        step()
    breakdown = fckl_profile_end()
    # every kernel of a step is recorded in the breakdown pass (two steps)
    launches_per_step = sum(p["launches"] for p in breakdown) // 2
    dom_kind = max(breakdown, key=lambda p: p["total_ms"])["name"] if breakdown else None

    clocks = ClockSampler(local)
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    # Timed region.  Events around the dominant kernel kind (its launch times
    # for the roofline) are recorded in the last quarter of the steps only: an
    # event between two kernels keeps the second from launching early
    # (programmatic dependent launch), so they cost a little of the step time.
    n_prof = max(1, min(args.steps, max(2, args.steps // 4)))
    e0.record(stream)
    for i in range(args.steps):
        if i == args.steps - n_prof:
            fckl_profile_begin([dom_kind] if dom_kind else None)
        out = step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    prof = fckl_profile_end()
    clk = clocks.stop()
    ms_total = e0.elapsed_time(e1)
    peak_gib = torch.cuda.max_memory_allocated(dev) / 2**30
    loss_val = float(out[0].item())
    del out
    st = fckl_check(ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    if st != 0:
        raise SystemExit(f"device error in the timed steps: status {st}")

    ms_total = max_over_ranks(torch, dev, ms_total, world)
    ms_step = ms_total / args.steps
    tokens = cfg.N * world
    value = tokens / (ms_step / 1e3)
    flops_step = 8.0 * cfg.H * cfg.V * n_valid
    tflops = flops_step * world / (ms_step / 1e3) / 1e12

    peaks = load_peaks()
    burst = peaks["bf16_tflops"]
    sustained = peaks.get("bf16_tflops_sustained") or burst
    # dominant kernel: its launches were event-timed inside the timed region
    bd_total = sum(p["total_ms"] for p in breakdown) or 1.0
    dom = max(prof, key=lambda p: p["total_ms"]) if prof else None
    roofline = None
    if dom is not None:
        avg_ms = dom["total_ms"] / dom["launches"]
        share = dom["total_ms"] / n_prof / ms_step
        traffic = MEASURED_TRAFFIC.get(cfg.name, {}).get(dom["name"])
        if dom["flops"] > 0:
            ach = dom["flops"] / dom["launches"] / (avg_ms / 1e3) / 1e12
            roofline = {"kernel": dom["name"], "bound": "tensor", "achieved": ach, "peak": burst,
                        "unit": "TFLOP/s", "frac": ach / burst,
                        "peak_kind": f"bf16_tflops burst ({peaks['source']})",
                        "frac_of_sustained_peak": ach / sustained,
                        "sustained_peak": sustained,
                        "traffic": traffic,
                        "algorithmic_bytes": dom["bytes"] / dom["launches"],
                        "algorithmic_flops": dom["flops"] / dom["launches"],
                        "launch_ms": avg_ms, "share": share,
                        "timed_steps_with_events": n_prof}
        else:
            peak = peaks["hbm_gbs"]
            ach = dom["bytes"] / dom["launches"] / (avg_ms / 1e3) / 1e9
            roofline = {"kernel": dom["name"], "bound": "hbm", "achieved": ach, "peak": peak,
                        "unit": "GB/s", "frac": ach / peak, "peak_kind": f"hbm_gbs ({peaks['source']})",
                        "traffic": traffic, "launch_ms": avg_ms, "share": share}
    kernels = [{"name": p["name"], "launches": p["launches"] // 2, "ms_per_step": p["total_ms"] / 2,
                "share": p["total_ms"] / bd_total,
                "tflops": (p["flops"] / (p["total_ms"] / 1e3) / 1e12) if p["flops"] else None}
               for p in breakdown]

    graph = None
    if args.graph and mode != "dp":
        graph = measure_graph(torch, dev, step, args.steps, cfg, world)

    # A workload whose explicit chunk is below 4096 rows also runs with chunks
    # grouped so that each dW GEMM covers >= 4096 rows (fckl_problem.dw_rows):
    # the speed the library's memory/speed knob buys back, same box, same inputs.
    grouped = None
    if (not args.no_grouped and mode == "single" and args.dw_rows == 0 and 0 < C < 4096
            and cfg.N > C):
        grouped = measure_grouped(torch, dev, d, cfg, args.steps, outs, flops_step, burst)

    e2e = None
    if not args.no_e2e:
        if mode == "dp":
            e2e = measure_e2e_dp(torch, dev, inp, cfg, ws, args, world, outs, d)
        else:
            e2e = measure_e2e(torch, dev, inp, cfg, ws, args.steps, world, outs, args.dw_rows)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_rows = args.cpu_rows or auto_cpu_rows(cfg)
        rps, n, dt = oracle_rows_per_sec(inp, n_rows)
        cpu = {"value": rps, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
               "sample": f"{n} seeded valid rows of the workload, fwd+bwd incl. dW contribution, "
                         f"{dt:.1f} s"}

    if rank == 0:
        par = {"single": "1 GPU", "replicas": f"replicas{world}",
               "dp": f"dp{world} (row shards, dW all-reduce overlapped)"}[mode]
        line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic",
                "config": dict(workload_config(cfg, C, args.dw_rows), parallelism=par,
                               global_batch=cfg.N * world, flush="inputs larger than L2"),
                "tflops": tflops,
                "frac_of_peak": {"burst": tflops / world / burst,
                                 "sustained": tflops / world / sustained,
                                 "dense_spec_2250": tflops / world / 2250.0,
                                 "burst_sustained_source": peaks["source"]},
                "peaks_source": peaks["source"],
                "peak_mem_gib": peak_gib, "loss": loss_val,
                "roofline": roofline, "kernels": kernels,
                "cpu_baseline": cpu, "e2e": e2e, "clocks": clk, "graph": graph,
                "dw_grouped": grouped,
                "gpu_launches": launches_per_step * args.steps}
        print(json.dumps(line), flush=True)
        if args.profile_json:
            with open(args.profile_json, "w") as fh:
                json.dump(line, fh, indent=1)
    if use_pg:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def measure_grouped(torch, dev, d, cfg, steps, outs, flops_step, burst):
    """The same workload with dw_rows = 4096 (two or more chunks per dW GEMM; the
    workspace then holds that many rows of dlogits): step time and the dW GEMM's
    rate, its launches event-timed in the last quarter of the steps."""
    from chunked_kl_loss_tcgen05_b200 import (FcklProblem, fckl_profile_begin, fckl_profile_end,
                                              fckl_workspace_bytes)
    from chunked_kl_loss_tcgen05_b200.torch_api import alloc_workspace, fused_kl_fwd_bwd
    prob = FcklProblem(cfg.N, cfg.H, cfg.V, cfg.K, cfg.T, cfg.chunk, dw_rows=4096)
    ws = alloc_workspace(prob, dev)

    def step():
        return fused_kl_fwd_bwd(*d, T=cfg.T, chunk=cfg.chunk, workspace=ws, check=False, out=outs,
                                dw_rows=4096)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n_prof = max(1, min(steps, max(2, steps // 4)))
    e0.record(stream)
    for i in range(steps):
        if i == steps - n_prof:
            fckl_profile_begin(["dW_gemm"])
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    prof = fckl_profile_end()
    ms = e0.elapsed_time(e1) / steps
    dw = next((p for p in prof if p["name"] == "dW_gemm"), None)
    dw_tflops = dw["flops"] / (dw["total_ms"] / 1e3) / 1e12 if dw and dw["total_ms"] > 0 else None
    out = {"dw_rows": 4096, "ms_per_step": ms, "value": cfg.N / (ms / 1e3), "unit": "tokens/s",
           "tflops": flops_step / (ms / 1e3) / 1e12, "frac_of_burst": flops_step / (ms / 1e3) / 1e12 / burst,
           "dW_gemm_tflops": dw_tflops, "steps": steps,
           "workspace_gib": fckl_workspace_bytes(prob) / 2**30}
    del ws
    torch.cuda.empty_cache()
    return out


def max_over_ranks(torch, dev, ms, world):
    """The slowest rank's time (every rank calls this at the same point)."""
    if world == 1:
        return ms
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measure_graph(torch, dev, step, steps, cfg, world):
    """The same step captured once into a CUDA graph and replayed (no per-launch
    host work); timed like the main region."""
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream(dev).wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        g.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dev, e0.elapsed_time(e1) / steps, world)
    del g
    return {"value": cfg.N * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms}


def measure_e2e(torch, dev, inp, cfg, ws, steps, world, outs, dw_rows=0):
    """Same metric through the host-input C-ABI call: every step the library
    copies that step's inputs (hidden states, teacher top-K ids and logits, row
    mask) from pinned host memory to the device, overlapped chunk by chunk with
    the kernels, and the loss is read back on the host.  W is the student's
    resident parameter and stays on the device."""
    from chunked_kl_loss_tcgen05_b200.torch_api import alloc_host_workspace, fused_kl_fwd_bwd_host
    from chunked_kl_loss_tcgen05_b200 import FcklProblem
    host = {"hidden": torch.from_numpy(inp.hidden.view(np.int16)).view(torch.bfloat16).pin_memory(),
            "topk_idx": torch.from_numpy(inp.topk_idx).pin_memory(),
            "topk_logit": torch.from_numpy(inp.topk_logit).pin_memory(),
            "row_mask": torch.from_numpy(inp.row_mask).pin_memory()}
    W = torch.from_numpy(inp.W.view(np.int16)).view(torch.bfloat16).to(dev)
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    prob = FcklProblem(cfg.N, cfg.H, cfg.V, cfg.K, cfg.T, cfg.chunk, dw_rows=dw_rows)
    hws = alloc_host_workspace(prob, dev)
    loss_host = torch.empty(1, dtype=torch.float32, pin_memory=True)
    out = (outs[1], outs[2])

    def call():
        return fused_kl_fwd_bwd_host(host["hidden"], W, host["topk_idx"], host["topk_logit"],
                                     host["row_mask"], T=cfg.T, chunk=cfg.chunk, workspace=hws,
                                     out=out, loss_host=loss_host, check=False, dw_rows=dw_rows)
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        call()  # returns after the loss has reached the host
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dev, e0.elapsed_time(e1) / steps, world)
    del hws, W
    return {"value": cfg.N * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4, "steps": steps,
            "path": "fckl_fwd_bwd_host (inputs pinned on the host, W resident)"}


def measure_e2e_dp(torch, dev, inp, cfg, ws, args, world, outs, d):
    """dp mode end to end through the data-parallel API: every step copies the
    rank's shard (hidden states, teacher top-K ids and logits, row mask) from
    pinned host memory into the device buffers, runs fused_kl_fwd_bwd_dp
    (valid-count and dW all-reduces included) and reads the loss back."""
    from chunked_kl_loss_tcgen05_b200.dp import fused_kl_fwd_bwd_dp
    host = [torch.from_numpy(inp.hidden.view(np.int16)).view(torch.bfloat16).pin_memory(), None,
            torch.from_numpy(inp.topk_idx).pin_memory(),
            torch.from_numpy(inp.topk_logit).pin_memory(),
            torch.from_numpy(inp.row_mask).pin_memory()]
    h2d = sum(t.numel() * t.element_size() for t in host if t is not None)
    loss_host = torch.empty(1, dtype=torch.float32, pin_memory=True)

    def call():
        for i, t in enumerate(host):
            if t is not None:
                d[i].copy_(t, non_blocking=True)
        loss, _, _ = fused_kl_fwd_bwd_dp(*d, T=cfg.T, chunk=cfg.chunk, workspace=ws,
                                         n_slices=args.dp_slices, out=outs, dw_rows=args.dw_rows)
        loss_host.copy_(loss, non_blocking=True)
        torch.cuda.current_stream(dev).synchronize()
        return float(loss_host[0])
    for _ in range(2):
        call()
    torch.cuda.synchronize()
    import torch.distributed as dist
    dist.barrier()
    stream = torch.cuda.current_stream(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        call()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(torch, dev, e0.elapsed_time(e1) / args.steps, world)
    return {"value": cfg.N * world / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": 4, "steps": args.steps,
            "path": "fused_kl_fwd_bwd_dp after host->device copies of the shard from pinned memory"}


def run_mem_sweep(args):
    """Peak device memory of one fused forward+backward call vs sequence length
    at the 32K toy-projection shape (H=4096, V=128256, K=100, chunk
    --sweep-chunk): inputs, outputs and workspace all counted
    (torch.cuda.max_memory_allocated)."""
    import torch
    from chunked_kl_loss_tcgen05_b200.torch_api import fused_kl_fwd_bwd
    torch.cuda.set_device(0)
    H, V, K, C = 4096, 128256, 100, args.sweep_chunk
    pts = []
    for S in [int(x) for x in args.sweep_s.split(",") if x]:
        torch.cuda.empty_cache()
        base = torch.cuda.memory_allocated()
        g = torch.Generator(device="cuda").manual_seed(S)
        hidden = torch.randn(S, H, device="cuda", dtype=torch.bfloat16, generator=g)
        W = (torch.randn(V, H, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
        ids = torch.randint(0, V, (S, K), device="cuda", dtype=torch.int32, generator=g)
        lg = torch.randn(S, K, device="cuda", generator=g) * 3
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()  # inputs stay counted, their fp32 temporaries do not
        loss, _, dH, dW = fused_kl_fwd_bwd(hidden, W, ids, lg, None, T=1.0, chunk=C,
                                           dw_rows=args.dw_rows)
        torch.cuda.synchronize()
        peak = (torch.cuda.max_memory_allocated() - base) / 2**30
        pts.append((S, peak))
        del hidden, W, ids, lg, loss, dH, dW
    xs = np.array([p[0] for p in pts], dtype=np.float64)
    ys = np.array([p[1] for p in pts], dtype=np.float64)
    b, a = np.polyfit(xs, ys, 1)
    r2 = 1 - ((ys - (a + b * xs)) ** 2).sum() / ((ys - ys.mean()) ** 2).sum()
    line = {"metric": f"peak GiB vs seq len (fused fwd+bwd, H=4096 V=128256 K=100 chunk={C}, "
                      f"dw_rows={args.dw_rows})",
            "points": [{"S": s, "peak_gib": round(p, 4)} for s, p in pts],
            "fit": {"intercept_gib": a, "slope_kib_per_row": b * 2**20, "r2": r2}}
    print(json.dumps(line), flush=True)
    return 0


def run_vs_cublas(args):
    """Same-conditions comparison: the fused forward+backward step against the
    four plain cuBLAS bf16 GEMMs of the same shapes (logits, their recompute,
    dH, dW; no loss arithmetic, bf16 outputs), each run back to back for the
    same time with clocks and power sampled, so that both see the same power
    cap.  A measurement aid, not part of the contract line."""
    import torch
    from chunked_kl_loss_tcgen05_b200 import FcklProblem, fckl_resolved_chunk
    from chunked_kl_loss_tcgen05_b200.torch_api import (alloc_workspace, arrays_to_device,
                                                        fused_kl_fwd_bwd)
    torch.cuda.set_device(0)
    cfg = workload(args)
    inp = synth.make_inputs(cfg)
    d = arrays_to_device(inp.hidden, inp.W, inp.topk_idx, inp.topk_logit, inp.row_mask)
    prob = FcklProblem(cfg.N, cfg.H, cfg.V, cfg.K, cfg.T, cfg.chunk, dw_rows=args.dw_rows)
    C = fckl_resolved_chunk(prob)
    ws = alloc_workspace(prob, d[0].device)
    outs = (torch.empty(1, device="cuda"), torch.empty(cfg.N, cfg.H, device="cuda"),
            torch.empty(cfg.V, cfg.H, device="cuda"))
    n_valid = int(inp.row_mask.sum())

    def fused():
        fused_kl_fwd_bwd(*d, T=cfg.T, chunk=cfg.chunk, workspace=ws, check=False, out=outs,
                         dw_rows=args.dw_rows)

    h = d[0][:C].contiguous()
    W = d[1]
    g = torch.Generator(device="cuda").manual_seed(7)
    dl = torch.randn(C, cfg.V, device="cuda", dtype=torch.bfloat16, generator=g)
    pieces = -(-n_valid // C)

    def gemms():
        for _ in range(pieces):
            h @ W.t()
            h @ W.t()
            dl @ W
            dl.t() @ h

    def timed(fn):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        clocks = ClockSampler(0)
        clocks.start()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.time()
        n = 0
        e0.record()
        while time.time() - t0 < args.vs_cublas:
            fn()
            n += 1
            if n % 4 == 0:
                torch.cuda.synchronize()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n, n, clocks.stop()

    ms_f, n_f, clk_f = timed(fused)
    ms_c, n_c, clk_c = timed(gemms)
    fl_f = 8.0 * cfg.H * cfg.V * n_valid
    fl_c = 4 * 2.0 * C * cfg.V * cfg.H * pieces
    line = {"workload": cfg.name, "chunk": C,
            "fused": {"ms_per_step": ms_f, "tflops": fl_f / ms_f / 1e9, "steps": n_f, "clocks": clk_f,
                      "rows": n_valid},
            "cublas_4_gemms": {"ms_per_step": ms_c, "tflops": fl_c / ms_c / 1e9, "steps": n_c,
                               "clocks": clk_c, "rows": C * pieces},
            "fused_over_cublas_tflops": (fl_f / ms_f) / (fl_c / ms_c)}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.mem_sweep:
        return run_mem_sweep(args)
    if args.vs_cublas > 0:
        return run_vs_cublas(args)
    return run_cuda(args)


if __name__ == "__main__":
    sys.exit(main())
