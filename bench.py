#!/usr/bin/env python
"""Training-step throughput of the B200 forward+backward step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload d20]
    python bench.py --impl reference ...     (the float64 CPU oracle, timed)

One step = one forward+backward pass (loss and every weight gradient) over one
batch of synthetic token ids, through the C ABI (nc_forward_backward).  The
default workload is the depth-20 model at seq 2048, batch 16 (32768 tokens per
step).  Rank 0 prints one JSON line: device-timed tokens/s with inputs
resident (`value`), the same through the host-buffer entry point with the
H2D/D2H copies inside the timed region (`e2e`), MFU, the roofline of the
dominant kernel class, the oracle on host cores (`cpu_baseline`), and the SM
clocks sampled during the timed region.

With --gpus N (launched by torchrun) every rank runs an independent replica on
its own batch: the step has no collective (weak scaling); NCCL is used only
for the barrier and the max-over-ranks of the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "train tokens/s (fwd+bwd) at depth-20, seq 2048, 1×B200; MFU vs BF16 peak"
NOMINAL_BF16_TFLOPS = 2250.0
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def step_flops_per_token(cfg, T, causal=True):
    """6 * matmul params (layer linears + LM head) + 6*L*H*hd*T causal attention;
    with causal=False the PaLM convention 12*L*H*hd*T (no causal halving)."""
    d, hd, F = cfg.d_model, cfg.head_dim, cfg.mlp_mult * cfg.d_model
    per_layer = d * (cfg.n_head * hd + 2 * cfg.n_kv_head * hd) + cfg.n_head * hd * d + 2 * F * d
    n_mm = cfg.n_layer * per_layer + cfg.vocab * d
    return 6.0 * n_mm + (6.0 if causal else 12.0) * cfg.n_layer * cfg.n_head * hd * T


def workload_desc(wl):
    c = wl.model
    return (f"{wl.name}: vocab {c.vocab}, d_model {c.d_model}, {c.n_layer} layers, {c.n_head}x{c.head_dim} MQA "
            f"({c.n_kv_head} kv head), mlp {c.mlp_mult * c.d_model} relu^2, softcap {c.softcap:g}, "
            f"seq {wl.seq_len}, batch {wl.batch}, {wl.ids} ids")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK}, "measured"
    except Exception:
        return dict(FALLBACK), "fallback"


def profile_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or
    None when absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_traffic.md")
    if not os.path.exists(path):
        return None
    vals = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.startswith("- "):
                k, v = line[2:].split(":", 1)
                vals[k.strip()] = v.strip().strip("`")
    src = vals.get("source")
    if not src or "bytes_per_launch" not in vals:
        return None
    fn, digest = src.split("@")
    fp = os.path.join(ROOT, fn)
    if not os.path.exists(fp) or hashlib.sha256(open(fp, "rb").read()).hexdigest()[:16] != digest:
        return None
    return float(vals["bytes_per_launch"])


def max_over_ranks(x, world, dist=None, device="cuda"):
    """The maximum of x over all ranks: the slowest rank sets the timed region."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, tokens_per_rank_step, steps, ms):
    """Whole-job tokens/s over `ms` milliseconds: every rank runs its own batch
    (independent replicas, weak scaling)."""
    return world * tokens_per_rank_step * steps / (ms / 1e3)


def roofline_of(rows, pk, src, traffic_of=None):
    """Roofline of the dominant kernel class from the profiler rows (one row per
    class: launches, ms, flops, bytes).  The gemm_* classes are the roles
    (forward, input grad, weight grad, LM head) of one tcgen05 GEMM kernel and
    are aggregated; a class with FLOPs is tensor-bound against the sustained
    bf16 peak, otherwise HBM-bound against the copy bandwidth."""
    traffic_of = traffic_of or profile_traffic
    by_kernel = {}
    for r in rows:
        k = "gemm_tcgen05" if r["kernel"].startswith("gemm_") and r["kernel"] != "gemm_fma" else r["kernel"]
        a = by_kernel.setdefault(k, {"kernel": k, "launches": 0, "ms": 0.0, "flops": 0.0, "bytes": 0.0})
        for f in ("launches", "ms", "flops", "bytes"):
            a[f] += r[f]
    dom = max(by_kernel.values(), key=lambda r: r["ms"])
    if dom["flops"] > 0:
        achieved = dom["flops"] / (dom["ms"] / 1e3) / 1e12
        peak, unit, bound = pk["bf16_tflops_sustained"], "TFLOP/s", "tensor"
    else:
        achieved = dom["bytes"] / (dom["ms"] / 1e3) / 1e9
        peak, unit, bound = pk["hbm_gbs"], "GB/s", "hbm"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "traffic": traffic_of(dom["kernel"]), "kernel": dom["kernel"], "launches": dom["launches"],
            "peak_source": f"{src} ({'sustained' if bound == 'tensor' else 'copy'})"}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.out = None

    def __enter__(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200", "-i", str(self.gpu)], stdout=self.out,
                                         stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.out is None:
            return None
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.out.name)
        if not rows:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 200.0] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "power_w_max": max(r[2] for r in rows)}


def time_workload(wl, steps, warmup):
    """Device-timed throughput of one workload at its full batch (inputs
    resident, no profiler): tokens/s, TFLOP/s and MFU.  Frees its buffers."""
    import torch
    from bwd_step_b200 import Model
    cfg = wl.model
    B, T = wl.batch, wl.seq_len
    bits, _ = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1)
    model = Model(cfg.as_dict(), "bf16")
    W = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    del bits
    grads = torch.empty(model.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(model.workspace_bytes(B, T), dtype=torch.uint8, device="cuda")
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        model.forward_backward(tok_d, tgt_d, W, grads, loss, ws, stream)
    if model.check(stream) != 0:
        raise RuntimeError(f"{wl.name}: device status")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        model.forward_backward(tok_d, tgt_d, W, grads, loss, ws, stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    out = {"workload": wl.name, "tokens_per_step": B * T, "ms_per_step": ms,
           "tokens_per_s": B * T / (ms / 1e3)}
    out["tflops"] = out["tokens_per_s"] * step_flops_per_token(cfg, T) / 1e12
    out["mfu"] = out["tflops"] / NOMINAL_BF16_TFLOPS
    out["loss"] = float(loss.item())
    model.close()
    del W, grads, loss, ws, tok_d, tgt_d
    torch.cuda.empty_cache()
    return out


def cpu_oracle_sample(wl, tokens_in_sample):
    """Times the float64 oracle on the first `tokens_in_sample` positions of
    row 0 (causal: identical to those positions of the full row)."""
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = None
    _, w = synth.make_weights(wl.model, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1, batch=1)
    S = min(tokens_in_sample, wl.seq_len)
    W64 = w.astype(np.float64)
    del w
    t0 = time.perf_counter()
    oracle.step(wl.model, W64, tok[:, :S], tgt[:, :S])
    dt = time.perf_counter() - t0
    return S, dt, threads


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    _, w = synth.make_weights(wl.model, seed=0, dtype="bf16")
    W64 = w.astype(np.float64)
    del w
    tok, tgt = synth.make_tokens(wl, seed=1, batch=1)
    S = min(args.reference_tokens, wl.seq_len)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.step(wl.model, W64, tok[:, :S], tgt[:, :S])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    per = sum(times) / len(times)
    value = S / per
    cores = len(os.sched_getaffinity(0))
    sample = f"positions 0..{S - 1} of one sequence of the {wl.name} workload per step (float64 numpy oracle)"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": per * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(wl), "global_batch": 1, "seq_len": S, "parallelism": "none"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="d20", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--cpu-sample-tokens", type=int, default=2048)
    ap.add_argument("--reference-tokens", type=int, default=512)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--table", action="store_true", help="print the per-kernel table to stderr")
    ap.add_argument("--profile-steps", type=int, default=5,
                    help="steps of the separate per-kernel profiling pass")
    ap.add_argument("--no-lm-modes", action="store_true",
                    help="skip timing the materialised LM-head strategy next to the fused default")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the short per-workload throughput lines (all five workloads)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    wl = synth.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
        return

    import torch
    import torch.distributed as dist
    from bwd_step_b200 import Model, launch_count

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    cfg = wl.model
    B, T = wl.batch, wl.seq_len
    M = B * T

    bits, _ = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1 + rank)
    model = Model(cfg.as_dict(), "bf16")
    W = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    del bits
    grads = torch.empty(model.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(model.workspace_bytes(B, T), dtype=torch.uint8, device="cuda")
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    # ---------------- device-resident timing (no per-launch events inside the timed region)
    for _ in range(args.warmup):
        model.forward_backward(tok_d, tgt_d, W, grads, loss, ws, stream)
    code = model.check(stream)
    if code != 0:
        raise RuntimeError(f"device status {code}")
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        barrier()
        l0 = launch_count()
        e0.record(stream)
        for _ in range(args.steps):
            model.forward_backward(tok_d, tgt_d, W, grads, loss, ws, stream)
        e1.record(stream)
        barrier()
        launches = launch_count() - l0
    ms = e0.elapsed_time(e1)
    code = model.check(stream)
    if code != 0:
        raise RuntimeError(f"device status {code}")
    ms = max_over_ranks(ms, world, dist)
    ms_step = ms / args.steps
    value = job_throughput(world, M, args.steps, ms)
    final_loss = float(loss.item())

    # ---------------- the LM head's two strategies, same inputs (fused is the default)
    lm_modes = None
    if not args.no_lm_modes:
        lm_modes = {"fused": ms_step}
        model.set_lm_head("materialised")
        ws2 = torch.empty(model.workspace_bytes(B, T), dtype=torch.uint8, device="cuda")
        for _ in range(2):
            model.forward_backward(tok_d, tgt_d, W, grads, loss, ws2, stream)
        barrier()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        for _ in range(max(3, min(args.steps, 10))):
            model.forward_backward(tok_d, tgt_d, W, grads, loss, ws2, stream)
        g1.record(stream)
        barrier()
        lm_modes["materialised"] = max_over_ranks(g0.elapsed_time(g1), world, dist) / max(3, min(args.steps, 10))
        lm_modes["materialised_loss"] = float(loss.item())
        lm_modes["unit"] = "ms per step"
        model.set_lm_head("fused")
        del ws2
        torch.cuda.empty_cache()

    # ---------------- per-kernel table: a separate pass with an event pair
    # around every launch (the library's profiler), same inputs and stream
    prof_steps = max(1, min(args.steps, args.profile_steps))
    model.profile(True)
    for _ in range(prof_steps):
        model.forward_backward(tok_d, tgt_d, W, grads, loss, ws, stream)
    model.profile(False)
    rows = model.profile_read(stream)
    barrier()

    # ---------------- end to end through the host-buffer entry point
    h_tok = torch.from_numpy(tok).pin_memory()
    h_tgt = torch.from_numpy(tgt).pin_memory()
    for _ in range(args.warmup):
        model.forward_backward_host(h_tok, h_tgt, W, grads, ws, stream)
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(args.steps):
        model.forward_backward_host(h_tok, h_tgt, W, grads, ws, stream)
    f1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(f0.elapsed_time(f1), world, dist)
    e2e_value = job_throughput(world, M, args.steps, e2e_ms)

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    # ---------------- every workload, briefly (one GPU only: keeps the run short)
    configs = None
    if world == 1 and not args.no_configs:
        model.close()
        del W, grads, loss, ws, tok_d, tgt_d
        torch.cuda.empty_cache()
        configs = []
        for name in ("tiny", "gpt2_124m", "d20", "d30", "long"):
            if name == args.workload:
                configs.append({"workload": name, "tokens_per_step": M, "ms_per_step": ms_step,
                                "tokens_per_s": value, "tflops": value * step_flops_per_token(cfg, T) / 1e12,
                                "mfu": value * step_flops_per_token(cfg, T) / 1e12 / NOMINAL_BF16_TFLOPS,
                                "loss": final_loss, "note": "the headline measurement above"})
            else:
                configs.append(time_workload(synth.WORKLOADS[name], steps=5, warmup=3))

    # ---------------- roofline of the dominant kernel
    pk, src = peaks()
    roofline = roofline_of(rows, pk, src)

    fpt = step_flops_per_token(cfg, T)
    tflops = value * fpt / 1e12
    clocks = clk.summary()

    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        S, dt, threads = cpu_oracle_sample(wl, args.cpu_sample_tokens)
        cpu = {"value": S / dt, "unit": "tokens/s", "cores": threads or len(os.sched_getaffinity(0)),
               "host_cores": len(os.sched_getaffinity(0)), "kind": "oracle",
               "sample": f"one sequence ({S} positions) of the {wl.name} workload, float64 numpy, {dt:.1f} s"}

    kernels = []
    for r in sorted(rows, key=lambda r: -r["ms"]):
        k = {"kernel": r["kernel"], "launches": r["launches"], "ms_per_step": r["ms"] / prof_steps,
             "share": r["ms"] / sum(x["ms"] for x in rows)}
        if r["flops"] > 0:
            k["tflops"] = r["flops"] / (r["ms"] / 1e3) / 1e12
        if r["bytes"] > 0:
            k["gbs"] = r["bytes"] / (r["ms"] / 1e3) / 1e9
        kernels.append(k)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded Zipf(1.1) ids, N(0,0.02) bf16 weights)",
        "config": {"workload": workload_desc(wl), "global_batch": B * world, "seq_len": T,
                   "parallelism": "replicas" if world > 1 else "single",
                   "l2": "no flush: per-step working set (weights, activations, grads) far exceeds the 126 MB L2"},
        "tflops": tflops, "mfu": tflops / NOMINAL_BF16_TFLOPS,
        "tflops_palm_convention": value * step_flops_per_token(cfg, T, causal=False) / 1e12,
        "mfu_vs_measured": tflops / pk["bf16_tflops"], "gflop_per_token": fpt / 1e9,
        "loss": final_loss,
        "roofline": roofline,
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": 2 * 4 * M, "d2h_bytes_per_step": 4},
        "gpu_launches": int(launches),
        "clocks": clocks,
        "kernels": kernels,
        "kernel_table_source": f"separate pass of {prof_steps} steps with an event pair around every launch",
        "configs": configs,
        "lm_head_modes": lm_modes,
    }
    if args.table:
        for k in kernels:
            print(f"{k['kernel']:18s} {k['launches'] / prof_steps:6.0f}/step {k['ms_per_step']:8.3f} ms "
                  f"{100 * k['share']:5.1f}%  " + (f"{k['tflops']:7.1f} TFLOP/s" if "tflops" in k else "") +
                  (f"{k['gbs']:8.0f} GB/s" if "gbs" in k else ""), file=sys.stderr)
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
