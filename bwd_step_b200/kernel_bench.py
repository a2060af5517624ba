"""Per-kernel timing of the step's building blocks on synthetic inputs.

    python -m bwd_step_b200.kernel_bench gemm [--only NAME] [--iters N]
    python -m bwd_step_b200.kernel_bench attention [--iters N]
    python -m bwd_step_b200.kernel_bench step [--workload d20] [--batch B] [--layers L] [--lm-rows R] [--warmup W] [--iters K]
    python -m bwd_step_b200.kernel_bench adamw|decode|recompute [--workload d20] [--iters K]

`gemm` runs every GEMM shape of one depth-20 step (32768 tokens, d 1280,
MLP 5120, 10x128 MQA, vocab 65536 with a 4096-row LM-head chunk) through the
testing ABI with its real operand layouts and fused epilogue, and prints
TFLOP/s from CUDA events.  `attention` times the tcgen05 attention forward and
backward at seq 2048, batch 16.  `step` runs W warm-up steps and then K
steps of a workload (optionally at a smaller batch, for profiler captures
that must stay small) and prints the library's kernel launches per step.
`adamw` times one AdamW update of every parameter of a workload (fp32 master
and moments, bf16 copy; 30 bytes per parameter); `decode` prefills 1024 tokens
in 16 rows and times one-token decode steps over the KV cache; `recompute`
times the step with the MLP hidden saved and recomputed, with both workspaces.
Each case holds at most a few GB on the device, except `step` at full batch.
"""
from __future__ import annotations

import argparse
import ctypes
import json

import torch

from . import lib

P = ctypes.c_void_p

M, D, F, NQKV, HHD, V, R = 32768, 1280, 5120, 1536, 1280, 65536, 4096

# name: (M, N, K, a_kmajor, b_kmajor, epi, c_bf16)
GEMMS = {
    "fwd_qkv": (M, NQKV, D, 1, 1, 0, 1),
    "fwd_oproj": (M, D, HHD, 1, 1, 1, 0),
    "fwd_fc_relu2": (M, F, D, 1, 1, 2, 1),
    "fwd_proj": (M, D, F, 1, 1, 1, 0),
    "dgrad_fc_relu2bwd": (M, F, D, 1, 0, 3, 1),
    "dgrad_mlp_in": (M, D, F, 1, 0, 0, 0),
    "dgrad_oproj": (M, HHD, D, 1, 0, 0, 1),
    "dgrad_qkv": (M, D, NQKV, 1, 0, 0, 0),
    "wgrad_proj": (D, F, M, 0, 0, 0, 0),
    "wgrad_fc": (F, D, M, 0, 0, 0, 0),
    "wgrad_oproj": (D, HHD, M, 0, 0, 0, 0),
    "wgrad_qkv": (NQKV, D, M, 0, 0, 0, 0),
    "lmhead_z": (R, V, D, 1, 1, 4, 1),
    "lmhead_dx": (R, D, V, 1, 0, 0, 0),
    "lmhead_dw": (V, D, R, 0, 0, 1, 0),
}


def _timed(fn, iters):
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(iters):
        fn()
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / iters


def bench_gemm(name, iters):
    m, n, k, ak, bk, epi, cbf = GEMMS[name]
    g = torch.Generator(device="cuda").manual_seed(0)
    A = (torch.randn(m * k, device="cuda", generator=g) * 0.1).to(torch.bfloat16)
    B = (torch.randn(n * k, device="cuda", generator=g) * 0.1).to(torch.bfloat16)
    C = torch.zeros(m * n, device="cuda", dtype=torch.bfloat16 if cbf else torch.float32)
    C2 = torch.zeros(m * n, device="cuda", dtype=torch.bfloat16) if epi == 2 else None
    aux = torch.rand(m * n, device="cuda", generator=g).to(torch.bfloat16) if epi == 3 else None
    scratch = torch.empty(8 * 4 * max(R * D, F * D), dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    lda = k if ak else m
    ldb = k if bk else n
    stream = P(torch.cuda.current_stream().cuda_stream)

    def run():
        r = lib().nc_test_gemm(m, n, k, 1, P(A.data_ptr()), lda, ak, P(B.data_ptr()), ldb, bk, epi, P(C.data_ptr()),
                               n, cbf, P(C2.data_ptr() if C2 is not None else 0), n,
                               P(aux.data_ptr() if aux is not None else 0), n, ctypes.c_float(15.0), 1,
                               P(scratch.data_ptr()), scratch.numel(), P(status.data_ptr()), stream)
        assert r == 0, r

    ms = _timed(run, iters)
    assert status.item() == 0
    return {"kernel": f"gemm_{name}", "M": m, "N": n, "K": k, "ms": ms, "tflops": 2.0 * m * n * k / ms / 1e9}


def bench_attention(iters, B=16, T=2048, H=10, nkv=1, hd=128):
    g = torch.Generator(device="cuda").manual_seed(0)
    nq = (H + 2 * nkv) * hd
    qkv = torch.randn(B * T * nq, device="cuda", generator=g).to(torch.bfloat16)
    dO = torch.randn(B * T * H * hd, device="cuda", generator=g).to(torch.bfloat16)
    o = torch.empty(B * T * H * hd, device="cuda", dtype=torch.bfloat16)
    lse = torch.empty(B * H * ((T + 127) // 128 * 128), device="cuda", dtype=torch.float32)
    dqkv = torch.empty_like(qkv)
    Dbuf = torch.empty(2 * lse.numel(), device="cuda", dtype=torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    nws = lib().nc_test_attention_workspace_bytes(B, T, H, nkv, hd)
    ws = torch.empty(nws, device="cuda", dtype=torch.uint8)
    stream = P(torch.cuda.current_stream().cuda_stream)

    def fwd():
        assert lib().nc_test_attention(B, T, H, nkv, hd, P(qkv.data_ptr()), P(o.data_ptr()), P(lse.data_ptr()),
                                       P(0), P(0), P(0), P(0), 0, 1, P(status.data_ptr()), stream) == 0

    def both():
        assert lib().nc_test_attention(B, T, H, nkv, hd, P(qkv.data_ptr()), P(o.data_ptr()), P(lse.data_ptr()),
                                       P(dO.data_ptr()), P(dqkv.data_ptr()), P(Dbuf.data_ptr()), P(ws.data_ptr()),
                                       nws, 1, P(status.data_ptr()), stream) == 0

    flops = 4.0 * B * H * hd * T * (T + 1) / 2
    t_f = _timed(fwd, iters)
    t_b = _timed(both, iters) - t_f
    assert status.item() == 0
    return [{"kernel": "attention_fwd", "ms": t_f, "tflops": flops / t_f / 1e9},
            {"kernel": "attention_bwd", "ms": t_b, "tflops": 2 * flops / t_b / 1e9}]


def run_steps(workload, batch, warmup, iters, layers=0, lm_rows=0):
    import numpy as np
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from . import Model, launch_count
    wl = synth.WORKLOADS[workload]
    if layers:
        # same shapes with fewer layers: full-size activations in a smaller workspace
        cfg = synth.ModelConfig(**{**wl.model.as_dict(), "n_layer": layers})
        wl = synth.Workload(wl.name, cfg, wl.seq_len, wl.batch, wl.ids)
    B = batch or wl.batch
    bits, _ = synth.make_weights(wl.model, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1, batch=B)
    m = Model(wl.model.as_dict(), "bf16")
    if lm_rows:
        m.set_lm_head("fused", lm_rows)
    W = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    grads = torch.empty(m.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(m.workspace_bytes(B, wl.seq_len), dtype=torch.uint8, device="cuda")
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    for _ in range(warmup):
        m.forward_backward(tok_d, tgt_d, W, grads, loss, ws)
    torch.cuda.synchronize()
    l0 = launch_count()
    t = _timed(lambda: m.forward_backward(tok_d, tgt_d, W, grads, loss, ws), iters) if iters else 0.0
    per = (launch_count() - l0) // max(iters + 2, 1) if iters else 0
    assert m.check() == 0
    return {"workload": workload, "batch": B, "lm_rows": lm_rows, "ms_per_step": t, "launches_per_step": per, "loss": float(loss.item())}


def _setup(workload):
    import numpy as np
    import os
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import synth
    from . import Model
    wl = synth.WORKLOADS[workload]
    bits, _ = synth.make_weights(wl.model, seed=0, dtype="bf16")
    m = Model(wl.model.as_dict(), "bf16")
    W = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
    return synth, wl, m, W


def bench_adamw(workload, iters):
    """One AdamW update of every parameter (two groups), fp32 master and moments,
    bf16 compute copy: 30 bytes of HBM traffic per parameter."""
    from . import adamw_step
    _, _, m, W = _setup(workload)
    n = m.num_params()
    g = torch.Generator(device="cuda").manual_seed(0)
    master = W.float()
    grads = torch.randn(n, device="cuda", generator=g) * 1e-3
    mom, vel = torch.zeros(n, device="cuda"), torch.zeros(n, device="cuda")
    half = n // 2
    groups = [(0, half, 3e-4, 0.9, 0.95, 1e-8, 0.0), (half, n - half, 1e-3, 0.8, 0.95, 1e-10, 0.01)]
    step = [0]

    def run():
        step[0] += 1
        adamw_step(groups, step[0], master, W, grads, mom, vel)

    ms = _timed(run, iters)
    m.close()
    return {"kernel": "adamw", "workload": workload, "params": n, "ms": ms, "gbs": 30.0 * n / ms / 1e6}


def bench_decode(workload, iters, B=16, T0=1024):
    """Prefill T0 tokens per row, then time one-token decode steps (every row
    one new token at the next position) through the KV cache."""
    synth, wl, m, W = _setup(workload)
    T_max = T0 + iters + 8
    tok, _ = synth.make_tokens(synth.Workload("dec", wl.model, T_max, B, "uniform"), seed=1)
    tok_d = torch.from_numpy(tok).cuda()
    cache = torch.empty(m.kv_cache_bytes(B, T_max), dtype=torch.uint8, device="cuda")
    ws = torch.empty(m.inference_workspace_bytes(B, T_max), dtype=torch.uint8, device="cuda")
    logits = torch.empty((B, wl.model.vocab), dtype=torch.bfloat16, device="cuda")
    cols = [tok_d[:, t].contiguous() for t in range(T_max)]
    m.prefill(tok_d[:, :T0].contiguous(), W, cache, T_max, logits, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t_p = _timed(lambda: m.prefill(tok_d[:, :T0].contiguous(), W, cache, T_max, logits, ws), 3)
    pos = [T0]
    for _ in range(3):  # warm-up steps
        m.decode_step(cols[pos[0]], pos[0], W, cache, T_max, logits, ws)
        pos[0] += 1
    torch.cuda.synchronize()
    e0.record()
    for _ in range(iters):
        m.decode_step(cols[pos[0]], pos[0], W, cache, T_max, logits, ws)
        pos[0] += 1
    e1.record()
    torch.cuda.synchronize()
    assert m.check() == 0
    ms = e0.elapsed_time(e1) / iters
    weight_bytes = 2.0 * m.num_params()
    m.close()
    return {"kernel": "decode_step", "workload": workload, "batch": B, "prompt": T0, "prefill_ms": t_p,
            "ms": ms, "tokens_per_s": B / ms * 1e3, "weight_gbs": weight_bytes / ms / 1e6}


def bench_recompute(workload, warmup, iters):
    """The step with and without recomputing the MLP hidden in the backward."""
    synth, wl, m, W = _setup(workload)
    tok, tgt = synth.make_tokens(wl, seed=1)
    tok_d, tgt_d = torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda()
    grads = torch.empty(m.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    out = {"workload": workload}
    for name, flag in (("saved", False), ("recompute", True), ("saved_again", False)):
        m.set_recompute(flag)
        nb = m.workspace_bytes(wl.batch, wl.seq_len)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        for _ in range(warmup):
            m.forward_backward(tok_d, tgt_d, W, grads, loss, ws)
        out[name] = {"ms_per_step": _timed(lambda: m.forward_backward(tok_d, tgt_d, W, grads, loss, ws), iters),
                     "workspace_gib": nb / 2**30}
        del ws
        torch.cuda.empty_cache()
    assert m.check() == 0
    m.close()
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("what", choices=["gemm", "attention", "step", "adamw", "decode", "recompute"])
    ap.add_argument("--workload", default="d20")
    ap.add_argument("--batch", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--lm-rows", type=int, default=0, help="LM-head chunk rows (0 = default)")
    ap.add_argument("--only", default=None)
    ap.add_argument("--iters", type=int, default=10)
    args = ap.parse_args()
    if args.what == "gemm":
        for name in GEMMS:
            if args.only and args.only != name:
                continue
            print(json.dumps(bench_gemm(name, args.iters)), flush=True)
            torch.cuda.empty_cache()
    elif args.what == "attention":
        for r in bench_attention(args.iters):
            print(json.dumps(r), flush=True)
    elif args.what == "adamw":
        print(json.dumps(bench_adamw(args.workload, args.iters)), flush=True)
    elif args.what == "decode":
        print(json.dumps(bench_decode(args.workload, args.iters)), flush=True)
    elif args.what == "recompute":
        print(json.dumps(bench_recompute(args.workload, args.warmup, args.iters)), flush=True)
    else:
        print(json.dumps(run_steps(args.workload, args.batch, args.warmup, args.iters, args.layers, args.lm_rows)), flush=True)


if __name__ == "__main__":
    main()
