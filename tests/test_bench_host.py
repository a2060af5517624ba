"""Host-side logic of bench.py without a GPU: the max-over-ranks reduction of the
timed region and the whole-job throughput on two gloo ranks (the N > 1 path),
the roofline aggregation of the profiler rows, the source-hash check of the
committed DRAM-traffic summary, and the two FLOP-per-token conventions."""
import hashlib
import importlib.util
import json
import os
import socket

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import torch.distributed as dist
    from datetime import timedelta
    bench = _bench()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        # each rank's own timed region; the slowest one sets the job's time
        ms = bench.max_over_ranks(100.0 + 25.0 * rank, world, dist, device="cpu")
        value = bench.job_throughput(world, 32768, 10, ms)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"ms": ms, "value": value}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_time(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    got = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    for g in got:
        assert g["ms"] == 125.0
        # two replicas of 32768 tokens, 10 steps in 125 ms
        assert g["value"] == pytest.approx(2 * 32768 * 10 / 0.125)


def test_single_rank_needs_no_process_group():
    bench = _bench()
    assert bench.max_over_ranks(42.0, 1) == 42.0
    assert bench.job_throughput(1, 32768, 20, 2000.0) == pytest.approx(32768 * 20 / 2.0)


def test_roofline_aggregates_the_gemm_roles():
    bench = _bench()
    rows = [
        {"kernel": "gemm_fwd", "launches": 80, "ms": 20.0, "flops": 20e12, "bytes": 1e9},
        {"kernel": "gemm_dgrad", "launches": 80, "ms": 20.0, "flops": 20e12, "bytes": 1e9},
        {"kernel": "attention_bwd_dkv", "launches": 20, "ms": 30.0, "flops": 3e12, "bytes": 0.0},
        {"kernel": "rmsnorm_bwd", "launches": 41, "ms": 5.0, "flops": 0.0, "bytes": 25e9},
    ]
    pk = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    r = bench.roofline_of(rows, pk, "measured", traffic_of=lambda k: 123.0 if k == "gemm_tcgen05" else None)
    # the two GEMM roles together (40 ms) outweigh the attention class (30 ms)
    assert r["kernel"] == "gemm_tcgen05" and r["launches"] == 160
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(40e12 / 0.040 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1400.0)
    assert r["traffic"] == 123.0
    # a memory-bound class is measured against the copy bandwidth
    r2 = bench.roofline_of(rows[3:], pk, "measured", traffic_of=lambda k: None)
    assert r2["bound"] == "hbm" and r2["achieved"] == pytest.approx(25e9 / 0.005 / 1e9)


def test_traffic_is_reported_only_for_the_profiled_source(tmp_path):
    bench = _bench()
    src = tmp_path / "k.cu"
    src.write_text("// kernel v1\n")
    digest = hashlib.sha256(src.read_bytes()).hexdigest()[:16]
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "demo_traffic.md").write_text(
        f"# demo\n\n- source: `k.cu@{digest}`\n- bytes_per_launch: 4096\n")
    bench.ROOT = str(tmp_path)
    assert bench.profile_traffic("demo") == 4096.0
    src.write_text("// kernel v2\n")
    assert bench.profile_traffic("demo") is None
    assert bench.profile_traffic("absent") is None


def test_flops_per_token_conventions():
    import synth
    bench = _bench()
    cfg = synth.WORKLOADS["d20"].model
    causal = bench.step_flops_per_token(cfg, 2048)
    palm = bench.step_flops_per_token(cfg, 2048, causal=False)
    assert causal / 1e9 == pytest.approx(2.823, abs=1e-3)
    # the PaLM convention counts the full T x T attention: 6 L H hd T more per token
    assert palm - causal == pytest.approx(6.0 * 20 * 10 * 128 * 2048)
