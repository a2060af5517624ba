"""The data-parallel step end to end (bwd_step_b200.dp.DataParallelStep): two
ranks, each a process on cuda:0 with the gloo backend, run the library step
on their half of the batch with the per-bucket events and the overlapped
gradient / loss averaging on a communication stream; the averaged result
must equal the float64 oracle on the whole batch.

The ranks' kernels never wait on one another: gloo stages every bucket
through host memory, so two processes may share one GPU here.  On several
GPUs the same class runs over NCCL."""
import os
import socket

import numpy as np
import pytest

import oracle
import synth
from harness import compare

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, T):
    wl = synth.WORKLOADS["tiny"]
    cfg = wl.model
    bits, w = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(synth.Workload("dp", cfg, T, B, "uniform"), seed=B * 100 + T)
    return cfg, bits, w, tok, tgt


def _rank_main(rank, world, port, out_dir, B, T):
    from datetime import timedelta
    import torch.distributed as dist
    from bwd_step_b200 import Model
    from bwd_step_b200.dp import DataParallelStep
    from harness import to_device_weights
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=120))
    try:
        torch.cuda.set_device(0)
        cfg, bits, w, tok, tgt = _inputs(B, T)
        per = B // world
        rows = slice(rank * per, (rank + 1) * per)
        m = Model(cfg.as_dict(), "bf16")
        W = to_device_weights(bits, w, "bf16")
        grads = torch.full((m.num_params(),), float("nan"), dtype=torch.float32, device="cuda")
        loss = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
        ws = torch.empty(m.workspace_bytes(per, T), dtype=torch.uint8, device="cuda")
        dp = DataParallelStep(m)
        tok_d = torch.from_numpy(np.ascontiguousarray(tok[rows])).cuda()
        tgt_d = torch.from_numpy(np.ascontiguousarray(tgt[rows])).cuda()
        for _ in range(2):  # the second step reuses the events and the communication stream
            dp.step(tok_d, tgt_d, W, grads, loss, ws)
        torch.cuda.synchronize()
        assert m.check() == 0
        dp.close()
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), grads=grads.cpu().numpy(), loss=loss.cpu().numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("B,T", [(2, 32), (4, 37)])
def test_two_ranks_average_to_the_whole_batch(tmp_path, B, T):
    import torch.multiprocessing as mp
    world = 2
    mp.start_processes(_rank_main, args=(world, _free_port(), str(tmp_path), B, T), nprocs=world, join=True,
                       start_method="spawn")
    cfg, bits, w, tok, tgt = _inputs(B, T)
    ref_loss, ref_g = oracle.step(cfg, w, tok, tgt)
    got = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert np.array_equal(got[0]["grads"], got[1]["grads"]) and got[0]["loss"][0] == got[1]["loss"][0]
    compare(cfg, float(got[0]["loss"][0]), got[0]["grads"], ref_loss, ref_g, "bf16")
