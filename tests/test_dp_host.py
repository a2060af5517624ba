"""Host logic of the data-parallel step (bwd_step_b200.dp) without a GPU: the
gradient buckets tile the flat layout in backward order, and two gloo ranks
average every bucket (and the loss) in bucket order."""
import json
import os
import socket

import numpy as np
import pytest

import synth
from bwd_step_b200.dp import average_buckets, grad_buckets_from_layout


@pytest.mark.parametrize("name", ["tiny", "d20"])
def test_buckets_tile_the_layout_in_backward_order(name):
    cfg = synth.WORKLOADS[name].model
    layout = synth.param_layout(cfg)
    b = grad_buckets_from_layout(layout, cfg.n_layer)
    assert len(b) == cfg.n_layer + 2
    n = synth.num_params(cfg)
    # LM head first, token embedding last, layers from last to first in between
    assert b[0] == (layout[-1][3], cfg.vocab * cfg.d_model)
    assert b[-1] == (0, cfg.vocab * cfg.d_model)
    assert [off for off, _ in b[1:-1]] == sorted((off for off, _ in b[1:-1]), reverse=True)
    covered = np.zeros(n, dtype=np.int8)
    for off, cnt in b:
        covered[off:off + cnt] += 1
    assert np.all(covered == 1)


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    from datetime import timedelta
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=timedelta(seconds=60))
    try:
        cfg = synth.WORKLOADS["tiny"].model
        buckets = grad_buckets_from_layout(synth.param_layout(cfg), cfg.n_layer)
        n = synth.num_params(cfg)
        # rank r's "gradients": a ramp scaled by (r + 1); its loss: 2 + r
        grads = torch.arange(n, dtype=torch.float32) * (rank + 1)
        loss = torch.tensor([2.0 + rank])
        order = []
        views = [grads[off:off + cnt] for off, cnt in buckets] + [loss]
        average_buckets(views, None, before=order.append)
        with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
            json.dump({"grads": grads.tolist(), "loss": float(loss.item()), "order": order}, f)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_average_every_bucket(tmp_path):
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    cfg = synth.WORKLOADS["tiny"].model
    n = synth.num_params(cfg)
    want = np.arange(n, dtype=np.float64) * 1.5  # mean of 1x and 2x the ramp
    for r in range(world):
        got = json.load(open(tmp_path / f"rank{r}.json"))
        assert np.allclose(np.asarray(got["grads"]), want, rtol=1e-6)
        assert got["loss"] == pytest.approx(2.5)
        assert got["order"] == list(range(cfg.n_layer + 3))  # every bucket, then the loss
