"""The library side of the data-parallel step on one GPU: the gradient buckets
agree with the flat layout, and the per-bucket events are recorded in bucket
order without changing the step's results."""
import numpy as np
import pytest

import synth
from harness import gpu_step, to_device_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import Model, NcError  # noqa: E402
from bwd_step_b200.dp import grad_buckets_from_layout  # noqa: E402


def _tiny():
    wl = synth.WORKLOADS["tiny"]
    cfg = wl.model
    bits, values = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(wl, seed=1)
    m = Model(cfg, "bf16")
    return cfg, m, to_device_weights(bits, values, "bf16"), tok, tgt


def test_grad_buckets_match_the_layout():
    cfg, m, _, _, _ = _tiny()
    assert m.grad_buckets() == grad_buckets_from_layout(synth.param_layout(cfg), cfg.n_layer)


def test_grad_events_are_recorded_in_bucket_order_and_change_nothing():
    cfg, m, W, tok, tgt = _tiny()
    loss0, g0 = gpu_step(m, W, tok, tgt)
    events = [torch.cuda.Event(enable_timing=True) for _ in m.grad_buckets()]
    for e in events:
        e.record()
    m.set_grad_events(events)
    loss1, g1 = gpu_step(m, W, tok, tgt)
    torch.cuda.synchronize()
    assert all(e.query() for e in events)
    t = [events[0].elapsed_time(e) for e in events]
    assert all(b >= a for a, b in zip(t, t[1:])), t
    assert loss1 == loss0 and np.array_equal(g0, g1)
    m.set_grad_events([])
    loss2, g2 = gpu_step(m, W, tok, tgt)
    assert loss2 == loss0 and np.array_equal(g0, g2)


def test_grad_events_reject_a_wrong_count():
    _, m, _, _, _ = _tiny()
    e = torch.cuda.Event()
    e.record()
    with pytest.raises(NcError):
        m.set_grad_events([e])
