"""KV-cache inference through the C ABI (nc_prefill, nc_decode_step): the
logits after the prompt and after every decoded token must match the float64
oracle's full forward over the extended sequence (oracle.forward_logits, which
the oracle's own incremental decode is pinned to), within the forward-logits
tolerances of each precision."""
import numpy as np
import pytest

import oracle
import synth
from harness import to_device_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import Model, NcError  # noqa: E402

TOL = {"bf16": 2e-2, "fp32": 1e-4}


def _cfg(base="tiny", **kw):
    d = synth.WORKLOADS[base].model.as_dict()
    d.update(kw)
    return synth.ModelConfig(**d)


def _run(cfg, precision, B, T0, steps, T_max, std=0.02, seed=0):
    bits, w = synth.make_weights(cfg, seed=seed, dtype=precision, std=std)
    tok, _ = synth.make_tokens(synth.Workload("dec", cfg, T0 + steps, B, "uniform"), seed=seed + 1)
    full = oracle.forward_logits(cfg, w, tok)  # [B, T0 + steps, V]
    m = Model(cfg.as_dict(), precision)
    W = to_device_weights(bits, w, precision)
    cache = torch.full((m.kv_cache_bytes(B, T_max) // 2,), float("nan"), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(m.inference_workspace_bytes(B, T_max), dtype=torch.uint8, device="cuda")
    logits = torch.empty((B, cfg.vocab), dtype=m.weight_dtype, device="cuda")
    tok_d = torch.from_numpy(tok).cuda()
    m.prefill(tok_d[:, :T0].contiguous(), W, cache, T_max, logits, ws)
    assert m.check() == 0

    def close(t):
        got = logits.float().cpu().numpy().astype(np.float64)
        ref = full[:, t]
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= TOL[precision], (t, err)
        assert np.all(np.abs(got) <= cfg.softcap + 1e-3)

    close(T0 - 1)
    for i in range(steps):
        pos = T0 + i
        m.decode_step(tok_d[:, pos].contiguous(), pos, W, cache, T_max, logits, ws)
        assert m.check() == 0
        close(pos)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_tiny_prefill_then_decode(precision):
    _run(_cfg(), precision, B=2, T0=20, steps=6, T_max=40, std=0.3)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("hd,H,nkv", [(64, 4, 1), (128, 2, 1), (32, 4, 2)])
def test_head_dims_prefill_then_decode(precision, hd, H, nkv):
    _run(_cfg(head_dim=hd, n_head=H, n_kv_head=nkv, d_model=128), precision, B=3, T0=130, steps=4, T_max=200,
         std=0.1, seed=hd)


def test_gpt2_124m_shape_prefill_then_decode():
    _run(synth.WORKLOADS["gpt2_124m"].model, "bf16", B=2, T0=200, steps=3, T_max=256)


def test_decode_rejects_positions_outside_the_cache():
    cfg = _cfg()
    m = Model(cfg.as_dict(), "bf16")
    bits, w = synth.make_weights(cfg, seed=0, dtype="bf16")
    W = to_device_weights(bits, w, "bf16")
    cache = torch.empty(m.kv_cache_bytes(1, 8), dtype=torch.uint8, device="cuda")
    ws = torch.empty(m.inference_workspace_bytes(1, 8), dtype=torch.uint8, device="cuda")
    logits = torch.empty((1, cfg.vocab), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(NcError):
        m.decode_step(torch.zeros(1, dtype=torch.int32, device="cuda"), 8, W, cache, 8, logits, ws)
    with pytest.raises(NcError):
        m.prefill(torch.zeros((1, 9), dtype=torch.int32, device="cuda"), W, cache, 8, logits, ws)
