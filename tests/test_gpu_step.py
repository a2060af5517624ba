"""GPU parity of the forward+backward step against the float64 oracle,
through the C ABI, plus the step's error paths.

Tolerances (per tensor relative L2 of every gradient, absolute loss):
bf16 path 3e-2 / 2e-2, fp32 debug path 1e-3 / 1e-4.
"""
import numpy as np
import pytest

import oracle
import synth
from harness import TOL, compare, gpu_step, to_device_weights

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

from bwd_step_b200 import Model, NcError  # noqa: E402
from bwd_step_b200 import _lib  # noqa: E402


def _cfg(base="tiny", **kw):
    d = synth.WORKLOADS[base].model.as_dict()
    d.update(kw)
    return synth.ModelConfig(**d)


def _case(cfg, B, T, precision, ids="uniform", seed_w=0, seed_t=1, std=0.02):
    bits, w = synth.make_weights(cfg, seed=seed_w, dtype=precision, std=std)
    tok, tgt = synth.make_tokens(synth.Workload("case", cfg, T, B, ids), seed=seed_t)
    return bits, w, tok, tgt


def _parity(cfg, B, T, precision, lm_head=None, chunk_rows=0, **kw):
    bits, w, tok, tgt = _case(cfg, B, T, precision, **kw)
    ref_loss, ref_g = oracle.step(cfg, w, tok, tgt)
    m = Model(cfg.as_dict(), precision)
    if lm_head is not None:
        m.set_lm_head(lm_head, chunk_rows)
    loss, g = gpu_step(m, to_device_weights(bits, w, precision), tok, tgt)
    return compare(cfg, loss, g, ref_loss, ref_g, precision)


@pytest.mark.parametrize("lm_head", ["fused", "materialised"])
@pytest.mark.parametrize("B,T,chunk_rows,std", [(2, 32, 0, 0.02), (3, 37, 128, 0.02), (2, 200, 128, 0.3),
                                                (1, 129, 0, 0.3)])
def test_lm_head_modes(lm_head, B, T, chunk_rows, std):
    # several row chunks (chunk_rows < B*T), a ragged last chunk, and weights that
    # drive the logits into the softcap's curved range
    _parity(_cfg(), B, T, "bf16", lm_head=lm_head, chunk_rows=chunk_rows, std=std, seed_w=B + T,
            seed_t=7 * T)


def test_lm_head_fused_needs_the_bf16_path():
    m = Model(_cfg().as_dict(), "fp32")
    with pytest.raises(NcError):
        m.set_lm_head("fused")
    m.set_lm_head("materialised", 256)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_tiny_workload(precision):
    wl = synth.WORKLOADS["tiny"]
    _parity(wl.model, wl.batch, wl.seq_len, precision)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("B,T", [(1, 1), (3, 37), (1, 200), (2, 129)])
def test_tiny_shapes_ragged(precision, B, T):
    _parity(_cfg(), B, T, precision, seed_t=B * 1000 + T)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("hd,H,nkv", [(32, 2, 1), (64, 2, 1), (128, 2, 1), (16, 4, 2)])
def test_head_dims(precision, hd, H, nkv):
    cfg = _cfg(head_dim=hd, n_head=H, n_kv_head=nkv, d_model=128)
    _parity(cfg, 2, 70, precision)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_large_weights_exercise_softcap(precision):
    # std 0.3 drives logits well into the tanh's curved range
    _parity(_cfg(), 2, 48, precision, std=0.3, seed_w=5)


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
def test_gpt2_124m_shape_one_row(precision):
    wl = synth.WORKLOADS["gpt2_124m"]
    _parity(wl.model, 1, wl.seq_len, precision, ids="zipf")


def _full_launch(name, patterns, min_layer=0):
    """The bench's launch configuration (full B and T) with `patterns` distinct
    seeded rows repeated in turn over the batch (row b holds pattern
    b % patterns), against the oracle on the distinct rows: repeating rows
    leaves the mean loss and the gradients unchanged (a pinned property), so
    a kernel that mixes batch rows or takes an offset from the wrong row
    fails here while the host cost stays that of `patterns` rows.  With
    min_layer > 0 only the LM head and the layers >= min_layer are compared."""
    wl = synth.WORKLOADS[name]
    cfg = wl.model
    assert wl.batch % patterns == 0
    bits, w = synth.make_weights(cfg, seed=0, dtype="bf16")
    tok_p, tgt_p = synth.make_tokens(wl, seed=1, batch=patterns)
    assert patterns == 1 or not np.array_equal(tok_p[0], tok_p[1])
    ref_loss, ref_g = oracle.step(cfg, w, tok_p, tgt_p, min_layer=min_layer)
    tok = np.tile(tok_p, (wl.batch // patterns, 1))
    tgt = np.tile(tgt_p, (wl.batch // patterns, 1))
    m = Model(cfg.as_dict(), "bf16")
    loss, g = gpu_step(m, to_device_weights(bits, w, "bf16"), tok, tgt)
    if min_layer == 0:
        return compare(cfg, loss, g, ref_loss, ref_g, "bf16")
    lay = [x for x in synth.param_layout(cfg) if x[0] == "wlm" or
           (x[0].startswith("h.") and int(x[0].split(".")[1]) >= min_layer)]
    tl, tg = TOL["bf16"]
    assert abs(loss - ref_loss) <= tl
    for n, r, c, off in lay:
        rel = np.linalg.norm(g[off:off + r * c] - ref_g[off:off + r * c]) / np.linalg.norm(ref_g[off:off + r * c])
        assert rel <= tg, (n, rel)


def test_gpt2_124m_full_launch_configuration_distinct_rows():
    _full_launch("gpt2_124m", patterns=8)


def test_d20_full_launch_configuration():
    _full_launch("d20", patterns=2)


def test_d30_full_launch_configuration_every_layer():
    _full_launch("d30", patterns=2)


def test_long_context_full_launch_configuration_every_layer():
    _full_launch("long", patterns=1)


def test_fp32_debug_full_d20_row():
    wl = synth.WORKLOADS["d20"]
    _parity(wl.model, 1, wl.seq_len, "fp32", ids="zipf")


def test_forward_logits_match_oracle():
    cfg = _cfg()
    for precision in ("bf16", "fp32"):
        bits, w, tok, tgt = _case(cfg, 2, 33, precision, std=0.2)
        ref = oracle.forward_logits(cfg, w, tok)
        m = Model(cfg.as_dict(), precision)
        out = torch.empty((2, 33, cfg.vocab), dtype=m.weight_dtype, device="cuda")
        ws = torch.empty(m.workspace_bytes(2, 33), dtype=torch.uint8, device="cuda")
        m.forward_logits(torch.from_numpy(tok).cuda(), to_device_weights(bits, w, precision), out, ws)
        assert m.check() == 0
        got = out.float().cpu().numpy()
        err = np.linalg.norm(got - ref) / np.linalg.norm(ref)
        assert err <= (2e-2 if precision == "bf16" else 1e-4), err
        assert np.all(np.abs(got) <= cfg.softcap)


def test_bitwise_deterministic():
    wl = synth.WORKLOADS["gpt2_124m"]
    cfg = wl.model
    bits, w, tok, tgt = _case(cfg, 2, 256, "bf16", ids="zipf")
    m = Model(cfg.as_dict(), "bf16")
    W = to_device_weights(bits, w, "bf16")
    l1, g1 = gpu_step(m, W, tok, tgt)
    l2, g2 = gpu_step(m, W, tok, tgt)
    assert l1 == l2
    assert np.array_equal(g1.view(np.uint32), g2.view(np.uint32))


def test_host_buffer_entry_point_equals_device_entry_point():
    cfg = _cfg()
    bits, w, tok, tgt = _case(cfg, 2, 40, "bf16")
    m = Model(cfg.as_dict(), "bf16")
    W = to_device_weights(bits, w, "bf16")
    l1, g1 = gpu_step(m, W, tok, tgt)
    grads = torch.empty(m.num_params(), dtype=torch.float32, device="cuda")
    ws = torch.empty(m.workspace_bytes(2, 40), dtype=torch.uint8, device="cuda")
    l2 = m.forward_backward_host(torch.from_numpy(tok).pin_memory(), torch.from_numpy(tgt).pin_memory(), W, grads,
                                 ws)
    assert l1 == l2
    assert np.array_equal(g1, grads.cpu().numpy())


def test_bad_token_is_reported_and_context_survives():
    cfg = _cfg()
    bits, w, tok, tgt = _case(cfg, 2, 16, "bf16")
    m = Model(cfg.as_dict(), "bf16")
    W = to_device_weights(bits, w, "bf16")
    bad = tok.copy()
    bad[1, 3] = cfg.vocab + 7
    grads = torch.empty(m.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = torch.empty(m.workspace_bytes(2, 16), dtype=torch.uint8, device="cuda")
    m.forward_backward(torch.from_numpy(bad).cuda(), torch.from_numpy(tgt).cuda(), W, grads, loss, ws)
    assert m.check() == _lib.NC_ERR_BAD_TOKEN
    badt = tgt.copy()
    badt[0, 0] = -1
    m.forward_backward(torch.from_numpy(tok).cuda(), torch.from_numpy(badt).cuda(), W, grads, loss, ws)
    assert m.check() == _lib.NC_ERR_BAD_TOKEN
    assert m.check() == 0  # cleared
    gpu_step(m, W, tok, tgt)


def test_bounded_wait_expires_without_trapping():
    cfg = _cfg()
    m = Model(cfg.as_dict(), "bf16")
    m.debug_expired_wait(200)
    assert m.check() == _lib.NC_ERR_DEVICE_TIMEOUT
    bits, w, tok, tgt = _case(cfg, 1, 8, "bf16")
    gpu_step(m, to_device_weights(bits, w, "bf16"), tok, tgt)


def test_argument_errors():
    cfg = _cfg()
    m = Model(cfg.as_dict(), "bf16")
    bits, w, tok, tgt = _case(cfg, 2, 16, "bf16")
    W = to_device_weights(bits, w, "bf16")
    grads = torch.empty(m.num_params(), dtype=torch.float32, device="cuda")
    loss = torch.empty(1, dtype=torch.float32, device="cuda")
    small = torch.empty(m.workspace_bytes(2, 16) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(NcError) as e:
        m.forward_backward(torch.from_numpy(tok).cuda(), torch.from_numpy(tgt).cuda(), W, grads, loss, small)
    assert e.value.code == _lib.NC_ERR_WORKSPACE_TOO_SMALL
    assert m.workspace_bytes(0, 16) == 0 and m.workspace_bytes(2, -1) == 0


@pytest.mark.parametrize("precision", ["bf16", "fp32"])
@pytest.mark.parametrize("base,B,T", [("tiny", 3, 37), ("gpt2_124m", 1, 256)])
def test_recompute_mlp_is_bitwise_equal_and_smaller(precision, base, B, T):
    """Recomputing relu(u), relu(u)^2 in the backward runs the same GEMM on the
    same operands: loss and gradients are bitwise those of the saved path, and
    the workspace shrinks by 2 * 2 (or 4) * B*T*F bytes per layer but one."""
    cfg = _cfg(base) if base == "tiny" else synth.WORKLOADS[base].model
    bits, w, tok, tgt = _case(cfg, B, T, precision, ids="zipf" if base != "tiny" else "uniform")
    m = Model(cfg.as_dict(), precision)
    W = to_device_weights(bits, w, precision)
    n0 = m.workspace_bytes(B, T)
    l0, g0 = gpu_step(m, W, tok, tgt)
    m.set_recompute(True)
    n1 = m.workspace_bytes(B, T)
    l1, g1 = gpu_step(m, W, tok, tgt)
    assert l1 == l0 and np.array_equal(g0.view(np.uint32), g1.view(np.uint32))
    es = 2 if precision == "bf16" else 4
    assert n0 - n1 >= 2 * es * B * T * cfg.mlp_mult * cfg.d_model * (cfg.n_layer - 1)
    if base == "tiny":
        ref_loss, ref_g = oracle.step(cfg, w, tok, tgt)
        compare(cfg, l1, g1, ref_loss, ref_g, precision)
