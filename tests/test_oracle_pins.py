"""Pins for the float64 CPU oracle: it is checked against facts that do not
come from the oracle itself (closed forms, invariants the architecture fixes,
library routines the special cases reduce to, finite differences), so a
dropped term, a wrong sign or index, or a transposed operand fails here.

Architecture items cited as "arch list, item n" are the bullets of the model
section of the nanochat announcement (vpshk.cn).
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
TINY = synth.WORKLOADS["tiny"]


def _cfg(**kw):
    base = TINY.model.as_dict()
    base.update(kw)
    return synth.ModelConfig(**base)


def _tiny_inputs(seed_w=0, seed_t=1, dtype="bf16", cfg=None, B=None, T=None):
    cfg = cfg or TINY.model
    _, w = synth.make_weights(cfg, seed=seed_w, dtype=dtype)
    wl = synth.Workload("t", cfg, T or TINY.seq_len, B or TINY.batch, "uniform")
    tok, tgt = synth.make_tokens(wl, seed=seed_t)
    return cfg, w.astype(np.float64), tok, tgt


# ---------------------------------------------------------------- RMSNorm
def test_rmsnorm_unit_rms():
    """Parameter-free RMSNorm (arch list, item 7): rms(y) = sqrt(ms/(ms+eps))."""
    rng = np.random.default_rng(3)
    for scale in (1e-3, 0.02, 1.0, 50.0):
        x = rng.standard_normal((7, 96)) * scale
        y, r = oracle.rmsnorm(x)
        ms = np.mean(x * x, axis=-1)
        np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)),
                                   np.sqrt(ms / (ms + oracle.RMS_EPS)), rtol=1e-13)
        if scale >= 1.0:
            np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-6)
        np.testing.assert_allclose(y / x, np.broadcast_to(r, x.shape), rtol=1e-13)


def test_rmsnorm_backward_finite_difference():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 48))
    g = rng.standard_normal((5, 48))
    y, r = oracle.rmsnorm(x)
    dx = oracle.rmsnorm_backward(g, y, r)
    h = 1e-6
    fd = np.empty_like(x)
    for idx in np.ndindex(*x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += h
        xm[idx] -= h
        fd[idx] = (np.sum(g * oracle.rmsnorm(xp)[0]) - np.sum(g * oracle.rmsnorm(xm)[0])) / (2 * h)
    np.testing.assert_allclose(dx, fd, rtol=1e-7, atol=1e-9)


# ---------------------------------------------------------------- RoPE
def test_rope_preserves_pair_norms():
    """Rotary embedding (arch list, item 2) rotates each (j, j+hd/2) pair."""
    rng = np.random.default_rng(5)
    T, nh, hd = 11, 3, 16
    cos, sin = oracle.rope_tables(T, hd, 10000.0)
    x = rng.standard_normal((T, nh, hd))
    y = oracle.rope(x, cos, sin)
    h = hd // 2
    np.testing.assert_allclose(x[..., :h] ** 2 + x[..., h:] ** 2,
                               y[..., :h] ** 2 + y[..., h:] ** 2, rtol=1e-13)
    np.testing.assert_allclose(y[0], x[0], rtol=0, atol=0)  # position 0: identity


def test_rope_is_complex_rotation_with_published_frequencies():
    """Pair j as a complex number x_j + i x_{j+hd/2} is multiplied by
    exp(i * pos * base^(-2j/hd)): the textbook rotary form, which pins the
    pairing, the sign of the rotation and the frequency index."""
    rng = np.random.default_rng(6)
    T, hd, base = 9, 32, 10000.0
    cos, sin = oracle.rope_tables(T, hd, base)
    x = rng.standard_normal((T, 1, hd))
    y = oracle.rope(x, cos, sin)[:, 0]
    z = x[:, 0, :hd // 2] + 1j * x[:, 0, hd // 2:]
    pos = np.arange(T)[:, None]
    freq = np.array([base ** (-2.0 * j / hd) for j in range(hd // 2)])
    zr = z * np.exp(1j * pos * freq[None, :])
    np.testing.assert_allclose(y[:, :hd // 2], zr.real, atol=1e-13)
    np.testing.assert_allclose(y[:, hd // 2:], zr.imag, atol=1e-13)
    assert freq[0] == 1.0 and abs(freq[1] - base ** (-2 / hd)) < 1e-18


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(7)
    hd, T = 16, 40
    cos, sin = oracle.rope_tables(T, hd, 10000.0)
    q = rng.standard_normal(hd)
    k = rng.standard_normal(hd)
    Q = oracle.rope(np.broadcast_to(q, (T, 1, hd)).copy(), cos, sin)[:, 0]
    K = oracle.rope(np.broadcast_to(k, (T, 1, hd)).copy(), cos, sin)[:, 0]
    for m, n, delta in [(5, 2, 7), (3, 3, 30), (0, 9, 11), (20, 1, 19)]:
        assert abs(Q[m] @ K[n] - Q[m + delta] @ K[n + delta]) < 1e-12


def test_rope_commutes_with_qk_norm():
    """QK-norm (arch list, item 3) and RoPE commute: norm(R q) = R norm(q)."""
    rng = np.random.default_rng(8)
    T, nh, hd = 13, 4, 16
    cos, sin = oracle.rope_tables(T, hd, 10000.0)
    x = rng.standard_normal((T, nh, hd)) * 3.0
    a = oracle.rmsnorm(oracle.rope(x, cos, sin))[0]
    b = oracle.rope(oracle.rmsnorm(x)[0], cos, sin)
    np.testing.assert_allclose(a, b, atol=1e-14)


def test_rope_backward_is_adjoint():
    rng = np.random.default_rng(9)
    T, nh, hd = 6, 2, 16
    cos, sin = oracle.rope_tables(T, hd, 500.0)
    x = rng.standard_normal((T, nh, hd))
    g = rng.standard_normal((T, nh, hd))
    assert abs(np.sum(oracle.rope(x, cos, sin) * g) - np.sum(x * oracle.rope_backward(g, cos, sin))) < 1e-12


# ---------------------------------------------------------------- attention
def _sdpa(q, k, v):
    """torch's scaled-dot-product attention, float64, causal; kv heads
    repeated across query heads (MQA as MHA with copied K/V)."""
    T, H, hd = q.shape
    rep = H // k.shape[1]
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(rep, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(rep, 0)[None]
    return qt, kt, vt


@pytest.mark.parametrize("T,H,nkv,hd", [(1, 4, 1, 16), (17, 4, 1, 16), (33, 3, 1, 8),
                                        (12, 1, 1, 32), (10, 4, 2, 8), (8, 2, 2, 4)])
def test_attention_matches_library_sdpa(T, H, nkv, hd):
    """Causal MQA (arch list, item 9) equals torch SDPA with K/V copied to every head."""
    rng = np.random.default_rng(T * 100 + H)
    q = rng.standard_normal((T, H, hd))
    k = rng.standard_normal((T, nkv, hd))
    v = rng.standard_normal((T, nkv, hd))
    o = oracle.attention(q, k, v)
    qt, kt, vt = _sdpa(q, k, v)
    qt.requires_grad_(True)
    kt0 = torch.from_numpy(k).permute(1, 0, 2).clone().requires_grad_(True)
    vt0 = torch.from_numpy(v).permute(1, 0, 2).clone().requires_grad_(True)
    rep = H // nkv
    ref = F.scaled_dot_product_attention(qt, kt0.repeat_interleave(rep, 0)[None],
                                         vt0.repeat_interleave(rep, 0)[None], is_causal=True)
    np.testing.assert_allclose(o, ref[0].permute(1, 0, 2).detach().numpy(), atol=1e-13)
    g = rng.standard_normal(o.shape)
    ref.backward(torch.from_numpy(g).permute(1, 0, 2)[None])
    dq, dk, dv = oracle.attention_backward(q, k, v, g)
    np.testing.assert_allclose(dq, qt.grad[0].permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dk, kt0.grad.permute(1, 0, 2).numpy(), atol=1e-12)
    np.testing.assert_allclose(dv, vt0.grad.permute(1, 0, 2).numpy(), atol=1e-12)


def test_attention_single_position_returns_v():
    rng = np.random.default_rng(10)
    q = rng.standard_normal((1, 5, 8))
    k = rng.standard_normal((1, 1, 8))
    v = rng.standard_normal((1, 1, 8))
    o = oracle.attention(q, k, v)
    np.testing.assert_array_equal(o, np.broadcast_to(v, o.shape))


# ---------------------------------------------------------------- whole model
def test_causal_invariance_whole_model():
    """Changing tokens after position t leaves every loss at positions <= t
    exactly unchanged (causal mask, arch list item 9)."""
    cfg, w, tok, tgt = _tiny_inputs()
    base = oracle.position_losses(cfg, w, tok, tgt)
    rng = np.random.default_rng(11)
    for t in (0, 5, 20, 30):
        tok2 = tok.copy()
        tok2[:, t + 1:] = rng.integers(0, cfg.vocab, size=tok2[:, t + 1:].shape)
        tgt2 = tgt.copy()
        tgt2[:, t + 1:] = rng.integers(0, cfg.vocab, size=tgt2[:, t + 1:].shape)
        pl = oracle.position_losses(cfg, w, tok2, tgt2)
        np.testing.assert_array_equal(pl[:, :t + 1], base[:, :t + 1])
        assert not np.array_equal(pl[:, t + 1:], base[:, t + 1:])


def test_softcap_bound_and_limit():
    """|z| < c for the tanh softcap (arch list, item 10); c -> inf gives z = l."""
    rng = np.random.default_rng(12)
    l = rng.uniform(-249.0, 249.0, size=10000)
    z = oracle.softcap(l, 15.0)
    assert np.all(np.abs(z) < 15.0)
    l2 = rng.standard_normal(1000) * 30
    np.testing.assert_allclose(oracle.softcap(l2, 1e9), l2, rtol=1e-12)


def _golden_lnv():
    vals = {}
    with open(os.path.join(GOLDEN, "uniform_logits_loss.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                V, val = line.split()
                vals[int(V)] = float(val)
    return vals


def test_zero_lm_head_gives_ln_v_and_closed_form_gradient():
    """Wlm = 0 makes every softcapped logit 0, so the loss is ln V exactly and
    dWlm[v] = (1/M) sum_m (1/V - [target_m = v]) xf_m, with xf the final-norm
    output.  ln V values come from the golden fixture."""
    cfg, w, tok, tgt = _tiny_inputs()
    P = oracle.views(cfg, w)
    P["wlm"][:] = 0.0
    loss, g = oracle.step(cfg, w, tok, tgt)
    lnv = _golden_lnv()
    assert abs(loss - lnv[cfg.vocab]) < 1e-13
    assert abs(math.log(cfg.vocab) - lnv[cfg.vocab]) < 1e-15
    # final-norm output from the independent torch forward below
    xf = _torch_forward(cfg, torch.from_numpy(w), tok, tgt, return_xf=True).numpy()
    M = tok.size
    onehot = np.zeros((M, cfg.vocab))
    onehot[np.arange(M), tgt.reshape(-1)] = 1.0
    expect = ((1.0 / cfg.vocab - onehot).T @ xf.reshape(M, -1)) / M
    np.testing.assert_allclose(oracle.views(cfg, g)["wlm"], expect, atol=1e-15, rtol=1e-11)
    # d(loss)/d(xf) = 0 because Wlm = 0: all other gradients vanish too
    G = oracle.views(cfg, g)
    assert np.all(G["wte"] == 0) and np.all(G["h.0.wq"] == 0)


def _torch_forward(cfg, W, tok, tgt, return_xf=False):
    """Independent float64 torch forward of the same model (not the oracle's
    code): library rms_norm, complex-number RoPE, library SDPA and
    cross_entropy.  Its autograd gradients are the library reduction the
    oracle's hand-written backward is checked against."""
    d, H, nkv, hd = cfg.d_model, cfg.n_head, cfg.n_kv_head, cfg.head_dim
    B, T = tok.shape
    P = {name: W[off:off + r * c].view(r, c) for name, r, c, off in synth.param_layout(cfg)}
    eps = 1e-6
    tok_t = torch.from_numpy(tok.astype(np.int64))
    theta = cfg.rope_base ** (-torch.arange(0, hd, 2, dtype=torch.float64) / hd)
    ang = torch.arange(T, dtype=torch.float64)[:, None] * theta[None, :]
    rot = torch.polar(torch.ones_like(ang), ang)

    def rot_emb(t):
        zc = torch.complex(t[..., :hd // 2], t[..., hd // 2:]) * rot[None, :, None, :]
        return torch.cat([zc.real, zc.imag], dim=-1)

    x = F.rms_norm(P["wte"][tok_t], (d,), eps=eps)
    for i in range(cfg.n_layer):
        a = F.rms_norm(x, (d,), eps=eps)
        q = (a @ P[f"h.{i}.wq"].T).view(B, T, H, hd)
        k = (a @ P[f"h.{i}.wk"].T).view(B, T, nkv, hd)
        v = (a @ P[f"h.{i}.wv"].T).view(B, T, nkv, hd)
        q = rot_emb(F.rms_norm(q, (hd,), eps=eps)).transpose(1, 2)
        k = rot_emb(F.rms_norm(k, (hd,), eps=eps)).transpose(1, 2).repeat_interleave(H // nkv, 1)
        v = v.transpose(1, 2).repeat_interleave(H // nkv, 1)
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True)
        x = x + o.transpose(1, 2).reshape(B, T, H * hd) @ P[f"h.{i}.wo"].T
        m = F.rms_norm(x, (d,), eps=eps)
        x = x + F.relu(m @ P[f"h.{i}.wfc"].T).square() @ P[f"h.{i}.wproj"].T
    xf = F.rms_norm(x, (d,), eps=eps)
    if return_xf:
        return xf.detach()
    z = cfg.softcap * torch.tanh((xf @ P["wlm"].T) / cfg.softcap)
    return F.cross_entropy(z.reshape(B * T, -1), torch.from_numpy(tgt.astype(np.int64)).reshape(-1))


@pytest.mark.parametrize("variant", ["tiny", "tiny_gqa", "tiny_hd32"])
def test_oracle_matches_library_autograd(variant):
    cfg = {"tiny": TINY.model, "tiny_gqa": _cfg(n_kv_head=2),
           "tiny_hd32": _cfg(n_head=2, head_dim=32, rope_base=500.0, softcap=5.0)}[variant]
    cfg, w, tok, tgt = _tiny_inputs(cfg=cfg, seed_w=21)
    # larger weights so the softcap and relu^2 are exercised away from linear regimes
    w = w * 10.0
    loss, g = oracle.step(cfg, w, tok, tgt)
    W = torch.from_numpy(w.copy()).requires_grad_(True)
    ref = _torch_forward(cfg, W, tok, tgt)
    ref.backward()
    assert abs(loss - ref.item()) < 1e-12 * max(1.0, abs(loss))
    G, R = oracle.views(cfg, g), oracle.views(cfg, W.grad.numpy())
    for name in G:
        num = np.linalg.norm(G[name] - R[name])
        den = np.linalg.norm(R[name])
        assert num <= 1e-10 * den + 1e-300, (name, num, den)


def test_oracle_backward_finite_differences():
    """Central differences of the oracle's own forward, h = 1e-5, 50 random
    entries per tensor: relative error of the sampled vector <= 1e-6."""
    cfg, w, tok, tgt = _tiny_inputs(seed_w=31)
    w = w * 8.0
    loss, g = oracle.step(cfg, w, tok, tgt)
    rng = np.random.default_rng(13)
    h = 1e-5

    def f(wv):
        return oracle.position_losses(cfg, wv, tok, tgt).mean()

    assert abs(f(w) - loss) < 1e-13
    for name, r, c, off in oracle.layout(cfg)[0]:
        n = r * c
        if name == "wte":
            rows = np.unique(tok)
            cand = (rows[:, None] * c + np.arange(c)[None, :]).reshape(-1)
            pick = rng.choice(cand, size=50, replace=False) + off
        else:
            pick = rng.choice(n, size=min(50, n), replace=False) + off
        fd = np.empty(len(pick))
        for j, p in enumerate(pick):
            wp, wm = w.copy(), w.copy()
            wp[p] += h
            wm[p] -= h
            fd[j] = (f(wp) - f(wm)) / (2 * h)
        an = g[pick]
        assert np.linalg.norm(fd - an) <= 1e-6 * np.linalg.norm(an), name


def test_duplicate_rows_leave_loss_and_grads_unchanged():
    cfg, w, tok, tgt = _tiny_inputs(seed_w=41)
    loss, g = oracle.step(cfg, w, tok, tgt)
    loss2, g2 = oracle.step(cfg, w, np.concatenate([tok, tok]), np.concatenate([tgt, tgt]))
    assert abs(loss - loss2) < 1e-13
    np.testing.assert_allclose(g2, g, rtol=1e-11, atol=1e-17)


def test_unused_embedding_rows_get_zero_gradient():
    cfg, w, tok, tgt = _tiny_inputs(seed_w=51)
    _, g = oracle.step(cfg, w, tok, tgt)
    G = oracle.views(cfg, g)["wte"]
    used = np.zeros(cfg.vocab, dtype=bool)
    used[np.unique(tok)] = True
    assert np.all(G[~used] == 0.0)
    assert np.all(np.linalg.norm(G[used], axis=1) > 0)


def test_layouts_agree():
    for wl in synth.WORKLOADS.values():
        a = [(n, r, c, o) for n, r, c, o in synth.param_layout(wl.model)]
        b, total = oracle.layout(wl.model)
        assert a == b and total == synth.num_params(wl.model)


def test_tiny_golden_regression():
    """Loss and gradient fingerprints of the tiny workload, written by
    tests/golden/make_golden.py from the oracle alone."""
    path = os.path.join(GOLDEN, "tiny_step.txt")
    vals = {}
    with open(path) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                k, v = line.split()
                vals[k] = float(v)
    _, wb = synth.make_weights(TINY.model, seed=0, dtype="bf16")
    tok, tgt = synth.make_tokens(TINY, seed=1)
    loss, g = oracle.step(TINY.model, wb, tok, tgt)
    assert abs(loss - vals["loss"]) < 1e-12
    G = oracle.views(TINY.model, g)
    for name in G:
        assert abs(np.linalg.norm(G[name]) - vals["norm." + name]) <= 1e-12 * vals["norm." + name] + 1e-300


def test_truncated_backward_matches_full_on_the_layers_it_keeps():
    cfg, w, tok, tgt = _tiny_inputs(seed_w=61)
    loss, g = oracle.step(cfg, w, tok, tgt)
    loss1, g1 = oracle.step(cfg, w, tok, tgt, min_layer=1)
    assert loss1 == loss
    G, G1 = oracle.views(cfg, g), oracle.views(cfg, g1)
    for name in G:
        if name.startswith("h.1.") or name == "wlm":
            np.testing.assert_array_equal(G1[name], G[name])
        else:
            assert np.all(G1[name] == 0)


# ---------------------------------------------------------------- forward logits
def test_forward_logits_match_library_forward():
    """oracle.forward_logits equals the softcapped LM-head output of the
    independent torch float64 forward (library rms_norm, complex RoPE, SDPA):
    a swapped weight, a dropped softcap or a missing final norm fails here."""
    cfg, w, tok, tgt = _tiny_inputs(seed_w=71)
    w = w * 10.0
    oracle.views(cfg, w)["wlm"][:] *= 5.0  # drive the logits into the curved range of the tanh
    z = oracle.forward_logits(cfg, w, tok)
    xf = _torch_forward(cfg, torch.from_numpy(w), tok, tgt, return_xf=True).numpy()
    wlm = oracle.views(cfg, w)["wlm"]
    expect = cfg.softcap * np.tanh((xf @ wlm.T) / cfg.softcap)
    assert z.shape == (tok.shape[0], tok.shape[1], cfg.vocab)
    np.testing.assert_allclose(z, expect, rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(z)) > 0.5 * cfg.softcap  # the cap is exercised


def test_forward_logits_log_softmax_gives_position_losses():
    """-log softmax(z)[target] of the returned logits is the per-position loss
    (whose LM head is the separately pinned lm_head_loss)."""
    cfg, w, tok, tgt = _tiny_inputs(seed_w=72)
    w = w * 5.0
    z = oracle.forward_logits(cfg, w, tok)
    zmax = z.max(axis=-1, keepdims=True)
    lse = zmax[..., 0] + np.log(np.exp(z - zmax).sum(axis=-1))
    ce = lse - np.take_along_axis(z, tgt[..., None], axis=-1)[..., 0]
    np.testing.assert_allclose(ce, oracle.position_losses(cfg, w, tok, tgt), rtol=1e-12, atol=1e-13)


def test_forward_logits_zero_lm_head_are_zero():
    """Wlm = 0 gives z = c tanh(0) = 0 exactly at every position."""
    cfg, w, tok, _ = _tiny_inputs(seed_w=73)
    oracle.views(cfg, w)["wlm"][:] = 0.0
    z = oracle.forward_logits(cfg, w, tok)
    assert np.all(z == 0.0)
