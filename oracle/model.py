"""Float64 CPU oracle of the pretraining forward+backward step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
links this module: only the tests, the smoke check in ``__graft_entry__`` and
the CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA
library; the two meet only on the seeded arrays from ``synth``.

What it computes (the model of the nanochat announcement, vpshk.cn, section
on the model architecture, whose bullet list is cited below as "arch list"):

* a dense decoder stack, Llama-like but simpler (arch list, item 1);
* token embedding then a parameter-free RMSNorm of it (items 4, 5, 7);
* per block, pre-norm residual attention then pre-norm residual MLP;
* bias-free linears y = x W^T (item 8);
* multi-query attention: H query heads share n_kv key/value heads (item 9);
* rotary position embedding as the only positional signal (item 2);
* QK-norm: parameter-free RMSNorm of every q and k head vector (item 3);
* relu(u)^2 MLP with hidden width mlp_mult * d (item 6);
* a final RMSNorm, then an untied LM head (item 4);
* a tanh logit softcap z = c * tanh(l / c) (item 10);
* mean next-token cross-entropy over all B*T positions, and the gradient of
  that mean with respect to every weight matrix.

Readings where the pages are silent (each is also listed in the design notes):
RMSNorm eps = 1e-6; a final norm before the LM head; RoPE pairs (j, j+hd/2)
with theta_j = base**(-2j/hd), angle = position * theta_j, rotation
(x1 cos - x2 sin, x1 sin + x2 cos), positions 0..T-1 per row; QK-norm before
RoPE (the two commute); scale 1/sqrt(hd); causal mask j <= i within a row;
kv head of query head h is h // (H / n_kv); relu^2 derivative 2*relu(u);
no dropout, no biases, no ignore index, natural log.

Everything runs in float64 on whatever weights it is given (bf16 weights
are passed exactly, upcast).  Rows of the batch are processed one at a time
so host memory stays bounded; attention is the naive full T x T product per
head; the LM head is evaluated over chunks of positions.
"""
from __future__ import annotations

import math
import numpy as np

RMS_EPS = 1e-6


# ----------------------------------------------------------------------------
# parameter views
# ----------------------------------------------------------------------------
def layout(cfg):
    """(name, rows, cols, offset) in the flat storage order used by both sides."""
    d, hd = cfg.d_model, cfg.head_dim
    F = cfg.mlp_mult * d
    out, off = [], 0
    for name, r, c in ([("wte", cfg.vocab, d)]
                       + [x for i in range(cfg.n_layer) for x in (
                           (f"h.{i}.wq", cfg.n_head * hd, d),
                           (f"h.{i}.wk", cfg.n_kv_head * hd, d),
                           (f"h.{i}.wv", cfg.n_kv_head * hd, d),
                           (f"h.{i}.wo", d, cfg.n_head * hd),
                           (f"h.{i}.wfc", F, d),
                           (f"h.{i}.wproj", d, F))]
                       + [("wlm", cfg.vocab, d)]):
        out.append((name, r, c, off))
        off += r * c
    return out, off


def views(cfg, flat):
    """Dict name -> 2-D view of a flat parameter (or gradient) vector."""
    lay, n = layout(cfg)
    assert flat.size == n, (flat.size, n)
    return {name: flat[off:off + r * c].reshape(r, c) for name, r, c, off in lay}


# ----------------------------------------------------------------------------
# building blocks
# ----------------------------------------------------------------------------
def rmsnorm(x):
    """Parameter-free RMSNorm over the last axis (arch list, item 7).

    y = x * r with r = (mean(x^2) + eps)^(-1/2).  Returns (y, r), r keeps the
    reduced axis as size 1.
    """
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + RMS_EPS)
    return x * r, r


def rmsnorm_backward(dy, y, r):
    """Gradient of the parameter-free RMSNorm: dx = r * (dy - y * mean(dy*y))."""
    return r * (dy - y * np.mean(dy * y, axis=-1, keepdims=True))


def rope_tables(T, hd, base):
    """cos/sin [T, hd/2] of angle pos * base**(-2j/hd) (arch list, item 2)."""
    j = np.arange(hd // 2, dtype=np.float64)
    theta = base ** (-2.0 * j / hd)
    ang = np.arange(T, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang), np.sin(ang)


def rope(x, cos, sin):
    """Rotate each (j, j+hd/2) pair of x [T, n_heads, hd] by its position's angle."""
    h = x.shape[-1] // 2
    x1, x2 = x[..., :h], x[..., h:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([x1 * c - x2 * s, x1 * s + x2 * c], axis=-1)


def rope_backward(dy, cos, sin):
    """Adjoint of rope: the inverse rotation applied to the gradient."""
    h = dy.shape[-1] // 2
    d1, d2 = dy[..., :h], dy[..., h:]
    c, s = cos[:, None, :], sin[:, None, :]
    return np.concatenate([d1 * c + d2 * s, -d1 * s + d2 * c], axis=-1)


def _kv_of(h, H, nkv):
    return h // (H // nkv)


def _causal_probs(qh, kg):
    """Softmax of the causal, 1/sqrt(hd)-scaled scores of one head: [T, T]."""
    T, hd = qh.shape
    s = (qh @ kg.T) / math.sqrt(hd)
    s = np.where(np.tril(np.ones((T, T), dtype=bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def attention(q, k, v):
    """Causal multi-query attention (arch list, item 9).

    q [T, H, hd]; k, v [T, n_kv, hd].  Query head h reads kv head
    h // (H / n_kv); key j is visible to query i iff j <= i.  Returns o [T, H, hd].
    """
    T, H, hd = q.shape
    nkv = k.shape[1]
    o = np.empty_like(q)
    for h in range(H):
        g = _kv_of(h, H, nkv)
        o[:, h] = _causal_probs(q[:, h], k[:, g]) @ v[:, g]
    return o


def attention_backward(q, k, v, do):
    """Gradients of `attention` (probabilities are recomputed, not stored).

    dv_g = sum_h P_h^T do_h;  dS = P * (dP - rowsum(dP * P)) with dP = do v^T;
    dq_h = dS k_g / sqrt(hd);  dk_g = sum_h dS^T q_h / sqrt(hd).
    """
    T, H, hd = q.shape
    nkv = k.shape[1]
    dq = np.empty_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    sc = 1.0 / math.sqrt(hd)
    for h in range(H):
        g = _kv_of(h, H, nkv)
        p = _causal_probs(q[:, h], k[:, g])
        dv[:, g] += p.T @ do[:, h]
        dp = do[:, h] @ v[:, g].T
        ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
        dq[:, h] = (ds @ k[:, g]) * sc
        dk[:, g] += (ds.T @ q[:, h]) * sc
    return dq, dk, dv


def softcap(l, c):
    """Logit softcap z = c * tanh(l / c) (arch list, item 10)."""
    return c * np.tanh(l / c)


def lm_head_loss(xf, wlm, targets, c, grad_scale, chunk=256, want_grad=True):
    """Untied LM head + softcap + cross-entropy for one row of positions.

    xf [T, d]; wlm [V, d]; targets [T].  Returns (per-position losses [T],
    dxf [T, d], dwlm [V, d]) where the gradients are of grad_scale * sum(losses).
    loss_t = logsumexp(z_t) - z_t[target_t]; dz = grad_scale*(softmax(z) - onehot);
    dl = dz * (1 - (z/c)^2) since d/dl [c tanh(l/c)] = 1 - tanh^2(l/c).
    """
    T = xf.shape[0]
    losses = np.empty(T)
    dxf = np.zeros_like(xf) if want_grad else None
    dwlm = np.zeros_like(wlm) if want_grad else None
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        rows = np.arange(t1 - t0)
        tg = targets[t0:t1]
        z = softcap(xf[t0:t1] @ wlm.T, c)
        zmax = z.max(axis=1, keepdims=True)
        lse = zmax[:, 0] + np.log(np.sum(np.exp(z - zmax), axis=1))
        losses[t0:t1] = lse - z[rows, tg]
        if want_grad:
            p = np.exp(z - lse[:, None])
            p[rows, tg] -= 1.0
            dl = grad_scale * p * (1.0 - (z / c) ** 2)
            dxf[t0:t1] = dl @ wlm
            dwlm += dl.T @ xf[t0:t1]
    return losses, dxf, dwlm


# ----------------------------------------------------------------------------
# the model, one batch row at a time
# ----------------------------------------------------------------------------
def _row_forward(cfg, P, idx, cos, sin, keep):
    T = idx.shape[0]
    H, nkv, hd, L = cfg.n_head, cfg.n_kv_head, cfg.head_dim, cfg.n_layer
    e = P["wte"][idx]
    x, r0 = rmsnorm(e)
    saved = {"x0": x, "r0": r0, "layers": []}
    for i in range(L):
        wq, wk, wv = P[f"h.{i}.wq"], P[f"h.{i}.wk"], P[f"h.{i}.wv"]
        a, r1 = rmsnorm(x)
        qn, rq = rmsnorm((a @ wq.T).reshape(T, H, hd))
        kn, rk = rmsnorm((a @ wk.T).reshape(T, nkv, hd))
        v = (a @ wv.T).reshape(T, nkv, hd)
        qr, kr = rope(qn, cos, sin), rope(kn, cos, sin)
        o = attention(qr, kr, v).reshape(T, H * hd)
        x = x + o @ P[f"h.{i}.wo"].T
        m, r2 = rmsnorm(x)
        u = m @ P[f"h.{i}.wfc"].T
        hh = np.maximum(u, 0.0) ** 2
        x = x + hh @ P[f"h.{i}.wproj"].T
        if keep:
            saved["layers"].append(dict(a=a, r1=r1, qn=qn, rq=rq, kn=kn, rk=rk, v=v,
                                        qr=qr, kr=kr, o=o, m=m, r2=r2, u=u, h=hh))
    xf, rf = rmsnorm(x)
    saved["xf"], saved["rf"] = xf, rf
    return saved


def _row_backward(cfg, P, G, idx, saved, dxf, cos, sin, min_layer=0):
    T = idx.shape[0]
    H, nkv, hd = cfg.n_head, cfg.n_kv_head, cfg.head_dim
    dx = rmsnorm_backward(dxf, saved["xf"], saved["rf"])
    for i in reversed(range(min_layer, cfg.n_layer)):
        s = saved["layers"][i]
        # x_out = x_mid + relu(m Wfc^T)^2 Wproj^T
        dh = dx @ P[f"h.{i}.wproj"]
        G[f"h.{i}.wproj"] += dx.T @ s["h"]
        du = dh * 2.0 * np.maximum(s["u"], 0.0)
        G[f"h.{i}.wfc"] += du.T @ s["m"]
        dx = dx + rmsnorm_backward(du @ P[f"h.{i}.wfc"], s["m"], s["r2"])
        # x_mid = x_in + attn(...) Wo^T
        do = dx @ P[f"h.{i}.wo"]
        G[f"h.{i}.wo"] += dx.T @ s["o"]
        dqr, dkr, dv = attention_backward(s["qr"], s["kr"], s["v"], do.reshape(T, H, hd))
        dq = rmsnorm_backward(rope_backward(dqr, cos, sin), s["qn"], s["rq"]).reshape(T, H * hd)
        dk = rmsnorm_backward(rope_backward(dkr, cos, sin), s["kn"], s["rk"]).reshape(T, nkv * hd)
        dv = dv.reshape(T, nkv * hd)
        a = s["a"]
        G[f"h.{i}.wq"] += dq.T @ a
        G[f"h.{i}.wk"] += dk.T @ a
        G[f"h.{i}.wv"] += dv.T @ a
        da = dq @ P[f"h.{i}.wq"] + dk @ P[f"h.{i}.wk"] + dv @ P[f"h.{i}.wv"]
        dx = dx + rmsnorm_backward(da, a, s["r1"])
    if min_layer > 0:
        return
    de = rmsnorm_backward(dx, saved["x0"], saved["r0"])
    np.add.at(G["wte"], idx, de)


def step(cfg, weights, tokens, targets, min_layer=0):
    """Mean cross-entropy loss and the gradient of every weight.

    weights: flat vector in `layout` order (any float dtype; used as float64).
    tokens, targets: int [B, T].  Returns (loss: float, grads: flat float64).
    min_layer > 0 stops the backward after layer min_layer (used to bound the
    cost on large shapes): gradients of layers below it and of wte stay zero.
    """
    tokens = np.asarray(tokens)
    targets = np.asarray(targets)
    B, T = tokens.shape
    if tokens.min() < 0 or tokens.max() >= cfg.vocab:
        raise ValueError("token id out of range")
    W = np.asarray(weights, dtype=np.float64)
    P = views(cfg, W)
    grads = np.zeros_like(W)
    G = views(cfg, grads)
    cos, sin = rope_tables(T, cfg.head_dim, cfg.rope_base)
    scale = 1.0 / (B * T)
    total = 0.0
    for b in range(B):
        saved = _row_forward(cfg, P, tokens[b], cos, sin, keep=True)
        losses, dxf, dwlm = lm_head_loss(saved["xf"], P["wlm"], targets[b], cfg.softcap, scale)
        G["wlm"] += dwlm
        total += losses.sum()
        _row_backward(cfg, P, G, tokens[b], saved, dxf, cos, sin, min_layer)
    return total * scale, grads


def position_losses(cfg, weights, tokens, targets):
    """Per-position cross-entropy [B, T] of the forward pass alone."""
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    P = views(cfg, np.asarray(weights, dtype=np.float64))
    cos, sin = rope_tables(T, cfg.head_dim, cfg.rope_base)
    out = np.empty((B, T))
    for b in range(B):
        saved = _row_forward(cfg, P, tokens[b], cos, sin, keep=False)
        out[b], _, _ = lm_head_loss(saved["xf"], P["wlm"], np.asarray(targets)[b],
                                    cfg.softcap, 1.0, want_grad=False)
    return out


def forward_logits(cfg, weights, tokens):
    """Softcapped logits z [B, T, V] of the forward pass."""
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    P = views(cfg, np.asarray(weights, dtype=np.float64))
    cos, sin = rope_tables(T, cfg.head_dim, cfg.rope_base)
    out = np.empty((B, T, cfg.vocab))
    for b in range(B):
        saved = _row_forward(cfg, P, tokens[b], cos, sin, keep=False)
        out[b] = softcap(saved["xf"] @ P["wlm"].T, cfg.softcap)
    return out
