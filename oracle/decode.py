"""Float64 KV-cache inference: prefill and one-token decode (test
infrastructure, like the rest of ``oracle``).

The nanochat pipeline ends in an inference engine with a KV cache and
prefill / decode (tianqi.csdn.net nanochat article, pipeline paragraph).  With
multi-query attention (vpshk.cn, architecture list) the cache holds one K and
one V head per K/V group, after QK-norm and RoPE for K.  Decoding position p
appends that position's k and v and attends the new query to positions
0..p; the result must equal the last position of the full forward over the
extended sequence (``forward_logits``), which the tests check.

This module restates the forward one position at a time on its own (it does
not call the batched row forward), using only the pinned building blocks.
"""
from __future__ import annotations

import math

import numpy as np

from .model import rmsnorm, rope, rope_tables, softcap, views


def _params(cfg, weights):
    return views(cfg, np.asarray(weights, dtype=np.float64))


def _position(cfg, P, cache, idx, pos):
    """Forward of one position of one row: appends its k, v to `cache` (a list
    of per-layer dicts of python lists) and returns the softcapped logits [V]."""
    H, nkv, hd = cfg.n_head, cfg.n_kv_head, cfg.head_dim
    cos, sin = rope_tables(pos + 1, hd, cfg.rope_base)
    c1, s1 = cos[pos:pos + 1], sin[pos:pos + 1]
    x, _ = rmsnorm(P["wte"][idx])
    for i in range(cfg.n_layer):
        a, _ = rmsnorm(x)
        q, _ = rmsnorm((a @ P[f"h.{i}.wq"].T).reshape(1, H, hd))
        k, _ = rmsnorm((a @ P[f"h.{i}.wk"].T).reshape(1, nkv, hd))
        v = (a @ P[f"h.{i}.wv"].T).reshape(nkv, hd)
        q = rope(q, c1, s1)[0]
        k = rope(k, c1, s1)[0]
        cache[i]["k"].append(k)
        cache[i]["v"].append(v)
        K = np.stack(cache[i]["k"])  # [pos + 1, nkv, hd]
        V = np.stack(cache[i]["v"])
        o = np.empty((H, hd))
        for h in range(H):
            g = h // (H // nkv)
            s = K[:, g] @ q[h] / math.sqrt(hd)  # every cached position is visible
            p = np.exp(s - s.max())
            o[h] = (p / p.sum()) @ V[:, g]
        x = x + o.reshape(H * hd) @ P[f"h.{i}.wo"].T
        m, _ = rmsnorm(x)
        x = x + np.maximum(m @ P[f"h.{i}.wfc"].T, 0.0) ** 2 @ P[f"h.{i}.wproj"].T
    xf, _ = rmsnorm(x)
    return softcap(P["wlm"] @ xf, cfg.softcap)


def prefill(cfg, weights, tokens):
    """Runs the prompt tokens [B, T] one position at a time.  Returns (cache,
    logits of the last position [B, V]); cache[b][layer] holds lists "k", "v"
    of [n_kv, hd] arrays, one per position."""
    P = _params(cfg, weights)
    tokens = np.asarray(tokens)
    B, T = tokens.shape
    caches, out = [], np.empty((B, cfg.vocab))
    for b in range(B):
        cache = [{"k": [], "v": []} for _ in range(cfg.n_layer)]
        for t in range(T):
            out[b] = _position(cfg, P, cache, tokens[b, t], t)
        caches.append(cache)
    return caches, out


def decode_step(cfg, weights, caches, tokens):
    """One new token per row (tokens [B]) at position len(cache): appends to
    the caches and returns the logits [B, V]."""
    P = _params(cfg, weights)
    out = np.empty((len(caches), cfg.vocab))
    for b, cache in enumerate(caches):
        out[b] = _position(cfg, P, cache, int(tokens[b]), len(cache[0]["k"]))
    return out
