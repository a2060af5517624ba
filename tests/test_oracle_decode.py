"""Pins for the oracle's KV-cache decode: prefill plus one-token decode steps,
computed one position at a time from the cache, must equal the last position
of the full batched forward over the extended sequence (forward_logits, itself
pinned to the torch float64 forward), and the cached k must carry RoPE at its
own position (a relative-position property of the cached scores)."""
import numpy as np
import pytest

import oracle
import synth

TINY = synth.WORKLOADS["tiny"]


def _cfg(**kw):
    d = TINY.model.as_dict()
    d.update(kw)
    return synth.ModelConfig(**d)


@pytest.mark.parametrize("cfg", [_cfg(), _cfg(n_kv_head=2), _cfg(n_head=2, head_dim=32, softcap=5.0)])
def test_prefill_and_decode_equal_the_full_forward(cfg):
    _, w = synth.make_weights(cfg, seed=9, dtype="bf16")
    w = w.astype(np.float64) * 5.0
    wl = synth.Workload("t", cfg, 12, 2, "uniform")
    tok, _ = synth.make_tokens(wl, seed=4)
    T0 = 7
    caches, last = oracle.prefill(cfg, w, tok[:, :T0])
    full = oracle.forward_logits(cfg, w, tok)
    np.testing.assert_allclose(last, full[:, T0 - 1], rtol=1e-10, atol=1e-10)
    for t in range(T0, tok.shape[1]):
        got = oracle.decode_step(cfg, w, caches, tok[:, t])
        np.testing.assert_allclose(got, full[:, t], rtol=1e-10, atol=1e-10)
    assert len(caches[0][0]["k"]) == tok.shape[1]


def test_decode_does_not_depend_on_future_tokens():
    cfg = _cfg()
    _, w = synth.make_weights(cfg, seed=10, dtype="bf16")
    tok, _ = synth.make_tokens(synth.Workload("t", cfg, 6, 1, "uniform"), seed=5)
    a, _ = oracle.prefill(cfg, w, tok[:, :4])
    b, _ = oracle.prefill(cfg, w, tok[:, :5])
    for layer in range(cfg.n_layer):
        for p in range(4):
            assert np.array_equal(a[0][layer]["k"][p], b[0][layer]["k"][p])
            assert np.array_equal(a[0][layer]["v"][p], b[0][layer]["v"][p])
