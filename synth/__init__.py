"""Seeded synthetic inputs shared by the tests, the oracle checks and the bench.

This module holds only workload definitions (model shapes, batch sizes, token
distributions), the flat parameter layout, and seeded random draws.  It holds
none of the model's arithmetic: the CPU oracle and the CUDA library each
implement the step on their own and are fed the arrays made here.

Workloads follow the five shapes the pages' model family is run at: a tiny
correctness model, a GPT-2-124M-shaped stack (the llm.c article, qian.cx,
section on the 12-layer / 12-head / 768-wide / 1024-token model), the
depth-20 speedrun model and the depth-30 model (nanochat announcement,
tianqi.csdn.net, data-shard section for depth 20; vpshk.cn, the $1000-tier
paragraph for depth 30), and a seq-8192 variant of depth 20.

Vocabulary 65536 = 2**16 is the tokenizer size of the nanochat announcement
(tianqi.csdn.net, tokenizer-training section).  The training text itself
(FineWeb-EDU shards) is not available, so token ids are drawn from a Zipf
law, P(id = k-1) proportional to k**-s for k = 1..V (s = 1.1), which gives the
heavy-headed id frequencies of natural text, or uniformly for the tiny and
long-context workloads.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict
import numpy as np

__all__ = [
    "ModelConfig", "Workload", "WORKLOADS", "param_layout", "num_params",
    "make_weights", "make_tokens", "bf16_round", "bf16_bits_to_f32",
]


@dataclass(frozen=True)
class ModelConfig:
    vocab: int
    d_model: int
    n_layer: int
    n_head: int
    n_kv_head: int
    head_dim: int
    mlp_mult: int = 4
    softcap: float = 15.0
    rope_base: float = 10000.0

    def as_dict(self):
        return asdict(self)


@dataclass(frozen=True)
class Workload:
    name: str
    model: ModelConfig
    seq_len: int
    batch: int
    ids: str  # "uniform" or "zipf"
    zipf_s: float = 1.1

    @property
    def tokens_per_step(self) -> int:
        return self.seq_len * self.batch


def _d(depth: int, n_head: int) -> ModelConfig:
    return ModelConfig(vocab=65536, d_model=64 * depth, n_layer=depth, n_head=n_head,
                       n_kv_head=1, head_dim=128)


WORKLOADS = {
    "tiny": Workload("tiny", ModelConfig(vocab=512, d_model=64, n_layer=2, n_head=4,
                                         n_kv_head=1, head_dim=16), 32, 2, "uniform"),
    "gpt2_124m": Workload("gpt2_124m", ModelConfig(vocab=65536, d_model=768, n_layer=12,
                                                   n_head=12, n_kv_head=1, head_dim=64),
                          1024, 8, "zipf"),
    "d20": Workload("d20", _d(20, 10), 2048, 16, "zipf"),
    "d30": Workload("d30", _d(30, 15), 2048, 8, "zipf"),
    "long": Workload("long", _d(20, 10), 8192, 2, "uniform"),
}


def param_layout(cfg: ModelConfig):
    """Flat parameter layout: list of (name, rows, cols, offset) in storage order.

    Every matrix is row-major [out, in] so that a linear is y = x W^T.  Order:
    wte[V,d]; per layer wq[H*hd,d], wk[nkv*hd,d], wv[nkv*hd,d], wo[d,H*hd],
    wfc[F,d], wproj[d,F]; then wlm[V,d].  wq/wk/wv are adjacent, so together
    they form one [(H+2*nkv)*hd, d] matrix.
    """
    d, hd = cfg.d_model, cfg.head_dim
    F = cfg.mlp_mult * d
    out = []
    off = 0

    def add(name, r, c):
        nonlocal off
        out.append((name, r, c, off))
        off += r * c

    add("wte", cfg.vocab, d)
    for i in range(cfg.n_layer):
        add(f"h.{i}.wq", cfg.n_head * hd, d)
        add(f"h.{i}.wk", cfg.n_kv_head * hd, d)
        add(f"h.{i}.wv", cfg.n_kv_head * hd, d)
        add(f"h.{i}.wo", d, cfg.n_head * hd)
        add(f"h.{i}.wfc", F, d)
        add(f"h.{i}.wproj", d, F)
    add("wlm", cfg.vocab, d)
    return out


def num_params(cfg: ModelConfig) -> int:
    name, r, c, off = param_layout(cfg)[-1]
    return off + r * c


def bf16_round(x: np.ndarray):
    """Round fp32 values to bf16, round-to-nearest-even.

    Returns (bits uint16, values fp32).  Inputs are finite.
    """
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bits = ((u + (((u >> 16) & 1) + np.uint32(0x7FFF))) >> 16).astype(np.uint16)
    return bits, bf16_bits_to_f32(bits)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def make_weights(cfg: ModelConfig, seed: int = 0, dtype: str = "bf16", std: float = 0.02):
    """Flat weights drawn fp32 from N(0, std) with PCG64(seed), in param_layout order.

    dtype "bf16": returns (bits uint16 [N], values fp32 [N]) with values the
    exact bf16 numbers.  dtype "fp32": returns (None, values fp32 [N]).
    """
    n = num_params(cfg)
    rng = np.random.Generator(np.random.PCG64(seed))
    w = rng.standard_normal(n, dtype=np.float32)
    w *= np.float32(std)
    if dtype == "bf16":
        return bf16_round(w)
    if dtype == "fp32":
        return None, w
    raise ValueError(dtype)


def make_tokens(wl: Workload, seed: int = 1, batch: int | None = None):
    """Token ids and next-token targets, int32 [B, T] each.

    Each row draws T+1 ids s; tokens = s[:T], targets = s[1:].
    """
    B = wl.batch if batch is None else batch
    T, V = wl.seq_len, wl.model.vocab
    rng = np.random.Generator(np.random.PCG64(seed))
    if wl.ids == "uniform":
        s = rng.integers(0, V, size=(B, T + 1), dtype=np.int64)
    elif wl.ids == "zipf":
        k = np.arange(1, V + 1, dtype=np.float64)
        p = k ** (-wl.zipf_s)
        cdf = np.cumsum(p)
        cdf /= cdf[-1]
        u = rng.random(size=(B, T + 1))
        s = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1)
    else:
        raise ValueError(wl.ids)
    s = s.astype(np.int32)
    return np.ascontiguousarray(s[:, :T]), np.ascontiguousarray(s[:, 1:])
