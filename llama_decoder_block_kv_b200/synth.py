"""Seeded synthetic inputs shared by the tests, the bench and ``smoke()``.

This module only draws random numbers (torch generators with fixed seeds) and
casts them to a storage dtype. It holds no arithmetic of the model: sizes such
as the FFN width are stated per workload, not derived here.

Recipe (all workloads): linear weights ~ N(0, 0.02^2) drawn in fp32 and cast
(round-to-nearest-even) to the storage dtype; RMSNorm weights are 1 (the
workloads' statement), or, for parity cases that must exercise the learned
norm weight, 1 + N(0, 0.1^2) drawn per layer and per norm and cast to the
storage dtype (``Workload.norm_weights = "random"``); hidden
states ~ N(0, 1) cast to the activation dtype and handed over as fp32; token ids
uniform in [0, vocab); prefilled cache entries ~ N(0, 1) in the cache dtype;
ragged cache lengths uniform over an inclusive integer range. Every tensor has
its own seed, derived from the workload seed and the tensor's role, so any one
tensor can be regenerated without drawing the others.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch

WEIGHT_STD = 0.02
NORM_WEIGHT_STD = 0.1
LAYER_WEIGHT_NAMES = ("wq", "wk", "wv", "wo", "w1", "w2", "w3")


@dataclass(frozen=True)
class Workload:
    """A synthetic LLaMA-shaped workload: model shape plus the calls made on it."""
    name: str
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    ffn_hidden: int          # as the workload states it (checked against the library's rule)
    vocab_size: int          # 0 for single-layer workloads
    multiple_of: int
    ffn_dim_multiplier: Optional[float]
    norm_eps: float
    rope_theta: float
    max_batch_size: int
    max_seq_len: int
    act: str                 # "fp32" or "bf16"
    batch: int
    prefill_len: int = 0     # tokens per sequence in the prefill call
    decode_steps: int = 0
    cache_len: int = 0       # prefilled cache length (fixed) for decode-only workloads
    ragged_lo: int = 0       # ragged cache lengths, inclusive range
    ragged_hi: int = 0
    seed: int = 0
    norm_weights: str = "unit"   # "unit" (all 1) or "random" (1 + N(0, 0.1^2), per layer and per norm)

    @property
    def head_dim(self) -> int:
        return self.dim // self.n_heads

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: a tiny fp32 model, two single bf16 layers (LLaMA-1-7B and
# LLaMA-2-70B shapes), and a LLaMA-3-8B-shaped whole model in decode and prefill.
TINY_FP32 = Workload(
    name="tiny-fp32 (dim 256, 2 layers, 4 heads / 2 kv heads, vocab 1000)",
    dim=256, n_layers=2, n_heads=4, n_kv_heads=2, ffn_hidden=768, vocab_size=1000,
    multiple_of=256, ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0,
    max_batch_size=1, max_seq_len=64, act="fp32", batch=1, prefill_len=32, decode_steps=16)

LLAMA7B_LAYER = Workload(
    name="llama-7b-layer (dim 4096, MHA 32 heads, ffn 11008) prefill 512 + 128 decode, batch 1",
    dim=4096, n_layers=1, n_heads=32, n_kv_heads=32, ffn_hidden=11008, vocab_size=0,
    multiple_of=256, ffn_dim_multiplier=None, norm_eps=1e-6, rope_theta=10000.0,
    max_batch_size=1, max_seq_len=2048, act="bf16", batch=1, prefill_len=512, decode_steps=128)

LLAMA70B_LAYER = Workload(
    name="llama-70b-layer (dim 8192, 64 heads / 8 kv heads, ffn 28672) decode batch 16 at 4096",
    dim=8192, n_layers=1, n_heads=64, n_kv_heads=8, ffn_hidden=28672, vocab_size=0,
    multiple_of=4096, ffn_dim_multiplier=1.3, norm_eps=1e-5, rope_theta=10000.0,
    max_batch_size=16, max_seq_len=8192, act="bf16", batch=16, decode_steps=1, cache_len=4096)

LLAMA3_8B_DECODE = Workload(
    name="llama3-8b decode (32 layers, dim 4096, 32/8 heads, ffn 14336, vocab 128256) batch 32 ragged",
    dim=4096, n_layers=32, n_heads=32, n_kv_heads=8, ffn_hidden=14336, vocab_size=128256,
    multiple_of=1024, ffn_dim_multiplier=1.3, norm_eps=1e-5, rope_theta=500000.0,
    max_batch_size=32, max_seq_len=8192, act="bf16", batch=32, decode_steps=64,
    ragged_lo=1024, ragged_hi=8192 - 64)

LLAMA3_8B_PREFILL = LLAMA3_8B_DECODE.with_(
    name="llama3-8b prefill 4 x 8192 from start_pos 0",
    max_batch_size=4, batch=4, prefill_len=8192, decode_steps=0, ragged_lo=0, ragged_hi=0)

WORKLOADS = {
    "tiny-fp32": TINY_FP32,
    "llama7b-layer": LLAMA7B_LAYER,
    "llama70b-layer": LLAMA70B_LAYER,
    "llama3-8b-decode": LLAMA3_8B_DECODE,
    "llama3-8b-prefill": LLAMA3_8B_PREFILL,
}


def sub_seed(seed: int, *keys: int) -> int:
    """A stable 63-bit seed for one tensor role (a 64-bit multiply-xorshift mix)."""
    x = (seed * 0x9E3779B97F4A7C15 + 0x632BE59BD9B4E019) & 0xFFFFFFFFFFFFFFFF
    for k in keys:
        x ^= (k + 0x85EBCA77C2B2AE63) & 0xFFFFFFFFFFFFFFFF
        x = (x * 0xBF58476D1CE4E5B9) & 0xFFFFFFFFFFFFFFFF
        x ^= x >> 31
    return x & 0x7FFFFFFFFFFFFFFF


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32 from a seeded generator, then cast to ``dtype``."""
    x = torch.randn(shape, generator=_gen(seed, device), dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def storage_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.act == "fp32" else torch.bfloat16


# roles used in sub_seed
_ROLE_LAYER, _ROLE_EMBED, _ROLE_NORM, _ROLE_HEAD, _ROLE_TOKENS, _ROLE_HIDDEN, _ROLE_CACHE, _ROLE_LENS = range(8)


def norm_weight(w: Workload, which: int, layer: int = 0, device="cpu") -> torch.Tensor:
    """One RMSNorm weight vector [dim]: all 1, or 1 + N(0, 0.1^2) with its own seed
    (which = 0 attention_norm, 1 ffn_norm, 2 the final norm)."""
    dt = storage_dtype(w)
    if w.norm_weights == "unit":
        return torch.ones(w.dim, dtype=dt, device=device)
    if w.norm_weights != "random":
        raise ValueError(f"unknown norm_weights {w.norm_weights!r}")
    x = torch.randn((w.dim,), generator=_gen(sub_seed(w.seed, _ROLE_NORM, layer, which), device),
                    dtype=torch.float32, device=device)
    return (1.0 + NORM_WEIGHT_STD * x).to(dt)


def layer_weights(w: Workload, layer: int, device="cpu") -> dict:
    """Weights of one block as [out, in] tensors (the nn.Linear layout) and its two norm weights."""
    D, H, Hkv, F = w.head_dim, w.n_heads, w.n_kv_heads, w.ffn_hidden
    shapes = {"wq": (H * D, w.dim), "wk": (Hkv * D, w.dim), "wv": (Hkv * D, w.dim),
              "wo": (w.dim, H * D), "w1": (F, w.dim), "w2": (w.dim, F), "w3": (F, w.dim)}
    dt = storage_dtype(w)
    out = {name: normal(shapes[name], WEIGHT_STD, sub_seed(w.seed, _ROLE_LAYER, layer, i), dt, device)
           for i, name in enumerate(LAYER_WEIGHT_NAMES)}
    out["attn_norm"] = norm_weight(w, 0, layer, device)
    out["ffn_norm"] = norm_weight(w, 1, layer, device)
    return out


def embed_norm_head(w: Workload, device="cpu") -> dict:
    """Token embedding [vocab, dim], final norm weight [dim], LM head [vocab, dim]."""
    dt = storage_dtype(w)
    return {
        "tok_embeddings": normal((w.vocab_size, w.dim), WEIGHT_STD, sub_seed(w.seed, _ROLE_EMBED), dt, device),
        "norm": norm_weight(w, 2, 0, device),
        "output": normal((w.vocab_size, w.dim), WEIGHT_STD, sub_seed(w.seed, _ROLE_HEAD), dt, device),
    }


def tokens(w: Workload, shape, call: int = 0, device="cpu") -> torch.Tensor:
    """Token ids uniform in [0, vocab), int32."""
    return torch.randint(0, w.vocab_size, shape, generator=_gen(sub_seed(w.seed, _ROLE_TOKENS, call), device),
                         dtype=torch.int64, device=device).to(torch.int32)


def hidden(w: Workload, shape, call: int = 0, device="cpu") -> torch.Tensor:
    """Hidden states N(0, 1) rounded to the activation dtype, returned as fp32."""
    return normal(shape, 1.0, sub_seed(w.seed, _ROLE_HIDDEN, call), storage_dtype(w), device).to(torch.float32)


def cache_values(w: Workload, layer: int, which: int, shape, device="cpu") -> torch.Tensor:
    """Prefilled cache contents N(0, 1) in the cache dtype; which = 0 for K, 1 for V."""
    return normal(shape, 1.0, sub_seed(w.seed, _ROLE_CACHE, layer, which), storage_dtype(w), device)


def ragged_lengths(w: Workload, device="cpu") -> torch.Tensor:
    """Per-sequence cache lengths uniform in [ragged_lo, ragged_hi], int32."""
    return torch.randint(w.ragged_lo, w.ragged_hi + 1, (w.batch,),
                         generator=_gen(sub_seed(w.seed, _ROLE_LENS), device),
                         dtype=torch.int64, device=device).to(torch.int32)
