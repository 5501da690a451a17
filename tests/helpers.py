"""Glue between the seeded inputs (synth) and the oracle: tensor conversion only."""
from __future__ import annotations

import numpy as np
import torch

from oracle import ModelArgs, OracleModel
from llama_decoder_block_kv_b200 import synth


def t2np(t: torch.Tensor) -> np.ndarray:
    """Any float tensor -> float64 numpy (bf16 and fp32 values convert exactly)."""
    return t.detach().to("cpu", torch.float64).numpy()


def t2bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> raw uint16 bit patterns (keeps host memory at 2 bytes/value)."""
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def oracle_args(w: synth.Workload, **over) -> ModelArgs:
    a = ModelArgs(dim=w.dim, n_layers=w.n_layers, n_heads=w.n_heads, n_kv_heads=w.n_kv_heads,
                  vocab_size=w.vocab_size, multiple_of=w.multiple_of,
                  ffn_dim_multiplier=w.ffn_dim_multiplier, norm_eps=w.norm_eps,
                  rope_theta=w.rope_theta, max_batch_size=w.max_batch_size,
                  max_seq_len=w.max_seq_len, act=w.act)
    for k, v in over.items():
        setattr(a, k, v)
    return a


def _conv(t: torch.Tensor, bits: bool):
    if bits and t.dtype == torch.bfloat16:
        return t2bits(t)
    return t2np(t)


def build_oracle(w: synth.Workload, layer_weights, enh=None, bits: bool = False, **over) -> OracleModel:
    """An OracleModel holding the given synth weights (lists/dicts of torch tensors)."""
    m = OracleModel(oracle_args(w, **over))
    for i, lw in enumerate(layer_weights):
        m.layers[i] = {k: _conv(v, bits) for k, v in lw.items()}
    if enh is not None:
        m.tok_embeddings = _conv(enh["tok_embeddings"], bits)
        m.norm = t2np(enh["norm"])
        m.output = _conv(enh["output"], bits)
    return m
