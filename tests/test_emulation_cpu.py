"""The fp32 restatement that sizes the full-size parity bound (tests/emulation.py)
computes the oracle's function: on small blocks it stays within the bf16 bound
of the oracle, its cache rows match the oracle's up to one bf16 step, and a
planted mistake (a dropped residual, a transposed head map) is far outside."""
import numpy as np
import pytest
import torch

import oracle as O
from llama_decoder_block_kv_b200 import synth
from tests import emulation as E
from tests.helpers import build_oracle, oracle_args, t2np


def _wl(H, Hkv, dim=256):
    return synth.Workload(name="emu", dim=dim, n_layers=1, n_heads=H, n_kv_heads=Hkv,
                          ffn_hidden=O.ffn_hidden_dim(dim, 256), vocab_size=0, multiple_of=256,
                          ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_batch_size=2,
                          max_seq_len=64, act="bf16", batch=2, seed=3, norm_weights="random")


@pytest.mark.parametrize("H,Hkv", [(4, 2), (4, 4), (8, 1)])
def test_emulation_tracks_the_oracle(H, Hkv):
    w = _wl(H, Hkv)
    lw = synth.layer_weights(w, 0)
    om = build_oracle(w, [lw])
    args = oracle_args(w)
    em = E.EmuBlock(lw, args, om.cos, om.sin)
    ck = torch.zeros((2, 64, Hkv, w.head_dim))
    cv = torch.zeros_like(ck)
    for call, (T, sp) in enumerate([(20, 0), (7, np.array([20, 11])), (1, np.array([27, 30]))]):
        h = synth.hidden(w, (2, T, w.dim), call=call)
        ref = om.block(0, t2np(h), sp)
        got = E.EmuBlock.forward(em, h, ck, cv, sp).double().numpy()
        assert np.abs(got - ref).max() <= 2e-2
        # a rows subset gives the same rows
        rows = [(0, T - 1), (1, 0)]
        sub = em.forward(h, ck.clone(), cv.clone(), sp, rows=rows).double().numpy()
        assert np.abs(sub - got[[0, 1], [T - 1, 0]]).max() <= 2e-2   # other sum orders, same rows
    spacing = np.exp2(np.floor(np.log2(np.maximum(np.abs(om.cache_k[0]), 2.0 ** -126))) - 7)
    assert np.all(np.abs(ck.double().numpy() - om.cache_k[0]) <= spacing * 1.0000001)


def test_emulation_mistakes_are_visible():
    """A block that drops the attention residual, or maps query heads to kv heads
    modulo instead of by division, is far outside the bound: the comparison
    resolves such mistakes."""
    w = _wl(8, 2)
    lw = synth.layer_weights(w, 0)
    om = build_oracle(w, [lw])
    h = synth.hidden(w, (2, 12, w.dim), call=0)
    ref = om.block(0, t2np(h), 0)
    bad = dict(lw)
    bad["wo"] = torch.zeros_like(lw["wo"])
    em = E.EmuBlock(bad, oracle_args(w), om.cos, om.sin)
    got = em.forward(h, torch.zeros((2, 64, 2, w.head_dim)), torch.zeros((2, 64, 2, w.head_dim)), 0)
    assert np.abs(got.double().numpy() - ref).max() > 0.1
    perm = torch.arange(8).view(2, 4).T.reshape(-1)          # head h -> kv head h % 2 instead of h // 4
    bad = dict(lw)
    bad["wq"] = lw["wq"].view(8, w.head_dim, w.dim)[perm].reshape(8 * w.head_dim, w.dim)
    bad["wo"] = lw["wo"].view(w.dim, 8, w.head_dim)[:, perm].reshape(w.dim, 8 * w.head_dim)
    em = E.EmuBlock(bad, oracle_args(w), om.cos, om.sin)
    got = em.forward(h, torch.zeros((2, 64, 2, w.head_dim)), torch.zeros((2, 64, 2, w.head_dim)), 0)
    assert np.abs(got.double().numpy() - ref).max() > 0.1
