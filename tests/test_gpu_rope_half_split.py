"""The half-split RoPE convention (the HuggingFace port: q*cos + rotate_half(q)*sin,
pairs (i, i + D/2)): weights given in that convention with rope_half_split = 1
must give the logits the oracle computes from the interleaved-convention
weights they were converted from (rows of each head of wq, wk reordered
i <- 2i, i + D/2 <- 2i + 1), and the K cache must read back in the half-split
order."""
import dataclasses

import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import BF16_LOGITS_ABS, assert_abs_close, assert_fp32_close
from tests.helpers import build_oracle, t2np
import oracle as O

pytestmark = pytest.mark.gpu


def _to_half_split(w: torch.Tensor, n_heads: int, D: int) -> torch.Tensor:
    perm = torch.cat([torch.arange(0, D, 2), torch.arange(1, D, 2)])
    idx = torch.cat([h * D + perm for h in range(n_heads)])
    return w[idx].contiguous()


@pytest.mark.parametrize("act", ["fp32", "bf16"])
def test_half_split_weights_match_interleaved_oracle(act):
    w = synth.Workload(name="half-split rope model", dim=256, n_layers=2, n_heads=4, n_kv_heads=2,
                       ffn_hidden=O.ffn_hidden_dim(256, 256), vocab_size=512, multiple_of=256,
                       ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_batch_size=2, max_seq_len=64,
                       act=act, batch=2, seed=13, norm_weights="random")
    D = w.head_dim
    lws = [synth.layer_weights(w, i) for i in range(w.n_layers)]
    enh = synth.embed_norm_head(w)
    args = dataclasses.replace(B.ModelArgs.from_workload(w), rope_half_split=True)
    model = B.Llama(args)
    try:
        for i, lw in enumerate(lws):
            hf = dict(lw)
            hf["wq"] = _to_half_split(lw["wq"], w.n_heads, D)
            hf["wk"] = _to_half_split(lw["wk"], w.n_kv_heads, D)
            B.llama_set_layer(model.ctx, i, {k: v.cuda().contiguous() for k, v in hf.items()})
        B.llama_set_embed_norm_head(model.ctx, enh["tok_embeddings"].cuda(), enh["norm"].cuda(),
                                    enh["output"].cuda())
        om = build_oracle(w, lws, enh)
        tok = synth.tokens(w, (2, 21))
        for t0, t1 in ((0, 20), (20, 21)):
            out = torch.empty((2, t1 - t0, w.vocab_size), device="cuda")
            B.llama_forward(model.ctx, tok[:, t0:t1].cuda().contiguous(), t0, out, True)
            torch.cuda.synchronize()
            assert B.llama_get_error(model.ctx)[0] == B.LLAMA_OK
            ref = om.forward(t2np(tok[:, t0:t1]).astype(np.int64), t0)
            if act == "fp32":
                assert_fp32_close(t2np(out), ref, "logits")
            else:
                assert_abs_close(t2np(out), ref, BF16_LOGITS_ABS, "logits")
        # K reads back in the half-split order: the oracle's K with each head's pairs de-interleaved
        dt = torch.float32 if act == "fp32" else torch.bfloat16
        shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, D)
        k = torch.empty(shape, dtype=dt, device="cuda")
        v = torch.empty(shape, dtype=dt, device="cuda")
        B.llama_kv_read(model.ctx, 0, k, v)
        torch.cuda.synchronize()
        perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])
        kref = om.cache_k[0][..., perm]
        tol = 1e-4 * np.abs(kref).max() if act == "fp32" else 2e-2
        assert np.abs(t2np(k)[:2, :21] - kref[:2, :21]).max() <= tol
        assert np.abs(t2np(v)[:2, :21] - om.cache_v[0][:2, :21]).max() <= tol
        # and a round trip through kv_write leaves the cache as it was
        B.llama_kv_write(model.ctx, 0, k, v)
        k2 = torch.empty_like(k)
        v2 = torch.empty_like(v)
        B.llama_kv_read(model.ctx, 0, k2, v2)
        torch.cuda.synchronize()
        assert torch.equal(k, k2) and torch.equal(v, v2)
    finally:
        model.close()
