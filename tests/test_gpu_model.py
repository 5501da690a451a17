"""Whole-model calls (llama_forward, llama_forward_ragged) against the oracle:
the tiny fp32 model of the workload list (prefill 32 + 16 decode steps,
logits and caches at 1e-4 relative) and a small bf16 model with GQA,
ragged decode positions and last-position-only logits."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import BF16_LOGITS_ABS, Pair, assert_abs_close, assert_cache_matches, assert_fp32_close
from tests.helpers import t2np
import oracle as O

pytestmark = pytest.mark.gpu


def _forward(pair, tok, start_pos, all_positions=True):
    Bsz, T = tok.shape
    V = pair.w.vocab_size
    out = torch.full((Bsz, T, V) if all_positions else (Bsz, V), float("nan"), device="cuda")
    B.llama_forward(pair.ctx, tok.to("cuda").contiguous(), start_pos, out, all_positions)
    torch.cuda.synchronize()
    pair.check_error()
    ref = pair.oracle.forward(t2np(tok).astype(np.int64), start_pos, all_positions)
    return t2np(out), ref


@pytest.mark.parametrize("norms", ["unit", "random"])
def test_tiny_fp32_prefill_then_decode(norms):
    """The tiny fp32 workload as stated (norm weights 1), and with learned-looking
    norm weights so the weight multiply of every RMSNorm is checked too."""
    w = synth.TINY_FP32.with_(norm_weights=norms)
    pair = Pair(w)
    try:
        tok = synth.tokens(w, (1, 32 + 16))
        got, ref = _forward(pair, tok[:, :32], 0)
        assert_fp32_close(got, ref, "prefill logits")
        for s in range(32, 48):
            got, ref = _forward(pair, tok[:, s:s + 1], s)
            assert_fp32_close(got, ref, f"decode logits at {s}")
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:1, :48] = True
        for layer in range(w.n_layers):
            assert_cache_matches(pair, layer, written, None)
    finally:
        pair.close()


def _small_bf16(**kw):
    base = dict(name="small bf16 model", dim=512, n_layers=2, n_heads=8, n_kv_heads=2,
                ffn_hidden=O.ffn_hidden_dim(512, 256), vocab_size=1000, multiple_of=256, ffn_dim_multiplier=None,
                norm_eps=1e-5, rope_theta=500000.0, max_batch_size=3, max_seq_len=256, act="bf16", batch=3, seed=9,
                norm_weights="random")
    base.update(kw)
    return synth.Workload(**base)


def test_small_bf16_model_prefill_decode_last_only():
    w = _small_bf16()
    pair = Pair(w)
    try:
        tok = synth.tokens(w, (3, 70))
        got, ref = _forward(pair, tok[:, :60], 0)
        assert_abs_close(got, ref, BF16_LOGITS_ABS, "prefill logits")
        for s in range(60, 66):
            got, ref = _forward(pair, tok[:, s:s + 1], s)
            assert_abs_close(got, ref, BF16_LOGITS_ABS, f"decode logits at {s}")
        got, ref = _forward(pair, tok[:, 66:70], 66, all_positions=False)
        assert got.shape == (3, w.vocab_size)
        assert_abs_close(got, ref, BF16_LOGITS_ABS, "last-position logits")
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:3, :70] = True
        for layer in range(w.n_layers):
            assert_cache_matches(pair, layer, written, 2e-2)
    finally:
        pair.close()


def test_small_bf16_ragged_decode():
    w = _small_bf16(max_batch_size=4, batch=4)
    pair = Pair(w)
    try:
        Bsz = 4
        tok = synth.tokens(w, (Bsz, 40))
        _forward(pair, tok[:, :20], 0)
        pos = np.array([20, 20, 20, 20])
        for step in range(5):
            t = tok[:, 20 + step]
            logits = torch.full((Bsz, w.vocab_size), float("nan"), device="cuda")
            B.llama_forward_ragged(pair.ctx, t.to("cuda").contiguous(),
                                   torch.from_numpy(pos.astype(np.int32)).to("cuda"), logits)
            torch.cuda.synchronize()
            pair.check_error()
            ref = pair.oracle.forward(t2np(t).astype(np.int64)[:, None], pos)
            assert_abs_close(t2np(logits), ref[:, 0], BF16_LOGITS_ABS, f"ragged step {step}")
            pos = pos + np.array([1, 3, 7, 2])
    finally:
        pair.close()


def test_token_out_of_range_sets_flag():
    w = _small_bf16(n_layers=1)
    pair = Pair(w)
    try:
        tok = torch.tensor([[1, 5, w.vocab_size]], dtype=torch.int32, device="cuda")
        out = torch.empty((1, 3, w.vocab_size), device="cuda")
        B.llama_forward(pair.ctx, tok, 0, out, True)
        code, flags = B.llama_get_error(pair.ctx)
        assert code == B.LLAMA_ERR_TOKEN_RANGE and flags & 1
    finally:
        pair.close()
