"""Parity at the workloads' full sizes, in the launch configuration the bench
times (llama_block_forward, batch and positions of the workload), against
the oracle run on the same seeded inputs."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import (CacheSnapshot, Pair, assert_bf16_cache_close, assert_hidden_close_floor, oracle_floor)
from tests.helpers import t2np

pytestmark = pytest.mark.gpu


def test_llama7b_layer_prefill_512_then_decode():
    """LLaMA-1-7B-shaped layer: prefill 512 tokens (all outputs compared), then decode
    steps at positions 512.. (first 4 of the 128 compared element by element)."""
    w = synth.LLAMA7B_LAYER
    pair = Pair(w)
    try:
        h = synth.hidden(w, (1, 512, w.dim), 0)
        hd = h.cuda()
        B.llama_block_forward(pair.ctx, 0, hd, 0)
        torch.cuda.synchronize()
        pair.check_error()
        snap = CacheSnapshot(pair.oracle, [0])

        def run(x):
            snap.restore()
            return pair.oracle.block(0, x, 0)
        ref, floor = oracle_floor(run, t2np(h))
        assert_hidden_close_floor(t2np(hd), ref, floor, "prefill hidden")
        hdec = synth.hidden(w, (128, 1, 1, w.dim), 1)
        for i in range(4):
            x = hdec[i].cuda().contiguous()
            B.llama_block_forward(pair.ctx, 0, x, 512 + i)
            torch.cuda.synchronize()
            pair.check_error()
            snap = CacheSnapshot(pair.oracle, [0])

            def run(xx):
                snap.restore()
                return pair.oracle.block(0, xx, 512 + i)
            r, floor = oracle_floor(run, t2np(hdec[i]))
            assert_hidden_close_floor(t2np(x), r, floor, f"decode hidden at {512 + i}")
        # the cache rows the calls wrote: slots 0..515 of sequence 0, nothing else
        k, v = pair.kv(0)
        for got, refc in ((k, pair.oracle.cache_k[0]), (v, pair.oracle.cache_v[0])):
            assert np.all(got[0, 516:] == 0)
            assert_bf16_cache_close(got[0, :516], refc[0, :516], "cache")
    finally:
        pair.close()


def test_llama70b_layer_decode_batch16_at_4096():
    """LLaMA-2-70B-shaped layer (GQA 64/8): cache prefilled with N(0,1) to 4096,
    batch 16, one new token per sequence at start_pos 4096."""
    w = synth.LLAMA70B_LAYER
    pair = Pair(w, bits=True)
    try:
        shape = (w.max_batch_size, w.cache_len, w.n_kv_heads, w.head_dim)
        kc = synth.cache_values(w, 0, 0, shape)
        vc = synth.cache_values(w, 0, 1, shape)
        full = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
        k = torch.zeros(full, dtype=torch.bfloat16, device="cuda")
        v = torch.zeros_like(k)
        k[:, :w.cache_len] = kc.cuda()
        v[:, :w.cache_len] = vc.cuda()
        B.llama_kv_write(pair.ctx, 0, k, v)
        del k, v
        pair.oracle.cache_k[0] = np.zeros(full, dtype=np.float32)   # bf16 values are exact in fp32
        pair.oracle.cache_v[0] = np.zeros(full, dtype=np.float32)
        pair.oracle.cache_k[0][:, :w.cache_len] = kc.float().numpy()
        pair.oracle.cache_v[0][:, :w.cache_len] = vc.float().numpy()
        h = synth.hidden(w, (16, 1, w.dim), 1)
        hd = h.cuda()
        B.llama_block_forward(pair.ctx, 0, hd, w.cache_len)
        torch.cuda.synchronize()
        pair.check_error()
        snap = CacheSnapshot(pair.oracle, [0])

        def run(x):
            snap.restore()
            return pair.oracle.block(0, x, w.cache_len)
        ref, floor = oracle_floor(run, t2np(h))
        assert_hidden_close_floor(t2np(hd), ref, floor, "decode hidden")
        # repeating the step rewrites the same slot: identical result
        hd2 = h.cuda()
        B.llama_block_forward(pair.ctx, 0, hd2, w.cache_len)
        torch.cuda.synchronize()
        assert torch.equal(hd, hd2)
    finally:
        pair.close()
