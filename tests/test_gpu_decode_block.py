"""The persistent decode-block kernel (LLAMA_DECODE_PERSISTENT: one launch per
block and decode step) against the oracle: every batch-size class of the
kernel (1..8, 9..16, 17..24, 25..32 tokens), MHA / GQA / MQA head maps, scalar
and per-sequence positions, a long history split over many attention chunks,
repeated launches (self-resetting counters and grid barrier), and the error
paths. The kernel-per-step path (LLAMA_DECODE_LAYERED) runs the same steps on
the same inputs and must agree with the oracle too."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import BF16_HIDDEN_ABS, Pair, assert_abs_close, assert_cache_matches
from tests.helpers import t2np
import oracle as O

pytestmark = pytest.mark.gpu


def _wl(dim, H, Hkv, Bm, S=256, mo=256, seed=11):
    F = O.ffn_hidden_dim(dim, mo)
    return synth.Workload(name=f"decode block dim {dim} H {H}/{Hkv}", dim=dim, n_layers=1, n_heads=H, n_kv_heads=Hkv,
                          ffn_hidden=F, vocab_size=0, multiple_of=mo, ffn_dim_multiplier=None, norm_eps=1e-5,
                          rope_theta=10000.0, max_batch_size=Bm, max_seq_len=S, act="bf16", batch=Bm, seed=seed,
                          norm_weights="random")


def _step(pair, h, start_pos):
    hd = h.to("cuda").contiguous()
    sp = start_pos
    if isinstance(start_pos, np.ndarray):
        sp = torch.from_numpy(start_pos.astype(np.int32)).to("cuda")
    B.llama_block_forward(pair.ctx, 0, hd, sp)
    torch.cuda.synchronize()
    pair.check_error()
    ref = pair.oracle.block(0, t2np(h), start_pos)
    got = t2np(hd)
    assert_abs_close(got, ref, BF16_HIDDEN_ABS, "hidden")
    return got


@pytest.mark.parametrize("mode", [B.LLAMA_DECODE_PERSISTENT, B.LLAMA_DECODE_LAYERED])
@pytest.mark.parametrize("dim,H,Hkv,Bsz", [(512, 4, 2, 1), (512, 4, 4, 2), (1024, 8, 1, 3), (2048, 16, 2, 5),
                                           (1024, 8, 8, 9), (512, 4, 2, 17), (512, 4, 1, 32)])
def test_decode_steps_match_oracle(mode, dim, H, Hkv, Bsz):
    w = _wl(dim, H, Hkv, Bsz)
    pair = Pair(w)
    try:
        B.llama_set_decode_kernel(pair.ctx, mode)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        h = synth.hidden(w, (Bsz, 70, dim), call=0)       # prefill (T > 1 always takes the prefill kernels)
        _step(pair, h, 0)
        written[:Bsz, :70] = True
        for i in range(4):                                 # decode steps, scalar position
            h = synth.hidden(w, (Bsz, 1, dim), call=1 + i)
            _step(pair, h, 70 + i)
            written[:Bsz, 70 + i] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


def test_ragged_positions_and_many_chunks():
    """Per-sequence device positions: one sequence attends over ~3.9k keys (many
    128-key chunks merged by the last-arriving CTA), the others over a few."""
    w = _wl(512, 4, 1, 4, S=4096)
    pair = Pair(w)
    try:
        B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_PERSISTENT)
        h = synth.hidden(w, (4, 5, 512), call=0)
        _step(pair, h, 0)
        pos = np.array([5, 3900, 130, 1000])   # skipped slots stay zero on both sides
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:4, :5] = True
        for step in range(3):
            h = synth.hidden(w, (4, 1, 512), call=1 + step)
            _step(pair, h, pos)
            for b in range(4):
                written[b, pos[b]] = True
            pos = pos + np.array([1, 64, 7, 129])
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


def test_repeated_launches_rearm_counters():
    """Thirty decode launches in a row through the same workspace, mixed with
    kernel-per-step launches; every one must match the oracle."""
    w = _wl(512, 4, 2, 2, S=128)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (2, 8, 512), call=0)
        _step(pair, h, 0)
        for i in range(30):
            B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_LAYERED if i % 7 == 3 else B.LLAMA_DECODE_PERSISTENT)
            h = synth.hidden(w, (2, 1, 512), call=1 + i)
            _step(pair, h, 8 + i)
    finally:
        pair.close()


def test_graph_replay_of_persistent_steps():
    """Decode steps captured once in a CUDA graph and replayed on new inputs."""
    w = _wl(1024, 8, 2, 2, S=128)
    pair = Pair(w)
    try:
        B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_PERSISTENT)
        h = synth.hidden(w, (2, 16, 1024), call=0)
        _step(pair, h, 0)
        _step(pair, synth.hidden(w, (2, 1, 1024), call=9), 16)   # first launch outside the capture
        pos = torch.tensor([16, 16], dtype=torch.int32, device="cuda")
        hd = torch.zeros((2, 1, 1024), device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            B.llama_block_forward(pair.ctx, 0, hd, pos, stream=s)
        torch.cuda.synchronize()
        for i in range(3):
            hin = synth.hidden(w, (2, 1, 1024), call=1 + i)
            hd.copy_(hin.to("cuda"))
            pos.fill_(16 + i)
            g.replay()
            torch.cuda.synchronize()
            pair.check_error()
            ref = pair.oracle.block(0, t2np(hin), 16 + i)
            assert_abs_close(t2np(hd), ref, BF16_HIDDEN_ABS, f"replay {i}")
        del g
    finally:
        pair.close()


def test_ineligible_shape_and_position_errors():
    # head_dim 64: the persistent kernel does not apply; forcing it is an argument error
    w = _wl(256, 4, 1, 2, S=64)
    pair = Pair(w)
    try:
        B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_PERSISTENT)
        with pytest.raises(B.LlamaError) as e:
            B.llama_block_forward(pair.ctx, 0, torch.zeros((2, 1, 256), device="cuda"), 3)
        assert e.value.code == B.LLAMA_ERR_INVALID_ARGS
        B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_AUTO)   # AUTO runs the per-step kernels here
        B.llama_block_forward(pair.ctx, 0, torch.zeros((2, 1, 256), device="cuda"), 3)
        assert B.llama_get_error(pair.ctx)[0] == B.LLAMA_OK
        with pytest.raises(B.LlamaError):
            B.llama_set_decode_kernel(pair.ctx, 7)
    finally:
        pair.close()
    # a device position past the cache raises the position flag; that slot is not written
    w = _wl(512, 4, 2, 2, S=128)
    pair = Pair(w)
    try:
        B.llama_set_decode_kernel(pair.ctx, B.LLAMA_DECODE_PERSISTENT)
        sp = torch.tensor([5, 128], dtype=torch.int32, device="cuda")
        B.llama_block_forward(pair.ctx, 0, synth.hidden(w, (2, 1, 512), call=0).to("cuda").contiguous(), sp)
        code, flags = B.llama_get_error(pair.ctx)
        assert code == B.LLAMA_ERR_POS_RANGE and flags & 2
        k, _ = pair.kv(0)
        assert np.all(k[1] == 0.0) and np.any(k[0, 5] != 0.0)
    finally:
        pair.close()
