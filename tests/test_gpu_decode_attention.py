"""The two decode attention kernels of the per-step launches (LLAMA_ATTN_CHUNKED
and LLAMA_ATTN_STREAMK) against the oracle: MHA / GQA / MQA head maps (16 query
heads per kv head: one CTA group of 16; 24 at head_dim 64: three groups of 8;
3 and 6, where the prefill attention takes groups of 1 and 2; 12, 20 and 17,
served in groups of 12, 10 and 1), head_dim 64 and
128, scalar and per-sequence positions, histories split over many CTAs (the
stream-K split cuts one sequence's tiles over up to 16 CTAs), batches of up to
96 sequences, repeated launches through the same counters, CUDA-graph replay
with device positions, and the mode switch's errors.
The oracle's block (TransformerBlock.forward of the notes) is the reference,
held to the flat 2e-2 bound on hidden states; the two kernels' outputs are also
compared with each other (1e-2), which bounds a difference the block's output
would dilute."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import BF16_HIDDEN_ABS, Pair, assert_abs_close, assert_cache_matches
from tests.helpers import t2np
import oracle as O

pytestmark = pytest.mark.gpu

KERNELS = [B.LLAMA_ATTN_CHUNKED, B.LLAMA_ATTN_STREAMK]


def _wl(dim, H, Hkv, Bm, S=256, mo=256, seed=23):
    F = O.ffn_hidden_dim(dim, mo)
    return synth.Workload(name=f"decode attention dim {dim} H {H}/{Hkv}", dim=dim, n_layers=1, n_heads=H,
                          n_kv_heads=Hkv, ffn_hidden=F, vocab_size=0, multiple_of=mo, ffn_dim_multiplier=None,
                          norm_eps=1e-5, rope_theta=10000.0, max_batch_size=Bm, max_seq_len=S, act="bf16", batch=Bm,
                          seed=seed, norm_weights="random")


def _run(pair, h, start_pos):
    hd = h.to("cuda").contiguous()
    sp = start_pos
    if isinstance(start_pos, np.ndarray):
        sp = torch.from_numpy(start_pos.astype(np.int32)).to("cuda")
    B.llama_block_forward(pair.ctx, 0, hd, sp)
    torch.cuda.synchronize()
    pair.check_error()
    return t2np(hd)


def _oracle(pair, h, start_pos):
    """The oracle's output for this call (its cache advances like the library's)."""
    return pair.oracle.block(0, t2np(h), start_pos)


def _step(pair, h, start_pos):
    """One call through the library and the oracle (which keeps its own cache)."""
    ref = _oracle(pair, h, start_pos)
    got = _run(pair, h, start_pos)
    assert_abs_close(got, ref, BF16_HIDDEN_ABS, "call")
    return got


def _decode_both(pair, h, start_pos):
    """One decode step through each kernel from the same cache (the step's own
    slot is rewritten with the same values), each checked against the oracle;
    compares the two outputs with each other."""
    ref = _oracle(pair, h, start_pos)
    outs = []
    for k in KERNELS:
        B.llama_set_decode_attention(pair.ctx, k)
        got = _run(pair, h, start_pos)
        assert_abs_close(got, ref, BF16_HIDDEN_ABS, f"kernel {k}")
        outs.append(got)
    diff = np.abs(outs[0] - outs[1]).max()
    assert diff <= BF16_HIDDEN_ABS / 2, f"kernels differ by {diff:.4g}"
    return outs


@pytest.mark.parametrize("dim,H,Hkv,Bsz", [(512, 4, 2, 1), (512, 4, 4, 2), (1024, 8, 1, 3), (2048, 16, 2, 5),
                                           (1024, 8, 8, 9), (256, 4, 1, 4), (512, 8, 2, 6), (2048, 16, 4, 2),
                                           (1536, 24, 1, 2), (2048, 16, 1, 3), (768, 6, 2, 2), (768, 12, 2, 3),
                                           (768, 12, 1, 2), (1280, 20, 1, 2), (1088, 17, 1, 2)])
def test_decode_steps_match_oracle(dim, H, Hkv, Bsz):
    w = _wl(dim, H, Hkv, Bsz)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (Bsz, 70, dim), call=0)
        _step(pair, h, 0)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:Bsz, :70] = True
        for i in range(3):
            h = synth.hidden(w, (Bsz, 1, dim), call=1 + i)
            _decode_both(pair, h, 70 + i)
            written[:Bsz, 70 + i] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("dim,H,Hkv", [(768, 6, 2), (768, 12, 2)])
def test_long_prefill_then_decode_odd_head_ratios(dim, H, Hkv):
    """3 and 6 query heads per kv head: the prefill attention serves one or two
    heads per CTA, so a CTA holds 128 or 64 positions. A 300-token prefill of
    two sequences spans several query blocks, puts the causal diagonal inside
    later blocks, and has Q boxes that run past one sequence's end."""
    w = _wl(dim, H, Hkv, 2, S=512)
    pair = Pair(w)
    try:
        _step(pair, synth.hidden(w, (2, 300, dim), call=0), 0)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:2, :300] = True
        for i in range(2):
            _decode_both(pair, synth.hidden(w, (2, 1, dim), call=1 + i), 300 + i)
            written[:2, 300 + i] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("dim,H,Hkv", [(512, 4, 1), (1024, 8, 2), (256, 4, 2)])
def test_long_ragged_histories_split_over_many_ctas(dim, H, Hkv):
    """Per-sequence device positions, one history of ~3.9k keys next to short
    ones: the stream-K split gives a unit's tiles to many CTAs whose partials
    the last of them merges."""
    w = _wl(dim, H, Hkv, 4, S=4096)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (4, 5, dim), call=0)
        _step(pair, h, 0)
        pos = np.array([5, 3900, 130, 1000])   # skipped slots stay zero on both sides
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:4, :5] = True
        for step in range(3):
            h = synth.hidden(w, (4, 1, dim), call=1 + step)
            _decode_both(pair, h, pos)
            for s in range(4):
                written[s, pos[s]] = True
            pos = pos + np.array([1, 64, 63, 129])
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


def test_single_sequence_long_history():
    """One sequence, one kv head group, 4000 keys: every CTA of the stream-K grid
    holds a piece of the same unit."""
    w = _wl(512, 4, 1, 1, S=4096)
    pair = Pair(w)
    try:
        _step(pair, synth.hidden(w, (1, 3, 512), call=0), 0)
        for step, p in enumerate((3999, 4000, 4095)):
            h = synth.hidden(w, (1, 1, 512), call=1 + step)
            _decode_both(pair, h, np.array([p]))
    finally:
        pair.close()


def test_wide_ragged_batch():
    """96 sequences with lengths spread over 1 .. 1200 keys."""
    w = _wl(512, 4, 2, 96, S=1280)
    pair = Pair(w)
    try:
        _step(pair, synth.hidden(w, (96, 2, 512), call=0), 0)
        rng = np.random.default_rng(5)
        for step in range(2):
            pos = rng.integers(2, 1200, size=96)
            _decode_both(pair, synth.hidden(w, (96, 1, 512), call=1 + step), pos)
    finally:
        pair.close()


def test_repeated_launches_rearm_counters():
    """Forty launches through one workspace, alternating the kernels."""
    w = _wl(512, 4, 2, 3, S=512)
    pair = Pair(w)
    try:
        _step(pair, synth.hidden(w, (3, 200, 512), call=0), 0)
        for i in range(40):
            B.llama_set_decode_attention(pair.ctx, KERNELS[(i // 3) % 2])
            h = synth.hidden(w, (3, 1, 512), call=1 + i)
            pos = np.array([200 + i, 17 + i, 300 + 2 * i])
            _step(pair, h, pos)
    finally:
        pair.close()


def test_graph_replay_with_device_positions():
    w = _wl(1024, 8, 2, 2, S=256)
    pair = Pair(w)
    try:
        B.llama_set_decode_attention(pair.ctx, B.LLAMA_ATTN_STREAMK)
        _step(pair, synth.hidden(w, (2, 100, 1024), call=0), 0)
        _step(pair, synth.hidden(w, (2, 1, 1024), call=9), 100)   # first launch outside the capture
        pos = torch.tensor([100, 100], dtype=torch.int32, device="cuda")
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
            p = np.array([100 + 30 * i, 101 + 60 * i])
            pos.copy_(torch.from_numpy(p.astype(np.int32)))
            g.replay()
            torch.cuda.synchronize()
            pair.check_error()
            ref = pair.oracle.block(0, t2np(hin), p)
            assert_abs_close(t2np(hd), ref, BF16_HIDDEN_ABS, f"replay {i}")
        del g
    finally:
        pair.close()


def test_mode_errors():
    w = _wl(512, 4, 2, 2, S=64)
    pair = Pair(w)
    try:
        with pytest.raises(B.LlamaError):
            B.llama_set_decode_attention(pair.ctx, 3)
        B.llama_set_decode_attention(pair.ctx, B.LLAMA_ATTN_AUTO)
        _step(pair, synth.hidden(w, (2, 4, 512), call=0), 0)
        _step(pair, synth.hidden(w, (2, 1, 512), call=1), 4)
    finally:
        pair.close()


def test_24_query_heads_per_kv_head_at_head_dim_128():
    """dim 3072, 24 query heads on one kv head, head_dim 128 (three decode groups
    of 8, prefill groups of 8): a 70-token prefill and three decode steps through
    both kernels. At ffn 8192 the fp32 accumulation alone comes near the flat
    2e-2, so the bound is the one of the full-size tests: the flat one, or 2 x
    the fp32 emulation's distance from the oracle on the same inputs."""
    from tests import emulation as E
    from tests.gpu_util import assert_close_emulated
    w = _wl(3072, 24, 1, 2)
    pair = Pair(w)
    try:
        em = E.EmuBlock(pair.oracle.layers[0], pair.oracle.args, pair.oracle.cos, pair.oracle.sin)
        ek = torch.zeros((2, w.max_seq_len, 1, 128))
        ev = torch.zeros_like(ek)
        h = synth.hidden(w, (2, 70, 3072), call=0)
        ref = _oracle(pair, h, 0)
        emu = em.forward(h, ek, ev, 0).double().numpy()
        assert_close_emulated(_run(pair, h, 0), ref, emu, BF16_HIDDEN_ABS, "dim 3072, 24/1 heads, prefill 70")
        for i in range(3):
            h = synth.hidden(w, (2, 1, 3072), call=1 + i)
            ref = _oracle(pair, h, 70 + i)
            emu = em.forward(h, ek, ev, 70 + i).double().numpy()
            outs = []
            for k in KERNELS:
                B.llama_set_decode_attention(pair.ctx, k)
                got = _run(pair, h, 70 + i)
                assert_close_emulated(got, ref, emu, BF16_HIDDEN_ABS, f"dim 3072 decode {70 + i}, kernel {k}")
                outs.append(got)
            assert np.abs(outs[0] - outs[1]).max() <= BF16_HIDDEN_ABS / 2
    finally:
        pair.close()
