"""One decoder block (llama_block_forward) against the oracle at sizes that span
several tiles and ragged tails: prefill (tcgen05 GEMMs + flash prefill),
chunked prefill at start_pos > 0, decode (GEMV + split-K decode attention)
with scalar and per-sequence positions, and the cache slots written."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.gpu_util import BF16_HIDDEN_ABS, Pair, assert_abs_close, assert_cache_matches, assert_fp32_close
from tests.helpers import t2np
import oracle as O

pytestmark = pytest.mark.gpu


def _wl(dim, H, Hkv, act="bf16", Bm=2, S=256, mo=256, seed=5):
    F = O.ffn_hidden_dim(dim, mo)
    return synth.Workload(name=f"block dim {dim} H {H}/{Hkv}", dim=dim, n_layers=1, n_heads=H, n_kv_heads=Hkv,
                          ffn_hidden=F, vocab_size=0, multiple_of=mo, ffn_dim_multiplier=None, norm_eps=1e-5,
                          rope_theta=10000.0, max_batch_size=Bm, max_seq_len=S, act=act, batch=Bm, seed=seed,
                          norm_weights="random")


def _run(pair: Pair, h: torch.Tensor, start_pos, tol_hidden):
    """One block call on both sides; returns the library's output."""
    hd = h.to("cuda").contiguous()
    sp = start_pos
    if isinstance(start_pos, np.ndarray):
        sp = torch.from_numpy(start_pos.astype(np.int32)).to("cuda")
    B.llama_block_forward(pair.ctx, 0, hd, sp)
    torch.cuda.synchronize()
    pair.check_error()
    ref = pair.oracle.block(0, t2np(h), start_pos)
    got = t2np(hd)
    if pair.w.act == "fp32":
        assert_fp32_close(got, ref, "hidden")
    else:
        assert_abs_close(got, ref, tol_hidden, "hidden")
    return got


@pytest.mark.parametrize("dim,H,Hkv", [(512, 4, 2), (512, 4, 4), (256, 4, 1), (1024, 8, 1), (1024, 8, 8),
                                       (2048, 16, 1), (2048, 32, 1)])
def test_block_prefill_chunk_and_decode(dim, H, Hkv):
    w = _wl(dim, H, Hkv)
    pair = Pair(w)
    try:
        Bsz = 2
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        # prefill 77 tokens (ragged: 64 + 13), then a chunk of 40 at start_pos 77
        h = synth.hidden(w, (Bsz, 77, dim), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        written[:Bsz, :77] = True
        h = synth.hidden(w, (Bsz, 40, dim), call=1)
        _run(pair, h, 77, BF16_HIDDEN_ABS)
        written[:Bsz, 77:117] = True
        # three decode steps with a scalar position
        for i in range(3):
            h = synth.hidden(w, (Bsz, 1, dim), call=2 + i)
            _run(pair, h, 117 + i, BF16_HIDDEN_ABS)
            written[:Bsz, 117 + i] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("dim,H,Hkv,Bsz", [(1024, 8, 2, 1), (1024, 8, 2, 4), (1024, 8, 2, 5), (2048, 16, 16, 1),
                                           (2048, 16, 4, 3), (192, 3, 1, 2)])
def test_decode_rmsnorm_inside_the_gemv(dim, H, Hkv, Bsz):
    """Decode calls of at most 4 tokens at dim <= 4096 compute both RMSNorms
    inside the GEMVs that read them (the norm weight copied into shared memory,
    the normalised rows kept resident); 5 tokens take the RMSNorm launches.
    Both against the oracle over a few steps with per-sequence positions and
    random norm weights, including dim 192 (K of 3 stages, most consumer
    threads holding no chunk of the row). dim 4096, the largest fused K, is
    the 7B-layer workload test (test_gpu_workloads.py, batch-1 decode under
    the full-size bound)."""
    w = _wl(dim, H, Hkv, Bm=Bsz, S=128)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (Bsz, 21, dim), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        pos = np.full(Bsz, 21) if Bsz > 1 else 21  # device positions for batches, a scalar for one
        for i in range(3):
            h = synth.hidden(w, (Bsz, 1, dim), call=1 + i)
            _run(pair, h, pos + i, BF16_HIDDEN_ABS)
    finally:
        pair.close()


def test_block_ragged_decode_positions():
    w = _wl(512, 4, 2, Bm=4, S=512)
    pair = Pair(w)
    try:
        lens = np.array([7, 300, 64, 129])
        # fill each sequence's history with one prefill at its own length (T differs -> separate calls
        # would need B=1; use the device-position path with T=1 after a shared prefill instead)
        h = synth.hidden(w, (4, 7, 512), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        # sequences advance to different lengths by chunked prefill of sequence-specific sizes is not
        # expressible in one call; emulate ragged histories with per-sequence positions for T = 1:
        pos = np.array([7, 7, 7, 7])
        for step in range(4):
            h = synth.hidden(w, (4, 1, 512), call=10 + step)
            _run(pair, h, pos, BF16_HIDDEN_ABS)
            pos = pos + np.array([1, 50, 20, 30])   # jump ahead: skipped slots stay zero on both sides
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:4, :7] = True
        p = np.array([7, 7, 7, 7])
        for step in range(4):
            for b in range(4):
                written[b, p[b]] = True
            p = p + np.array([1, 50, 20, 30])
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("dim,H,Hkv,Bsz", [(1024, 8, 2, 2), (1024, 8, 8, 1)])
def test_long_prefill_on_cta_pairs(dim, H, Hkv, Bsz):
    """A prefill long enough for the CTA-pair attention kernel (2048 keys or more),
    against the oracle: GQA (4 query heads per kv head, 32 positions per block) and
    MHA (128 positions per block); T = 2080 gives an odd number of query blocks in
    both (65 and 17), so the last pair's second block lies wholly past the
    sequence; device start positions put the second sequence 40 positions on."""
    T = 2080
    w = _wl(dim, H, Hkv, Bm=Bsz, S=2176)
    pair = Pair(w)
    try:
        sp = np.array([0, 40][:Bsz])
        h = synth.hidden(w, (Bsz, T, dim), call=0)
        _run(pair, h, sp, BF16_HIDDEN_ABS)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        for b in range(Bsz):
            written[b, sp[b]:sp[b] + T] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


def test_block_fp32_mode():
    w = _wl(256, 4, 2, act="fp32", S=64)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (2, 33, 256), call=0)
        _run(pair, h, 0, None)
        h = synth.hidden(w, (2, 1, 256), call=1)
        _run(pair, h, 33, None)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:2, :34] = True
        assert_cache_matches(pair, 0, written, None)
    finally:
        pair.close()


def test_position_past_cache_raises_device_flag():
    w = _wl(512, 4, 2, Bm=2, S=128)
    pair = Pair(w)
    try:
        h = torch.zeros((2, 1, 512), device="cuda")
        sp = torch.tensor([5, 128], dtype=torch.int32, device="cuda")
        B.llama_block_forward(pair.ctx, 0, h, sp)
        code, flags = B.llama_get_error(pair.ctx)
        assert code == B.LLAMA_ERR_POS_RANGE and flags & 2
        # the flag clears after it has been read
        assert B.llama_get_error(pair.ctx)[0] == B.LLAMA_OK
        # host-checked scalar positions are rejected before any launch
        with pytest.raises(B.LlamaError) as e:
            B.llama_block_forward(pair.ctx, 0, torch.zeros((2, 4, 512), device="cuda"), 126)
        assert e.value.code == B.LLAMA_ERR_INVALID_ARGS
        with pytest.raises(B.LlamaError):
            B.llama_block_forward(pair.ctx, 0, torch.zeros((3, 1, 512), device="cuda"), 0)  # B > max_batch
    finally:
        pair.close()


def test_long_context_prefill_rows_and_decode():
    """A 16384-position cache (RoPE table of 32768 positions): a 4096-token chunk
    appended at start_pos 12000 after a prefill, then a decode step at 16383."""
    w = _wl(512, 4, 1, Bm=1, S=16384)
    pair = Pair(w)
    try:
        h = synth.hidden(w, (1, 1000, 512), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        # jump: positions 1000..11999 stay zero on both sides (zero keys and values)
        h = synth.hidden(w, (1, 4096, 512), call=1)
        _run(pair, h, 12000, BF16_HIDDEN_ABS)
        h = synth.hidden(w, (1, 1, 512), call=2)
        _run(pair, h, 16383, BF16_HIDDEN_ABS)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[0, :1000] = True
        written[0, 12000:16096] = True
        written[0, 16383] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("dim,H,Hkv", [(512, 4, 2), (1024, 8, 1)])
def test_chunked_prefill_with_per_sequence_positions(dim, H, Hkv):
    """T > 1 with a device vector of start positions (chunked prefill of sequences
    at different offsets in one call). Query s of sequence b sits at position
    start_pos[b] + s and sees keys j <= start_pos[b] + s ("灵哥讲llama3(中)",
    Transformer class, mask comment). The offsets are chosen so that query blocks
    start mid-tile, the diagonal crosses key tiles, and one sequence starts at 0."""
    w = _wl(dim, H, Hkv, Bm=3, S=512)
    pair = Pair(w)
    try:
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        h = synth.hidden(w, (3, 150, dim), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        written[:3, :150] = True
        sp = np.array([150, 37, 0])          # sequence 1 and 2 rewrite part of their history
        h = synth.hidden(w, (3, 70, dim), call=1)
        _run(pair, h, sp, BF16_HIDDEN_ABS)
        for b in range(3):
            written[b, sp[b]:sp[b] + 70] = True
        sp = np.array([220, 300, 70])        # a jump: positions 107..299 of sequence 1 stay as they are
        h = synth.hidden(w, (3, 129, dim), call=2)
        _run(pair, h, sp, BF16_HIDDEN_ABS)
        for b in range(3):
            written[b, sp[b]:sp[b] + 129] = True
        # a decode step after the ragged chunks
        pos = np.array([349, 429, 199])
        _run(pair, synth.hidden(w, (3, 1, dim), call=3), pos, BF16_HIDDEN_ABS)
        for b in range(3):
            written[b, pos[b]] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        pair.close()


@pytest.mark.parametrize("mma", [B.LLAMA_GEMV_MMA_WARP, B.LLAMA_GEMV_MMA_TCGEN05])
@pytest.mark.parametrize("Bsz", [16, 19, 32])
def test_batched_decode_with_either_gemv_product(mma, Bsz):
    """Decode steps of 16, 19 and 32 sequences run the batched decode GEMV with
    every epilogue (RoPE and the cache append on wqkv, the residual add on wo
    and w2, SiLU times the gate on w1|w3); either product of that kernel
    (warp-level mma.sync, or tcgen05.mma into tensor memory with 19 tokens in
    a 32-row box) against the oracle, with per-sequence positions, and the
    cache slots written."""
    w = _wl(1024, 8, 2, Bm=Bsz, S=64)
    pair = Pair(w)
    B.llama_set_decode_linear_mma(mma)
    try:
        h = synth.hidden(w, (Bsz, 9, 1024), call=0)
        _run(pair, h, 0, BF16_HIDDEN_ABS)
        pos = 9 + (np.arange(Bsz) % 5)
        written = np.zeros((w.max_batch_size, w.max_seq_len), dtype=bool)
        written[:Bsz, :9] = True
        for i in range(3):
            h = synth.hidden(w, (Bsz, 1, 1024), call=1 + i)
            _run(pair, h, pos + i, BF16_HIDDEN_ABS)
            written[np.arange(Bsz), pos + i] = True
        assert_cache_matches(pair, 0, written, 2e-2)
    finally:
        B.llama_set_decode_linear_mma(B.LLAMA_GEMV_MMA_AUTO)
        pair.close()
