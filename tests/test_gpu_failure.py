"""Failure detection on the device without a fault: a bounded wait that
nothing completes (an mbarrier phase; the persistent kernel's grid barrier with
a CTA that never arrives) gives up after its limit (~1 s), records the timeout
bit, and the device stays usable for the next call."""
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up_and_reports(which):
    flags, secs = B.llama_selftest_bounded_wait(which)
    assert flags == 4, flags              # LLAMA_DEV_TIMEOUT, nothing else
    assert 0.9 <= secs <= 5.0, secs       # the one-second bound, not an early exit
    # the context is intact: an ordinary GEMM right after runs and is correct
    x = synth.normal((3, 256), 1.0, 1, torch.bfloat16, "cuda")
    w = synth.normal((384, 256), 0.02, 2, torch.bfloat16, "cuda")
    y = torch.empty((3, 384), device="cuda")
    B.llama_linear(x, w, y, B.LLAMA_PATH_GEMV)
    torch.cuda.synchronize()
    assert torch.allclose(y, x.float() @ w.float().T, rtol=1e-3, atol=1e-3)


def test_selftest_rejects_unknown_case():
    with pytest.raises(B.LlamaError) as e:
        B.llama_selftest_bounded_wait(7)
    assert e.value.code == B.LLAMA_ERR_INVALID_ARGS


def test_allocation_cap_mid_create_and_workspace_growth():
    """Injected allocation failure on the device: a cap at half of a model's
    footprint makes llama_create fail part-way with LLAMA_ERR_OOM and leave
    nothing allocated; a cap that blocks workspace growth makes a forward call
    fail with LLAMA_ERR_OOM, after which lifting the cap lets the same context
    run normally."""
    import oracle as O
    w = synth.Workload(name="cap model", dim=512, n_layers=2, n_heads=4, n_kv_heads=2,
                       ffn_hidden=O.ffn_hidden_dim(512, 256), vocab_size=512, multiple_of=256,
                       ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_batch_size=2, max_seq_len=64,
                       act="bf16", batch=2, seed=4)
    args = B.ModelArgs.from_workload(w)
    base = B.llama_allocated_bytes()
    m = B.Llama(args)
    need = B.llama_allocated_bytes() - base
    m.close()
    assert B.llama_allocated_bytes() == base and need > 0
    B.llama_set_alloc_limit(base + need // 2)
    try:
        with pytest.raises(B.LlamaError) as e:
            B.Llama(args)
        assert e.value.code == B.LLAMA_ERR_OOM
        assert B.llama_allocated_bytes() == base
    finally:
        B.llama_set_alloc_limit(0)
    m = B.Llama(args)
    try:
        for i in range(w.n_layers):
            B.llama_set_layer(m.ctx, i, synth.layer_weights(w, i, device="cuda"))
        enh = synth.embed_norm_head(w, device="cuda")
        B.llama_set_embed_norm_head(m.ctx, enh["tok_embeddings"], enh["norm"], enh["output"])
        tok = synth.tokens(w, (2, 16), 0, "cuda")
        logits = torch.empty((2, w.vocab_size), device="cuda")
        B.llama_set_alloc_limit(B.llama_allocated_bytes())  # no room for the activation workspace
        try:
            with pytest.raises(B.LlamaError) as e:
                B.llama_forward(m.ctx, tok, 0, logits, False)
            assert e.value.code == B.LLAMA_ERR_OOM
        finally:
            B.llama_set_alloc_limit(0)
        B.llama_forward(m.ctx, tok, 0, logits, False)
        torch.cuda.synchronize()
        assert B.llama_get_error(m.ctx)[0] == B.LLAMA_OK and torch.isfinite(logits).all()
    finally:
        m.close()
