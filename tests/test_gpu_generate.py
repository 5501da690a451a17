"""Next-token selection and the device-side generation loop through the C ABI.

llama_sample is compared with the oracle's select_next on the same fp32 logits
(integer results: equal, except where the oracle's own decision sits within
rounding of a boundary). llama_generate is compared with a host loop of
llama_forward + llama_sample (same kernels: identical tokens) and, for the fp32
tiny model, with the oracle's generate."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.helpers import build_oracle, t2np
import oracle as O

pytestmark = pytest.mark.gpu


def _near_boundary(logits, temperature, top_p, u, eps=1e-5):
    """True when the oracle's draw for u is within eps of a decision boundary."""
    z = np.exp((logits - logits.max()) / temperature)
    p = z / z.sum()
    order = np.argsort(-p, kind="stable")
    ps = p[order]
    cum = np.cumsum(ps)
    keep_margin = np.abs((cum - ps) - top_p).min()
    ps = np.where(cum - ps > top_p, 0.0, ps)
    c = np.cumsum(ps / ps.sum())
    return keep_margin < eps or np.abs(c - u).min() < eps


@pytest.mark.parametrize("V", [1000, 128256])
def test_greedy_matches_oracle_argmax(V):
    g = torch.Generator().manual_seed(V)
    logits = torch.randn((5, V), generator=g) * 3.0
    logits[2, 17] = logits[2, 99] = logits[2].max() + 1.0  # a tie: lowest index wins
    out = torch.full((5,), -1, dtype=torch.int32, device="cuda")
    B.llama_sample(logits.cuda(), out, 0.0)
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    for b in range(5):
        assert got[b] == O.select_next(logits[b].numpy(), 0.0, 1.0)
    assert got[2] == 17


@pytest.mark.parametrize("V,T,top_p", [(1000, 1.0, 0.9), (1000, 0.6, 0.5), (128256, 0.8, 0.95), (257, 1.3, 1.0),
                                       (128256, 0.2, 0.3)])
def test_top_p_matches_oracle(V, T, top_p):
    g = torch.Generator().manual_seed(V + int(100 * top_p))
    Bsz = 16
    logits = torch.randn((Bsz, V), generator=g) * 2.5
    u = torch.rand((Bsz,), generator=g) * 0.999
    out = torch.full((Bsz,), -1, dtype=torch.int32, device="cuda")
    B.llama_sample(logits.cuda(), out, T, top_p, u.cuda())
    torch.cuda.synchronize()
    got = out.cpu().numpy()
    lg = logits.double().numpy()
    mism = 0
    for b in range(Bsz):
        ref = O.select_next(lg[b], T, top_p, float(u[b]))
        if got[b] != ref:
            assert _near_boundary(lg[b], T, top_p, float(u[b])), (b, got[b], ref)
            mism += 1
    assert mism <= 1


def _small_model(act, seed=21):
    return synth.Workload(name="generation model", dim=256, n_layers=2, n_heads=4, n_kv_heads=2,
                          ffn_hidden=O.ffn_hidden_dim(256, 256), vocab_size=512, multiple_of=256,
                          ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_batch_size=3,
                          max_seq_len=64, act=act, batch=3, seed=seed, norm_weights="random")


def _load(w):
    m = B.Llama(B.ModelArgs.from_workload(w))
    lws = [synth.layer_weights(w, i) for i in range(w.n_layers)]
    enh = synth.embed_norm_head(w)
    for i, lw in enumerate(lws):
        B.llama_set_layer(m.ctx, i, {k: v.cuda() for k, v in lw.items()})
    B.llama_set_embed_norm_head(m.ctx, enh["tok_embeddings"].cuda(), enh["norm"].cuda(), enh["output"].cuda())
    return m, lws, enh


def _prompts(w, total):
    g = torch.Generator().manual_seed(5)
    lens = [6, 9, 13]
    tokens = torch.zeros((3, total), dtype=torch.int32)
    mask = torch.zeros((3, total), dtype=torch.uint8)
    for b, n in enumerate(lens):
        tokens[b, :n] = torch.randint(0, w.vocab_size, (n,), generator=g, dtype=torch.int32)
        mask[b, :n] = 1
    return tokens, mask, min(lens)


@pytest.mark.parametrize("temperature,top_p", [(0.0, 1.0), (0.8, 0.9)])
def test_generate_equals_host_loop_of_forward_and_sample(temperature, top_p):
    w = _small_model("bf16")
    total = 30
    tokens, mask, min_len = _prompts(w, total)
    uni = torch.rand((total, 3), generator=torch.Generator().manual_seed(8)) * 0.999
    m, _, _ = _load(w)
    try:
        t_dev = tokens.cuda()
        B.llama_generate(m.ctx, t_dev, mask.cuda(), min_len, temperature, top_p, uni.cuda())
        torch.cuda.synchronize()
        assert B.llama_get_error(m.ctx)[0] == B.LLAMA_OK
        got = t_dev.cpu()
        # the same steps issued from the host
        B.llama_reset(m.ctx)
        ref = tokens.clone().cuda()
        prev = 0
        for cur in range(min_len, total):
            logits = torch.empty((3, w.vocab_size), device="cuda")
            B.llama_forward(m.ctx, ref[:, prev:cur].contiguous(), prev, logits, False)
            nxt = torch.empty((3,), dtype=torch.int32, device="cuda")
            B.llama_sample(logits, nxt, temperature, top_p, uni[cur].cuda().contiguous())
            keep = mask[:, cur].cuda().bool()
            ref[:, cur] = torch.where(keep, ref[:, cur], nxt)
            prev = cur
        torch.cuda.synchronize()
        assert torch.equal(got, ref.cpu())
        # prompts are untouched and every generated id is a valid token
        assert torch.equal(got[mask.bool()], tokens[mask.bool()])
        assert int(got.min()) >= 0 and int(got.max()) < w.vocab_size
    finally:
        m.close()


def test_greedy_generate_matches_oracle_fp32():
    w = _small_model("fp32")
    total = 24
    tokens, mask, min_len = _prompts(w, total)
    m, lws, enh = _load(w)
    try:
        t_dev = tokens.cuda()
        B.llama_generate(m.ctx, t_dev, mask.cuda(), min_len, 0.0, 1.0, None)
        torch.cuda.synchronize()
        got = t_dev.cpu().numpy()
    finally:
        m.close()
    om = build_oracle(w, lws, enh)
    ref = O.generate(om, t2np(tokens).astype(np.int64), mask.numpy().astype(bool), min_len, 0.0, 1.0)
    np.testing.assert_array_equal(got, ref)
