"""Pins for the CPU oracle against facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (tests/golden), closed forms and invariants, library routines that
compute a special case (torch's bf16 cast, rms_norm, silu,
scaled_dot_product_attention, Python complex arithmetic, the transformers
Llama model), and brute-force restatements on tiny inputs.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle as O
from llama_decoder_block_kv_b200 import synth
from tests.helpers import build_oracle, t2np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------- rounding

def test_bf16_round_matches_torch_cast():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(200000, generator=g, dtype=torch.float32) * 10.0
    x = torch.cat([x, torch.tensor([0.0, -0.0, 1e-30, -1e-30, 3.0e38, 65504.0, 1.0 + 2 ** -8])])
    ref = x.to(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_round(x.numpy().astype(np.float64))
    np.testing.assert_array_equal(got, ref)


def test_bf16_round_ties_to_even():
    # bf16 keeps 7 fraction bits: the spacing at 1.0 is 2^-7.
    assert O.bf16_round(1.0 + 2 ** -8) == 1.0                    # tie, even neighbour is 1.0
    assert O.bf16_round(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6       # tie, even neighbour is up
    assert O.bf16_round(-(1.0 + 2 ** -8)) == -1.0
    assert O.bf16_round(1.0 + 2 ** -8 + 2 ** -20) == 1.0 + 2 ** -7  # above the tie


# ----------------------------------------------------------------------------- sizes

def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_ffn_hidden_matches_stated_sizes():
    rows = _golden_rows("ffn_hidden.txt")
    assert len(rows) == 4
    for dim, mult_of, mult, expect, _src in rows:
        m = None if mult == "None" else float(mult)
        assert O.ffn_hidden_dim(int(dim), int(mult_of), m) == int(expect)


def test_ffn_hidden_is_rounded_multiple():
    for dim in (128, 256, 1000, 4096, 5120, 8192):
        for mo in (1, 64, 256, 1024):
            hdim = O.ffn_hidden_dim(dim, mo)
            assert hdim % mo == 0
            assert 0 <= hdim - int(8 * dim / 3) < mo


# ----------------------------------------------------------------------------- RoPE

def test_rope_table_shapes_and_first_frequency():
    for row in _golden_rows("rope_examples.txt"):
        if row[0] == "table_shape":
            d, end, r0, r1 = map(int, row[1:])
            cos, sin = O.rope_tables(d, end, 10000.0)
            assert cos.shape == (r0, r1) and sin.shape == (r0, r1)
    cos, sin = O.rope_tables(128, 64, 10000.0)
    t = np.arange(64, dtype=np.float32)
    # freq_0 = theta^0 = 1, so column 0 holds cos/sin of the position itself
    np.testing.assert_allclose(cos[:, 0], np.cos(t.astype(np.float64)), rtol=0, atol=1e-7)
    np.testing.assert_allclose(sin[:, 0], np.sin(t.astype(np.float64)), rtol=0, atol=1e-7)
    # the last frequency is theta^(-(d-2)/d)
    cos2, sin2 = O.rope_tables(128, 2, 10000.0)
    f_last = 1.0 / 10000.0 ** (126 / 128)
    assert abs(math.atan2(sin2[1, 63], cos2[1, 63]) - f_last) < 1e-9


def test_rope_polar_convention_and_complex_product():
    row = [r for r in _golden_rows("rope_examples.txt") if r[0] == "polar_half_pi"][0]
    c, s = math.cos(math.pi / 2), math.sin(math.pi / 2)
    # rotating the unit vector (1, 0) by pi/2 gives (cos, sin) = (6.1232e-17, 1)
    out = O.apply_rope(np.array([[[1.0, 0.0]]]), np.array([0]), np.array([[c]]), np.array([[s]]))
    assert abs(out[0, 0, 0] - float(row[1])) < 1e-20 and out[0, 0, 1] == float(row[2])
    # general pairs: equal to Python's complex multiplication (x0 + i x1)(c + i s)
    rng = np.random.default_rng(0)
    D, T = 16, 5
    x = rng.standard_normal((T, 1, D))
    cos, sin = O.rope_tables(D, 32, 10000.0)
    pos = np.array([0, 1, 7, 19, 31])
    got = O.apply_rope(x, pos, cos, sin)
    for t in range(T):
        for i in range(D // 2):
            z = complex(x[t, 0, 2 * i], x[t, 0, 2 * i + 1]) * complex(float(cos[pos[t], i]), float(sin[pos[t], i]))
            assert abs(got[t, 0, 2 * i] - z.real) < 1e-14 and abs(got[t, 0, 2 * i + 1] - z.imag) < 1e-14


def test_rope_block_diagonal_matrix_form():
    # the rotation as the sparse block-diagonal matrix of the LLaMA walk-through, section 2.3
    D = 8
    rng = np.random.default_rng(1)
    cos, sin = O.rope_tables(D, 16, 10000.0)
    m = 11
    R = np.zeros((D, D))
    for i in range(D // 2):
        c, s = float(cos[m, i]), float(sin[m, i])
        R[2 * i:2 * i + 2, 2 * i:2 * i + 2] = [[c, -s], [s, c]]
    x = rng.standard_normal(D)
    got = O.apply_rope(x[None, None, :], np.array([m]), cos, sin)[0, 0]
    np.testing.assert_allclose(got, R @ x, rtol=0, atol=1e-14)


def test_rope_invariants():
    D = 64
    cos, sin = O.rope_tables(D, 256, 10000.0)
    rng = np.random.default_rng(2)
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)

    def rot(v, p):
        return O.apply_rope(v[None, None, :], np.array([p]), cos, sin)[0, 0]

    # position 0 is the identity; norms are preserved (each pair is rotated)
    np.testing.assert_array_equal(rot(q, 0), q)
    for p in (1, 5, 100, 255):
        assert abs(np.linalg.norm(rot(q, p)) - np.linalg.norm(q)) < 1e-6
    # <RoPE(q, m), RoPE(k, n)> depends on m - n only (up to the fp32 table)
    for (m, n, d) in ((10, 3, 5), (50, 50, 70), (7, 90, 33)):
        a = rot(q, m) @ rot(k, n)
        b = rot(q, m + d) @ rot(k, n + d)
        assert abs(a - b) < 1e-4 * (np.linalg.norm(q) * np.linalg.norm(k))
    # and differs for different offsets
    assert abs(rot(q, 10) @ rot(k, 3) - rot(q, 10) @ rot(k, 4)) > 1e-3


def test_rope_matches_half_split_form_on_permuted_vectors():
    # The HuggingFace form (section RoPE of "LLaMa-1/2/3 原理+源码——拆解"): q*cos + rotate_half(q)*sin
    # on vectors whose pairs sit at (i, i + D/2). De-interleaving q and k by the same
    # permutation gives the same dot products as the interleaved form.
    D = 32
    cos, sin = O.rope_tables(D, 64, 10000.0)
    rng = np.random.default_rng(3)
    q = rng.standard_normal(D)
    k = rng.standard_normal(D)
    perm = np.concatenate([np.arange(0, D, 2), np.arange(1, D, 2)])

    def half_split(v, p):
        c = np.concatenate([cos[p], cos[p]]).astype(np.float64)
        s = np.concatenate([sin[p], sin[p]]).astype(np.float64)
        rh = np.concatenate([-v[D // 2:], v[:D // 2]])
        return v * c + rh * s

    for m, n in ((3, 1), (40, 17), (63, 0)):
        a = O.apply_rope(q[None, None], np.array([m]), cos, sin)[0, 0] @ \
            O.apply_rope(k[None, None], np.array([n]), cos, sin)[0, 0]
        b = half_split(q[perm], m) @ half_split(k[perm], n)
        assert abs(a - b) < 1e-12


# ----------------------------------------------------------------------------- RMSNorm, SiLU

def test_rmsnorm_matches_torch_rms_norm():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 256)) * 3.0
    w = rng.standard_normal(256)
    got = O.rmsnorm(x, w, 1e-5, O.ACT_FP32)
    ref = F.rms_norm(torch.from_numpy(x), (256,), torch.from_numpy(w), 1e-5).numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=1e-13)


def test_rmsnorm_unit_weight_closed_form_and_scale_invariance():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((5, 4096))
    eps = 1e-5
    y = O.rmsnorm(x, np.ones(4096), eps, O.ACT_FP32)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), np.sqrt(ms / (ms + eps)), rtol=1e-12)
    # RMSNorm(a x) = RMSNorm(x) when eps = 0
    np.testing.assert_allclose(O.rmsnorm(7.5 * x, np.ones(4096), 0.0, O.ACT_FP32),
                               O.rmsnorm(x, np.ones(4096), 0.0, O.ACT_FP32), rtol=1e-12)
    # bf16 mode with unit weight: the fp32-mode result rounded once (rounding is idempotent)
    yb = O.rmsnorm(x, np.ones(4096), eps, O.ACT_BF16)
    np.testing.assert_array_equal(yb, O.bf16_round(y))


def _golden_fields(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].split()
            if line:
                out[line[0]] = np.array([float(v) for v in line[1:]])
    return out


def test_rmsnorm_bf16_weight_after_cast_back_golden():
    """The notes' RMSNorm.forward casts the normalised row back, then multiplies by
    the weight in the activation type; the HuggingFace order (weight first, one
    cast) gives a different bf16 result on the hand-worked row of the golden file."""
    g = _golden_fields("rmsnorm_bf16_order.txt")
    eps = float(g["eps"][0])
    got = O.rmsnorm(g["h"][None], g["w"], eps, O.ACT_BF16)[0]
    np.testing.assert_array_equal(got, g["bf16_notes_order"])
    assert np.all(got != g["bf16_hf_order"])
    np.testing.assert_allclose(O.rmsnorm(g["h"][None], g["w"], eps, O.ACT_FP32)[0], g["fp32"], rtol=1e-8)


def test_rmsnorm_bf16_non_unit_weight_rounding_points():
    """bf16 mode with non-unit weights: every output is a bf16 value, equals the
    (rounded) product of a bf16 value and the weight, and the weight is applied
    per column (a row of equal inputs reproduces the weight vector's pattern)."""
    rng = np.random.default_rng(9)
    dim = 512
    w = O.bf16_round(1.0 + 0.1 * rng.standard_normal(dim))
    x = rng.standard_normal((6, dim)) * 2.0
    y = O.rmsnorm(x, w, 1e-5, O.ACT_BF16)
    np.testing.assert_array_equal(y, O.bf16_round(y))
    # a constant row normalises to 1 (up to eps) in every column: the output is bf16(w)
    c = O.rmsnorm(np.full((1, dim), 3.0), w, 0.0, O.ACT_BF16)[0]
    np.testing.assert_array_equal(c, w)
    # the result differs from the weight-first (one-rounding) order somewhere on random data
    yhf = O.bf16_round(x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + 1e-5) * w)
    assert np.any(y != yhf)
    # a permuted weight vector permutes nothing else: swapping two columns of x and w swaps the output
    xs, ws = x.copy(), w.copy()
    xs[:, [3, 77]] = xs[:, [77, 3]]
    ws[[3, 77]] = ws[[77, 3]]
    ys = O.rmsnorm(xs, ws, 1e-5, O.ACT_BF16)
    np.testing.assert_array_equal(ys[:, [3, 77]], y[:, [77, 3]])


def test_silu_identities_and_library():
    a = np.linspace(-30, 30, 601)
    s = O.silu(a)
    assert O.silu(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(O.silu(-a), s - a, atol=1e-12)      # silu(-x) = silu(x) - x
    assert abs(O.silu(np.array([40.0]))[0] - 40.0) < 1e-12
    np.testing.assert_allclose(s, F.silu(torch.from_numpy(a)).numpy(), rtol=1e-14, atol=1e-300)


# ----------------------------------------------------------------------------- attention

def _sdpa_reference(q, ck, cv, start_pos, n_rep):
    """torch's scaled_dot_product_attention on the pages' additive mask (float64)."""
    B, T, H, D = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        L = int(start_pos[b]) + T
        qt = torch.from_numpy(q[b]).permute(1, 0, 2)[None]              # [1, H, T, D]
        kt = torch.from_numpy(ck[b, :L]).permute(1, 0, 2)[None]        # [1, Hkv, L, D]
        vt = torch.from_numpy(cv[b, :L]).permute(1, 0, 2)[None]
        # the mask of the LLaMA-2/3 Transformer.forward: zeros for the cached columns,
        # then an upper-triangular -inf block over the new tokens
        tri = torch.triu(torch.full((T, T), float("-inf"), dtype=torch.float64), diagonal=1)
        mask = torch.hstack([torch.zeros((T, int(start_pos[b])), dtype=torch.float64), tri])
        o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, enable_gqa=(n_rep > 1))
        out[b] = o[0].permute(1, 0, 2).numpy()
    return out


@pytest.mark.parametrize("H,Hkv,T,start", [(4, 4, 6, [0, 0]), (8, 2, 5, [3, 9]), (6, 1, 1, [12, 4]),
                                            (4, 2, 7, [0, 5])])
def test_attention_matches_library_sdpa(H, Hkv, T, start):
    rng = np.random.default_rng(6)
    B, D, S = 2, 16, 32
    q = rng.standard_normal((B, T, H, D))
    ck = rng.standard_normal((B, S, Hkv, D))
    cv = rng.standard_normal((B, S, Hkv, D))
    sp = np.array(start)
    got = O.causal_gqa_attention(q, ck, cv, sp, H // Hkv)
    ref = _sdpa_reference(q, ck, cv, sp, H // Hkv)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_attention_equal_keys_give_mean_of_visible_values():
    rng = np.random.default_rng(7)
    B, T, H, D, S = 1, 3, 2, 8, 16
    q = rng.standard_normal((B, T, H, D))
    ck = np.tile(rng.standard_normal(D), (B, S, H, 1))
    cv = rng.standard_normal((B, S, H, D))
    got = O.causal_gqa_attention(q, ck, cv, np.array([4]), 1)
    for s in range(T):
        np.testing.assert_allclose(got[0, s], np.broadcast_to(cv[0, :4 + s + 1].mean(axis=0), (H, D)), atol=1e-12)


def test_attention_two_token_hand_example():
    # one head, D = 2; query at position 1 sees keys 0 and 1
    q = np.array([1.0, 0.0])
    k = np.array([[1.0, 0.0], [0.0, 1.0]])
    v = np.array([[1.0, 2.0], [3.0, 4.0]])
    e0, e1 = math.exp(1.0 / math.sqrt(2.0)), math.exp(0.0)
    expect = (e0 * v[0] + e1 * v[1]) / (e0 + e1)
    qq = np.zeros((1, 1, 1, 2)); qq[0, 0, 0] = q
    ck = np.zeros((1, 4, 1, 2)); ck[0, :2, 0] = k
    cv = np.zeros((1, 4, 1, 2)); cv[0, :2, 0] = v
    got = O.causal_gqa_attention(qq, ck, cv, np.array([1]), 1)
    np.testing.assert_allclose(got[0, 0, 0], expect, rtol=1e-15)
    # at position 0 only key 0 is visible
    got0 = O.causal_gqa_attention(qq, ck, cv, np.array([0]), 1)
    np.testing.assert_allclose(got0[0, 0, 0], v[0], rtol=1e-15)


# ----------------------------------------------------------------------------- block / model

def _tiny(act="fp32", **kw):
    base = dict(name="pin", dim=64, n_layers=2, n_heads=4, n_kv_heads=2, ffn_hidden=O.ffn_hidden_dim(64, 32),
                vocab_size=97, multiple_of=32, ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0,
                max_batch_size=2, max_seq_len=32, act=act, batch=2, seed=3)
    base.update(kw)
    w = synth.Workload(**base)
    return w, [synth.layer_weights(w, i) for i in range(w.n_layers)], synth.embed_norm_head(w)


def _repeat_kv_rows(wk, Hkv, n_rep, D):
    # an MHA projection whose head h is the GQA kv head h // n_rep (rows repeated per group)
    blocks = [wk[g * D:(g + 1) * D] for g in range(Hkv) for _ in range(n_rep)]
    return torch.cat(blocks, 0)


@pytest.mark.parametrize("Hkv", [2, 1])
def test_gqa_and_mqa_equal_mha_with_repeated_kv(Hkv):
    w, lws, enh = _tiny(n_kv_heads=Hkv)
    n_rep = w.n_heads // Hkv
    m_gqa = build_oracle(w, lws, enh)
    lws_mha = []
    for lw in lws:
        lw2 = dict(lw)
        lw2["wk"] = _repeat_kv_rows(lw["wk"], Hkv, n_rep, w.head_dim)
        lw2["wv"] = _repeat_kv_rows(lw["wv"], Hkv, n_rep, w.head_dim)
        lws_mha.append(lw2)
    m_mha = build_oracle(w.with_(n_kv_heads=w.n_heads), lws_mha, enh)
    tok = t2np(synth.tokens(w, (2, 9))).astype(np.int64)
    a = m_gqa.forward(tok, 0)
    b = m_mha.forward(tok, 0)
    np.testing.assert_allclose(a, b, rtol=1e-12, atol=1e-12)
    # and the MHA cache holds each GQA kv head n_rep times
    for layer in range(w.n_layers):
        for h in range(w.n_heads):
            # equal up to the float64 summation order of differently shaped matmuls
            np.testing.assert_allclose(m_mha.cache_k[layer][:, :, h], m_gqa.cache_k[layer][:, :, h // n_rep],
                                       rtol=0, atol=1e-14)


@pytest.mark.parametrize("act", ["fp32", "bf16"])
def test_decode_with_cache_equals_recompute(act):
    w, lws, enh = _tiny(act=act)
    tok = t2np(synth.tokens(w, (2, 16))).astype(np.int64)
    full = build_oracle(w, lws, enh).forward(tok, 0)                    # [2, 16, V]
    inc = build_oracle(w, lws, enh)
    parts = [inc.forward(tok[:, :8], 0)]
    for s in range(8, 16):
        parts.append(inc.forward(tok[:, s:s + 1], s))
    got = np.concatenate(parts, axis=1)
    tol = 1e-10 if act == "fp32" else 2e-2
    np.testing.assert_allclose(got, full, rtol=0, atol=tol)
    # chunked prefill (chunks of 4 at start_pos 0, 4, 8, 12) equals one prefill
    ch = build_oracle(w, lws, enh)
    got2 = np.concatenate([ch.forward(tok[:, c:c + 4], c) for c in range(0, 16, 4)], axis=1)
    np.testing.assert_allclose(got2, full, rtol=0, atol=tol)


def test_ragged_start_positions_equal_per_sequence_calls():
    w, lws, enh = _tiny()
    m = build_oracle(w, lws, enh)
    tok = t2np(synth.tokens(w, (2, 12))).astype(np.int64)
    m.forward(tok[:, :6], 0)
    m.forward(tok[:1, 6:9], 6)          # sequence 0 runs ahead by 3 tokens
    got = m.forward(np.stack([tok[0, 9:10], tok[1, 6:7]]), np.array([9, 6]))
    ref = build_oracle(w, lws, enh)
    r0 = ref.forward(tok[:1, :10], 0)[0, -1]
    ref2 = build_oracle(w, lws, enh)
    r1 = ref2.forward(tok[1:2, :7], 0)[0, -1]
    np.testing.assert_allclose(got[0, 0], r0, atol=1e-10)
    np.testing.assert_allclose(got[1, 0], r1, atol=1e-10)


def test_causality_later_tokens_do_not_change_earlier_logits():
    w, lws, enh = _tiny()
    tok = t2np(synth.tokens(w, (1, 10))).astype(np.int64)
    a = build_oracle(w, lws, enh).forward(tok, 0)
    tok2 = tok.copy()
    tok2[0, 6] = (tok2[0, 6] + 1) % w.vocab_size
    b = build_oracle(w, lws, enh).forward(tok2, 0)
    np.testing.assert_array_equal(a[0, :6], b[0, :6])
    assert np.abs(a[0, 6:] - b[0, 6:]).max() > 1e-6


def test_cache_slots_written_exactly():
    w, lws, enh = _tiny(act="bf16")
    m = build_oracle(w, lws, enh)
    sentinel = 12345.0
    for layer in range(w.n_layers):
        m.cache_k[layer][:] = sentinel
        m.cache_v[layer][:] = sentinel
    # sequence b's cache is valid below start_pos[b]; fill that part with finite values
    sp = np.array([5, 9])
    rng = np.random.default_rng(8)
    for layer in range(w.n_layers):
        for b in range(2):
            m.cache_k[layer][b, :sp[b]] = O.bf16_round(rng.standard_normal(m.cache_k[layer][b, :sp[b]].shape))
            m.cache_v[layer][b, :sp[b]] = O.bf16_round(rng.standard_normal(m.cache_v[layer][b, :sp[b]].shape))
    before = [(k.copy(), v.copy()) for k, v in zip(m.cache_k, m.cache_v)]
    tok = t2np(synth.tokens(w, (2, 3))).astype(np.int64)
    m.forward(tok, sp)
    for layer in range(w.n_layers):
        for c_new, c_old in ((m.cache_k[layer], before[layer][0]), (m.cache_v[layer], before[layer][1])):
            changed = np.any(c_new != c_old, axis=(2, 3))        # [B_max, S_max]
            expect = np.zeros_like(changed)
            for b in range(2):
                expect[b, sp[b]:sp[b] + 3] = True
            np.testing.assert_array_equal(changed, expect)


@pytest.mark.slow
def test_whole_model_matches_transformers_llama():
    """The fp32-mode oracle equals the transformers Llama model run in float64.

    That model uses the half-split RoPE pairing; the interleaved weights map onto it
    by permuting each head's rows of wq and wk (pairs (2i, 2i+1) -> (i, i + D/2)),
    which leaves every q.k dot product unchanged.
    """
    transformers = pytest.importorskip("transformers")
    w, lws, enh = _tiny(n_layers=2, n_kv_heads=2, max_seq_len=32)
    cfg = transformers.LlamaConfig(
        vocab_size=w.vocab_size, hidden_size=w.dim, intermediate_size=w.ffn_hidden,
        num_hidden_layers=w.n_layers, num_attention_heads=w.n_heads, num_key_value_heads=w.n_kv_heads,
        rms_norm_eps=w.norm_eps, max_position_embeddings=2 * w.max_seq_len, tie_word_embeddings=False,
        rope_parameters={"rope_type": "default", "rope_theta": w.rope_theta}, attention_bias=False,
        mlp_bias=False)
    hf = transformers.LlamaForCausalLM(cfg).double().eval()
    D = w.head_dim
    perm_head = torch.cat([torch.arange(0, D, 2), torch.arange(1, D, 2)])

    def permute_rows(wt, n_heads):
        idx = torch.cat([h * D + perm_head for h in range(n_heads)])
        return wt.double()[idx]

    with torch.no_grad():
        hf.model.embed_tokens.weight.copy_(enh["tok_embeddings"].double())
        hf.model.norm.weight.copy_(enh["norm"].double())
        hf.lm_head.weight.copy_(enh["output"].double())
        for i, lw in enumerate(lws):
            L = hf.model.layers[i]
            L.self_attn.q_proj.weight.copy_(permute_rows(lw["wq"], w.n_heads))
            L.self_attn.k_proj.weight.copy_(permute_rows(lw["wk"], w.n_kv_heads))
            L.self_attn.v_proj.weight.copy_(lw["wv"].double())
            L.self_attn.o_proj.weight.copy_(lw["wo"].double())
            L.mlp.gate_proj.weight.copy_(lw["w1"].double())
            L.mlp.up_proj.weight.copy_(lw["w3"].double())
            L.mlp.down_proj.weight.copy_(lw["w2"].double())
            L.input_layernorm.weight.copy_(lw["attn_norm"].double())
            L.post_attention_layernorm.weight.copy_(lw["ffn_norm"].double())
    tok = synth.tokens(w, (2, 20))
    ref = hf(input_ids=tok.long()).logits.detach().numpy()
    got = build_oracle(w, lws, enh).forward(t2np(tok).astype(np.int64), 0)
    # the library keeps its RMSNorm statistics and RoPE angles in fp32
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()


def test_block_forward_rows_is_block_forward_restricted():
    w, lws, enh = _tiny(act="bf16", n_layers=1)
    m = build_oracle(w, lws, enh)
    h = t2np(synth.hidden(w, (2, 7, w.dim)))
    sp = np.array([0, 5])
    full = m.block(0, h, sp)
    rows = [(0, 0), (0, 6), (1, 0), (1, 3), (1, 6)]
    got = O.block_forward_rows(h, m.layers[0], sp, m.args, m.cos, m.sin, rows)
    for i, (b, s) in enumerate(rows):
        np.testing.assert_allclose(got[i], full[b, s], rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------- next-token selection

def test_select_next_greedy_is_first_argmax():
    logits = np.array([0.1, 3.0, -1.0, 3.0, 2.9])
    assert O.select_next(logits, 0.0, 0.9) == 1          # first of the tied maxima
    assert O.select_next(logits, -1.0, 0.9) == 1


def test_select_next_top_p_hand_example():
    # probabilities 0.5, 0.3, 0.2 (logits are their logs, temperature 1): with top_p = 0.6 the
    # sorted cumulative sums are 0.5, 0.8, 1.0 and cum - p = 0, 0.5, 0.8, so the third token is
    # dropped; the kept pair renormalises to 0.625, 0.375.
    logits = np.log(np.array([0.2, 0.5, 0.3]))           # indices 1, 2, 0 in descending order
    assert O.select_next(logits, 1.0, 0.6, 0.10) == 1
    assert O.select_next(logits, 1.0, 0.6, 0.62) == 1
    assert O.select_next(logits, 1.0, 0.6, 0.63) == 2
    assert O.select_next(logits, 1.0, 0.6, 0.99) == 2    # token 0 never drawn
    # top_p = 1 keeps everything: plain inverse CDF over 0.5, 0.3, 0.2
    assert O.select_next(logits, 1.0, 1.0, 0.85) == 0


def test_select_next_frequencies_follow_renormalised_top_p():
    rng = np.random.default_rng(11)
    logits = rng.standard_normal(40) * 2.0
    T, top_p = 0.7, 0.8
    z = np.exp((logits - logits.max()) / T)
    probs = z / z.sum()
    order = np.argsort(-probs, kind="stable")
    cum = np.cumsum(probs[order])
    keep = order[(cum - probs[order]) <= top_p]
    target = np.zeros(40)
    target[keep] = probs[keep] / probs[keep].sum()
    us = (np.arange(20000) + 0.5) / 20000                 # a uniform grid of draws
    counts = np.bincount([O.select_next(logits, T, top_p, u) for u in us], minlength=40) / len(us)
    np.testing.assert_allclose(counts, target, atol=2e-4)


def test_generate_keeps_prompts_and_matches_stepwise_forward():
    w, lws, enh = _tiny(n_layers=1)
    m = build_oracle(w, lws, enh)
    rng = np.random.default_rng(12)
    total = 12
    tokens = np.zeros((2, total), dtype=np.int64)
    tokens[0, :5] = rng.integers(0, w.vocab_size, 5)
    tokens[1, :8] = rng.integers(0, w.vocab_size, 8)
    mask = np.zeros((2, total), dtype=bool)
    mask[0, :5] = True
    mask[1, :8] = True
    out = O.generate(m, tokens, mask, 5, 0.0, 1.0)
    np.testing.assert_array_equal(out[0, :5], tokens[0, :5])
    np.testing.assert_array_equal(out[1, :8], tokens[1, :8])
    # greedy continuation of sequence 0 equals argmax of a one-sequence recompute at each step
    m2 = build_oracle(w, lws, enh)
    for cur in range(5, total):
        logits = m2.forward(out[:1, :cur], 0, all_positions=False)
        m2 = build_oracle(w, lws, enh)
        assert out[0, cur] == int(np.argmax(logits[0]))
