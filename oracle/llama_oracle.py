"""CPU oracle for the LLaMA decoder block with a KV-cache.

TEST INFRASTRUCTURE ONLY. This module is the plain, slow, obviously correct
definition that the CUDA library is checked against. Only the tests, the
package's ``smoke()`` entry and the bench's CPU-baseline / reference legs may
import it; the CUDA product path never calls it and shares no code with it.

Everything is computed in float64 with numpy (a matmul is the only library
primitive used as a step). The one place where precision is a *definition*
rather than an accuracy choice is the bfloat16 rounding applied where the
pages cast back to the activation dtype (``act="bf16"``); in ``act="fp32"``
mode nothing is rounded.

Sources, cited by page title and section throughout:

[P1] "LLaMa-1/2/3 原理+源码——拆解 (KV-Cache, RoPE, RMSNorm, GQA, SwiGLU)"
     (aitechtogether.com/it/357112): sections RMS Norm, RoPE, SwiGLU Function,
     KV-Cache, Grouped Query Attention.
[P2] "LLaMA v1/2模型结构总览" (aitechtogether.com/it/312168): size table,
     GQA, RMSNorm, SwiGLU.
[P3] LLaMA-1 model.py walk-through (linkmax.top/l/4uqMqwhr28): §2.3 RoPE
     (element-wise form of the rotation), §3.2 model.
[P4] "LLaMA: Open and Efficient Foundation Language Models" notes
     (unpurerationalist.github.io): §3 code (ModelArgs, RMSNorm,
     precompute_freqs_cis, apply_rotary_emb, repeat_kv, Attention,
     FeedForward, TransformerBlock, Transformer).
[P5] "灵哥讲llama3(中)" (blog.csdn.net/RussellTheRush/article/details/139664760):
     Transformer class (rope_theta, the cached causal-mask comment).

Readings where the pages are silent or disagree are stated at the function
that applies them.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np

ACT_FP32 = "fp32"
ACT_BF16 = "bf16"


# ----------------------------------------------------------------------------
# Rounding and storage helpers
# ----------------------------------------------------------------------------

def bf16_round(x) -> np.ndarray:
    """Round to the nearest bfloat16 value, ties to even; return float64.

    The value is first taken to float32 (the GPU computes in fp32), then the low
    16 bits of the fp32 pattern are rounded away: add 0x7FFF plus the lowest
    kept bit, then truncate. This is the IEEE round-to-nearest-even rule on the
    8-bit-exponent / 7-bit-mantissa format.
    """
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = x32.view(np.uint32).astype(np.uint64)
    keep_lsb = (u >> np.uint64(16)) & np.uint64(1)
    u = ((u + np.uint64(0x7FFF) + keep_lsb) >> np.uint64(16)) << np.uint64(16)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def act_round(x, act: str) -> np.ndarray:
    """Cast back to the activation dtype ([P4] ``.type_as(x)``): bf16 rounds, fp32 keeps float64."""
    if act == ACT_BF16:
        return bf16_round(x)
    if act == ACT_FP32:
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"unknown activation type {act!r}")


def bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    """Widen raw bfloat16 bit patterns (uint16) to float64 values (exact)."""
    u = np.ascontiguousarray(u16, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def as_f64(w) -> np.ndarray:
    """Weights may be held as raw bf16 bits (uint16) to save host memory; widen on use."""
    w = np.asarray(w)
    if w.dtype == np.uint16:
        return bf16_bits_to_f64(w)
    return w.astype(np.float64, copy=False)


# ----------------------------------------------------------------------------
# ModelArgs and the derived sizes
# ----------------------------------------------------------------------------

def ffn_hidden_dim(dim: int, multiple_of: int, ffn_dim_multiplier: Optional[float] = None) -> int:
    """SwiGLU hidden size, [P4] FeedForward.__init__ called from TransformerBlock with 4*dim.

    Two thirds of 4*dim, truncated; scaled by ffn_dim_multiplier when given and
    truncated again; then rounded up to a multiple of ``multiple_of``.
    """
    hidden = 4 * dim
    hidden = int(2 * hidden / 3)
    if ffn_dim_multiplier is not None:
        hidden = int(ffn_dim_multiplier * hidden)
    return multiple_of * ((hidden + multiple_of - 1) // multiple_of)


@dataclass
class ModelArgs:
    """[P4] ModelArgs plus rope_theta ([P5] Transformer class) and the activation dtype."""
    dim: int = 4096
    n_layers: int = 32
    n_heads: int = 32
    n_kv_heads: Optional[int] = None
    vocab_size: int = -1
    multiple_of: int = 256
    ffn_dim_multiplier: Optional[float] = None
    norm_eps: float = 1e-5
    rope_theta: float = 10000.0
    max_batch_size: int = 32
    max_seq_len: int = 2048
    act: str = ACT_BF16

    @property
    def kv_heads(self) -> int:
        return self.n_heads if self.n_kv_heads is None else self.n_kv_heads

    @property
    def head_dim(self) -> int:
        return self.dim // self.n_heads

    @property
    def n_rep(self) -> int:
        return self.n_heads // self.kv_heads

    @property
    def ffn_hidden(self) -> int:
        return ffn_hidden_dim(self.dim, self.multiple_of, self.ffn_dim_multiplier)


# ----------------------------------------------------------------------------
# The ops
# ----------------------------------------------------------------------------

def rope_tables(head_dim: int, end: int, theta: float):
    """cos/sin of the rotation angles, float32 arrays of shape [end, head_dim // 2].

    [P4] precompute_freqs_cis: freq_i = 1 / theta^(2i/d) for i < d/2; the angle
    at position t is the outer product t * freq_i (taken in fp32, as torch.outer
    of fp32 vectors); polar(1, angle) = cos(angle) + i sin(angle) ([P3] §3.2,
    torch.polar). Reading: freq_i is evaluated in double and rounded to fp32;
    the angle is one fp32 multiply; cos/sin are evaluated in double on that fp32
    angle and rounded to fp32. The table spans ``end`` positions; the model
    uses end = 2 * max_seq_len ([P4] Transformer.__init__).
    """
    i = np.arange(head_dim // 2, dtype=np.float64)
    freqs = (1.0 / np.power(np.float64(theta), 2.0 * i / head_dim)).astype(np.float32)
    t = np.arange(end, dtype=np.float32)
    angles = np.multiply.outer(t, freqs)  # float32 x float32 -> float32, one rounding
    cos = np.cos(angles.astype(np.float64)).astype(np.float32)
    sin = np.sin(angles.astype(np.float64)).astype(np.float32)
    return cos, sin


def rmsnorm(h: np.ndarray, weight: np.ndarray, eps: float, act: str) -> np.ndarray:
    """[P4] RMSNorm.forward: ``_norm(x.float()).type_as(x) * weight``.

    _norm(x) = x * rsqrt(mean(x^2) + eps) over the last axis, with the statistics
    in (at least) fp32; the result is cast back to the activation dtype, then
    multiplied by the weight in that dtype (so it is rounded once more).
    """
    h = np.asarray(h, dtype=np.float64)
    ms = np.mean(h * h, axis=-1, keepdims=True)
    xhat = act_round(h / np.sqrt(ms + eps), act)
    return act_round(xhat * as_f64(weight), act)


def apply_rope(x: np.ndarray, pos: np.ndarray, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """Rotate interleaved pairs (x[2i], x[2i+1]) by the angle of position ``pos``.

    [P3] §2.3: out = x * [c0,c0,c1,c1,...] + [-x1,x0,-x3,x2,...] * [s0,s0,s1,s1,...],
    i.e. out[2i] = x[2i] c_i - x[2i+1] s_i and out[2i+1] = x[2i+1] c_i + x[2i] s_i,
    which is the complex product (x[2i] + i x[2i+1]) * (c_i + i s_i) of [P4]
    apply_rotary_emb. ``x`` has shape [..., heads, D]; ``pos`` has the leading
    shape [...] of x without the last two axes.
    """
    x = np.asarray(x, dtype=np.float64)
    c = cos[pos].astype(np.float64)[..., None, :]
    s = sin[pos].astype(np.float64)[..., None, :]
    xe = x[..., 0::2]
    xo = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xo * c + xe * s
    return out


def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + e^-a) ([P1] SwiGLU Function; [P4] FeedForward)."""
    a = np.asarray(a, dtype=np.float64)
    return a / (1.0 + np.exp(-a))


def causal_gqa_attention(q: np.ndarray, cache_k: np.ndarray, cache_v: np.ndarray,
                         start_pos: np.ndarray, n_rep: int) -> np.ndarray:
    """Scaled dot-product attention of new queries over the cache, causal and grouped.

    q: [B, T, H, D]; cache_k, cache_v: [B_max, S_max, Hkv, D] (the pages' cache
    layout, [P4] Attention.__init__), already holding this call's keys/values.
    Query s of sequence b sits at position p = start_pos[b] + s and sees keys
    j <= p ([P5] mask comment: row i is token cache_len + i and the masked
    entries are j > cache_len + i; [P4] Transformer.forward). Query head h reads
    kv head h // n_rep ([P4] repeat_kv expands kv head j to q heads
    j*n_rep ... j*n_rep + n_rep - 1). Scores are scaled by 1/sqrt(D) and
    soft-maxed ([P4] Attention.forward). A dense loop over all visible keys:
    no tiling, no splitting.
    """
    B, T, H, D = q.shape
    out = np.zeros((B, T, H, D), dtype=np.float64)
    scale = 1.0 / np.sqrt(D)
    n_kv = H // n_rep
    for b in range(B):
        for s in range(T):
            p = int(start_pos[b]) + s
            for g in range(n_kv):
                K = np.asarray(cache_k[b, :p + 1, g, :], dtype=np.float64)  # [p+1, D]
                V = np.asarray(cache_v[b, :p + 1, g, :], dtype=np.float64)
                qg = q[b, s, g * n_rep:(g + 1) * n_rep, :]                 # [n_rep, D]
                scores = (qg @ K.T) * scale                                # [n_rep, p+1]
                scores = scores - scores.max(axis=-1, keepdims=True)
                w = np.exp(scores)
                w = w / w.sum(axis=-1, keepdims=True)
                out[b, s, g * n_rep:(g + 1) * n_rep, :] = w @ V
    return out


# ----------------------------------------------------------------------------
# The block and the model
# ----------------------------------------------------------------------------

LAYER_KEYS = ("wq", "wk", "wv", "wo", "w1", "w2", "w3", "attn_norm", "ffn_norm")


def _positions(start_pos, B: int) -> np.ndarray:
    sp = np.asarray(start_pos, dtype=np.int64)
    if sp.ndim == 0:
        sp = np.full((B,), int(sp), dtype=np.int64)
    return sp


def block_forward(h: np.ndarray, lw: dict, cache_k: np.ndarray, cache_v: np.ndarray,
                  start_pos, args: ModelArgs, cos: np.ndarray, sin: np.ndarray) -> np.ndarray:
    """One decoder block, [P4] TransformerBlock.forward with Attention and FeedForward.

    h: [B, T, dim] residual stream (float64; the residual is kept unrounded,
    a reading: the GPU keeps it in fp32). Writes this call's k and v into the
    caches at positions start_pos[b] + s, s < T ([P4] Attention.forward cache
    slice assignment), then

        h   = h + wo( attention( rope(wq xn), rope(wk xn), wv xn ) ),  xn = attention_norm(h)
        out = h + w2( silu(w1 xn2) * w3 xn2 ),                          xn2 = ffn_norm(h)

    Activations are rounded to the activation dtype where the pages cast back or
    store: the norm outputs, q/k after RoPE and v (the cache dtype), the
    attention output and silu(w1 x) * w3 x.
    """
    act = args.act
    B, T, dim = h.shape
    H, Hkv, D = args.n_heads, args.kv_heads, args.head_dim
    sp = _positions(start_pos, B)
    pos = sp[:, None] + np.arange(T)[None, :]                  # [B, T]
    if np.any(pos >= cache_k.shape[1]):
        raise ValueError("start_pos + T exceeds max_seq_len")

    # attention half
    xn = rmsnorm(h, lw["attn_norm"], args.norm_eps, act)
    xq = (xn @ as_f64(lw["wq"]).T).reshape(B, T, H, D)
    xk = (xn @ as_f64(lw["wk"]).T).reshape(B, T, Hkv, D)
    xv = (xn @ as_f64(lw["wv"]).T).reshape(B, T, Hkv, D)
    xq = act_round(apply_rope(xq, pos, cos, sin), act)
    xk = act_round(apply_rope(xk, pos, cos, sin), act)
    xv = act_round(xv, act)
    for b in range(B):
        cache_k[b, sp[b]:sp[b] + T] = xk[b]
        cache_v[b, sp[b]:sp[b] + T] = xv[b]
    o = causal_gqa_attention(xq, cache_k, cache_v, sp, args.n_rep)
    o = act_round(o.reshape(B, T, H * D), act)
    h = h + o @ as_f64(lw["wo"]).T

    # feed-forward half
    xn2 = rmsnorm(h, lw["ffn_norm"], args.norm_eps, act)
    a = xn2 @ as_f64(lw["w1"]).T
    b3 = xn2 @ as_f64(lw["w3"]).T
    g = act_round(silu(a) * b3, act)
    return h + g @ as_f64(lw["w2"]).T


def block_forward_rows(h: np.ndarray, lw: dict, start_pos, args: ModelArgs, cos: np.ndarray,
                       sin: np.ndarray, rows) -> np.ndarray:
    """block_forward restricted to selected output rows (large prefills).

    The keys and values of every token of the call are computed (attention of a
    row needs all earlier positions); queries, the attention, the output
    projection and the feed-forward half are computed only for ``rows``, a list
    of (b, s) pairs. Returns [len(rows), dim]: row i equals
    block_forward(h, ...)[b_i, s_i]. Same definition, fewer rows.
    """
    act = args.act
    B, T, dim = h.shape
    H, Hkv, D = args.n_heads, args.kv_heads, args.head_dim
    sp = _positions(start_pos, B)
    pos = sp[:, None] + np.arange(T)[None, :]
    K = np.zeros((B, int(pos.max()) + 1, Hkv, D))
    V = np.zeros_like(K)
    xn = rmsnorm(h, lw["attn_norm"], args.norm_eps, act)
    xk = act_round(apply_rope((xn @ as_f64(lw["wk"]).T).reshape(B, T, Hkv, D), pos, cos, sin), act)
    xv = act_round((xn @ as_f64(lw["wv"]).T).reshape(B, T, Hkv, D), act)
    for b in range(B):
        K[b, sp[b]:sp[b] + T] = xk[b]
        V[b, sp[b]:sp[b] + T] = xv[b]
    out = np.zeros((len(rows), dim))
    for i, (b, s) in enumerate(rows):
        p = np.array([pos[b, s]])
        q = act_round(apply_rope((xn[b, s] @ as_f64(lw["wq"]).T).reshape(1, 1, H, D), p[None], cos, sin), act)
        o = causal_gqa_attention(q, K[b:b + 1], V[b:b + 1], p, args.n_rep)
        o = act_round(o.reshape(1, H * D), act)
        hr = h[b, s][None] + o @ as_f64(lw["wo"]).T
        xn2 = rmsnorm(hr, lw["ffn_norm"], args.norm_eps, act)
        g = act_round(silu(xn2 @ as_f64(lw["w1"]).T) * (xn2 @ as_f64(lw["w3"]).T), act)
        out[i] = (hr + g @ as_f64(lw["w2"]).T)[0]
    return out


@dataclass
class OracleModel:
    """The whole model of [P4] Transformer: embedding, blocks, final norm, LM head.

    Holds the weights (float64 or raw bf16 bits), one K and one V cache per
    layer of shape [max_batch_size, max_seq_len, n_kv_heads, head_dim]
    initialised to zero ([P4] Attention.__init__), and the RoPE table of
    2 * max_seq_len positions ([P4] Transformer.__init__).
    """
    args: ModelArgs
    layers: list = field(default_factory=list)
    tok_embeddings: Optional[np.ndarray] = None
    norm: Optional[np.ndarray] = None
    output: Optional[np.ndarray] = None

    def __post_init__(self):
        a = self.args
        if not self.layers:
            self.layers = [None] * a.n_layers
        shape = (a.max_batch_size, a.max_seq_len, a.kv_heads, a.head_dim)
        self.cache_k = [np.zeros(shape) for _ in range(a.n_layers)]
        self.cache_v = [np.zeros(shape) for _ in range(a.n_layers)]
        self.cos, self.sin = rope_tables(a.head_dim, 2 * a.max_seq_len, a.rope_theta)

    def block(self, layer: int, h: np.ndarray, start_pos) -> np.ndarray:
        """One block on hidden states h [B, T, dim] (single-layer configs)."""
        return block_forward(np.asarray(h, dtype=np.float64), self.layers[layer],
                             self.cache_k[layer], self.cache_v[layer], start_pos,
                             self.args, self.cos, self.sin)

    def forward(self, tokens: np.ndarray, start_pos, all_positions: bool = True,
                layers: Optional[Sequence[int]] = None) -> np.ndarray:
        """[P4] Transformer.forward: logits (float64 standing for fp32) of shape [B, T, V].

        With all_positions=False only the last position's logits are returned,
        shape [B, V] ([P3] §3.2, the LLaMA-1 form used by generate). ``layers``
        restricts the block stack (for reduced, stated samples of large configs).
        """
        a = self.args
        tokens = np.asarray(tokens)
        B, T = tokens.shape
        if B > a.max_batch_size:
            raise ValueError("batch exceeds max_batch_size")
        if np.any(tokens < 0) or np.any(tokens >= a.vocab_size):
            raise ValueError("token id out of range")
        h = as_f64(self.tok_embeddings[tokens.reshape(-1)]).reshape(B, T, a.dim)
        for layer in (range(a.n_layers) if layers is None else layers):
            h = self.block(layer, h, start_pos)
        self.last_hidden = h
        xn = rmsnorm(h, self.norm, a.norm_eps, a.act)
        if not all_positions:
            xn = xn[:, -1, :]
        return self._lm_head(xn)

    def _lm_head(self, xn: np.ndarray) -> np.ndarray:
        w = self.output
        V = w.shape[0]
        out = np.empty(xn.shape[:-1] + (V,), dtype=np.float64)
        step = 16384  # widen the (possibly bf16-bits) head in slices to bound host memory
        for v0 in range(0, V, step):
            out[..., v0:v0 + step] = xn @ as_f64(w[v0:v0 + step]).T
        return out


# ----------------------------------------------------------------------------
# Generation ([P3] §3.3 generate and sample_top_p)
# ----------------------------------------------------------------------------

def select_next(logits: np.ndarray, temperature: float, top_p: float, u: Optional[float] = None) -> int:
    """The next token from one row of logits.

    temperature <= 0: argmax (the first maximum). Otherwise probs =
    softmax(logits / temperature); sort descending (ties keep index order);
    zero the tokens whose predecessors' cumulative probability exceeds top_p
    (mask cum - p > top_p); renormalise; the multinomial draw is made with the
    given uniform u: the first token in that order whose cumulative
    renormalised probability exceeds u.
    """
    logits = np.asarray(logits, dtype=np.float64)
    if not temperature > 0:
        return int(np.argmax(logits))
    z = logits / temperature
    z = z - z.max()
    e = np.exp(z)
    probs = e / e.sum()
    order = np.argsort(-probs, kind="stable")
    ps = probs[order]
    cum = np.cumsum(ps)
    ps = np.where(cum - ps > top_p, 0.0, ps)
    ps = ps / ps.sum()
    c = np.cumsum(ps)
    k = min(int(np.searchsorted(c, u, side="right")), len(ps) - 1)
    return int(order[k])


def generate(model: "OracleModel", tokens: np.ndarray, prompt_mask: np.ndarray, min_prompt_len: int,
             temperature: float, top_p: float, uniforms: Optional[np.ndarray] = None) -> np.ndarray:
    """[P3] §3.3 generate on token ids: from cur = the shortest prompt's length,
    forward(tokens[:, prev:cur], prev) with last-position logits, select the
    next token, keep the prompt's own token where the prompt mask is set, then
    prev = cur. ``uniforms[cur, b]`` is the draw of sequence b at step cur.
    Returns the completed token array (a copy)."""
    tokens = np.array(tokens, dtype=np.int64, copy=True)
    B, total_len = tokens.shape
    prev = 0
    for cur in range(min_prompt_len, total_len):
        logits = model.forward(tokens[:, prev:cur], prev, all_positions=False)   # [B, V]
        for b in range(B):
            if not prompt_mask[b, cur]:
                u = None if uniforms is None else float(uniforms[cur, b])
                tokens[b, cur] = select_next(logits[b], temperature, top_p, u)
        prev = cur
    return tokens
