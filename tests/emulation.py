"""An fp32 restatement of the decoder block, used to size the parity bound at
the workloads' full sizes.

TEST INFRASTRUCTURE ONLY, like the oracle. It computes what the oracle computes
(TransformerBlock.forward of "LLaMA: Open and Efficient Foundation Language
Models" notes, section 3 code) with the same bf16 rounding points (the norm
outputs, q and k after RoPE, v, the attention output, silu(w1 x) * w3 x), but
with every sum and product in fp32, as any fp32-accumulating implementation
must: torch CPU float32 matmuls, an fp32 softmax with unrounded
probabilities, fp32 RoPE on the fp32 cos/sin table. Its distance from the
float64 oracle is the error that fp32 accumulation alone causes on given
inputs; a GPU result may not be much further from the oracle than that. It
shares no code with the CUDA library and does not call it.

The linears accumulate like the tensor-core MMA instructions (K = 16 per
instruction, accumulator in fp32): the sums of 16-term blocks of the inner
dimension are added to an fp32 accumulator one block after another. Measured
on the CPU, this order has 2-3 x the maximum error of a blocked fp32 matmul
against float64 at K = 4096 .. 11008 (products of bf16 values, N(0,1) x
N(0, 0.02^2)), so the blocked matmul would understate what the hardware's
fp32 accumulation does.
"""
from __future__ import annotations

import numpy as np
import torch

F32 = torch.float32


def _bf16(x: torch.Tensor) -> torch.Tensor:
    """Round fp32 to bf16 (round-to-nearest-even, torch's cast) and back to fp32."""
    return x.to(torch.bfloat16).to(F32)


def _t(x) -> torch.Tensor:
    if isinstance(x, torch.Tensor):
        return x.detach().to("cpu", F32)
    x = np.asarray(x)
    if x.dtype == np.uint16:   # raw bf16 bit patterns
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(F32)
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))


MMA_K = 16


def linear(x: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
    """x [..., K] @ w[N, K]^T with the K dimension summed in 16-term blocks added in turn to an fp32 accumulator."""
    K = x.shape[-1]
    acc = torch.zeros(x.shape[:-1] + (w.shape[0],), dtype=F32)
    for k0 in range(0, K, MMA_K):
        acc += x[..., k0:k0 + MMA_K] @ w[:, k0:k0 + MMA_K].T
    return acc


def rmsnorm(h: torch.Tensor, w: torch.Tensor, eps: float) -> torch.Tensor:
    """fp32 statistics, cast back, then times the weight in bf16 (the notes' RMSNorm.forward)."""
    ms = (h * h).mean(-1, keepdim=True)
    return _bf16(_bf16(h * torch.rsqrt(ms + eps)) * w)


def rope(x: torch.Tensor, cos: torch.Tensor, sin: torch.Tensor) -> torch.Tensor:
    """Interleaved pairs rotated in fp32; x [..., heads, D], cos/sin [..., D/2] for its positions."""
    c, s = cos[..., None, :], sin[..., None, :]
    xe, xo = x[..., 0::2], x[..., 1::2]
    out = torch.empty_like(x)
    out[..., 0::2] = xe * c - xo * s
    out[..., 1::2] = xo * c + xe * s
    return out


def attention(q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, pos: torch.Tensor, n_rep: int) -> torch.Tensor:
    """One sequence: q [T, H, D], K/V [L, Hkv, D] (rounded values), query t at position pos[t]
    sees keys j <= pos[t]; fp32 scores, softmax and P V."""
    T, H, D = q.shape
    L = K.shape[0]
    Kr = K.repeat_interleave(n_rep, dim=1).permute(1, 0, 2)       # [H, L, D]
    Vr = V.repeat_interleave(n_rep, dim=1).permute(1, 0, 2)
    s = torch.matmul(q.permute(1, 0, 2), Kr.transpose(1, 2)) * (1.0 / float(np.sqrt(D)))   # [H, T, L]
    mask = torch.arange(L)[None, :] > pos[:, None]                 # [T, L]
    s = s.masked_fill(mask[None], float("-inf"))
    p = torch.softmax(s, dim=-1)
    return torch.matmul(p, Vr).permute(1, 0, 2)                   # [T, H, D]


class EmuBlock:
    """One block's weights in fp32 and the fp32 cos/sin table."""

    def __init__(self, lw: dict, args, cos: np.ndarray, sin: np.ndarray):
        self.a = args
        self.w = {k: _t(v) for k, v in lw.items()}
        self.cos, self.sin = _t(cos), _t(sin)

    def forward(self, h, cache_k, cache_v, start_pos, rows=None) -> torch.Tensor:
        """h [B, T, dim]; cache_k/v [B, S, Hkv, D] (modified: this call's slots are
        written); returns the block output [B, T, dim], or only the (b, s) pairs
        of ``rows`` as [len(rows), dim]."""
        a, w = self.a, self.w
        h = _t(h)
        B, T, dim = h.shape
        H, Hkv, D = a.n_heads, a.kv_heads, a.head_dim
        sp = torch.as_tensor(np.broadcast_to(np.asarray(start_pos, dtype=np.int64), (B,)).copy())
        pos = sp[:, None] + torch.arange(T)[None, :]
        xn = rmsnorm(h, w["attn_norm"], a.norm_eps)
        k = _bf16(rope(linear(xn, w["wk"]).view(B, T, Hkv, D), self.cos[pos], self.sin[pos]))
        v = _bf16(linear(xn, w["wv"]).view(B, T, Hkv, D))
        for b in range(B):
            cache_k[b, sp[b]:sp[b] + T] = k[b]
            cache_v[b, sp[b]:sp[b] + T] = v[b]
        sel = [(b, s) for b in range(B) for s in range(T)] if rows is None else list(rows)
        out = torch.empty((len(sel), dim), dtype=F32)
        by_seq = {}
        for i, (b, s) in enumerate(sel):
            by_seq.setdefault(b, []).append((i, s))
        for b, items in by_seq.items():
            idx = torch.tensor([s for _, s in items])
            hb = h[b, idx]
            q = _bf16(rope(linear(xn[b, idx], w["wq"]).view(len(idx), H, D), self.cos[pos[b, idx]],
                           self.sin[pos[b, idx]]))
            n = int(pos[b, idx].max()) + 1
            o = _bf16(attention(q, _t(cache_k[b, :n]), _t(cache_v[b, :n]), pos[b, idx], a.n_rep).reshape(len(idx), -1))
            hr = hb + linear(o, w["wo"])
            xn2 = rmsnorm(hr, w["ffn_norm"], a.norm_eps)
            g = _bf16(torch.nn.functional.silu(linear(xn2, w["w1"])) * linear(xn2, w["w3"]))
            out[[i for i, _ in items]] = hr + linear(g, w["w2"])
        return out.view(B, T, dim) if rows is None else out


def lm_head(h: torch.Tensor, norm_w, output, eps: float) -> torch.Tensor:
    """Final RMSNorm and the LM head in fp32 (the head widened in slices)."""
    xn = rmsnorm(_t(h), _t(norm_w), eps)
    V = output.shape[0]
    return torch.cat([linear(xn, _t(output[v0:v0 + 16384])) for v0 in range(0, V, 16384)], dim=-1)
