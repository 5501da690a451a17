"""Shared set-up for the GPU parity tests: load synth weights into the library
and into the oracle, and compare results (tolerances stated once here)."""
from __future__ import annotations

import numpy as np
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
from tests.helpers import build_oracle, t2np

# Tolerances: fp32 mode max relative error 1e-4 (norm-wise and element-wise
# with a small absolute floor); bf16 mode max absolute error 2e-2 on hidden
# states and 5e-2 on logits, fp32 accumulation on both sides.
FP32_REL = 1e-4
BF16_HIDDEN_ABS = 2e-2
BF16_LOGITS_ABS = 5e-2


def assert_fp32_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    scale = np.abs(ref).max()
    err = np.abs(got - ref)
    assert err.max() <= FP32_REL * scale, f"{what}: norm-wise rel err {err.max() / scale:.3g}"
    assert np.all(err <= FP32_REL * np.abs(ref) + FP32_REL * 1e-2 * scale + 1e-6), f"{what}: element-wise"


def assert_abs_close(got: np.ndarray, ref: np.ndarray, tol: float, what: str = ""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref).max()
    assert err <= tol, f"{what}: max abs err {err:.4g} > {tol}"


def assert_bf16_ulp(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Stored bf16 values (the cache) equal the oracle's up to one rounding step:
    |got - ref| <= one bf16 spacing at |ref| (2^-7 relative at the bottom of a
    binade) plus 1e-4 * max|ref|. The absolute term covers values that are the
    small remainder of a cancelling sum, where fp32 accumulation error is large
    relative to the value itself."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    spacing = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    floor = 1e-4 * float(np.abs(ref).max())
    diff = np.abs(got - ref)
    bad = diff > spacing * 1.0000001 + floor
    assert not bad.any(), (f"{what}: {int(bad.sum())} values differ by more than one bf16 step; worst diff "
                           f"{diff[bad].max():.3g} at |ref| {np.abs(ref[bad]).max():.3g} (floor {floor:.3g})")


def assert_bf16_cache_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    """Cached bf16 values: within the 2e-2 bound, or within one bf16 rounding step
    where one step is larger than that (|value| >= 2.56, where a single rounding
    flip already moves a value by 2^-5 or more)."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    spacing = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -126))) - 7)
    diff = np.abs(got - ref)
    bad = diff > np.maximum(BF16_HIDDEN_ABS, spacing * 1.0000001)
    assert not bad.any(), (f"{what}: {int(bad.sum())} values off by more than max(2e-2, one bf16 step); "
                           f"worst {diff[bad].max():.3g} at |ref| {np.abs(ref[bad]).max():.3g}")


class Pair:
    """The same synthetic model loaded into the CUDA library and the oracle."""

    def __init__(self, w: synth.Workload, layers=None, bits: bool = False, weights_device="cpu"):
        self.w = w
        self.args = B.ModelArgs.from_workload(w)
        self.model = B.Llama(self.args)
        n = w.n_layers if layers is None else layers
        lws = []
        for i in range(n):
            lw = synth.layer_weights(w, i, device=weights_device)
            B.llama_set_layer(self.model.ctx, i, {k: v.to("cuda").contiguous() for k, v in lw.items()})
            lws.append({k: v.cpu() for k, v in lw.items()})
        enh = None
        if w.vocab_size > 0:
            enh = synth.embed_norm_head(w, device=weights_device)
            B.llama_set_embed_norm_head(self.model.ctx, *(enh[k].to("cuda").contiguous()
                                                          for k in ("tok_embeddings", "norm", "output")))
            enh = {k: v.cpu() for k, v in enh.items()}
        self.oracle = build_oracle(w, lws, enh, bits=bits)
        torch.cuda.synchronize()

    @property
    def ctx(self):
        return self.model.ctx

    def check_error(self):
        code, flags = B.llama_get_error(self.ctx)
        assert code == B.LLAMA_OK, (B.strerror(code), flags)

    def kv(self, layer: int):
        w = self.w
        dt = torch.float32 if w.act == "fp32" else torch.bfloat16
        shape = (w.max_batch_size, w.max_seq_len, w.n_kv_heads, w.head_dim)
        k = torch.empty(shape, dtype=dt, device="cuda")
        v = torch.empty(shape, dtype=dt, device="cuda")
        B.llama_kv_read(self.ctx, layer, k, v)
        torch.cuda.synchronize()
        return t2np(k), t2np(v)

    def close(self):
        self.model.close()


def assert_cache_matches(pair: Pair, layer: int, written: np.ndarray, tol: float):
    """written: bool [B_max, S_max] of slots this test wrote; others must still be 0 (bit-exact),
    written ones match the oracle within tol (fp32: relative)."""
    k, v = pair.kv(layer)
    ok_, ov_ = pair.oracle.cache_k[layer], pair.oracle.cache_v[layer]
    for got, ref, name in ((k, ok_, "K"), (v, ov_, "V")):
        untouched = ~written
        assert np.all(got[untouched] == 0.0), f"cache {name} layer {layer}: a slot outside the written ones changed"
        nz = np.any(got != 0.0, axis=(2, 3))
        assert np.all(nz[written]), f"cache {name} layer {layer}: a written slot is still zero"
        if pair.w.act == "fp32":
            assert_fp32_close(got[written], ref[written], f"cache {name}")
        else:
            # slots are exact (checked above); values within the mode's bound
            assert_bf16_cache_close(got[written], ref[written], f"cache {name}")


# ----------------------------------------------------------------------------- full-size bound
#
# At the workloads' full sizes the bf16 rounding points (norm outputs, q/k/v,
# attention output, silu*mul) make the block ill-conditioned: the rounding
# error of an fp32 accumulation flips a few bf16 roundings, and each flip fans
# out through 4096..28672-wide sums, so no fp32-accumulating implementation
# stays within a flat 2e-2 of the float64 oracle everywhere. The bound there is
# measured, not assumed: tests/emulation.py computes the same block with the
# same rounding points and fp32 sums on the CPU, and the GPU result must be
# within the flat bound, or within EMU_FACTOR x the emulation's own distance
# from the oracle on the same inputs, for the maximum and for the 99th
# percentile of |error| separately. The factor is 2: the tensor cores' fp32
# accumulation of bf16 products is measurably coarser than an IEEE fp32 sum
# (test_gpu_linear.py prints both against float64: the tcgen05 GEMM's rms
# error is 15-26 x that of sequential fp32 at K = 4096 .. 11008), so each
# linear feeds the bf16 rounding points a few more flips than the emulation's.

EMU_FACTOR = 2.0


def assert_close_emulated(got: np.ndarray, ref: np.ndarray, emu: np.ndarray, flat: float, what: str = ""):
    """|got - ref| within max(flat, EMU_FACTOR x |emu - ref|) in max and in p99; prints both."""
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    eemu = np.abs(emu - ref)
    p99, ep99 = float(np.quantile(err, 0.99)), float(np.quantile(eemu, 0.99))
    tol_max = max(flat, EMU_FACTOR * float(eemu.max()))
    tol_p99 = max(flat, EMU_FACTOR * ep99)
    print(f"[parity] {what}: GPU max {err.max():.4g} p99 {p99:.4g}; fp32 emulation max {eemu.max():.4g} "
          f"p99 {ep99:.4g}; bound max {tol_max:.4g} p99 {tol_p99:.4g}")
    assert p99 <= tol_p99, f"{what}: p99 abs err {p99:.4g} > {tol_p99:.4g} (emulation p99 {ep99:.4g})"
    assert err.max() <= tol_max, f"{what}: max abs err {err.max():.4g} > {tol_max:.4g} (emulation {eemu.max():.4g})"
    return float(err.max()), p99


class CacheSnapshot:
    """Save and restore an oracle's caches (so a perturbed run starts from the same state)."""

    def __init__(self, model, layers):
        self.model, self.layers = model, list(layers)
        self.k = [model.cache_k[i].copy() for i in self.layers]
        self.v = [model.cache_v[i].copy() for i in self.layers]

    def restore(self):
        for j, i in enumerate(self.layers):
            self.model.cache_k[i][...] = self.k[j]
            self.model.cache_v[i][...] = self.v[j]
