"""Python binding of the C ABI in include/llama_b200.h (argument marshalling only).

Every function here has the name of the C call it wraps, takes torch tensors
(or plain ints) and passes their device pointers, sizes and the current CUDA
stream to the library. No computation happens in Python: if the shared
library is missing the first call raises, there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libllama_b200.so")

LLAMA_FP32, LLAMA_BF16 = 0, 1
LLAMA_OK = 0
LLAMA_ERR_INVALID_ARGS = -1
LLAMA_ERR_OOM = -2
LLAMA_ERR_CUDA = -3
LLAMA_ERR_NOT_READY = -4
LLAMA_ERR_TOO_LARGE = -5
LLAMA_ERR_INTERNAL = -6
LLAMA_ERR_TOKEN_RANGE = -10
LLAMA_ERR_POS_RANGE = -11
LLAMA_ERR_TIMEOUT = -12
LLAMA_PATH_AUTO, LLAMA_PATH_TCGEN05, LLAMA_PATH_GEMV, LLAMA_PATH_SIMT = 0, 1, 2, 3
LLAMA_WEIGHTS_TILED = 16
LLAMA_DECODE_AUTO, LLAMA_DECODE_LAYERED, LLAMA_DECODE_PERSISTENT = 0, 1, 2
LLAMA_ATTN_AUTO, LLAMA_ATTN_CHUNKED, LLAMA_ATTN_STREAMK = 0, 1, 2
LLAMA_GEMV_MMA_AUTO, LLAMA_GEMV_MMA_WARP, LLAMA_GEMV_MMA_TCGEN05 = 0, 1, 2

# every symbol the header declares (checked by the CPU test suite)
EXPORTED = ("llama_ffn_hidden", "llama_create", "llama_destroy", "llama_set_layer", "llama_set_embed_norm_head",
            "llama_reserve", "llama_forward", "llama_forward_ragged", "llama_block_forward", "llama_kv_read",
            "llama_kv_write", "llama_reset", "llama_get_error", "llama_strerror", "llama_linear",
            "llama_linear_noalloc", "llama_linear_noalloc_status", "llama_sample", "llama_generate", "llama_set_decode_kernel",
            "llama_set_decode_attention", "llama_set_decode_linear_mma", "llama_tile_weights",
            "llama_selftest_bounded_wait", "llama_set_alloc_limit", "llama_allocated_bytes",
            "llama_selfcheck_plans")


class LlamaArgs(ctypes.Structure):
    _fields_ = [("dim", ctypes.c_int32), ("n_layers", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("vocab_size", ctypes.c_int32), ("multiple_of", ctypes.c_int32),
                ("ffn_dim_multiplier", ctypes.c_float), ("norm_eps", ctypes.c_float), ("rope_theta", ctypes.c_float),
                ("max_batch_size", ctypes.c_int32), ("max_seq_len", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("rope_half_split", ctypes.c_int32)]


class LlamaError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {strerror(code)} ({code})")
        self.code = code


_lib = None


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m llama_decoder_block_kv_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
        L.llama_ffn_hidden.argtypes = [ctypes.POINTER(LlamaArgs)]
        L.llama_create.argtypes = [ctypes.POINTER(LlamaArgs), ctypes.POINTER(vp)]
        L.llama_destroy.argtypes = [vp]
        L.llama_destroy.restype = None
        L.llama_set_layer.argtypes = [vp, i] + [vp] * 9
        L.llama_set_embed_norm_head.argtypes = [vp, vp, vp, vp]
        L.llama_reserve.argtypes = [vp, i]
        L.llama_forward.argtypes = [vp, vp, i, i, i, vp, i, vp]
        L.llama_forward_ragged.argtypes = [vp, vp, vp, i, vp, vp]
        L.llama_block_forward.argtypes = [vp, i, vp, i, i, vp, i, vp]
        L.llama_kv_read.argtypes = [vp, i, vp, vp, vp]
        L.llama_kv_write.argtypes = [vp, i, vp, vp, vp]
        L.llama_reset.argtypes = [vp]
        L.llama_get_error.argtypes = [vp, ctypes.POINTER(i)]
        L.llama_strerror.argtypes = [i]
        L.llama_strerror.restype = ctypes.c_char_p
        L.llama_linear.argtypes = [vp, vp, vp, i, i, i, i, i, vp]
        L.llama_linear_noalloc.argtypes = [vp, vp, vp, i, i, i, vp]
        L.llama_linear_noalloc_status.argtypes = [ctypes.POINTER(ctypes.c_int)]
        L.llama_sample.argtypes = [vp, i, i, f, f, vp, vp, vp]
        L.llama_generate.argtypes = [vp, vp, vp, i, i, i, f, f, vp, vp]
        L.llama_set_decode_kernel.argtypes = [vp, i]
        L.llama_set_decode_attention.argtypes = [vp, i]
        L.llama_set_decode_linear_mma.argtypes = [i]
        L.llama_tile_weights.argtypes = [vp, vp, i, i, vp]
        L.llama_selftest_bounded_wait.argtypes = [i, ctypes.POINTER(i), ctypes.POINTER(ctypes.c_double)]
        L.llama_set_alloc_limit.argtypes = [ctypes.c_uint64]
        L.llama_allocated_bytes.argtypes = []
        L.llama_selfcheck_plans.argtypes = [i] * 7
        for name in EXPORTED:
            if name not in ("llama_destroy", "llama_strerror"):
                getattr(L, name).restype = ctypes.c_int
        L.llama_allocated_bytes.restype = ctypes.c_uint64
        _lib = L
    return _lib


def strerror(code: int) -> str:
    return lib().llama_strerror(int(code)).decode()


def _check(code: int, what: str) -> int:
    if code != LLAMA_OK:
        raise LlamaError(code, what)
    return code


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


@dataclass
class ModelArgs:
    """The notes' ModelArgs plus rope_theta and the storage dtype ("fp32" / "bf16")."""
    dim: int
    n_layers: int
    n_heads: int
    n_kv_heads: int
    vocab_size: int
    multiple_of: int
    ffn_dim_multiplier: Optional[float]
    norm_eps: float
    rope_theta: float
    max_batch_size: int
    max_seq_len: int
    dtype: str = "bf16"
    rope_half_split: bool = False

    def c(self) -> LlamaArgs:
        return LlamaArgs(self.dim, self.n_layers, self.n_heads, self.n_kv_heads, self.vocab_size, self.multiple_of,
                         -1.0 if self.ffn_dim_multiplier is None else float(self.ffn_dim_multiplier),
                         float(self.norm_eps), float(self.rope_theta), self.max_batch_size, self.max_seq_len,
                         LLAMA_BF16 if self.dtype == "bf16" else LLAMA_FP32, int(bool(self.rope_half_split)))

    @classmethod
    def from_workload(cls, w) -> "ModelArgs":
        return cls(w.dim, w.n_layers, w.n_heads, w.n_kv_heads, w.vocab_size, w.multiple_of, w.ffn_dim_multiplier,
                   w.norm_eps, w.rope_theta, w.max_batch_size, w.max_seq_len, w.act)


def llama_ffn_hidden(args: ModelArgs) -> int:
    a = args.c()
    return lib().llama_ffn_hidden(ctypes.byref(a))


def llama_create(args: ModelArgs) -> ctypes.c_void_p:
    a = args.c()
    ctx = ctypes.c_void_p()
    _check(lib().llama_create(ctypes.byref(a), ctypes.byref(ctx)), "llama_create")
    return ctx


def llama_destroy(ctx) -> None:
    lib().llama_destroy(ctx)


def llama_set_layer(ctx, layer: int, w: dict) -> None:
    names = ("wq", "wk", "wv", "wo", "w1", "w2", "w3", "attn_norm", "ffn_norm")
    _check(lib().llama_set_layer(ctx, layer, *[_ptr(w[n]) for n in names]), "llama_set_layer")


def llama_set_embed_norm_head(ctx, tok_embeddings, norm, output) -> None:
    _check(lib().llama_set_embed_norm_head(ctx, _ptr(tok_embeddings), _ptr(norm), _ptr(output)),
           "llama_set_embed_norm_head")


def llama_reserve(ctx, max_tokens: int) -> None:
    _check(lib().llama_reserve(ctx, int(max_tokens)), "llama_reserve")


def llama_forward(ctx, tokens: torch.Tensor, start_pos: int, logits: torch.Tensor, all_positions: bool = True,
                  stream=None) -> None:
    B, T = tokens.shape
    _check(lib().llama_forward(ctx, _ptr(tokens), B, T, int(start_pos), _ptr(logits), int(bool(all_positions)),
                               _stream(stream)), "llama_forward")


def llama_forward_ragged(ctx, tokens: torch.Tensor, start_pos: torch.Tensor, logits: torch.Tensor,
                         stream=None) -> None:
    _check(lib().llama_forward_ragged(ctx, _ptr(tokens), _ptr(start_pos), tokens.shape[0], _ptr(logits),
                                      _stream(stream)), "llama_forward_ragged")


def llama_block_forward(ctx, layer: int, h: torch.Tensor, start_pos, stream=None) -> None:
    """start_pos: an int (same for every sequence) or an int32 device tensor [B]."""
    B, T = h.shape[0], h.shape[1]
    if isinstance(start_pos, torch.Tensor):
        code = lib().llama_block_forward(ctx, layer, _ptr(h), B, T, _ptr(start_pos), 0, _stream(stream))
    else:
        code = lib().llama_block_forward(ctx, layer, _ptr(h), B, T, None, int(start_pos), _stream(stream))
    _check(code, "llama_block_forward")


def llama_kv_read(ctx, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
    _check(lib().llama_kv_read(ctx, layer, _ptr(k), _ptr(v), _stream(stream)), "llama_kv_read")


def llama_kv_write(ctx, layer: int, k: torch.Tensor, v: torch.Tensor, stream=None) -> None:
    _check(lib().llama_kv_write(ctx, layer, _ptr(k), _ptr(v), _stream(stream)), "llama_kv_write")


def llama_reset(ctx) -> None:
    _check(lib().llama_reset(ctx), "llama_reset")


def llama_set_decode_kernel(ctx, mode: int) -> None:
    _check(lib().llama_set_decode_kernel(ctx, int(mode)), "llama_set_decode_kernel")


def llama_set_decode_linear_mma(mode: int) -> None:
    """Product of the 9..32-token decode GEMV (LLAMA_GEMV_MMA_*), process-wide."""
    _check(lib().llama_set_decode_linear_mma(int(mode)), "llama_set_decode_linear_mma")


def llama_set_decode_attention(ctx, mode: int) -> None:
    _check(lib().llama_set_decode_attention(ctx, int(mode)), "llama_set_decode_attention")


def llama_get_error(ctx):
    """Returns (code, flags) after synchronising; clears the device flags."""
    flags = ctypes.c_int(0)
    code = lib().llama_get_error(ctx, ctypes.byref(flags))
    return code, flags.value


def llama_set_alloc_limit(nbytes: int) -> None:
    """Cap the device memory the library may hold (0: no cap); see the header."""
    _check(lib().llama_set_alloc_limit(int(nbytes)), "llama_set_alloc_limit")


def llama_selfcheck_plans(M: int, dim: int, n_heads: int, n_kv_heads: int, ffn: int, max_seq_len: int,
                          num_sms: int = 148) -> int:
    """Host-only walk of the decode kernels' work partitions; returns the C code (0 = consistent)."""
    return lib().llama_selfcheck_plans(M, dim, n_heads, n_kv_heads, ffn, max_seq_len, num_sms)


def llama_allocated_bytes() -> int:
    return int(lib().llama_allocated_bytes())


def llama_selftest_bounded_wait(which: int):
    """Returns (flags, seconds) of a device wait that nothing completes (0: mbarrier, 1: grid barrier)."""
    flags, secs = ctypes.c_int(0), ctypes.c_double(0.0)
    _check(lib().llama_selftest_bounded_wait(int(which), ctypes.byref(flags), ctypes.byref(secs)),
           "llama_selftest_bounded_wait")
    return flags.value, secs.value


def llama_tile_weights(w: torch.Tensor, stream=None) -> torch.Tensor:
    """The library's tile layout of a bf16 [N][K] weight matrix (returned as a new tensor)."""
    N, K = w.shape
    out = torch.empty(((N + 127) // 128 * 128 * K,), dtype=torch.bfloat16, device=w.device)
    _check(lib().llama_tile_weights(_ptr(w), _ptr(out), N, K, _stream(stream)), "llama_tile_weights")
    return out


def llama_linear(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, path: int = LLAMA_PATH_AUTO, stream=None,
                 n: Optional[int] = None) -> None:
    """y = x w^T; w is [N][K], or with path | LLAMA_WEIGHTS_TILED the tiles of llama_tile_weights (pass n = N)."""
    M, K = x.shape
    N = w.shape[0] if n is None else n
    dt = LLAMA_BF16 if x.dtype == torch.bfloat16 else LLAMA_FP32
    _check(lib().llama_linear(_ptr(x), _ptr(w), _ptr(y), M, N, K, dt, int(path), _stream(stream)), "llama_linear")


def llama_sample(logits: torch.Tensor, out: torch.Tensor, temperature: float = 0.0, top_p: float = 1.0,
                 uniforms: Optional[torch.Tensor] = None, stream=None) -> None:
    B, V = logits.shape
    _check(lib().llama_sample(_ptr(logits), B, V, float(temperature), float(top_p), _ptr(uniforms), _ptr(out),
                              _stream(stream)), "llama_sample")


def llama_generate(ctx, tokens: torch.Tensor, prompt_mask: torch.Tensor, min_prompt_len: int,
                   temperature: float = 0.0, top_p: float = 1.0, uniforms: Optional[torch.Tensor] = None,
                   stream=None) -> None:
    B, total_len = tokens.shape
    _check(lib().llama_generate(ctx, _ptr(tokens), _ptr(prompt_mask), B, total_len, int(min_prompt_len),
                                float(temperature), float(top_p), _ptr(uniforms), _stream(stream)), "llama_generate")


def llama_linear_noalloc(x: torch.Tensor, w: torch.Tensor, y: torch.Tensor, stream=None) -> int:
    """The GEMV case of llama_linear without any allocation; returns the C return code."""
    M, K = x.shape
    N = w.shape[0]
    return lib().llama_linear_noalloc(_ptr(x), _ptr(w), _ptr(y), M, N, K, _stream(stream))


def llama_linear_noalloc_status():
    """(code, raw error bits) of llama_linear_noalloc on the current device; clears them."""
    flags = ctypes.c_int(0)
    code = lib().llama_linear_noalloc_status(ctypes.byref(flags))
    return code, flags.value


class Llama:
    """Owns one llama_ctx (create on construction, destroy on close)."""

    def __init__(self, args: ModelArgs):
        self.args = args
        self.ctx = llama_create(args)

    def close(self):
        if self.ctx is not None:
            llama_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
