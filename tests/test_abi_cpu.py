"""CPU checks of the C ABI: the library loads, exports every declared symbol,
and validates arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth
import oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "llama_b200.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(llama_[a-z_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("library not built")
    declared = _declared()
    assert len(declared) >= 15
    L = ctypes.CDLL(B.LIB_PATH)
    for name in declared:
        assert hasattr(L, name), name
    assert set(declared) == set(B.EXPORTED)


def test_binding_constants_equal_the_header_defines():
    """Every integer #define LLAMA_* of the header has the same value in the binding."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    defines = {m.group(1): int(m.group(2)) for m in re.finditer(r"#define\s+(LLAMA_[A-Z0-9_]+)\s+(-?\d+)\b", src)}
    assert len(defines) >= 20
    for name, value in defines.items():
        assert hasattr(B, name), name
        assert getattr(B, name) == value, (name, getattr(B, name), value)


def test_ffn_hidden_matches_oracle_rule():
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("library not built")
    for w in synth.WORKLOADS.values():
        a = B.ModelArgs.from_workload(w)
        assert B.llama_ffn_hidden(a) == w.ffn_hidden
        assert O.ffn_hidden_dim(w.dim, w.multiple_of, w.ffn_dim_multiplier) == w.ffn_hidden
    for dim in (256, 512, 1024, 5120, 6656, 8192):
        for mo in (32, 256, 1024):
            for mult in (None, 1.3, 1.5):
                a = B.ModelArgs(dim, 1, dim // 128, dim // 128, 0, mo, mult, 1e-5, 1e4, 1, 16)
                assert B.llama_ffn_hidden(a) == O.ffn_hidden_dim(dim, mo, mult)


@pytest.mark.parametrize("bad", [
    dict(dim=300),                 # not a multiple of n_heads * 64
    dict(n_heads=3),               # dim % n_heads
    dict(n_kv_heads=3),            # n_heads % n_kv_heads
    dict(dim=2048, n_heads=8),     # head_dim 256 unsupported
    dict(max_batch_size=0),
    dict(max_seq_len=0),
    dict(vocab_size=1001),         # vocab % 8
    dict(dtype="fp16"),
    dict(n_heads=32, n_kv_heads=2, dim=4096),  # bf16 GQA group of 16 is fine (multiple of 8)
    dict(n_heads=12, n_kv_heads=1, dim=768),   # bf16 group of 12 is fine (any ratio)
    dict(n_heads=24, n_kv_heads=1, dim=1536),  # bf16 group of 24 is fine (three CTA groups of 8)
    dict(n_heads=20, n_kv_heads=1, dim=1280),  # bf16 group of 20 is fine (two CTA groups of 10)
])
def test_create_rejects_invalid_args_on_host(bad):
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("library not built")
    base = dict(dim=512, n_layers=1, n_heads=4, n_kv_heads=2, vocab_size=1000, multiple_of=256,
                ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=1e4, max_batch_size=2, max_seq_len=64,
                dtype="bf16")
    base.update(bad)
    a = B.ModelArgs(**base)
    c = a.c()
    if base["dtype"] == "fp16":
        c.dtype = 7
    ctx = ctypes.c_void_p()
    code = B.lib().llama_create(ctypes.byref(c), ctypes.byref(ctx))
    if bad in (dict(n_heads=32, n_kv_heads=2, dim=4096), dict(n_heads=24, n_kv_heads=1, dim=1536),
               dict(n_heads=12, n_kv_heads=1, dim=768), dict(n_heads=20, n_kv_heads=1, dim=1280)):
        # valid shape: without a GPU the failure (if any) comes from CUDA, not validation
        assert code != B.LLAMA_ERR_INVALID_ARGS
        if code == B.LLAMA_OK:
            B.llama_destroy(ctx)
    else:
        assert code == B.LLAMA_ERR_INVALID_ARGS
        assert not ctx.value


def test_null_and_bad_calls_are_rejected_without_a_device():
    if not os.path.exists(B.LIB_PATH):
        pytest.skip("library not built")
    L = B.lib()
    assert L.llama_forward(None, None, 1, 1, 0, None, 1, None) == B.LLAMA_ERR_INVALID_ARGS
    assert L.llama_block_forward(None, 0, None, 1, 1, None, 0, None) == B.LLAMA_ERR_INVALID_ARGS
    assert L.llama_get_error(None, None) == B.LLAMA_ERR_INVALID_ARGS
    assert L.llama_linear(None, None, None, 1, 8, 8, 1, 0, None) == B.LLAMA_ERR_INVALID_ARGS
    assert L.llama_linear(ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), 1, 7, 8, 1, 0, None) \
        == B.LLAMA_ERR_INVALID_ARGS
    assert B.strerror(B.LLAMA_ERR_POS_RANGE).startswith("position")
    L.llama_destroy(None)


def test_wrappers_reach_the_library_without_a_device():
    """Wrappers whose C call rejects a NULL context before touching the device:
    the argument error comes back as LlamaError (checks the marshalling)."""
    with pytest.raises(B.LlamaError) as e:
        B.llama_set_decode_kernel(None, B.LLAMA_DECODE_LAYERED)
    assert e.value.code == B.LLAMA_ERR_INVALID_ARGS
    with pytest.raises(B.LlamaError) as e:
        B.llama_reset(None)
    assert e.value.code == B.LLAMA_ERR_INVALID_ARGS


def test_allocation_cap_fails_create_cleanly_on_the_host():
    """Injected allocation failure: with a one-byte cap the first device
    allocation of llama_create fails before cudaMalloc is reached, the call
    returns LLAMA_ERR_OOM and the library holds nothing afterwards."""
    args = B.ModelArgs(dim=256, n_layers=2, n_heads=4, n_kv_heads=2, vocab_size=1000, multiple_of=256,
                       ffn_dim_multiplier=None, norm_eps=1e-5, rope_theta=10000.0, max_batch_size=1,
                       max_seq_len=64, dtype="bf16").c()
    before = B.llama_allocated_bytes()
    B.llama_set_alloc_limit(1)
    try:
        ctx = ctypes.c_void_p()
        code = B.lib().llama_create(ctypes.byref(args), ctypes.byref(ctx))
        assert code == B.LLAMA_ERR_OOM
        assert not ctx.value
        assert B.llama_allocated_bytes() == before
    finally:
        B.llama_set_alloc_limit(0)
