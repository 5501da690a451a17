"""llama_linear_noalloc through the C ABI: the decode GEMV with its scratch in a
fixed array compiled into the library, for callers that cannot allocate device
memory when they call (an application whose device memory belongs to its own
pool allocator, so a cudaMalloc behind its back could fail or fragment it; a
loop where cudaMalloc/cudaFree and the device synchronisation they can cause
are not acceptable).

Checked here: the result against a float64 matmul of the same bf16 inputs,
call after call (the fixed array keeps the previous call's contents, so the
second call checks that the counters were cleared); that the calls take no
device memory (the library's tracked total and the device's free memory do
not move, and the calls still run under an allocation cap set to what the
library already holds); that the error word reads back clear; and that shapes
whose scratch would not fit are refused. Collected last so that a failure here
leaves every other test run."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth

pytestmark = pytest.mark.gpu

REL = 2e-5  # the GEMM-core tolerance of test_gpu_linear.py: of the largest output, fp32 accumulation


def _inputs(M, N, K, seed):
    x = synth.normal((M, K), 1.0, seed, torch.bfloat16, "cuda")
    w = synth.normal((N, K), 0.02, seed + 1, torch.bfloat16, "cuda")
    ref = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    return x, w, ref


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (7, 12288, 4096), (32, 4096, 11008), (3, 136, 192)])
def test_noalloc_matches_float64_matmul_twice_in_a_row(M, N, K):
    x, w, ref = _inputs(M, N, K, 41)
    scale = np.abs(ref).max()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), device="cuda")
        assert B.llama_linear_noalloc(x, w, y) == B.LLAMA_OK
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        err = np.abs(got - ref).max()
        assert err <= REL * scale, (err, scale)
    assert B.llama_linear_noalloc_status() == (B.LLAMA_OK, 0)


def test_noalloc_takes_no_device_memory():
    x, w, ref = _inputs(16, 8192, 4096, 43)
    y = torch.empty((16, 8192), device="cuda")
    assert B.llama_linear_noalloc(x, w, y) == B.LLAMA_OK     # warm-up (the per-device set-up)
    torch.cuda.synchronize()
    held, (free0, _) = B.llama_allocated_bytes(), torch.cuda.mem_get_info()
    try:
        B.llama_set_alloc_limit(max(held, 1))                # any allocation by the library would now fail
        for _ in range(3):
            y.fill_(float("nan"))
            assert B.llama_linear_noalloc(x, w, y) == B.LLAMA_OK
            torch.cuda.synchronize()
            got = y.cpu().double().numpy()   # copied out first: no device-side temporary
            assert np.abs(got - ref).max() <= REL * np.abs(ref).max()
    finally:
        B.llama_set_alloc_limit(0)
    assert B.llama_allocated_bytes() == held
    assert torch.cuda.mem_get_info()[0] == free0
    assert B.llama_linear_noalloc_status() == (B.LLAMA_OK, 0)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 32 tokens x a 128256-row head needs ~8.2 Mi partial sums, more than the 2 Mi it holds
    x = torch.zeros((32, 4096), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((128256, 4096), dtype=torch.bfloat16, device="cuda")
    y = torch.zeros((32, 128256), device="cuda")
    assert B.llama_linear_noalloc(x, w, y) == B.LLAMA_ERR_TOO_LARGE
    # K must be a multiple of 64 (argument check, nothing launched)
    xs = torch.zeros((2, 100), dtype=torch.bfloat16, device="cuda")
    ws = torch.zeros((8, 100), dtype=torch.bfloat16, device="cuda")
    ys = torch.zeros((2, 8), device="cuda")
    assert B.llama_linear_noalloc(xs, ws, ys) == B.LLAMA_ERR_INVALID_ARGS
