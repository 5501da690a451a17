"""llama_linear_noalloc through the C ABI: the decode GEMV with its scratch in a
fixed array compiled into the library, for callers that cannot allocate device
memory when they call (an application whose memory belongs to its own pool
allocator, a loop where cudaMalloc/cudaFree and their possible device
synchronisation are not acceptable). It must give the same result as
llama_linear's GEMV path, call after call, and refuse shapes whose scratch
would not fit. Collected last so a failure here leaves every other test run."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth

pytestmark = pytest.mark.gpu

REL = 2e-5  # the GEMM-core tolerance of test_gpu_linear.py


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (7, 12288, 4096), (32, 4096, 11008), (3, 136, 192)])
def test_noalloc_matches_linear_twice_in_a_row(M, N, K):
    x = synth.normal((M, K), 1.0, 41, torch.bfloat16, "cuda")
    w = synth.normal((N, K), 0.02, 42, torch.bfloat16, "cuda")
    ref = torch.empty((M, N), device="cuda")
    B.llama_linear(x, w, ref, B.LLAMA_PATH_GEMV)
    torch.cuda.synchronize()
    r = ref.double().cpu().numpy()
    for _ in range(2):
        y = torch.full((M, N), float("nan"), device="cuda")
        assert B.llama_linear_noalloc(x, w, y) == B.LLAMA_OK
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.abs(got - r).max() <= REL * np.abs(r).max()


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
