"""GEMM cores through the C ABI (llama_linear) against a float64 matmul of the
same bf16 / fp32 inputs (the library primitive the oracle uses for a linear)."""
import numpy as np
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _inputs(M, N, K, dtype, seed):
    x = synth.normal((M, K), 1.0, seed, dtype, "cuda")
    w = synth.normal((N, K), 0.02, seed + 1, dtype, "cuda")
    return x, w


def _check(x, w, y, rel=2e-5):
    ref = x.double().cpu().numpy() @ w.double().cpu().numpy().T
    got = y.double().cpu().numpy()
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    assert err <= rel * scale + 1e-6, (err, scale)


@pytest.mark.parametrize("M,N,K", [(1, 256, 64), (37, 384, 128), (128, 256, 4096), (129, 512, 448),
                                   (300, 1024, 1024), (512, 12288, 4096), (77, 128, 11008), (2, 2048, 256)])
def test_tcgen05_gemm(M, N, K):
    x, w = _inputs(M, N, K, torch.bfloat16, 11)
    y = torch.full((M, N), float("nan"), device="cuda")
    B.llama_linear(x, w, y, B.LLAMA_PATH_TCGEN05)
    torch.cuda.synchronize()
    _check(x, w, y)


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 1024), (1000, 22016, 4096), (8192, 6144, 4096)])
def test_tcgen05_gemm_on_cta_pairs(M, N, K):
    """Shapes large enough for the CTA-pair GEMM (2-SM MMAs over 256 x 256 tiles),
    which takes weights in the library's tile layout: against a float64 matmul of
    the same bf16 inputs, including a ragged M (1000 rows: the last pair tile holds
    rows past the matrix). Row-major weights of the same shapes run the single-CTA
    kernel; the two agree to the GEMM tolerance, not necessarily to the bit."""
    x, w = _inputs(M, N, K, torch.bfloat16, 13)
    wt = B.llama_tile_weights(w)
    y = torch.full((M, N), float("nan"), device="cuda")
    B.llama_linear(x, wt, y, B.LLAMA_PATH_TCGEN05 | B.LLAMA_WEIGHTS_TILED, n=N)
    torch.cuda.synchronize()
    _check(x, w, y)


@pytest.mark.parametrize("M,N,K", [(512, 4096, 11008), (300, 4096, 11008), (40, 512, 8192), (40, 512, 8256),
                                   (512, 12288, 4096), (512, 22016, 4096)])
def test_tcgen05_gemm_on_cta_pairs_with_k_halves(M, N, K):
    """Calls whose whole pair tiles fill less than one wave, with long k ranges
    (the LLaMA-7B layer's w2 at 512 tokens, a ragged 300 and 40, an odd number
    of 64-wide k steps), split each pair tile's k range in two, run on
    different pairs; the second half to finish adds the first's partial sums.
    The 7B layer's wqkv and w1|w3 at 512 tokens stay whole. Against a float64
    matmul, three calls in a row (the arrival counters and flags re-arm
    themselves)."""
    x, w = _inputs(M, N, K, torch.bfloat16, 17)
    wt = B.llama_tile_weights(w)
    for _ in range(3):
        y = torch.full((M, N), float("nan"), device="cuda")
        B.llama_linear(x, wt, y, B.LLAMA_PATH_TCGEN05 | B.LLAMA_WEIGHTS_TILED, n=N)
        torch.cuda.synchronize()
        _check(x, w, y)


@pytest.mark.parametrize("M,N,K", [(1, 128, 256), (5, 384, 4096), (8, 4096, 4096), (16, 12288, 4096),
                                   (17, 256, 11008), (32, 4096, 14336), (32, 28672, 4096), (3, 136, 192), (9, 8, 128)])
def test_gemv_split_k(M, N, K):
    x, w = _inputs(M, N, K, torch.bfloat16, 21)
    y = torch.full((M, N), float("nan"), device="cuda")
    for _ in range(2):  # the second call checks that the split-K counters were re-armed
        B.llama_linear(x, w, y, B.LLAMA_PATH_GEMV)
    torch.cuda.synchronize()
    _check(x, w, y)


@pytest.mark.parametrize("mode", [B.LLAMA_GEMV_MMA_WARP, B.LLAMA_GEMV_MMA_TCGEN05])
@pytest.mark.parametrize("M,N,K", [(9, 8, 128), (16, 12288, 4096), (17, 256, 11008), (24, 6144, 4096),
                                   (32, 4096, 14336), (32, 28672, 4096), (13, 1000, 640)])
def test_gemv_batched_both_products(mode, M, N, K):
    """The 9..32-token decode GEMV with either product (warp-level mma.sync, or
    tcgen05.mma into tensor memory with 17..24 tokens padded to a 32-row box):
    against a float64 matmul, twice in a row (counters re-armed), including row
    blocks that end inside one CTA's range and ragged N."""
    x, w = _inputs(M, N, K, torch.bfloat16, 23)
    y = torch.full((M, N), float("nan"), device="cuda")
    B.llama_set_decode_linear_mma(mode)
    try:
        for _ in range(2):
            B.llama_linear(x, w, y, B.LLAMA_PATH_GEMV)
        torch.cuda.synchronize()
    finally:
        B.llama_set_decode_linear_mma(B.LLAMA_GEMV_MMA_AUTO)
    _check(x, w, y)


def test_decode_linear_mma_mode_is_checked():
    with pytest.raises(Exception):
        B.llama_set_decode_linear_mma(3)


@pytest.mark.parametrize("M,N,K,dt", [(33, 136, 200, torch.float32), (64, 64, 64, torch.float32),
                                      (5, 256, 96, torch.bfloat16),
                                      # fp32 calls of up to 8 tokens take the warp-per-column GEMV
                                      (1, 1000, 256, torch.float32), (8, 1536, 768, torch.float32),
                                      (3, 136, 200, torch.float32), (7, 64, 1024, torch.float32),
                                      (9, 1536, 768, torch.float32), (2, 512, 1032, torch.float32)])
def test_simt_gemm(M, N, K, dt):
    x, w = _inputs(M, N, K, dt, 31)
    y = torch.full((M, N), float("nan"), device="cuda")
    B.llama_linear(x, w, y, B.LLAMA_PATH_SIMT)
    torch.cuda.synchronize()
    _check(x, w, y, rel=1e-5)


@pytest.mark.parametrize("path,M,N,K", [(B.LLAMA_PATH_GEMV, 1, 12288, 4096), (B.LLAMA_PATH_GEMV, 9, 136, 192),
                                        (B.LLAMA_PATH_GEMV, 32, 4096, 11008), (B.LLAMA_PATH_TCGEN05, 300, 1152, 1024),
                                        (B.LLAMA_PATH_TCGEN05, 512, 12160, 4096), (B.LLAMA_PATH_TCGEN05, 77, 384, 448)])
def test_tiled_weights_give_identical_results(path, M, N, K):
    """The tile layout only changes where a 128 x 64 stage is read from: the
    shared-memory image, hence every MMA and every sum, is the same as with
    row-major weights, so the outputs are bit-identical (for shapes that run the
    same kernel with both layouts, as these do: the CTA-pair GEMM takes only
    tiled weights with N a multiple of 256, test_tcgen05_gemm_on_cta_pairs, so
    the tcgen05 shapes here have N = 128 mod 256)."""
    x, w = _inputs(M, N, K, torch.bfloat16, 41)
    wt = B.llama_tile_weights(w)
    assert wt.numel() == (N + 127) // 128 * 128 * K
    # the layout itself: tile (n // 128, k // 64), row n % 128, column k % 64; rows past N zero
    nk = K // 64
    tiles = wt.view(-1, 128, 64)
    for n, k in [(0, 0), (N - 1, K - 1), (min(130, N - 1), 70 % K), (N // 2, K // 2)]:
        assert tiles[(n // 128) * nk + k // 64, n % 128, k % 64] == w[n, k]
    if N % 128:
        assert torch.all(tiles[(N // 128) * nk:, N % 128:, :] == 0)
    y0 = torch.full((M, N), float("nan"), device="cuda")
    y1 = torch.full((M, N), float("nan"), device="cuda")
    B.llama_linear(x, w, y0, path)
    B.llama_linear(x, wt, y1, path | B.LLAMA_WEIGHTS_TILED, n=N)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    _check(x, w, y1)


@pytest.mark.parametrize("M,N,K,path", [(512, 4096, 4096, B.LLAMA_PATH_TCGEN05), (512, 4096, 11008, B.LLAMA_PATH_TCGEN05),
                                        (16, 4096, 4096, B.LLAMA_PATH_GEMV), (1, 4096, 11008, B.LLAMA_PATH_GEMV)])
def test_accumulation_error_against_fp32_orders(M, N, K, path):
    """How far the tensor-core accumulation is from float64, next to an fp32 CPU
    sum taken in the same 16-term blocks: printed (the full-size parity bound
    is sized from it) and held to the GEMM-core tolerance."""
    x, w = _inputs(M, N, K, torch.bfloat16, 51)
    y = torch.empty((M, N), device="cuda")
    B.llama_linear(x, w, y, path)
    torch.cuda.synchronize()
    xd, wd = x.double().cpu(), w.double().cpu()
    ref = (xd @ wd.T).numpy()
    xf, wf = x.float().cpu(), w.float().cpu()
    seq = torch.zeros(M, N)
    for k0 in range(0, K, 16):
        seq += xf[:, k0:k0 + 16] @ wf[:, k0:k0 + 16].T
    eg = y.double().cpu().numpy() - ref
    es = seq.double().numpy() - ref
    rg, rs = float(np.sqrt(np.mean(eg ** 2))), float(np.sqrt(np.mean(es ** 2)))
    print(f"[accumulation] M={M} N={N} K={K} path={path}: GPU rms {rg:.3e} max {np.abs(eg).max():.3e}; "
          f"fp32 16-term blocks rms {rs:.3e} max {np.abs(es).max():.3e}; ratio {rg / rs:.1f}")
    assert np.abs(eg).max() <= 2e-5 * np.abs(ref).max() + 1e-6
