"""Host-only consistency of the decode kernels' work partitions
(llama_selfcheck_plans walks them with the kernels' own index functions):
every weight tile covered exactly once and in bounds, split-K partial slots
distinct and inside the workspace, for the workloads' shapes, the test shapes,
every batch of up to 32 tokens and several SM counts."""
import os
import random

import pytest

from llama_decoder_block_kv_b200 import binding as B
import oracle as O

pytestmark = pytest.mark.skipif(not os.path.exists(B.LIB_PATH), reason="library not built")

SHAPES = [  # dim, heads, kv heads, ffn, max_seq_len
    (4096, 32, 32, 11008, 2048),                          # LLaMA-7B layer
    (8192, 64, 8, 28672, 8192),                           # LLaMA-2-70B layer
    (4096, 32, 8, 14336, 8192),                           # LLaMA-3-8B
    (512, 4, 2, O.ffn_hidden_dim(512, 256), 256),
    (1024, 8, 1, O.ffn_hidden_dim(1024, 256), 4096),
    (2048, 16, 2, O.ffn_hidden_dim(2048, 256), 256),
    (2048, 32, 1, O.ffn_hidden_dim(2048, 256), 16384),
    (256, 4, 1, 768, 64),                                 # head_dim 64: GEMV only
]


@pytest.mark.parametrize("dim,H,Hkv,F,S", SHAPES)
def test_plans_of_the_workload_and_test_shapes(dim, H, Hkv, F, S):
    for M in (1, 2, 5, 8, 9, 16, 17, 24, 25, 32):
        for sms in (148, 132):
            assert B.llama_selfcheck_plans(M, dim, H, Hkv, F, S, sms) == B.LLAMA_OK, (M, sms)


def test_plans_of_random_shapes_and_grids():
    rng = random.Random(7)
    for _ in range(60):
        D = rng.choice([64, 128])
        Hkv = rng.choice([1, 2, 4, 8])
        H = Hkv * rng.choice([1, 2, 4, 8, 16])
        dim = H * D
        F = 64 * rng.randint(2, 200)
        M = rng.randint(1, 32)
        sms = rng.choice([1, 3, 7, 64, 100, 148, 160])
        assert B.llama_selfcheck_plans(M, dim, H, Hkv, F, 128 * rng.randint(1, 64), sms) == B.LLAMA_OK, \
            (M, dim, H, Hkv, F, sms)


def test_selfcheck_rejects_bad_sizes():
    assert B.llama_selfcheck_plans(0, 4096, 32, 32, 11008, 2048, 148) == B.LLAMA_ERR_INVALID_ARGS
    assert B.llama_selfcheck_plans(1, 4096, 32, 3, 11008, 2048, 148) == B.LLAMA_ERR_INVALID_ARGS


@pytest.mark.parametrize("M", [33, 96, 255, 1024])
def test_stream_k_attention_split_of_wide_batches(M):
    """The decode attention's stream-K split (walked inside llama_selfcheck_plans
    at ragged and uniform positions) for batches past the GEMV range."""
    for dim, H, Hkv, S in ((4096, 32, 8, 2048), (512, 4, 2, 1280), (2048, 32, 1, 512)):
        for sms in (148, 7):
            assert B.llama_selfcheck_plans(M, dim, H, Hkv, 1024, S, sms) == B.LLAMA_OK, (M, dim, H, Hkv, sms)


@pytest.mark.parametrize("H,Hkv", [(24, 1), (48, 2), (40, 1), (56, 7), (64, 2), (16, 1), (12, 3), (6, 2)])
def test_decode_attention_head_groups_cover_every_head(H, Hkv):
    """More than 16 query heads per kv head, not a multiple of 16 (groups of 8),
    next to the usual ratios: every query head in exactly one group of both
    decode attention kernels (checked inside llama_selfcheck_plans)."""
    for D in (64, 128):
        for M in (1, 7, 32):
            assert B.llama_selfcheck_plans(M, H * D, H, Hkv, 1024, 2048, 148) == B.LLAMA_OK, (H, Hkv, D, M)


@pytest.mark.parametrize("H,Hkv", [(20, 1), (17, 1), (34, 2), (36, 3), (44, 1), (12, 1), (10, 1), (9, 3)])
def test_head_groups_of_ratios_that_are_not_multiples_of_eight(H, Hkv):
    """Ratios above 8 that 8 does not divide (20 -> groups of 10, 17 -> groups
    of 1, 22 -> 11): every query head in exactly one group of each attention
    kernel, the prefill's rows holding whole positions."""
    for D in (64, 128):
        for M in (1, 5, 32):
            assert B.llama_selfcheck_plans(M, H * D, H, Hkv, 1024, 512, 148) == B.LLAMA_OK, (H, Hkv, D, M)


@pytest.mark.parametrize("H,Hkv", [(3, 1), (5, 1), (6, 1), (7, 1), (12, 4), (24, 8), (30, 5), (48, 6)])
def test_head_groups_of_every_ratio_up_to_eight(H, Hkv):
    """Ratios of 3, 5, 6 and 7 query heads per kv head: the prefill attention's
    128 MMA rows must hold whole positions (heads per CTA dividing 128) and
    every head must fall in exactly one group of each attention kernel."""
    for D in (64, 128):
        assert B.llama_selfcheck_plans(4, H * D, H, Hkv, 1024, 512, 148) == B.LLAMA_OK, (H, Hkv, D)
