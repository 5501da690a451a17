"""CPU oracle (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference
legs of ``bench.py`` may import this package. It shares no code with the CUDA
library in ``llama_decoder_block_kv_b200`` and never imports it.
"""
from .llama_oracle import (  # noqa: F401
    ACT_BF16,
    ACT_FP32,
    LAYER_KEYS,
    ModelArgs,
    OracleModel,
    act_round,
    apply_rope,
    as_f64,
    bf16_bits_to_f64,
    bf16_round,
    block_forward,
    block_forward_rows,
    causal_gqa_attention,
    ffn_hidden_dim,
    generate,
    rmsnorm,
    rope_tables,
    select_next,
    silu,
)
