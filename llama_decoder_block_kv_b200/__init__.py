"""LLaMA decoder block with a KV-cache, native to the B200 (sm_100a).

The compute path is the C-ABI shared library built from ``csrc/`` (declared in
``include/llama_b200.h``); ``binding`` marshals torch tensors into its calls.
The binding loads the library on first use and raises if it is missing: there
is no CPU fallback.
"""
__all__ = ["binding", "synth"]
