"""Failure detection on the device without a fault: a bounded wait that
nothing completes (an mbarrier phase; the persistent kernel's grid barrier with
a CTA that never arrives) gives up after its limit (~1 s), records the timeout
bit, and the device stays usable for the next call."""
import pytest
import torch

from llama_decoder_block_kv_b200 import binding as B
from llama_decoder_block_kv_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up_and_reports(which):
    flags, secs = B.llama_selftest_bounded_wait(which)
    assert flags == 4, flags              # LLAMA_DEV_TIMEOUT, nothing else
    assert 0.9 <= secs <= 5.0, secs       # the one-second bound, not an early exit
    # the context is intact: an ordinary GEMM right after runs and is correct
    x = synth.normal((3, 256), 1.0, 1, torch.bfloat16, "cuda")
    w = synth.normal((384, 256), 0.02, 2, torch.bfloat16, "cuda")
    y = torch.empty((3, 384), device="cuda")
    B.llama_linear(x, w, y, B.LLAMA_PATH_GEMV)
    torch.cuda.synchronize()
    assert torch.allclose(y, x.float() @ w.float().T, rtol=1e-3, atol=1e-3)


def test_selftest_rejects_unknown_case():
    with pytest.raises(B.LlamaError) as e:
        B.llama_selftest_bounded_wait(7)
    assert e.value.code == B.LLAMA_ERR_INVALID_ARGS
