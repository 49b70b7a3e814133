"""Failure detection on the GPU without a fault: a kernel's bounded wait on a
barrier that nothing signals gives up, the status word says so, and the
context stays usable for the next call."""
import pytest
import torch

import synth
import sparse_attention_20_b200 as dsa
from sparse_attention_20_b200 import build as dsa_build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    dsa_build.build()
    dsa.load_library()
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def test_bounded_wait_reports_timeout_and_context_survives():
    assert dsa.device_status() == 0
    status = dsa.selftest_bounded_wait(limit_ms=100)
    assert status == -4, dsa.last_error()
    assert "tag 999" in dsa.last_error()
    # the status word was cleared by the read, and the library still works
    assert dsa.device_status() == 0
    x = synth.prefill_inputs("tiny", device="cuda", seed=0)
    idx = dsa.indexer_topk(x.q_idx, x.w, x.k_idx, x.k)
    out, lse = dsa.sparse_mla_attn(x.q, x.kv, idx, x.scale, x.d_v)
    torch.cuda.synchronize()
    assert dsa.device_status() == 0
    assert torch.isfinite(lse).all()
