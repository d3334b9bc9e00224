"""Failure detection without faulting the GPU.

Every wait inside the tensor-core prefill is bounded.  A test switch makes the
MMA issuer withhold one completion, so the waits behind it run out after a short
limit: the kernel must record a timeout in its workspace (read back as
LIGER_ERR_TIMEOUT, with the site of the first wait that gave up), drain, free its
tensor memory and return -- and the CUDA context must stay usable for a normal
call right after."""
import os

import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from tests.parity_util import assert_close, np64
from oracle import oracle

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    wl = inputs.small("stall", B=1, Hq=4, Hkv=2, T=200, d=128, seed=41)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    need = ops.prefill_workspace_size(1, 4, 2, 200, 128, 1)
    ws = torch.zeros(need, dtype=torch.uint8, device=cuda_device)
    os.environ["LIGER_TEST_INJECT_STALL"] = "1"
    os.environ["LIGER_WAIT_LIMIT_NS"] = "50000000"   # 50 ms per wait
    try:
        ops.prefill(q, k, v, workspace=ws)
        torch.cuda.synchronize()
    finally:
        del os.environ["LIGER_TEST_INJECT_STALL"]
        del os.environ["LIGER_WAIT_LIMIT_NS"]
    assert ops.prefill_status(ws) == ops.LIGER_ERR_TIMEOUT
    msg = ops.last_error()
    assert "gave up waiting" in msg and any(f"role {r}," in msg for r in (2, 3, 4, 5))
    # the context is intact: a normal call right after is correct and reports OK
    out, fs = ops.prefill(q, k, v, workspace=ws)
    torch.cuda.synchronize()
    assert ops.prefill_status(ws) == ops.LIGER_OK
    ro, rfs, _, _ = oracle.prefill(np64(q.cpu()), np64(k.cpu()), np64(v.cpu()))
    assert_close(np64(out), ro, torch.bfloat16, "out after a timeout")
    assert_close(np64(fs), rfs, torch.bfloat16, "final state after a timeout")
