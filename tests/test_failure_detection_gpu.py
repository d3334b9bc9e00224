"""Failure detection without faulting the GPU.

Every wait inside the tensor-core prefill is bounded.  A test switch, read by the
library when it loads, makes the MMA issuer of the process's first tensor-core call
withhold one completion, so the waits behind it run out after a short limit: the
kernel must record a timeout in its workspace (read back as LIGER_ERR_TIMEOUT, with
the site of the first wait that gave up), drain, free its tensor memory and return --
and the CUDA context must stay usable for a normal call right after.  The switch is
set in a child process so that it never reaches the other tests."""
import pytest

from tests import child_scenarios

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(cuda_device):
    out = child_scenarios.run("stall_then_recover", child_scenarios.STALL_ENV)
    assert "timeout reported" in out
