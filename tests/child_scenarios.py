"""GPU scenarios that need library options set in the environment before the library
loads (the library reads them once, at load).  Each runs in a fresh child process
(``python -m tests.child_scenarios <name>``), checks its own results and exits
non-zero on a failure; ``run`` starts one from a test and returns its output.

Scenarios:
  stall_then_recover    LIGER_TEST_INJECT_STALL=1: the first tensor-core call
                        times out, reports LIGER_ERR_TIMEOUT with its site, and the
                        next call on the same context is correct.
  noalloc_stall_status  the same through liger_attn_prefill_noalloc and
                        liger_attn_prefill_noalloc_status.
  general_parity        LIGER_PREFILL_PATH=general: the general (CUDA-core)
                        prefill kernel on bf16 cases against the oracle.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

STALL_ENV = {"LIGER_TEST_INJECT_STALL": "1", "LIGER_WAIT_LIMIT_NS": "50000000"}   # 50 ms per wait
GENERAL_ENV = {"LIGER_PREFILL_PATH": "general"}


def run(name: str, env_extra: dict, timeout: float = 600.0) -> str:
    """Runs scenario `name` in a child process; raises AssertionError with its output on failure."""
    env = dict(os.environ)
    for key in ("LIGER_TEST_INJECT_STALL", "LIGER_WAIT_LIMIT_NS", "LIGER_PREFILL_PATH"):
        env.pop(key, None)
    env.update(env_extra)
    r = subprocess.run([sys.executable, "-m", "tests.child_scenarios", name], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=timeout)
    out = r.stdout + r.stderr
    assert r.returncode == 0, f"scenario {name} failed (rc {r.returncode}):\n{out[-4000:]}"
    return out


def _stall_then_recover():
    import torch

    from gated_linear_attention_liger_b200 import inputs, ops
    from oracle import oracle
    from tests.parity_util import assert_close, np64

    dev = torch.device("cuda:0")
    wl = inputs.small("stall", B=1, Hq=4, Hkv=2, T=200, d=128, seed=41)
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    need = ops.prefill_workspace_size(1, 4, 2, 200, 128, 1)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    ops.prefill(q, k, v, workspace=ws)   # the first call withholds a completion
    torch.cuda.synchronize()
    assert ops.prefill_status(ws) == ops.LIGER_ERR_TIMEOUT
    msg = ops.last_error()
    assert "gave up waiting" in msg and any(f"role {r}," in msg for r in (2, 3, 4, 5)), msg
    # the context is intact: a normal call right after is correct and reports OK
    out, fs = ops.prefill(q, k, v, workspace=ws)
    torch.cuda.synchronize()
    assert ops.prefill_status(ws) == ops.LIGER_OK
    ro, rfs, _, _ = oracle.prefill(np64(q.cpu()), np64(k.cpu()), np64(v.cpu()))
    assert_close(np64(out), ro, torch.bfloat16, "out after a timeout")
    assert_close(np64(fs), rfs, torch.bfloat16, "final state after a timeout")
    print("timeout reported:", msg)


def _noalloc_stall_status():
    import torch

    from gated_linear_attention_liger_b200 import inputs, ops

    lib = ops.load()
    dev = torch.device("cuda:0")
    wl = inputs.small("stall_na", B=1, Hq=4, Hkv=2, T=200, d=128, seed=43)
    q, k, v = (t.to(dev) for t in inputs.prefill_inputs(wl))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    vp = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    def call(out, fs):
        return lib.liger_attn_prefill_noalloc(vp(q), vp(k), vp(v), vp(out), vp(fs), 1, 4, 2, 200, 128, 64, 0.5,
                                              ops.LIGER_BF16, None, None, 1, None, None, stream)

    out = torch.empty_like(q)
    fs = torch.empty(1, 4, 128, 128, device=dev)
    assert call(out, fs) == ops.LIGER_OK, ops.last_error()   # the first call withholds a completion
    torch.cuda.synchronize()
    assert lib.liger_attn_prefill_noalloc_status() == ops.LIGER_ERR_TIMEOUT
    assert "gave up waiting" in ops.last_error(), ops.last_error()
    assert call(out, fs) == ops.LIGER_OK, ops.last_error()
    torch.cuda.synchronize()
    assert lib.liger_attn_prefill_noalloc_status() == ops.LIGER_OK, ops.last_error()
    ref_out, ref_fs = ops.prefill(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(fs, ref_fs)
    print("no-alloc timeout reported and cleared")


def _general_parity():
    import numpy as np
    import torch

    from tests.parity_util import assert_close, np64
    from tests.test_parity_gpu import SMALL, run_small

    dev = torch.device("cuda:0")
    cases = [c for c in SMALL if c[6] == torch.bfloat16][:6]
    for case in cases:
        (out, fs, ring, pos), (ro, rfs, rring, rpos), dtype = run_small(case, dev)
        assert_close(np64(out), ro, dtype, f"{case[0]} out")
        assert_close(np64(fs), rfs, dtype, f"{case[0]} final_state")
        np.testing.assert_array_equal(np64(ring), rring)
        np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
        print("general kernel ok:", case[0])


SCENARIOS = {"stall_then_recover": _stall_then_recover, "noalloc_stall_status": _noalloc_stall_status,
             "general_parity": _general_parity}

if __name__ == "__main__":
    if ROOT not in sys.path:
        sys.path.insert(0, ROOT)
    SCENARIOS[sys.argv[1]]()
