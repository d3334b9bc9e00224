"""The prefill entry point that allocates nothing (liger_attn_prefill_noalloc).

It serves callers that cannot call cudaMalloc where they run the prefill (a plugin
whose host framework owns every device allocation, a serving loop that reserved all
memory up front, a path that must not take cudaMalloc's implicit synchronisation):
its scratch is a fixed array inside the library.  These tests call it through the C
ABI.  On two calls in a row -- after a larger call of another shape has left its
contents in the shared scratch -- it must return exactly what the ordinary entry point
(with a caller-allocated workspace) returns, and agree with the oracle within the bf16
tolerance of the parity tests.  Sizes beyond its scratch are refused before anything
is launched; calls that the general kernel serves use no scratch and are not limited;
its status call reports a timeout of its own kernels.  The file sorts last so that a
run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests import child_scenarios
from tests.parity_util import assert_close, np64

pytestmark = pytest.mark.gpu


def _vp(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _noalloc(lib, q, k, v, out, fs, ring, pos, cu=None, n=None, alpha=0.5, w=64):
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    n = B if cu is None else n
    return lib.liger_attn_prefill_noalloc(
        _vp(q), _vp(k), _vp(v), _vp(out), _vp(fs), B, Hq, Hkv, T, d, w, alpha, ops.LIGER_BF16, None,
        _vp(cu), n, _vp(ring), _vp(pos), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _fill_scratch_with_a_larger_call(lib, device):
    """A call of another, larger shape, so the compared calls find the shared scratch full of
    that call's tables and states."""
    wl = inputs.small("filler", B=1, Hq=16, Hkv=4, T=2500, d=128, seed=5)
    q, k, v = (t.to(device) for t in inputs.prefill_inputs(wl))
    need = ops.prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, wl.B)
    assert need <= 16 * 1024 * 1024
    out = torch.empty_like(q)
    fs = torch.empty(1, wl.Hq, wl.d, wl.d, device=device)
    assert _noalloc(lib, q, k, v, out, fs, None, None) == ops.LIGER_OK, ops.last_error()
    torch.cuda.synchronize()
    return need


@pytest.mark.parametrize("case", [
    dict(name="batch", B=2, Hq=8, Hkv=2, T=1000, d=128, seqlens=()),
    dict(name="varlen", B=1, Hq=8, Hkv=4, T=700, d=64, seqlens=(100, 1, 465, 134)),
])
def test_noalloc_matches_workspace_entry_point_twice(case, cuda_device):
    lib = ops.load()
    filler_need = _fill_scratch_with_a_larger_call(lib, cuda_device)
    wl = inputs.small(case["name"], B=case["B"], Hq=case["Hq"], Hkv=case["Hkv"], T=case["T"], d=case["d"],
                      seed=77, seqlens=case["seqlens"])
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    cu = None if wl.cu_seqlens is None else torch.tensor(wl.cu_seqlens, dtype=torch.int32, device=cuda_device)
    n = wl.n_seqs
    need = ops.prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, n)
    assert 0 < need < filler_need
    ref_out, ref_fs, ref_ring, ref_pos = ops.prefill(q, k, v, cu_seqlens=cu, return_ring=True)
    ro, rfs, rring, rpos = oracle.prefill(np64(q), np64(k), np64(v), cu_seqlens=wl.cu_seqlens)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        fs = torch.full((n, wl.Hq, wl.d, wl.d), float("nan"), device=cuda_device)
        ring = torch.empty(n, wl.Hkv, 2, 64, wl.d, dtype=q.dtype, device=cuda_device)
        pos = torch.full((n,), -1, dtype=torch.int32, device=cuda_device)
        st = _noalloc(lib, q, k, v, out, fs, ring, pos, cu=cu, n=n)
        assert st == ops.LIGER_OK, ops.last_error()
        torch.cuda.synchronize()
        assert lib.liger_attn_prefill_noalloc_status() == ops.LIGER_OK, ops.last_error()
        # the prefill is deterministic: the same bits as with a workspace of its own
        assert torch.equal(out, ref_out) and torch.equal(fs, ref_fs)
        assert torch.equal(ring, ref_ring) and torch.equal(pos, ref_pos)
        assert_close(np64(out), ro, torch.bfloat16, "out vs oracle")
        assert_close(np64(fs), rfs, torch.bfloat16, "final_state vs oracle")
        np.testing.assert_array_equal(np64(ring), rring)
        np.testing.assert_array_equal(pos.cpu().numpy(), rpos)


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    # Null tensor pointers: the size check comes first, so the call is refused for its size;
    # were that check ever lost, the ordinary entry point would reject the null pointers on
    # the host and the assertion on the message would fail without anything being launched.
    lib = ops.load()
    B, Hq, Hkv, T, d = 1, 32, 8, 1 << 20, 128
    need = ops.prefill_workspace_size(B, Hq, Hkv, T, d, B)
    assert need > 16 * 1024 * 1024
    st = lib.liger_attn_prefill_noalloc(None, None, None, None, None, B, Hq, Hkv, T, d, 64, 0.5, ops.LIGER_BF16,
                                        None, None, B, None, None, None)
    assert st == ops.LIGER_ERR_UNSUPPORTED
    assert "scratch" in ops.last_error()


def test_noalloc_general_kernel_calls_are_not_size_limited(cuda_device):
    # w = 32 is served by the general kernel, which uses no scratch: the size limit does not
    # apply, and the call reaches the ordinary argument checks (null pointers: rejected there).
    lib = ops.load()
    B, Hq, Hkv, T, d = 1, 32, 8, 1 << 20, 128
    assert ops.prefill_workspace_size(B, Hq, Hkv, T, d, B) > 16 * 1024 * 1024
    st = lib.liger_attn_prefill_noalloc(None, None, None, None, None, B, Hq, Hkv, T, d, 32, 0.5, ops.LIGER_BF16,
                                        None, None, B, None, None, None)
    assert st == ops.LIGER_ERR_INVALID_ARG
    assert "scratch" not in ops.last_error()
    # and a real general-kernel call through it matches the workspace entry point
    wl = inputs.small("general_na", B=1, Hq=4, Hkv=2, T=150, d=64, seed=8)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    out = torch.empty_like(q)
    fs = torch.empty(1, 4, 64, 64, device=cuda_device)
    assert _noalloc(lib, q, k, v, out, fs, None, None, w=32) == ops.LIGER_OK, ops.last_error()
    torch.cuda.synchronize()
    assert lib.liger_attn_prefill_noalloc_status() == ops.LIGER_OK
    ref_out, ref_fs = ops.prefill(q, k, v, w=32)
    torch.cuda.synchronize()
    assert torch.equal(out, ref_out) and torch.equal(fs, ref_fs)


def test_noalloc_status_reports_a_timeout(cuda_device):
    """In a child process whose library was loaded with the stall switch: the first no-alloc call
    times out, liger_attn_prefill_noalloc_status says so, the next call is correct and clears it."""
    out = child_scenarios.run("noalloc_stall_status", child_scenarios.STALL_ENV)
    assert "no-alloc timeout reported and cleared" in out
