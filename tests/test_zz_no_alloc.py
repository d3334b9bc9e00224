"""The prefill entry point that allocates nothing (liger_attn_prefill_noalloc).

It serves callers that cannot call cudaMalloc where they run the prefill: its
scratch is a fixed array inside the library.  These tests call it through the
C ABI and check that, on two calls in a row, it returns what the ordinary
entry point (with a caller-allocated workspace) returns, within the bf16
tolerance used by the parity tests, and that sizes beyond its scratch are
refused.  The file sorts last so that a run stopping at the first failure has
already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
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


@pytest.mark.parametrize("case", [
    dict(name="batch", B=2, Hq=8, Hkv=2, T=1000, d=128, seqlens=()),
    dict(name="varlen", B=1, Hq=8, Hkv=4, T=700, d=64, seqlens=(100, 1, 465, 134)),
])
def test_noalloc_matches_workspace_entry_point_twice(case, cuda_device):
    lib = ops.load()
    wl = inputs.small(case["name"], B=case["B"], Hq=case["Hq"], Hkv=case["Hkv"], T=case["T"], d=case["d"],
                      seed=77, seqlens=case["seqlens"])
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    cu = None if wl.cu_seqlens is None else torch.tensor(wl.cu_seqlens, dtype=torch.int32, device=cuda_device)
    n = wl.n_seqs
    need = ops.prefill_workspace_size(wl.B, wl.Hq, wl.Hkv, wl.T, wl.d, n)
    assert 0 < need <= 16 * 1024 * 1024
    ref_out, ref_fs, ref_ring, ref_pos = ops.prefill(q, k, v, cu_seqlens=cu, return_ring=True)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        fs = torch.full((n, wl.Hq, wl.d, wl.d), float("nan"), device=cuda_device)
        ring = torch.empty(n, wl.Hkv, 2, 64, wl.d, dtype=q.dtype, device=cuda_device)
        pos = torch.full((n,), -1, dtype=torch.int32, device=cuda_device)
        st = _noalloc(lib, q, k, v, out, fs, ring, pos, cu=cu, n=n)
        assert st == ops.LIGER_OK, ops.last_error()
        torch.cuda.synchronize()
        assert_close(np64(out), np64(ref_out), torch.bfloat16, "out")
        assert_close(np64(fs), np64(ref_fs), torch.bfloat16, "final_state")
        assert torch.equal(ring, ref_ring) and torch.equal(pos, ref_pos)


def test_noalloc_refuses_sizes_beyond_its_scratch(cuda_device):
    lib = ops.load()
    B, Hq, Hkv, T, d = 1, 32, 8, 1 << 20, 128
    need = ops.prefill_workspace_size(B, Hq, Hkv, T, d, B)
    assert need > 16 * 1024 * 1024
    st = lib.liger_attn_prefill_noalloc(
        ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), ctypes.c_void_p(16), None, B, Hq, Hkv,
        T, d, 64, 0.5, ops.LIGER_BF16, None, None, B, None, None, None)
    assert st == ops.LIGER_ERR_UNSUPPORTED
    assert "scratch" in ops.last_error()
