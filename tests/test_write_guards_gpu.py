"""No entry point writes outside the tensors it is given: every input, output, ring, position
and workspace tensor sits inside a byte buffer with guard regions (tests/canary.py), checked
after each call.  The outputs are also compared with the oracle, so a call that wrote nothing
cannot pass."""
import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests.canary import Guarded, guarded_like
from tests.parity_util import assert_close, np64

pytestmark = pytest.mark.gpu

PREFILL = [
    # name, B, Hq, Hkv, T, d, dtype, seqlens
    ("tensor_core_d128_ragged", 2, 8, 2, 257, 128, torch.bfloat16, ()),
    ("tensor_core_d64_packed", 1, 4, 2, 150, 64, torch.bfloat16, (0, 77, 73, 0)),
    ("general_fp32", 1, 4, 2, 150, 128, torch.float32, ()),
]


@pytest.mark.parametrize("case", PREFILL, ids=[c[0] for c in PREFILL])
def test_prefill_writes_stay_inside_their_tensors(case, cuda_device):
    name, B, Hq, Hkv, T, d, dtype, seqlens = case
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, dtype=dtype, seed=41, seqlens=seqlens)
    q, k, v = inputs.prefill_inputs(wl)
    cu = wl.cu_seqlens
    n = wl.n_seqs
    dev = cuda_device
    gq, gk, gv = (guarded_like(t, dev) for t in (q, k, v))
    gout = Guarded(tuple(q.shape), dtype, dev)
    gfs = Guarded((n, Hq, d, d), torch.float32, dev)
    gring = Guarded((n, Hkv, 2, 64, d), dtype, dev)
    gpos = Guarded((n,), torch.int32, dev)
    gcu = None if cu is None else guarded_like(torch.tensor(cu, dtype=torch.int32), dev)
    need = ops.prefill_workspace_size(B, Hq, Hkv, T, d, n, dtype)
    gws = Guarded((need,), torch.uint8, dev) if need else None
    ops.prefill(gq.tensor, gk.tensor, gv.tensor, cu_seqlens=None if gcu is None else gcu.tensor,
                return_ring=True, out=gout.tensor, final_state=gfs.tensor, ring=gring.tensor,
                pos=gpos.tensor, workspace=None if gws is None else gws.tensor)
    torch.cuda.synchronize()
    for what, g in (("q", gq), ("k", gk), ("v", gv), ("out", gout), ("final_state", gfs),
                    ("ring", gring), ("pos", gpos), ("cu_seqlens", gcu), ("workspace", gws)):
        assert g is None or g.intact(), f"{what}: a write beyond the tensor"
    ro, rfs, rring, rpos = oracle.prefill(np64(q), np64(k), np64(v), cu_seqlens=cu)
    assert_close(np64(gout.tensor), ro, dtype, "out")
    assert_close(np64(gfs.tensor), rfs, dtype, "final_state")
    np.testing.assert_array_equal(np64(gring.tensor), rring)
    np.testing.assert_array_equal(gpos.tensor.cpu().numpy(), rpos)


@pytest.mark.parametrize("kvshared", [False, True], ids=["per_head", "kv_shared"])
def test_decode_writes_stay_inside_their_tensors(kvshared, cuda_device):
    B, Hq, Hkv, d, w = 3, 8, 2, 128, 64
    G = Hq // Hkv
    dev = cuda_device
    gen = torch.Generator().manual_seed(5)
    hs = Hkv if kvshared else Hq
    state = 0.05 * torch.randn(B, hs, d, d, generator=gen)
    ring = torch.randn(B, Hkv, 2, w, d, generator=gen).to(torch.bfloat16)
    pos = torch.tensor([0, 63, 700], dtype=torch.int32)
    q = torch.randn(B, Hq, d, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, Hkv, d, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, Hkv, d, generator=gen).to(torch.bfloat16)
    gq, gk, gv, gst, grg, gps = (guarded_like(t, dev) for t in (q, k, v, state, ring, pos))
    gout = Guarded((B, Hq, d), torch.bfloat16, dev)
    fn = ops.decode_kvshared if kvshared else ops.decode
    fn(gq.tensor, gk.tensor, gv.tensor, gst.tensor, grg.tensor, gps.tensor, out=gout.tensor)
    torch.cuda.synchronize()
    for what, g in (("q", gq), ("k", gk), ("v", gv), ("state", gst), ("ring", grg), ("pos", gps),
                    ("out", gout)):
        assert g.intact(), f"{what}: a write beyond the tensor"
    st = np64(state)
    if kvshared:
        st = np.repeat(st, G, axis=1)
    ro, rst, rrg, rps = oracle.decode(np64(q), np64(k), np64(v), st, np64(ring), pos.numpy(), w=w)
    assert_close(np64(gout.tensor), ro, torch.bfloat16, "out")
    got_state = np64(gst.tensor)
    if kvshared:
        got_state = np.repeat(got_state, G, axis=1)
    assert_close(got_state, rst, torch.bfloat16, "state")
    np.testing.assert_array_equal(np64(grg.tensor), rrg)
    np.testing.assert_array_equal(gps.tensor.cpu().numpy(), rps)
