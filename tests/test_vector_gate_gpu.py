"""The per-dimension (vector) gate on the GPU against the oracle: the prefill (segment-parallel
general kernels) and decode steps, bf16 and fp32, with ragged and packed sequences and an initial state; the
Llama-3-8B-shape prefill in full.  Tolerances: bf16 max-abs 2e-2 and rel-L2 5e-3, fp32 1e-4."""
import zlib

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests.parity_util import assert_close, np64

pytestmark = pytest.mark.gpu

CASES = [
    ("bf16_d128", 2, 8, 2, 200, 128, torch.bfloat16, (), False),
    ("bf16_d64_packed", 1, 4, 2, 230, 64, torch.bfloat16, (100, 0, 130), False),
    ("fp32_d64_s0", 1, 4, 4, 130, 64, torch.float32, (), True),
    ("fp32_d128", 1, 2, 1, 90, 128, torch.float32, (), False),
    # several 256-token segments (a ragged last one), packed sequences across segment
    # boundaries, an initial state shared by each group (the segment scan starts from it)
    ("bf16_d128_segments", 1, 8, 2, 700, 128, torch.bfloat16, (), False),
    ("bf16_d64_packed_segments", 1, 4, 2, 1100, 64, torch.bfloat16, (300, 0, 530, 270), False),
    ("fp32_d64_shared_s0_segments", 2, 4, 2, 600, 64, torch.float32, (), "shared"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_vector_gate_prefill_then_decode(case, cuda_device):
    name, B, Hq, Hkv, T, d, dtype, seqlens, with_s0 = case
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, dtype=dtype, seed=zlib.crc32(name.encode()) % 10000,
                      seqlens=seqlens)
    q, k, v = inputs.prefill_inputs(wl)
    n = wl.n_seqs
    s0 = inputs.random_state(n, Hq, d, seed=4, scale=0.05) if with_s0 else None
    if with_s0 == "shared":   # the copies of a group equal: one state per kv head
        s0 = s0.view(n, Hkv, Hq // Hkv, d, d)[:, :, :1].expand(n, Hkv, Hq // Hkv, d, d).reshape(n, Hq, d, d)
        s0 = s0.contiguous()
    cu = wl.cu_seqlens
    dev = cuda_device
    out, fs, ring, pos = ops.prefill_vector_gate(
        q.to(dev), k.to(dev), v.to(dev), initial_state=None if s0 is None else s0.to(dev),
        cu_seqlens=None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev), return_ring=True)
    torch.cuda.synchronize()
    ro, rfs, rring, rpos = oracle.prefill(np64(q), np64(k), np64(v), cu_seqlens=cu, vector_gate=True,
                                          initial_state=None if s0 is None else np64(s0))
    assert_close(np64(out), ro, dtype, "out")
    assert_close(np64(fs), rfs, dtype, "final_state")
    np.testing.assert_array_equal(np64(ring), rring)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
    if cu is not None:
        return
    # decode steps from the GPU prefill's state (both sides start from the same fp32 state)
    st = np.ascontiguousarray(np64(fs))
    rg = np.ascontiguousarray(np64(ring))
    ps = np.ascontiguousarray(pos.cpu().numpy().astype(np.int32))
    for step in range(6):
        qt, kt, vt = inputs.decode_step_inputs(inputs.Workload("vg", "decode", B, Hq, Hkv, T, d, dtype), step)
        o = ops.decode_vector_gate(qt.to(dev), kt.to(dev), vt.to(dev), fs, ring, pos)
        ro = oracle.decode_inplace(np64(qt), np64(kt), np64(vt), st, rg, ps, vector_gate=True)
        torch.cuda.synchronize()
        assert_close(np64(o), ro, dtype, f"decode step {step}")
    assert_close(np64(fs), st, dtype, "state after decode")


def test_vector_gate_llama8b_shape(cuda_device):
    """Llama-3-8B shape on one batch row (B=1, T=8192, Hq=32, Hkv=8, d=128), every element."""
    wl = inputs.WORKLOADS["llama8b_prefill"]
    q, k, v = (t[:1].contiguous() for t in inputs.prefill_inputs(wl))
    dev = cuda_device
    out, fs = ops.prefill_vector_gate(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v), vector_gate=True)
    assert_close(np64(out), ro, wl.dtype, "out")
    assert_close(np64(fs), rfs, wl.dtype, "final_state")
