"""Causal softmax attention (the standard attention layer of the inter-layer hybrid) on the
GPU against the oracle: every output of small cases (several 128-token blocks, ragged tails,
packed sequences with an empty one, MHA and GQA, d = 64 and 128), and at the Llama-3-8B shape
(B=2, T=8192, Hq=32, Hkv=8, d=128) the first 384 tokens in full plus sampled rows across the
whole sequence, the last ones included.  Tolerance: bf16, max-abs 2e-2 and rel-L2 5e-3."""
import zlib

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests.parity_util import assert_close, np64

pytestmark = pytest.mark.gpu

CASES = [
    # name, B, Hq, Hkv, T, d, seqlens
    ("d128_gqa_ragged", 2, 8, 2, 300, 128, ()),
    ("d64_mha", 1, 4, 4, 260, 64, ()),
    ("d128_one_token", 2, 4, 2, 1, 128, ()),
    ("d64_one_block", 1, 4, 1, 128, 64, ()),
    ("d128_packed_empty", 1, 4, 2, 400, 128, (130, 0, 1, 269)),
    ("d64_packed", 1, 6, 3, 333, 64, (200, 133)),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_full_causal_small(case, cuda_device):
    name, B, Hq, Hkv, T, d, seqlens = case
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, seed=zlib.crc32(name.encode()) % 10000, seqlens=seqlens)
    q, k, v = inputs.prefill_inputs(wl)
    cu = wl.cu_seqlens
    dev = cuda_device
    out = ops.full_causal_attention(q.to(dev), k.to(dev), v.to(dev),
                                    cu_seqlens=None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    assert ops.full_causal_status() == ops.LIGER_OK
    longest = max(seqlens) if seqlens else T
    ref = oracle.prefill(np64(q), np64(k), np64(v), w=max(longest, 1), alpha=0.0, cu_seqlens=cu)[0]
    assert_close(np64(out), ref, torch.bfloat16, "out")


def test_full_causal_llama8b_shape(cuda_device):
    wl = inputs.WORKLOADS["llama8b_prefill"]
    q, k, v = inputs.prefill_inputs(wl)
    dev = cuda_device
    out = ops.full_causal_attention(q.to(dev), k.to(dev), v.to(dev)).cpu()
    assert ops.full_causal_status() == ops.LIGER_OK
    T0 = 384   # rows < T0 depend on keys < T0 only
    ref = oracle.prefill(np64(q[:, :T0]), np64(k[:, :T0]), np64(v[:, :T0]), w=T0, alpha=0.0)[0]
    assert_close(np64(out[:, :T0]), ref, wl.dtype, "first 384 tokens")
    rng = np.random.default_rng(5)
    rows = [(int(b), int(t), int(h)) for b, t, h in zip(rng.integers(0, wl.B, 300), rng.integers(0, wl.T, 300),
                                                       rng.integers(0, wl.Hq, 300))]
    rows += [(b, wl.T - 1, h) for b in range(wl.B) for h in (0, 7, 31)]
    got = np.stack([np64(out[b, t, h]) for b, t, h in rows])
    assert_close(got, oracle.causal_attention_rows(np64(q), np64(k), np64(v), rows), wl.dtype, "sampled rows")
