"""Gradient of the bf16 prefill on the GPU against the oracle's gradient (reverse-mode
derivative of the token-by-token evaluation, pinned by finite differences), element by element:
dq, dk, dv and the gradient of the initial state, for L = sum(d_out * out) +
sum(d_final_state * final_state).  Small cases span several chunks, ragged tails, packed
sequences (with an empty one), both head dims, alpha at 0, 0.3 and 1, near-closed gates on both
sides of the factored-decay switch and an initial state; the Llama-3-8B-shape case runs the
backward in the benchmark's configuration and compares every element.  The initial state and
its gradient are one per (sequence, kv head): the oracle's per-head states are that state
repeated over the group, and its per-head gradients are summed over the group.  Tolerance:
bf16, max-abs 2e-2 and rel-L2 5e-3 on each gradient (scaled by the reference's largest
element, since the gradients' magnitudes differ by orders)."""
import zlib

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests.parity_util import errors, np64

pytestmark = pytest.mark.gpu


def assert_grad_close(got, ref, what):
    scale = max(float(np.abs(ref).max()), 1e-30)
    max_abs, rel = errors(got / scale, ref / scale)
    assert max_abs <= 2e-2 and rel <= 5e-3, f"{what}: max-abs/scale {max_abs:.3e}, rel-L2 {rel:.3e}"


CASES = [
    # name, B, Hq, Hkv, T, d, alpha, seqlens, key_bias, with_s0, with_dfs
    ("d128_ragged", 2, 4, 2, 200, 128, 0.5, (), 0.0, False, True),
    ("d64_gqa4", 1, 8, 2, 257, 64, 0.5, (), 0.0, False, False),
    ("d128_packed_empty", 1, 4, 1, 300, 128, 0.3, (70, 0, 130, 100), 0.0, False, True),
    ("d64_alpha1", 1, 4, 2, 150, 64, 1.0, (), 0.0, False, True),
    ("d128_alpha0", 1, 4, 2, 130, 128, 0.0, (), 0.0, False, False),
    ("d128_extreme_gates", 1, 4, 2, 200, 128, 0.5, (), 4.0, False, True),
    ("d64_initial_state", 2, 4, 2, 140, 64, 0.5, (), 0.0, True, True),
]


def run_case(name, B, Hq, Hkv, T, d, alpha, seqlens, kb, with_s0, with_dfs, dev, sharp=False):
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, seed=zlib.crc32(name.encode()) % 10000,
                      seqlens=seqlens, key_bias_std=kb)
    q, k, v = inputs.prefill_inputs(wl)
    if sharp:
        k += 3.0
        k[:, 30] = -50.0
        k[:, 100] = -70.0
        k[:, 150] = -55.0
    n = wl.n_seqs
    G = Hq // Hkv
    gen = torch.Generator().manual_seed(17)
    dout = torch.randn(q.shape, generator=gen).to(q.dtype)
    dfs = torch.randn(n, Hq, d, d, generator=gen) * 0.1 if with_dfs else None
    s0 = inputs.random_state(n, Hkv, d, seed=9, scale=0.05) if with_s0 else None
    cu = wl.cu_seqlens
    dq, dk, dv, ds0 = ops.prefill_backward(
        q.to(dev), k.to(dev), v.to(dev), dout.to(dev), alpha=alpha,
        d_final_state=None if dfs is None else dfs.to(dev), initial_state=None if s0 is None else s0.to(dev),
        cu_seqlens=None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev), want_d_initial_state=True)
    torch.cuda.synchronize()
    s0_heads = None if s0 is None else np.repeat(np64(s0), G, axis=1)
    rdq, rdk, rdv, rds0 = oracle.prefill_backward(
        np64(q), np64(k), np64(v), np64(dout), alpha=alpha, initial_state=s0_heads, cu_seqlens=cu,
        d_final_state=None if dfs is None else np64(dfs))
    rds0_kv = rds0.reshape(n, Hkv, G, d, d).sum(axis=2)
    assert_grad_close(np64(dq), rdq, f"{name} dq")
    assert_grad_close(np64(dk), rdk, f"{name} dk")
    assert_grad_close(np64(dv), rdv, f"{name} dv")
    assert_grad_close(np64(ds0), rds0_kv, f"{name} d_initial_state")


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_small(case, cuda_device):
    run_case(*case, dev=cuda_device)


def test_backward_sharp_gate_drops(cuda_device):
    """Chunks on both sides of the factored-decay switch (totals near -53, -58, -73)."""
    run_case("sharp_drops", 1, 4, 2, 260, 128, 0.5, (), 0.0, False, True, dev=cuda_device, sharp=True)


def test_backward_is_deterministic_in_dq(cuda_device):
    wl = inputs.small("bwd_det", B=1, Hq=4, Hkv=2, T=300, d=128)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    dout = torch.randn_like(q)
    a = ops.prefill_backward(q, k, v, dout)
    b = ops.prefill_backward(q, k, v, dout)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])


def test_backward_llama8b_shape(cuda_device):
    """B=2, T=8192, Hq=32, Hkv=8, d=128 with a final-state gradient: every element of dq, dk, dv
    and d_initial_state against the oracle."""
    wl = inputs.WORKLOADS["llama8b_prefill"]
    q, k, v = inputs.prefill_inputs(wl)
    gen = torch.Generator().manual_seed(23)
    dout = torch.randn(q.shape, generator=gen).to(q.dtype)
    dfs = torch.randn(wl.n_seqs, wl.Hq, wl.d, wl.d, generator=gen) * 0.1
    dev = cuda_device
    dq, dk, dv, ds0 = ops.prefill_backward(q.to(dev), k.to(dev), v.to(dev), dout.to(dev), alpha=wl.alpha,
                                           d_final_state=dfs.to(dev), want_d_initial_state=True)
    torch.cuda.synchronize()
    # the oracle keeps every state of a sequence (8192 x d x d doubles per head): 8 threads at a time
    rdq, rdk, rdv, rds0 = oracle.prefill_backward(np64(q), np64(k), np64(v), np64(dout), alpha=wl.alpha,
                                                  d_final_state=np64(dfs), nthreads=8)
    G = wl.Hq // wl.Hkv
    assert_grad_close(np64(dq), rdq, "dq")
    assert_grad_close(np64(dk), rdk, "dk")
    assert_grad_close(np64(dv), rdv, "dv")
    assert_grad_close(np64(ds0), rds0.reshape(wl.n_seqs, wl.Hkv, G, wl.d, wl.d).sum(axis=2), "d_initial_state")
