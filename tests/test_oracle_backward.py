"""Pins of the oracle's prefill gradient (CPU only).

The gradient is pinned to things other than itself:
- central finite differences of the forward oracle (itself pinned in test_oracle_pins.py) on
  every element of q, k, v and the initial state, for the loss
  sum(d_out * out) + sum(d_final_state * final_state);
- the window branch alone (alpha = 0) against torch's autograd through
  scaled_dot_product_attention with a band mask, in float64;
- invariants: grouped kv heads get the sum of the gradients of their repeated copies, and a
  packed batch gets the gradients of its sequences run one by one.
"""
import numpy as np
import pytest
import torch

from oracle import oracle

CASES = [
    # name, B, T, Hq, Hkv, d, w, alpha, cu_seqlens, with_s0, with_dfs, gate_off, key_bias
    ("gqa_state_in_and_out", 2, 6, 4, 2, 3, 3, 0.4, None, True, True, False, 0.0),
    ("packed_with_empty_sequence", 1, 9, 2, 1, 4, 2, 0.7, (0, 4, 4, 9), False, True, False, 0.0),
    ("window_wider_than_sequence", 1, 5, 1, 1, 3, 8, 0.5, None, True, False, False, 0.0),
    ("ungated_recurrence_only", 1, 7, 2, 1, 3, 3, 1.0, None, True, True, True, 0.0),
    ("window_only", 1, 7, 2, 2, 3, 4, 0.0, None, False, False, False, 0.0),
    ("saturated_gates", 1, 8, 2, 1, 3, 3, 0.5, None, True, True, False, 6.0),
]


def make(case, seed=0):
    name, B, T, Hq, Hkv, d, w, alpha, cu, with_s0, with_dfs, gate_off, kb = case
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(B, T, Hq, d))
    k = rng.normal(size=(B, T, Hkv, d))
    if kb:   # gates near 1 on even tokens, near 0 on odd ones
        k += np.where(np.arange(T) % 2 == 0, kb, -kb)[None, :, None, None]
    v = rng.normal(size=(B, T, Hkv, d))
    n = B if cu is None else len(cu) - 1
    s0 = 0.3 * rng.normal(size=(n, Hq, d, d)) if with_s0 else np.zeros((n, Hq, d, d))
    dout = rng.normal(size=q.shape)
    dfs = rng.normal(size=(n, Hq, d, d)) if with_dfs else None
    kw = dict(w=w, alpha=alpha, cu_seqlens=cu, gate_off=gate_off)
    return q, k, v, s0, dout, dfs, kw


def loss(q, k, v, s0, dout, dfs, kw):
    out, fs, _, _ = oracle.prefill(q, k, v, initial_state=s0, nthreads=1, **kw)
    L = float(np.sum(dout * out))
    if dfs is not None:
        L += float(np.sum(dfs * fs))
    return L


def numeric_grad(x, f, h=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + h
        fp = f()
        x[idx] = old - h
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * h)
    return g


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_gradient_matches_finite_differences(case):
    q, k, v, s0, dout, dfs, kw = make(case)
    dq, dk, dv, ds0 = oracle.prefill_backward(q, k, v, dout, initial_state=s0, d_final_state=dfs, **kw)
    f = lambda: loss(q, k, v, s0, dout, dfs, kw)   # noqa: E731  (reads the arrays as perturbed)
    for name, x, g in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("initial_state", s0, ds0)):
        np.testing.assert_allclose(g, numeric_grad(x, f), rtol=1e-6, atol=1e-7, err_msg=name)


def test_zero_initial_state_is_the_default():
    q, k, v, _, dout, dfs, kw = make(CASES[1])
    n = len(kw["cu_seqlens"]) - 1
    a = oracle.prefill_backward(q, k, v, dout, d_final_state=dfs, **kw)
    b = oracle.prefill_backward(q, k, v, dout, initial_state=np.zeros((n, 2, 4, 4)), d_final_state=dfs, **kw)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_window_branch_gradient_matches_torch_sdpa():
    """alpha = 0: the gradient of the band-masked softmax attention, from torch's autograd."""
    rng = np.random.default_rng(5)
    B, T, Hq, Hkv, d, w = 2, 11, 4, 2, 5, 4
    q = rng.normal(size=(B, T, Hq, d))
    k = rng.normal(size=(B, T, Hkv, d))
    v = rng.normal(size=(B, T, Hkv, d))
    dout = rng.normal(size=q.shape)
    dq, dk, dv, _ = oracle.prefill_backward(q, k, v, dout, w=w, alpha=0.0)

    qt, kt, vt = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
    G = Hq // Hkv
    kh = kt.repeat_interleave(G, dim=2).transpose(1, 2)
    vh = vt.repeat_interleave(G, dim=2).transpose(1, 2)
    i = torch.arange(T)[:, None]
    j = torch.arange(T)[None, :]
    band = (j <= i) & (j > i - w)
    o = torch.nn.functional.scaled_dot_product_attention(qt.transpose(1, 2), kh, vh, attn_mask=band)
    (o.transpose(1, 2) * torch.tensor(dout)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dk, kt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dv, vt.grad.numpy(), rtol=1e-10, atol=1e-12)


def test_grouped_kv_gets_the_sum_over_its_q_heads():
    """GQA = MHA with each kv head repeated G times: the shared kv head's gradient is the sum."""
    rng = np.random.default_rng(9)
    B, T, Hq, Hkv, d, w = 1, 9, 4, 2, 4, 3
    G = Hq // Hkv
    q = rng.normal(size=(B, T, Hq, d))
    k = rng.normal(size=(B, T, Hkv, d))
    v = rng.normal(size=(B, T, Hkv, d))
    dout = rng.normal(size=q.shape)
    dfs = rng.normal(size=(B, Hq, d, d))
    dq, dk, dv, ds0 = oracle.prefill_backward(q, k, v, dout, w=w, alpha=0.6, d_final_state=dfs)
    kr, vr = np.repeat(k, G, axis=2), np.repeat(v, G, axis=2)
    dq2, dk2, dv2, ds02 = oracle.prefill_backward(q, kr, vr, dout, w=w, alpha=0.6, d_final_state=dfs)
    np.testing.assert_allclose(dq, dq2, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dk, dk2.reshape(B, T, Hkv, G, d).sum(axis=3), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dv, dv2.reshape(B, T, Hkv, G, d).sum(axis=3), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ds0, ds02, rtol=1e-12, atol=1e-13)


def test_packed_sequences_get_their_separate_gradients():
    rng = np.random.default_rng(11)
    lens = (5, 0, 7, 3)
    cu = np.concatenate([[0], np.cumsum(lens)])
    T, Hq, Hkv, d, w = int(cu[-1]), 2, 1, 3, 3
    q = rng.normal(size=(1, T, Hq, d))
    k = rng.normal(size=(1, T, Hkv, d))
    v = rng.normal(size=(1, T, Hkv, d))
    dout = rng.normal(size=q.shape)
    n = len(lens)
    s0 = 0.2 * rng.normal(size=(n, Hq, d, d))
    dfs = rng.normal(size=(n, Hq, d, d))
    dq, dk, dv, ds0 = oracle.prefill_backward(q, k, v, dout, w=w, alpha=0.5, cu_seqlens=cu,
                                              initial_state=s0, d_final_state=dfs)
    for s in range(n):
        a, b = cu[s], cu[s + 1]
        if a == b:
            np.testing.assert_array_equal(ds0[s], dfs[s])   # nothing between the two states
            continue
        r = oracle.prefill_backward(q[:, a:b], k[:, a:b], v[:, a:b], dout[:, a:b], w=w, alpha=0.5,
                                    initial_state=s0[s:s + 1], d_final_state=dfs[s:s + 1])
        np.testing.assert_allclose(dq[:, a:b], r[0], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(dk[:, a:b], r[1], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(dv[:, a:b], r[2], rtol=1e-13, atol=1e-14)
        np.testing.assert_allclose(ds0[s], r[3][0], rtol=1e-13, atol=1e-14)


def test_backward_rejects_bad_arguments():
    q = np.zeros((1, 4, 3, 2))
    k = np.zeros((1, 4, 2, 2))   # Hq % Hkv != 0
    with pytest.raises(ValueError):
        oracle.prefill_backward(q, k, k, q, w=2)
