"""Pins of the fp64 oracle against what the Liger pages and mathematics fix.

Every check reaches the expected value by a route that shares nothing with
the oracle's token-by-token loop: scipy / torch library routines, quadratic
(parallel) forms of the recurrence, a closed form, or an invariant.  A dropped
term, a wrong sign or index, or a transposed operand in the oracle fails at
least one of them.

Sources: "Liger: Linearizing Large Language Models to Gated Recurrent
Structures" (Paper-Notes page) -- gate equation (section 核心思想), recurrence
(section 统一的门控线性循环框架), hybrid o = alpha*GRM + beta*SWA with w = 64
(section Liger Attention), ablation table rows "去掉SWA" (no SWA) and
"纯线性注意力(无Gate)" (no gate).
"""
import numpy as np
import pytest
import scipy.special as sps
import torch

from oracle import oracle

RNG = np.random.default_rng(12345)


def rand(*shape, scale=1.0):
    return RNG.standard_normal(shape) * scale


# ---------------------------------------------------------------- elementary

def test_feature_map_is_softmax_over_head_dim():
    x = rand(5, 3, 64, scale=3.0)
    np.testing.assert_allclose(oracle.feature_map(x), sps.softmax(x, axis=-1), rtol=1e-13, atol=0)
    # shift invariance and a huge input that would overflow a naive exp
    np.testing.assert_allclose(oracle.feature_map(x + 1000.0), sps.softmax(x, axis=-1), rtol=1e-12)


def test_log_gate_is_log_sigmoid_of_mean():
    k = rand(50, 128, scale=2.0) + rand(50, 1, scale=3.0)
    ref = sps.log_expit(k.mean(-1))
    np.testing.assert_allclose(oracle.log_gate(k), ref, rtol=1e-13, atol=1e-300)
    # extreme means: no overflow on either side
    big = np.array([[800.0] * 8, [-800.0] * 8, [0.0] * 8])
    np.testing.assert_allclose(oracle.log_gate(big), sps.log_expit(big.mean(-1)), rtol=1e-13)


# ------------------------------------------------------- reference routes

def phi(x):
    return sps.softmax(x, axis=-1)


def gates(k):
    return sps.expit(k.mean(-1))  # [.., T]


def grm_parallel(q, k, v, gate_on=True, s0=None):
    """Masked parallel form for one head: O = ((phiQ phiK^T) * D) V (+ decay * phiQ S0),
    D[t, s] = prod_{r=s+1..t} g_r for s <= t, else 0.  q, k, v [T, d]."""
    T = q.shape[0]
    pq, pk = phi(q), phi(k)
    g = gates(k) if gate_on else np.ones(T)
    D = np.zeros((T, T))
    for t in range(T):
        for s in range(t + 1):
            D[t, s] = np.prod(g[s + 1:t + 1])
    o = ((pq @ pk.T) * D) @ v
    if s0 is not None:
        o += (np.cumprod(g)[:, None]) * (pq @ s0)
    return o


def final_state_parallel(k, v, gate_on=True, s0=None):
    T = k.shape[0]
    g = gates(k) if gate_on else np.ones(T)
    pk = phi(k)
    w = np.array([np.prod(g[s + 1:]) for s in range(T)])
    S = (pk * w[:, None]).T @ v
    if s0 is not None:
        S += np.prod(g) * s0
    return S


def swa_sdpa(q, k, v, w):
    """Banded causal softmax attention through torch's SDPA (fp64, CPU).  q,k,v [T, d]."""
    T, d = q.shape
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    allowed = (j <= i) & (j > i - w)
    mask = torch.from_numpy(allowed)
    out = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None], torch.from_numpy(k)[None, None],
        torch.from_numpy(v)[None, None], attn_mask=mask[None, None], scale=1.0 / np.sqrt(d))
    return out[0, 0].numpy()


# ---------------------------------------------------------------- pins

@pytest.mark.parametrize("d", [8, 64])
def test_no_gate_equals_quadratic_causal_linear_attention(d):
    """Ablation "no gate" (g = 1) with alpha = 1: o_t = sum_{s<=t} (phi q_t . phi k_s) v_s."""
    T = 40
    q, k, v = rand(1, T, 1, d), rand(1, T, 1, d), rand(1, T, 1, d)
    out, fs, _, _ = oracle.prefill(q, k, v, w=64, alpha=1.0, gate_off=True)
    pq, pk = phi(q[0, :, 0]), phi(k[0, :, 0])
    ref = np.tril(pq @ pk.T) @ v[0, :, 0]
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(fs[0, 0], pk.T @ v[0, :, 0], rtol=1e-11, atol=1e-13)


@pytest.mark.parametrize("T", [1, 2, 7, 16])
def test_gated_recurrence_equals_masked_parallel_form(T):
    d = 16
    q, k, v = rand(1, T, 1, d), rand(1, T, 1, d, scale=2.0), rand(1, T, 1, d)
    out, fs, _, _ = oracle.prefill(q, k, v, w=64, alpha=1.0)
    np.testing.assert_allclose(out[0, :, 0], grm_parallel(q[0, :, 0], k[0, :, 0], v[0, :, 0]),
                               rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], final_state_parallel(k[0, :, 0], v[0, :, 0]),
                               rtol=1e-11, atol=1e-14)


def test_initial_state_enters_with_cumulative_decay():
    T, d = 12, 8
    q, k, v = rand(1, T, 1, d), rand(1, T, 1, d), rand(1, T, 1, d)
    s0 = rand(1, 1, d, d)
    out, fs, _, _ = oracle.prefill(q, k, v, alpha=1.0, initial_state=s0)
    ref = grm_parallel(q[0, :, 0], k[0, :, 0], v[0, :, 0], s0=s0[0, 0])
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(fs[0, 0], final_state_parallel(k[0, :, 0], v[0, :, 0], s0=s0[0, 0]),
                               rtol=1e-11, atol=1e-14)


@pytest.mark.parametrize("T,w", [(30, 64), (64, 64), (100, 64), (50, 7)])
def test_swa_branch_equals_banded_causal_softmax_attention(T, w):
    """alpha = 0 isolates the window branch; with w >= T it is full causal attention."""
    d = 32
    q, k, v = rand(1, T, 1, d, scale=2.0), rand(1, T, 1, d, scale=2.0), rand(1, T, 1, d)
    out, _, _, _ = oracle.prefill(q, k, v, w=w, alpha=0.0)
    np.testing.assert_allclose(out[0, :, 0], swa_sdpa(q[0, :, 0], k[0, :, 0], v[0, :, 0], w),
                               rtol=1e-10, atol=1e-12)
    if w >= T:
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[0, :, 0])[None], torch.from_numpy(k[0, :, 0])[None],
            torch.from_numpy(v[0, :, 0])[None], is_causal=True)[0].numpy()
        np.testing.assert_allclose(out[0, :, 0], ref, rtol=1e-10, atol=1e-12)


def test_mix_is_alpha_grm_plus_one_minus_alpha_swa():
    """alpha = 1 is GRM only (ablation "no SWA"), alpha = 0 is SWA only, and the hybrid
    is their convex combination with beta = 1 - alpha."""
    T, d = 90, 16
    q, k, v = rand(2, T, 2, d), rand(2, T, 1, d), rand(2, T, 1, d)
    o1 = oracle.prefill(q, k, v, alpha=1.0)[0]
    o0 = oracle.prefill(q, k, v, alpha=0.0)[0]
    for a in (0.5, 0.3):
        oa = oracle.prefill(q, k, v, alpha=a)[0]
        np.testing.assert_allclose(oa, a * o1 + (1 - a) * o0, rtol=1e-12, atol=1e-14)
    for b in range(2):
        for h in range(2):
            np.testing.assert_allclose(o1[b, :, h], grm_parallel(q[b, :, h], k[b, :, 0], v[b, :, 0]),
                                       rtol=1e-10, atol=1e-13)
            np.testing.assert_allclose(o0[b, :, h], swa_sdpa(q[b, :, h], k[b, :, 0], v[b, :, 0], 64),
                                       rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kappa,c,alpha", [(0.7, 1.5, 0.5), (-2.0, -0.25, 0.3), (0.0, 3.0, 1.0)])
def test_closed_form_constant_inputs(kappa, c, alpha):
    """q = 0, k = kappa*1, v = c*1: phi q = phi k = 1/d, g = sigmoid(kappa), so
    GRM_t = c (1 - g^(t+1)) / (d (1 - g)) (t counted from 0), SWA_t = c, and
    S_T = (1 - g^T) / (d (1 - g)) * 1 c^T."""
    T, d = 70, 16
    q = np.zeros((1, T, 1, d))
    k = np.full((1, T, 1, d), kappa)
    v = np.full((1, T, 1, d), c)
    out, fs, _, _ = oracle.prefill(q, k, v, alpha=alpha)
    g = 1.0 / (1.0 + np.exp(-kappa))
    t = np.arange(T)
    grm = c * (1 - g ** (t + 1)) / (d * (1 - g))
    ref = alpha * grm + (1 - alpha) * c
    np.testing.assert_allclose(out[0, :, 0], ref[:, None] * np.ones(d), rtol=1e-12)
    np.testing.assert_allclose(fs[0, 0], (1 - g ** T) / (d * (1 - g)) * c * np.ones((d, d)), rtol=1e-12)


def test_linear_in_v():
    T, d = 80, 16
    q, k = rand(1, T, 2, d), rand(1, T, 1, d)
    v1, v2 = rand(1, T, 1, d), rand(1, T, 1, d)
    o1, s1, _, _ = oracle.prefill(q, k, v1)
    o2, s2, _, _ = oracle.prefill(q, k, v2)
    o3, s3, _, _ = oracle.prefill(q, k, 2.0 * v1 - 3.0 * v2)
    np.testing.assert_allclose(o3, 2.0 * o1 - 3.0 * o2, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(s3, 2.0 * s1 - 3.0 * s2, rtol=1e-10, atol=1e-12)


def test_key_shift_moves_only_the_gate():
    """phi(k + c) = phi(k) and the window's scores shift by the same amount for every key,
    so with the gate off a constant key shift changes nothing; with the gate on it does."""
    T, d = 80, 16
    q, k, v = rand(1, T, 2, d), rand(1, T, 1, d), rand(1, T, 1, d)
    a = oracle.prefill(q, k, v, gate_off=True)[0]
    b = oracle.prefill(q, k + 1.75, v, gate_off=True)[0]
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)
    c = oracle.prefill(q, k + 1.75, v)[0]
    assert np.max(np.abs(c - oracle.prefill(q, k, v)[0])) > 1e-4


def test_gqa_equals_mha_with_repeated_kv():
    T, d, Hq, Hkv = 70, 16, 6, 2
    q, k, v = rand(2, T, Hq, d), rand(2, T, Hkv, d), rand(2, T, Hkv, d)
    a, sa, _, _ = oracle.prefill(q, k, v)
    G = Hq // Hkv
    b, sb, _, _ = oracle.prefill(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2))
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=0)
    np.testing.assert_allclose(sa, sb, rtol=1e-13, atol=0)


def test_varlen_equals_separate_runs():
    lens = [5, 70, 1, 33]
    T, d, Hq, Hkv = sum(lens), 16, 4, 2
    q, k, v = rand(1, T, Hq, d), rand(1, T, Hkv, d), rand(1, T, Hkv, d)
    cu = np.concatenate([[0], np.cumsum(lens)])
    s0 = rand(len(lens), Hq, d, d, scale=0.1)
    out, fs, ring, pos = oracle.prefill(q, k, v, w=16, cu_seqlens=cu, initial_state=s0)
    for i, n in enumerate(lens):
        sl = slice(cu[i], cu[i + 1])
        o, s, r, p = oracle.prefill(q[:, sl], k[:, sl], v[:, sl], w=16, initial_state=s0[i:i + 1])
        np.testing.assert_array_equal(out[:, sl], o)
        np.testing.assert_array_equal(fs[i], s[0])
        np.testing.assert_array_equal(ring[i], r[0])
        assert pos[i] == n == p[0]


def test_ring_holds_last_w_tokens_at_position_mod_w():
    T, d, w = 23, 4, 8
    q, k, v = rand(1, T, 2, d), rand(1, T, 2, d), rand(1, T, 2, d)
    _, _, ring, pos = oracle.prefill(q, k, v, w=w)
    assert pos[0] == T
    for p in range(T - w, T):
        np.testing.assert_array_equal(ring[0, :, 0, p % w], k[0, p])
        np.testing.assert_array_equal(ring[0, :, 1, p % w], v[0, p])
    _, _, ring2, _ = oracle.prefill(q[:, :3], k[:, :3], v[:, :3], w=w)
    assert np.all(ring2[0, :, :, 3:] == 0)


@pytest.mark.parametrize("T1,T2,w", [(0, 9, 4), (3, 12, 4), (20, 15, 8)])
def test_prefill_then_decode_equals_longer_prefill(T1, T2, w):
    """Constant-size state: decoding T2 tokens after a T1 prefill reproduces a T1 + T2
    prefill token for token, with the state and the ring as the whole resume point."""
    d, Hq, Hkv, B = 8, 4, 2, 2
    T = T1 + T2
    q, k, v = rand(B, T, Hq, d), rand(B, T, Hkv, d), rand(B, T, Hkv, d)
    full, fs_full, ring_full, _ = oracle.prefill(q, k, v, w=w)
    if T1:
        _, st, rg, ps = oracle.prefill(q[:, :T1], k[:, :T1], v[:, :T1], w=w)
    else:
        st, rg, ps = np.zeros((B, Hq, d, d)), np.zeros((B, Hkv, 2, w, d)), np.zeros(B, np.int32)
    for t in range(T1, T):
        o, st, rg, ps = oracle.decode(q[:, t], k[:, t], v[:, t], st, rg, ps, w=w)
        np.testing.assert_allclose(o, full[:, t], rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(st, fs_full, rtol=1e-11, atol=1e-13)
    np.testing.assert_array_equal(rg, ring_full)
    assert np.all(ps == T)


def test_decode_treats_each_query_head_state_independently():
    """A decode step only reads its own q head's state: perturbing head 1's state leaves
    head 0's output untouched, and its own output moves by exactly phi(q) dS * g."""
    B, Hq, Hkv, d, w = 1, 2, 1, 8, 4
    q, k, v = rand(B, Hq, d), rand(B, Hkv, d), rand(B, Hkv, d)
    st = rand(B, Hq, d, d)
    rg = rand(B, Hkv, 2, w, d)
    ps = np.array([9], np.int32)
    o1 = oracle.decode(q, k, v, st, rg, ps, alpha=1.0)[0]
    dS = rand(d, d)
    st2 = st.copy()
    st2[0, 1] += dS
    o2 = oracle.decode(q, k, v, st2, rg, ps, alpha=1.0)[0]
    np.testing.assert_array_equal(o1[0, 0], o2[0, 0])
    g = sps.expit(k[0, 0].mean())
    np.testing.assert_allclose(o2[0, 1] - o1[0, 1], g * (phi(q[0, 1]) @ dS), rtol=1e-9, atol=1e-12)


def test_oracle_rejects_bad_arguments():
    q, k, v = rand(1, 4, 3, 8), rand(1, 4, 2, 8), rand(1, 4, 2, 8)
    with pytest.raises(ValueError):
        oracle.prefill(q, k, v)  # Hq % Hkv != 0
    q = rand(2, 4, 2, 8)
    with pytest.raises(ValueError):
        oracle.prefill(q, rand(2, 4, 2, 8), rand(2, 4, 2, 8), cu_seqlens=[0, 4])  # B != 1


def test_golden_small_case():
    """Stored oracle output on a small case (written by tests/golden/make_golden.py)."""
    import json
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "oracle_small.json")
    with open(path) as f:
        g = json.load(f)
    out, fs, _, pos = oracle.prefill(np.array(g["q"]), np.array(g["k"]), np.array(g["v"]),
                                     w=g["shape"]["w"], alpha=g["shape"]["alpha"])
    np.testing.assert_allclose(out, np.array(g["out"]), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(fs, np.array(g["final_state"]), rtol=1e-12, atol=1e-15)
    assert pos.tolist() == g["pos"]


def test_decode_inplace_steps_equal_a_longer_prefill():
    """The in-place decode front end (no copies; used for long full-size runs) continues a prefill
    exactly as a longer prefill does, and updates its arrays in place."""
    B, Hq, Hkv, T1, T2, d, w = 2, 4, 2, 9, 5, 8, 4
    q, k, v = rand(B, T1 + T2, Hq, d), rand(B, T1 + T2, Hkv, d), rand(B, T1 + T2, Hkv, d)
    full, fs_full, ring_full, pos_full = oracle.prefill(q, k, v, w=w)
    _, st, rg, ps = oracle.prefill(q[:, :T1], k[:, :T1], v[:, :T1], w=w)
    st, rg, ps = np.ascontiguousarray(st), np.ascontiguousarray(rg), np.ascontiguousarray(ps.astype(np.int32))
    ids = (id(st), id(rg), id(ps))
    for t in range(T1, T1 + T2):
        o = oracle.decode_inplace(q[:, t], k[:, t], v[:, t], st, rg, ps)
        np.testing.assert_allclose(o, full[:, t], rtol=1e-12, atol=1e-14)
    assert (id(st), id(rg), id(ps)) == ids
    np.testing.assert_allclose(st, fs_full, rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(rg, ring_full)
    np.testing.assert_array_equal(ps, pos_full)
    with pytest.raises(ValueError):
        oracle.decode_inplace(q[:, 0], k[:, 0], v[:, 0], st.astype(np.float32), rg, ps)


def test_causal_attention_rows_equal_the_window_branch_and_sdpa():
    """The row-wise causal attention reference equals the C oracle's window branch with a window
    covering the sequence and alpha = 0, and torch's causal scaled_dot_product_attention (fp64);
    with packed sequences each row sees only its own sequence."""
    import torch
    B, T, Hq, Hkv, d = 2, 13, 4, 2, 8
    q, k, v = rand(B, T, Hq, d), rand(B, T, Hkv, d), rand(B, T, Hkv, d)
    rows = [(b, t, h) for b in range(B) for t in range(T) for h in range(Hq)]
    got = oracle.causal_attention_rows(q, k, v, rows)
    ref = oracle.prefill(q, k, v, w=T, alpha=0.0)[0]
    np.testing.assert_allclose(got, np.array([ref[b, t, h] for b, t, h in rows]), rtol=1e-12, atol=1e-13)
    G = Hq // Hkv
    qt = torch.tensor(q).permute(0, 2, 1, 3)
    kt = torch.tensor(np.repeat(k, G, axis=2)).permute(0, 2, 1, 3)
    vt = torch.tensor(np.repeat(v, G, axis=2)).permute(0, 2, 1, 3)
    sd = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True).permute(0, 2, 1, 3).numpy()
    np.testing.assert_allclose(got, np.array([sd[b, t, h] for b, t, h in rows]), rtol=1e-10, atol=1e-12)
    cu = [0, 5, 5, 13]
    q1, k1, v1 = q[:1], k[:1], v[:1]
    rows1 = [(0, t, h) for t in range(T) for h in range(Hq)]
    got1 = oracle.causal_attention_rows(q1, k1, v1, rows1, cu_seqlens=cu)
    for a, b_ in ((0, 5), (5, 13)):
        sep = oracle.causal_attention_rows(q1[:, a:b_], k1[:, a:b_], v1[:, a:b_],
                                           [(0, t, h) for t in range(b_ - a) for h in range(Hq)])
        np.testing.assert_allclose(got1[a * Hq:b_ * Hq], sep, rtol=1e-13, atol=1e-14)


# ---------------------------------------------------------------- per-dimension gate

def _sig(x):
    return 1.0 / (1.0 + np.exp(-x))


def _phi(x):
    e = np.exp(x - x.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def test_vector_gate_equals_scalar_gate_for_uniform_keys():
    """When every element of a key is the same value, its mean is that value: the per-dimension
    gate and the pooled scalar gate coincide."""
    B, T, Hq, Hkv, d = 1, 9, 2, 1, 6
    q, v = rand(B, T, Hq, d), rand(B, T, Hkv, d)
    k = np.repeat(rand(B, T, Hkv, 1), d, axis=-1)
    a = oracle.prefill(q, k, v, w=4, vector_gate=True)
    b = oracle.prefill(q, k, v, w=4)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(a[1], b[1], rtol=1e-12, atol=1e-14)


def test_vector_gate_equals_masked_parallel_form():
    """alpha = 1: o_t = sum_{s<=t} sum_r phi q_t[r] (prod_{u=s+1..t} g_u[r]) phi k_s[r] v_s, the gate
    acting on the key dimension r; the final state is sum_s (prod_{u>s} g_u[r]) phi k_s[r] v_s[c]
    plus the decayed initial state.  (A gate applied to the value dimension fails both.)"""
    T, d = 7, 5
    q, k, v = rand(1, T, 1, d), rand(1, T, 1, d), rand(1, T, 1, d)
    s0 = rand(1, 1, d, d, scale=0.3)
    out, fs, _, _ = oracle.prefill(q, k, v, w=3, alpha=1.0, vector_gate=True, initial_state=s0)
    pq, pk, g = _phi(q[0, :, 0]), _phi(k[0, :, 0]), _sig(k[0, :, 0])
    for t in range(T):
        ref = np.zeros(d)
        for s in range(t + 1):
            dec = np.prod(g[s + 1:t + 1], axis=0)                       # [d] over the key dim
            ref += (pq[t] * dec * pk[s]).sum() * v[0, s, 0]
        ref += (pq[t] * np.prod(g[:t + 1], axis=0)) @ s0[0, 0]
        np.testing.assert_allclose(out[0, t, 0], ref, rtol=1e-11, atol=1e-13)
    ref_s = np.prod(g, axis=0)[:, None] * s0[0, 0]
    for s in range(T):
        ref_s += np.outer(np.prod(g[s + 1:], axis=0) * pk[s], v[0, s, 0])
    np.testing.assert_allclose(fs[0, 0], ref_s, rtol=1e-11, atol=1e-13)


def test_vector_gate_decode_continues_prefill():
    B, Hq, Hkv, T1, T2, d, w = 2, 4, 2, 8, 4, 8, 4
    q, k, v = rand(B, T1 + T2, Hq, d), rand(B, T1 + T2, Hkv, d), rand(B, T1 + T2, Hkv, d)
    full = oracle.prefill(q, k, v, w=w, vector_gate=True)
    _, st, rg, ps = oracle.prefill(q[:, :T1], k[:, :T1], v[:, :T1], w=w, vector_gate=True)
    for t in range(T1, T1 + T2):
        o, st, rg, ps = oracle.decode(q[:, t], k[:, t], v[:, t], st, rg, ps, vector_gate=True)
        np.testing.assert_allclose(o, full[0][:, t], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(st, full[1], rtol=1e-12, atol=1e-14)
