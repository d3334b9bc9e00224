"""The chunk-level backward equations of the gated recurrent branch, checked against the
oracle's gradient (CPU only).

The backward kernels are to work chunk by chunk, like the forward: within a chunk of n tokens
with running log-gate sums b_0..b_{n-1} (b_C = b_{n-1}), entering state S and the gradient
dS' of the state the chunk hands on,

  A_ij    = e^{b_i - b_j} (phi q_i . phi k_j)              (j <= i)
  out_i   = alpha (e^{b_i} phi q_i S + sum_j A_ij v_j)
  S'      = e^{b_C} S + sum_j e^{b_C - b_j} phi k_j^T v_j

so that, with G = alpha dO V^T masked to j <= i and E the masked decay matrix,

  d phi q = alpha e^{b} (dO S^T) + (G * E) phi K
  d phi k = (G * E)^T phi Q + e^{b_C - b} (V dS'^T)
  dV      = A^T (alpha dO) + e^{b_C - b} (phi K dS')
  dS      = e^{b_C} dS' + (e^{b} phi Q)^T (alpha dO)
  d b_i   = alpha e^{b_i} (phi q_i S . dO_i) + sum_j A_ij G_ij - sum_i' A_i'i G_i'i
            - e^{b_C - b_i} (phi k_i dS' . v_i) + [i = n-1] <dS', S'>

and d log g_t is the sum of d b_i over i >= t in the chunk; the gate then gives
dk_t += d log g_t sigmoid(-m_t) / d.  The window branch's backward is the band-masked
softmax attention backward.  This model evaluates those equations in numpy for one head, in
the three passes planned for the kernels (states entering the chunks; their gradients from the
last chunk back; then every chunk on its own, in shuffled order), and must reproduce the
oracle's token-by-token gradient.
"""
import numpy as np
import pytest

from oracle import oracle


def softmax_rows(x):
    e = np.exp(x - x.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def log_sigmoid(m):
    return np.where(m >= 0, -np.log1p(np.exp(-np.abs(m))), m - np.log1p(np.exp(-np.abs(m))))


def chunked_backward(q, k, v, s0, dout, dfs, w, alpha, C, order_seed=None):
    """One head, one sequence: q, k, v, dout [T, d]; s0, dfs [d, d].  Returns dq, dk, dv, ds0.

    Three passes: (1) h_c, the state entering each chunk; (2) dh_c, the gradient of the state
    entering each chunk, from the last chunk back; (3) each chunk's gradients from h_c and
    dh_{c+1} alone, in any order (order_seed shuffles it)."""
    T, d = q.shape
    beta = 1.0 - alpha
    pq, pk = softmax_rows(q), softmax_rows(k)
    m = k.mean(axis=1)
    lg = log_sigmoid(m)
    starts = list(range(0, T, C))
    spans = [slice(c0, min(c0 + C, T)) for c0 in starts]
    bs = [np.cumsum(lg[sl]) for sl in spans]
    # pass 1: h[c] enters chunk c, h[len] is the final state
    h = [s0]
    for sl, b in zip(spans, bs):
        h.append(np.exp(b[-1]) * h[-1] + (np.exp(b[-1] - b)[:, None] * pk[sl]).T @ v[sl])
    # pass 2: dh[c] is the gradient of h[c]; it needs only e^{b_C} and (e^{b} phi Q)^T (alpha dO)
    dh = [None] * len(spans) + [dfs]
    for ci in range(len(spans) - 1, -1, -1):
        sl, b = spans[ci], bs[ci]
        dh[ci] = np.exp(b[-1]) * dh[ci + 1] + (np.exp(b)[:, None] * pq[sl]).T @ (alpha * dout[sl])
    # pass 3: per chunk, independent of the others
    dpq, dpk = np.zeros_like(q), np.zeros_like(k)
    dv = np.zeros_like(v)
    dlg = np.zeros(T)
    order = list(range(len(spans)))
    if order_seed is not None:
        np.random.default_rng(order_seed).shuffle(order)
    for ci in order:
        sl, b = spans[ci], bs[ci]
        n = b.shape[0]
        S, Sn, dS = h[ci], h[ci + 1], dh[ci + 1]
        bC = b[-1]
        Pq, Pk, V, dO = pq[sl], pk[sl], v[sl], alpha * dout[sl]
        mask = np.tril(np.ones((n, n), dtype=bool))
        E = np.where(mask, np.exp(np.where(mask, b[:, None] - b[None, :], 0.0)), 0.0)
        A = E * (Pq @ Pk.T)
        G = np.where(mask, dO @ V.T, 0.0)
        eb, ekey = np.exp(b), np.exp(bC - b)
        dpq[sl] = eb[:, None] * (dO @ S.T) + (G * E) @ Pk
        dpk[sl] = (G * E).T @ Pq + ekey[:, None] * (V @ dS.T)
        dv[sl] += A.T @ dO + ekey[:, None] * (Pk @ dS)
        db = (eb * np.sum((Pq @ S) * dO, axis=1) + np.sum(A * G, axis=1) - np.sum(A * G, axis=0)
              - ekey * np.sum((Pk @ dS) * V, axis=1))
        db[-1] += np.sum(dS * Sn)
        dlg[sl] = np.cumsum(db[::-1])[::-1]
    dq = pq * (dpq - np.sum(dpq * pq, axis=1, keepdims=True))
    dk = pk * (dpk - np.sum(dpk * pk, axis=1, keepdims=True))
    dk += (dlg * np.exp(log_sigmoid(-m)) / d)[:, None]
    # window branch: band-masked softmax attention backward
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    band = (j <= i) & (j > i - w)
    s = np.where(band, q @ k.T / np.sqrt(d), -np.inf)
    P = softmax_rows(s)
    dOs = beta * dout
    dP = dOs @ v.T
    dsc = P * (dP - np.sum(dP * P, axis=1, keepdims=True)) / np.sqrt(d)
    dq += dsc @ k
    dk += dsc.T @ q
    dv += P.T @ dOs
    return dq, dk, dv, dh[0]


@pytest.mark.parametrize("T,C,w,alpha,kb", [(23, 4, 5, 0.5, 0.0), (16, 8, 3, 0.8, 0.0),
                                            (19, 4, 64, 0.3, 2.5), (9, 16, 4, 1.0, 0.0)])
def test_chunk_equations_reproduce_the_oracle_gradient(T, C, w, alpha, kb):
    rng = np.random.default_rng(T * 7 + C)
    d = 5
    q = rng.normal(size=(T, d))
    k = rng.normal(size=(T, d)) + kb * np.where(np.arange(T) % 3 == 0, 1.0, -1.0)[:, None]
    v = rng.normal(size=(T, d))
    s0 = 0.3 * rng.normal(size=(d, d))
    dout = rng.normal(size=(T, d))
    dfs = rng.normal(size=(d, d))
    got = chunked_backward(q, k, v, s0, dout, dfs, w, alpha, C, order_seed=T)
    ref = oracle.prefill_backward(q[None, :, None], k[None, :, None], v[None, :, None], dout[None, :, None],
                                  w=w, alpha=alpha, initial_state=s0[None, None], d_final_state=dfs[None, None])
    for name, a, r in zip(("dq", "dk", "dv", "d_initial_state"), got,
                          (ref[0][0, :, 0], ref[1][0, :, 0], ref[2][0, :, 0], ref[3][0, 0])):
        np.testing.assert_allclose(a, r, rtol=1e-9, atol=1e-11, err_msg=name)
