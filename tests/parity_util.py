"""Helpers for GPU-vs-oracle parity tests: tolerances, comparison, sampled
oracle runs at full sizes.  Test infrastructure; the oracle is called here only."""
from __future__ import annotations

import numpy as np
import torch

from oracle import oracle

# Tolerances: bf16 inputs max-abs 2e-2 and relative L2 5e-3; fp32 inputs 1e-4 for both.
TOL = {torch.bfloat16: (2e-2, 5e-3), torch.float32: (1e-4, 1e-4)}


def errors(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in the CUDA result"
    diff = got - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    den = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def assert_close(got, ref, dtype, what=""):
    max_abs, rel = errors(got, ref)
    tol_abs, tol_rel = TOL[dtype]
    assert max_abs <= tol_abs and rel <= tol_rel, \
        f"{what}: max-abs {max_abs:.3e} (tol {tol_abs}), rel-L2 {rel:.3e} (tol {tol_rel})"
    return max_abs, rel


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_group(q, k, v, b, kv, G, w=64, alpha=0.5, cu=None, s0=None):
    """Oracle over one (batch row, kv head) group: q heads kv*G .. kv*G+G-1.
    q, k, v are CPU torch tensors [B, T, H, d]."""
    hs = slice(kv * G, (kv + 1) * G)
    qs = np64(q[b:b + 1, :, hs])
    ks = np64(k[b:b + 1, :, kv:kv + 1])
    vs = np64(v[b:b + 1, :, kv:kv + 1])
    s0s = None if s0 is None else np64(s0[:, hs]) if cu is not None else np64(s0[b:b + 1, hs])
    return oracle.prefill(qs, ks, vs, w=w, alpha=alpha, cu_seqlens=cu, initial_state=s0s)
