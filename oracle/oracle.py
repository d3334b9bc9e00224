"""Python front end of the fp64 CPU oracle (``oracle.c``): the prefill, its gradient, and
the decode step.

TEST INFRASTRUCTURE ONLY: the test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  The product path never imports this
module.  It shares no code with the CUDA library.

``build()`` compiles ``oracle.c`` with gcc into ``liboracle.so`` beside it (on
demand, when the library is missing or older than its source).  The functions
take numpy arrays of any float dtype, widen them to float64 (exact for bf16
and fp32 values) and return float64 results.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile the oracle with gcc if needed; return the library path."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off", "-pthread", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.oracle_prefill.restype = ctypes.c_int
            lib.oracle_prefill.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, _dp, _ip, ctypes.c_int, _dp, _dp, _dp, _ip,
                ctypes.c_int, ctypes.c_int]
            lib.oracle_decode.restype = ctypes.c_int
            lib.oracle_decode.argtypes = [
                _dp, _dp, _dp, _dp, _dp, _dp, _ip, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int]
            lib.oracle_prefill_backward.restype = ctypes.c_int
            lib.oracle_prefill_backward.argtypes = [
                _dp, _dp, _dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                ctypes.c_int, ctypes.c_double, _dp, _ip, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp,
                ctypes.c_int, ctypes.c_int]
            lib.oracle_feature_map.restype = None
            lib.oracle_feature_map.argtypes = [_dp, ctypes.c_int, _dp]
            lib.oracle_log_gate.restype = ctypes.c_double
            lib.oracle_log_gate.argtypes = [_dp, ctypes.c_int]
            _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a, t=_dp):
    return None if a is None else a.ctypes.data_as(t)


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def feature_map(x):
    """Softmax over the last axis, row by row, through the oracle's C routine."""
    lib = _load()
    x = _f64(x)
    d = x.shape[-1]
    flat = x.reshape(-1, d)
    y = np.empty_like(flat)
    for i in range(flat.shape[0]):
        row = np.ascontiguousarray(flat[i])
        out = np.empty(d)
        lib.oracle_feature_map(_ptr(row), d, _ptr(out))
        y[i] = out
    return y.reshape(x.shape)


def log_gate(k):
    """log sigmoid(mean over the last axis), row by row, through the C routine."""
    lib = _load()
    k = _f64(k)
    d = k.shape[-1]
    flat = k.reshape(-1, d)
    res = np.array([lib.oracle_log_gate(_ptr(np.ascontiguousarray(r)), d) for r in flat])
    return res.reshape(k.shape[:-1])


def _gate_mode(gate_off, vector_gate):
    if gate_off and vector_gate:
        raise ValueError("gate_off and vector_gate exclude each other")
    return 1 if gate_off else (2 if vector_gate else 0)


def prefill(q, k, v, w=64, alpha=0.5, initial_state=None, cu_seqlens=None, gate_off=False,
            nthreads=None, vector_gate=False):
    """Token-by-token prefill.  Returns (out, final_state, ring, pos).

    vector_gate: one gate per key dimension, sigmoid(k_t[r]) scaling row r of the state
    (the per-dimension form of the pooled key gate), instead of sigmoid(mean_d k_t).

    q [B, T, Hq, d]; k, v [B, T, Hkv, d]; cu_seqlens (optional, B == 1) lists
    n_seqs + 1 offsets into T.  out [B, T, Hq, d], final_state [n, Hq, d, d],
    ring [n, Hkv, 2, w, d], pos [n] int32.
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != (B, T, Hkv, d):
        raise ValueError("prefill: inconsistent shapes")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n = cu.shape[0] - 1
    else:
        cu = None
        n = B
    s0 = None if initial_state is None else _f64(initial_state)
    if s0 is not None and s0.shape != (n, Hq, d, d):
        raise ValueError("prefill: initial_state must be [n, Hq, d, d]")
    out = np.zeros_like(q)
    fs = np.zeros((n, Hq, d, d))
    ring = np.zeros((n, Hkv, 2, w, d))
    pos = np.zeros(n, dtype=np.int32)
    rc = lib.oracle_prefill(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, T, d, w, float(alpha), _ptr(s0),
        _ptr(cu, _ip), n, _ptr(out), _ptr(fs), _ptr(ring), _ptr(pos, _ip), _gate_mode(gate_off, vector_gate),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return out, fs, ring, pos


def prefill_backward(q, k, v, d_out, w=64, alpha=0.5, initial_state=None, cu_seqlens=None,
                     d_final_state=None, gate_off=False, nthreads=None):
    """Gradients of L = sum(d_out * out) + sum(d_final_state * final_state) of the prefill.

    Returns (dq, dk, dv, d_initial_state) with the shapes of q, k, v and [n, Hq, d, d]; the
    last is the gradient with respect to the initial state (a zero state when none is given).
    Arguments as in ``prefill``; d_out has the shape of out, d_final_state [n, Hq, d, d] or None.
    """
    lib = _load()
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(d_out)
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    if k.shape != (B, T, Hkv, d) or v.shape != (B, T, Hkv, d) or dout.shape != q.shape:
        raise ValueError("prefill_backward: inconsistent shapes")
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        n = cu.shape[0] - 1
    else:
        cu = None
        n = B
    s0 = None if initial_state is None else _f64(initial_state)
    dfs = None if d_final_state is None else _f64(d_final_state)
    for name, a in (("initial_state", s0), ("d_final_state", dfs)):
        if a is not None and a.shape != (n, Hq, d, d):
            raise ValueError(f"prefill_backward: {name} must be [n, Hq, d, d]")
    dq = np.empty_like(q)
    dk = np.empty_like(k)
    dv = np.empty_like(v)
    ds0 = np.zeros((n, Hq, d, d))
    rc = lib.oracle_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), B, Hq, Hkv, T, d, w, float(alpha), _ptr(s0), _ptr(cu, _ip), n,
        _ptr(dout), _ptr(dfs), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds0), int(bool(gate_off)),
        nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_prefill_backward rejected its arguments")
    return dq, dk, dv, ds0


def decode_inplace(q, k, v, state, ring, pos, alpha=0.5, gate_off=False, nthreads=None, vector_gate=False):
    """One decode step that updates state, ring and pos in place and returns out.

    state [B, Hq, d, d] and ring [B, Hkv, 2, w, d] must be C-contiguous float64 arrays and pos a
    C-contiguous int32 array [B] (they are handed to the C routine as they are, with no copy:
    for long runs at large B, where copying the state every step would dominate).
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    for name, a, dt in (("state", state, np.float64), ("ring", ring, np.float64), ("pos", pos, np.int32)):
        if not isinstance(a, np.ndarray) or a.dtype != dt or not a.flags["C_CONTIGUOUS"]:
            raise ValueError(f"decode_inplace: {name} must be a C-contiguous {np.dtype(dt).name} array")
    w = ring.shape[3]
    if k.shape != (B, Hkv, d) or v.shape != (B, Hkv, d) or state.shape != (B, Hq, d, d) \
            or ring.shape != (B, Hkv, 2, w, d) or pos.shape != (B,):
        raise ValueError("decode_inplace: inconsistent shapes")
    out = np.zeros_like(q)
    rc = lib.oracle_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(ring), _ptr(out), _ptr(pos, _ip), B, Hq, Hkv, d, w,
        float(alpha), _gate_mode(gate_off, vector_gate), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return out


def decode(q, k, v, state, ring, pos, w=None, alpha=0.5, gate_off=False, nthreads=None, vector_gate=False):
    """One decode step.  Returns (out, new_state, new_ring, new_pos); inputs are not modified.

    q [B, Hq, d]; k, v [B, Hkv, d]; state [B, Hq, d, d]; ring [B, Hkv, 2, w, d]; pos [B].
    The window w is the ring's slot count (a w argument, if given, must agree).
    """
    lib = _load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    st = _f64(state).copy()
    rg = _f64(ring).copy()
    if w is not None and w != rg.shape[3]:
        raise ValueError(f"w={w} but the ring has {rg.shape[3]} slots")
    w = rg.shape[3]
    if k.shape != (B, Hkv, d) or v.shape != (B, Hkv, d) or st.shape != (B, Hq, d, d) \
            or rg.shape != (B, Hkv, 2, w, d) or np.asarray(pos).shape != (B,):
        raise ValueError("decode: inconsistent shapes")
    ps = np.ascontiguousarray(np.asarray(pos, dtype=np.int32)).copy()
    out = np.zeros_like(q)
    rc = lib.oracle_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(st), _ptr(rg), _ptr(out), _ptr(ps, _ip), B, Hq, Hkv, d, w,
        float(alpha), _gate_mode(gate_off, vector_gate), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return out, st, rg, ps


def causal_attention_rows(q, k, v, rows, cu_seqlens=None):
    """Causal softmax attention o_t = sum_{j <= t} softmax_j(q_t . k_j / sqrt(d)) v_j, written out
    row by row for the requested rows only (numpy, float64); the sequence containing each row
    bounds its keys.

    q [B, T, Hq, d]; k, v [B, T, Hkv, d]; rows: iterable of (b, t, h).  Returns [len(rows), d].
    This is the standard attention layer of the inter-layer hybrid (news article on Liger, section
    ハイブリッドメカニズム: one full softmax attention layer after every seven Liger layers); it is
    also the window branch with a window covering the whole sequence.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, T, Hq, d = q.shape
    G = Hq // k.shape[2]
    starts = None if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    res = np.empty((len(rows), d))
    for n, (b, t, h) in enumerate(rows):
        t0 = 0 if starts is None else int(starts[np.searchsorted(starts, t, side="right") - 1])
        kv = h // G
        s = k[b, t0:t + 1, kv] @ q[b, t, h] / np.sqrt(d)
        p = np.exp(s - s.max())
        res[n] = (p / p.sum()) @ v[b, t0:t + 1, kv]
    return res
