"""ctypes binding of ``libliger_attn.so`` (C ABI in ``include/liger_attn.h``).

Argument marshalling only: every step of the forward pass runs in the CUDA
library.  PyTorch supplies device memory and streams.  The library is loaded
on first use; if it is missing this raises (there is no CPU fallback).
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libliger_attn.so")

LIGER_OK, LIGER_ERR_INVALID_ARG, LIGER_ERR_UNSUPPORTED, LIGER_ERR_CUDA, LIGER_ERR_TIMEOUT = range(5)
LIGER_BF16, LIGER_FP32 = 0, 1
STATUS_NAMES = {0: "LIGER_OK", 1: "LIGER_ERR_INVALID_ARG", 2: "LIGER_ERR_UNSUPPORTED",
                3: "LIGER_ERR_CUDA", 4: "LIGER_ERR_TIMEOUT"}

_vp = ctypes.c_void_p
_i = ctypes.c_int
_lock = threading.Lock()
_lib = None

# Entry points and their C signatures (restype, argtypes), as declared in the header.
SIGNATURES = {
    "liger_abi_version": (_i, []),
    "liger_last_error": (ctypes.c_char_p, []),
    "liger_attn_prefill_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i]),
    "liger_attn_prefill": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float, _i,
                                _vp, _vp, _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "liger_attn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float,
                               _i, _vp]),
    "liger_attn_decode_kvshared": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float,
                                        _i, _vp]),
    "liger_attn_prefill_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                                        _i, _vp, _vp, _i, _vp, _vp, _vp]),
    "liger_attn_prefill_status": (_i, [_vp, ctypes.c_size_t]),
    "liger_attn_prefill_noalloc_status": (_i, []),
    "liger_attn_prefill_plan": (_i, [_i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i),
                                     ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(ctypes.c_size_t)]),
    "liger_attn_prefill_backward_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i]),
    "liger_attn_prefill_backward": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float, _i,
                                         _vp, _i, _vp, _vp, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "liger_attn_prefill_vector_gate_workspace_size": (ctypes.c_size_t, [_i, _i, _i, _i, _i, _i, _i]),
    "liger_attn_prefill_vector_gate": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, ctypes.c_float,
                                            _i, _vp, _vp, _i, _vp, _vp, _vp, ctypes.c_size_t, _vp]),
    "liger_attn_decode_vector_gate": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_float,
                                           _i, _vp]),
    "liger_attn_full_causal": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _i, _i, _vp]),
    "liger_attn_full_causal_status": (_i, []),
    "liger_attn_decode_status": (_i, []),
    "liger_set_timing_events": (None, [_vp, _vp]),
    "liger_kernel_launches": (ctypes.c_uint64, []),
}


class LigerError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def load(path: Optional[str] = None):
    """Load the CUDA library (raises FileNotFoundError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            p = path or LIB_PATH
            if not os.path.exists(p):
                raise FileNotFoundError(
                    f"{p} is missing: build it with `python -m gated_linear_attention_liger_b200.build`"
                    " (the Liger Attention ops have no CPU fallback)")
            lib = ctypes.CDLL(p)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def set_timing_events(start=None, stop=None):
    """Bracket the dominant kernel of later calls (this thread) with two torch.cuda.Events."""
    load().liger_set_timing_events(None if start is None else ctypes.c_void_p(start.cuda_event),
                                   None if stop is None else ctypes.c_void_p(stop.cuda_event))


def kernel_launches() -> int:
    """Kernels this thread has launched through the library so far."""
    return int(load().liger_kernel_launches())


def last_error() -> str:
    return load().liger_last_error().decode()


def _check(status: int):
    if status != LIGER_OK:
        raise LigerError(status, last_error())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LIGER_BF16
    if t.dtype == torch.float32:
        return LIGER_FP32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or fp32)")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    ref = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if ref is None:
            ref = t.device
        elif t.device != ref:
            raise ValueError(f"tensors must be on one device ({ref} and {t.device})")


def _expect(t, name, shape, dtype):
    """The library sees only pointers: shapes and dtypes are checked here, so that a wrong
    output buffer is an error instead of an out-of-bounds write."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def prefill_workspace_size(B, Hq, Hkv, T, d, n_seqs, dtype=torch.bfloat16) -> int:
    return int(load().liger_attn_prefill_workspace_size(
        B, Hq, Hkv, T, d, n_seqs, LIGER_BF16 if dtype == torch.bfloat16 else LIGER_FP32))


def prefill_plan(B, Hq, Hkv, T, d, n_seqs=None, packed: bool = False) -> dict:
    """The tensor-core prefill's launch plan for these sizes (host only; see the header)."""
    lib = load()
    vals = [_i(), _i(), _i(), _i()]
    nbytes = ctypes.c_size_t()
    n = B if n_seqs is None else n_seqs
    st = lib.liger_attn_prefill_plan(B, Hq, Hkv, T, d, n, int(bool(packed)), *(ctypes.byref(x) for x in vals),
                                     ctypes.byref(nbytes))
    _check(st)
    return {"chunks_per_segment": vals[0].value, "max_segments": vals[1].value,
            "state_subsegments": vals[2].value, "sm_count": vals[3].value, "plan_bytes": nbytes.value}


def prefill(q, k, v, alpha: float = 0.5, w: int = 64, initial_state=None, cu_seqlens=None,
            return_ring: bool = False, out=None, final_state=None, ring=None, pos=None,
            workspace=None, want_final_state: bool = True, stream=None):
    """Liger Attention prefill.

    q [B, T, Hq, d], k and v [B, T, Hkv, d] (bf16 or fp32, CUDA).  Returns
    (out, final_state) or, with return_ring, (out, final_state, ring, pos).
    cu_seqlens: int32 CUDA tensor of n+1 offsets (B must be 1).
    """
    lib = load()
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, T, Hq, d] and k, v [B, T, Hkv, d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _expect(k, "k", (B, T, Hkv, d), q.dtype)
    _expect(v, "v", (B, T, Hkv, d), q.dtype)
    if cu_seqlens is not None and (cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2
                                   or cu_seqlens.dtype != torch.int32):
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of n + 1 offsets")
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    _expect(initial_state, "initial_state", (n, Hq, d, d), torch.float32)
    _expect(out, "out", (B, T, Hq, d), q.dtype)
    _expect(final_state, "final_state", (n, Hq, d, d), torch.float32)
    _expect(ring, "ring", (n, Hkv, 2, w, d), q.dtype)
    _expect(pos, "pos", (n,), torch.int32)
    _need_cuda(q, k, v, initial_state, cu_seqlens, out, final_state, ring, pos, workspace)
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if final_state is None and want_final_state:
        final_state = torch.empty(n, Hq, d, d, device=dev, dtype=torch.float32)
    if return_ring:
        if ring is None:
            ring = torch.empty(n, Hkv, 2, w, d, device=dev, dtype=q.dtype)
        if pos is None:
            pos = torch.empty(n, device=dev, dtype=torch.int32)
    need = prefill_workspace_size(B, Hq, Hkv, T, d, n, q.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.liger_attn_prefill(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(final_state), B, Hq, Hkv, T, d, w,
        float(alpha), _dt(q), _ptr(initial_state), _ptr(cu_seqlens), n, _ptr(ring), _ptr(pos),
        _ptr(workspace), ws_bytes, _stream_ptr(stream))
    _check(st)
    if return_ring:
        return out, final_state, ring, pos
    return out, final_state


def _check_decode(q, k, v, state, ring, pos, out, per_head: bool):
    if q.dim() != 3 or k.dim() != 3 or ring.dim() != 5:
        raise ValueError("q must be [B, Hq, d], k and v [B, Hkv, d], ring [B, Hkv, 2, w, d]")
    B, Hq, d = q.shape
    Hkv = k.shape[1]
    w = ring.shape[3]
    _expect(k, "k", (B, Hkv, d), q.dtype)
    _expect(v, "v", (B, Hkv, d), q.dtype)
    _expect(state, "state", (B, Hq if per_head else Hkv, d, d), torch.float32)
    _expect(ring, "ring", (B, Hkv, 2, w, d), q.dtype)
    _expect(pos, "pos", (B,), torch.int32)
    _expect(out, "out", (B, Hq, d), q.dtype)
    _need_cuda(q, k, v, state, ring, pos, out)
    return B, Hq, Hkv, d, w


def decode(q, k, v, state, ring, pos, alpha: float = 0.5, out=None, stream=None):
    """One Liger Attention decode step; updates state, ring and pos in place.

    q [B, Hq, d], k and v [B, Hkv, d]; state [B, Hq, d, d] fp32; ring
    [B, Hkv, 2, w, d]; pos [B] int32.  Returns out [B, Hq, d].
    """
    lib = load()
    B, Hq, Hkv, d, w = _check_decode(q, k, v, state, ring, pos, out, per_head=True)
    if out is None:
        out = torch.empty_like(q)
    st = lib.liger_attn_decode(
        _ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(ring), _ptr(out), _ptr(pos), B, Hq, Hkv, d, w,
        float(alpha), _dt(q), _stream_ptr(stream))
    _check(st)
    return out


def decode_kvshared(q, k, v, state, ring, pos, alpha: float = 0.5, out=None, stream=None):
    """One decode step over one state per (sequence, kv head): state [B, Hkv, d, d] fp32.

    Equivalent to `decode` when the per-head states of each group are equal (as
    prefill leaves them); moves G = Hq/Hkv times less state per step.
    """
    lib = load()
    B, Hq, Hkv, d, w = _check_decode(q, k, v, state, ring, pos, out, per_head=False)
    if out is None:
        out = torch.empty_like(q)
    st = lib.liger_attn_decode_kvshared(
        _ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(ring), _ptr(out), _ptr(pos), B, Hq, Hkv, d, w,
        float(alpha), _dt(q), _stream_ptr(stream))
    _check(st)
    return out


def prefill_status(workspace) -> int:
    """LIGER_OK, or LIGER_ERR_TIMEOUT if the last prefill on this workspace gave up waiting
    (call after its stream has completed)."""
    if workspace is None:
        return LIGER_OK
    return int(load().liger_attn_prefill_status(_ptr(workspace), workspace.numel() * workspace.element_size()))


def full_causal_attention(q, k, v, cu_seqlens=None, max_seqlen=None, out=None, stream=None):
    """Causal softmax attention (the hybrid's standard attention layer), bf16.

    q [B, T, Hq, d], k and v [B, T, Hkv, d]; cu_seqlens as for `prefill` (B must be 1), with
    max_seqlen the longest sequence (computed from cu_seqlens when not given, which reads it
    back to the host).  Returns out [B, T, Hq, d].
    """
    lib = load()
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, T, Hq, d] and k, v [B, T, Hkv, d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _expect(k, "k", (B, T, Hkv, d), q.dtype)
    _expect(v, "v", (B, T, Hkv, d), q.dtype)
    _expect(out, "out", (B, T, Hq, d), q.dtype)
    if cu_seqlens is not None and (cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2
                                   or cu_seqlens.dtype != torch.int32):
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of n + 1 offsets")
    _need_cuda(q, k, v, out, cu_seqlens)
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and max_seqlen is None:
        max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item())
    if out is None:
        out = torch.empty_like(q)
    st = lib.liger_attn_full_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(out), B, Hq, Hkv, T, d, _dt(q),
                                    _ptr(cu_seqlens), n, 0 if max_seqlen is None else int(max_seqlen),
                                    _stream_ptr(stream))
    _check(st)
    return out


def full_causal_status() -> int:
    """LIGER_OK, or LIGER_ERR_TIMEOUT if a causal attention call gave up waiting since the last query."""
    return int(load().liger_attn_full_causal_status())


def decode_status() -> int:
    """LIGER_OK, or LIGER_ERR_TIMEOUT if a decode step gave up waiting since the last query."""
    return int(load().liger_attn_decode_status())


def prefill_backward_workspace_size(B, Hq, Hkv, T, d, n_seqs, dtype=torch.bfloat16) -> int:
    return int(load().liger_attn_prefill_backward_workspace_size(
        B, Hq, Hkv, T, d, n_seqs, LIGER_BF16 if dtype == torch.bfloat16 else LIGER_FP32))


def prefill_backward(q, k, v, d_out, alpha: float = 0.5, w: int = 64, d_final_state=None,
                     initial_state=None, cu_seqlens=None, want_d_initial_state: bool = False,
                     workspace=None, stream=None):
    """Gradient of `prefill` for L = sum(d_out * out) + sum(d_final_state * final_state).

    initial_state and the returned d_initial_state are one per (sequence, kv head):
    [n, Hkv, d, d] fp32.  Returns (dq, dk, dv, d_initial_state or None).
    """
    lib = load()
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, T, Hq, d] and k, v [B, T, Hkv, d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _expect(k, "k", (B, T, Hkv, d), q.dtype)
    _expect(v, "v", (B, T, Hkv, d), q.dtype)
    _expect(d_out, "d_out", (B, T, Hq, d), q.dtype)
    if cu_seqlens is not None and (cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2
                                   or cu_seqlens.dtype != torch.int32):
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of n + 1 offsets")
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    _expect(d_final_state, "d_final_state", (n, Hq, d, d), torch.float32)
    _expect(initial_state, "initial_state", (n, Hkv, d, d), torch.float32)
    _need_cuda(q, k, v, d_out, d_final_state, initial_state, cu_seqlens, workspace)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ds0 = torch.empty(n, Hkv, d, d, device=q.device, dtype=torch.float32) if want_d_initial_state else None
    need = prefill_backward_workspace_size(B, Hq, Hkv, T, d, n, q.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = lib.liger_attn_prefill_backward(
        _ptr(q), _ptr(k), _ptr(v), _ptr(d_out), _ptr(d_final_state), _ptr(initial_state), B, Hq, Hkv, T, d, w,
        float(alpha), _dt(q), _ptr(cu_seqlens), n, _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ds0), _ptr(workspace),
        ws_bytes, _stream_ptr(stream))
    _check(st)
    return dq, dk, dv, ds0


def prefill_vector_gate_workspace_size(B, Hq, Hkv, T, d, n_seqs, dtype=torch.bfloat16) -> int:
    return int(load().liger_attn_prefill_vector_gate_workspace_size(
        B, Hq, Hkv, T, d, n_seqs, LIGER_BF16 if dtype == torch.bfloat16 else LIGER_FP32))


def prefill_vector_gate(q, k, v, alpha: float = 0.5, w: int = 64, initial_state=None, cu_seqlens=None,
                        return_ring: bool = False, workspace=None, stream=None):
    """The prefill with one gate per key dimension (sigmoid(k_t[r]) on row r of the state).
    Returns (out, final_state) or, with return_ring, (out, final_state, ring, pos).
    workspace: uint8 CUDA tensor of prefill_vector_gate_workspace_size() bytes (allocated
    here when None)."""
    lib = load()
    if q.dim() != 4 or k.dim() != 4:
        raise ValueError("q must be [B, T, Hq, d] and k, v [B, T, Hkv, d]")
    B, T, Hq, d = q.shape
    Hkv = k.shape[2]
    _expect(k, "k", (B, T, Hkv, d), q.dtype)
    _expect(v, "v", (B, T, Hkv, d), q.dtype)
    if cu_seqlens is not None and (cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2
                                   or cu_seqlens.dtype != torch.int32):
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of n + 1 offsets")
    n = B if cu_seqlens is None else cu_seqlens.numel() - 1
    _expect(initial_state, "initial_state", (n, Hq, d, d), torch.float32)
    _need_cuda(q, k, v, initial_state, cu_seqlens)
    out = torch.empty_like(q)
    fs = torch.empty(n, Hq, d, d, device=q.device, dtype=torch.float32)
    ring = torch.empty(n, Hkv, 2, w, d, device=q.device, dtype=q.dtype) if return_ring else None
    pos = torch.empty(n, device=q.device, dtype=torch.int32) if return_ring else None
    need = lib.liger_attn_prefill_vector_gate_workspace_size(B, Hq, Hkv, T, d, n, _dt(q))
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=q.device, dtype=torch.uint8)
    _need_cuda(workspace)
    if workspace.dtype != torch.uint8 or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous uint8 tensor")
    st = lib.liger_attn_prefill_vector_gate(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(fs), B, Hq, Hkv, T, d, w, float(alpha), _dt(q),
        _ptr(initial_state), _ptr(cu_seqlens), n, _ptr(ring), _ptr(pos), _ptr(workspace), workspace.numel(),
        _stream_ptr(stream))
    _check(st)
    return (out, fs, ring, pos) if return_ring else (out, fs)


def decode_vector_gate(q, k, v, state, ring, pos, alpha: float = 0.5, out=None, stream=None):
    """One decode step with one gate per key dimension; updates state, ring and pos in place."""
    lib = load()
    B, Hq, Hkv, d, w = _check_decode(q, k, v, state, ring, pos, out, per_head=True)
    if out is None:
        out = torch.empty_like(q)
    st = lib.liger_attn_decode_vector_gate(
        _ptr(q), _ptr(k), _ptr(v), _ptr(state), _ptr(ring), _ptr(out), _ptr(pos), B, Hq, Hkv, d, w,
        float(alpha), _dt(q), _stream_ptr(stream))
    _check(st)
    return out
