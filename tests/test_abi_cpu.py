"""The C-ABI library: builds for sm_100a, loads without a GPU, exports every
symbol the header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest
import torch

from gated_linear_attention_liger_b200 import build as libbuild
from gated_linear_attention_liger_b200 import ops

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include",
                      "liger_attn.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"\b([a-z_][a-z0-9_]*)\s*\(", src)
    keywords = {"if", "sizeof", "defined", "return"}
    return sorted({n for n in names if n.startswith("liger_") and n not in keywords})


@pytest.fixture(scope="module")
def lib():
    libbuild.build()
    return ops.load()


def test_header_declares_the_entry_points():
    names = declared_functions()
    for required in ("liger_attn_prefill", "liger_attn_decode", "liger_attn_prefill_workspace_size",
                     "liger_last_error", "liger_abi_version"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in ops.SIGNATURES, f"binding lacks {name}"
    assert lib.liger_abi_version() == 1


def _prefill(lib, **kw):
    a = dict(q=16, k=16, v=16, out=16, fs=None, B=1, Hq=4, Hkv=2, T=8, d=64, w=64, alpha=0.5, dt=0,
             s0=None, cu=None, n=1, ring=None, pos=None, ws=None, wsb=0)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.liger_attn_prefill(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["out"]), vp(a["fs"]), a["B"],
                                  a["Hq"], a["Hkv"], a["T"], a["d"], a["w"], a["alpha"], a["dt"],
                                  vp(a["s0"]), vp(a["cu"]), a["n"], vp(a["ring"]), vp(a["pos"]),
                                  vp(a["ws"]), a["wsb"], None)


def _decode(lib, **kw):
    a = dict(q=16, k=16, v=16, st=16, ring=16, out=16, pos=16, B=2, Hq=4, Hkv=2, d=128, w=64,
             alpha=0.5, dt=0)
    a.update(kw)
    vp = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.liger_attn_decode(vp(a["q"]), vp(a["k"]), vp(a["v"]), vp(a["st"]), vp(a["ring"]),
                                 vp(a["out"]), vp(a["pos"]), a["B"], a["Hq"], a["Hkv"], a["d"], a["w"],
                                 a["alpha"], a["dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=3, Hkv=2), ops.LIGER_ERR_INVALID_ARG),
    (dict(Hkv=0), ops.LIGER_ERR_INVALID_ARG),
    (dict(w=0), ops.LIGER_ERR_INVALID_ARG),
    (dict(alpha=1.5), ops.LIGER_ERR_INVALID_ARG),
    (dict(alpha=float("nan")), ops.LIGER_ERR_INVALID_ARG),
    (dict(dt=7), ops.LIGER_ERR_INVALID_ARG),
    (dict(d=96), ops.LIGER_ERR_UNSUPPORTED),
    (dict(w=65), ops.LIGER_ERR_UNSUPPORTED),
    (dict(B=0), ops.LIGER_ERR_INVALID_ARG),
    (dict(T=-1), ops.LIGER_ERR_INVALID_ARG),
    (dict(B=2, cu=16, n=2), ops.LIGER_ERR_INVALID_ARG),
    (dict(cu=16, n=0), ops.LIGER_ERR_INVALID_ARG),
    (dict(B=2, n=1), ops.LIGER_ERR_INVALID_ARG),
    (dict(q=None), ops.LIGER_ERR_INVALID_ARG),
    (dict(out=8), ops.LIGER_ERR_INVALID_ARG),
    (dict(fs=24), ops.LIGER_ERR_INVALID_ARG),
    (dict(cu=18), ops.LIGER_ERR_INVALID_ARG),
])
def test_prefill_rejects_bad_arguments(lib, kw, status):
    assert _prefill(lib, **kw) == status
    assert lib.liger_last_error().decode() != ""


def test_prefill_rejects_short_workspace(lib):
    need = lib.liger_attn_prefill_workspace_size(2, 32, 8, 8192, 128, 2, 0)
    if need == 0:
        pytest.skip("no workspace needed on this path")
    assert _prefill(lib, B=2, Hq=32, Hkv=8, T=8192, d=128, n=2, ws=16, wsb=need - 16) == \
        ops.LIGER_ERR_INVALID_ARG


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=5), ops.LIGER_ERR_INVALID_ARG),
    (dict(B=0), ops.LIGER_ERR_INVALID_ARG),
    (dict(st=None), ops.LIGER_ERR_INVALID_ARG),
    (dict(pos=None), ops.LIGER_ERR_INVALID_ARG),
    (dict(pos=18), ops.LIGER_ERR_INVALID_ARG),
    (dict(ring=40), ops.LIGER_ERR_INVALID_ARG),
    (dict(d=32), ops.LIGER_ERR_UNSUPPORTED),
    (dict(alpha=-0.1), ops.LIGER_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status
    assert lib.liger_last_error().decode() != ""


def test_workspace_size_is_zero_for_rejected_sizes(lib):
    assert lib.liger_attn_prefill_workspace_size(0, 32, 8, 128, 128, 0, 0) == 0
    assert lib.liger_attn_prefill_workspace_size(1, 3, 2, 128, 128, 1, 0) == 0
    assert lib.liger_attn_prefill_workspace_size(1, 4, 2, 128, 128, 1, 1) == 0  # fp32 needs none


def test_binding_refuses_host_tensors(lib):
    """No CPU fallback: host tensors are an error, not a slow path."""
    import torch
    q = torch.zeros(1, 8, 2, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 8, 1, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ops.prefill(q, kv, kv)
    with pytest.raises(ValueError, match="CUDA"):
        ops.decode(q[:, 0], kv[:, 0], kv[:, 0], torch.zeros(1, 2, 64, 64),
                   torch.zeros(1, 1, 2, 64, 64, dtype=torch.bfloat16), torch.zeros(1, dtype=torch.int32))


def test_missing_library_raises():
    saved = ops._lib
    ops._lib = None
    try:
        with pytest.raises(FileNotFoundError, match="no CPU fallback"):
            ops.load(os.path.join(os.path.dirname(HEADER), "no_such_library.so"))
    finally:
        ops._lib = saved


def test_package_never_imports_the_oracle():
    """The oracle is test infrastructure: no module or source of the package refers to it."""
    pkg = os.path.join(os.path.dirname(os.path.dirname(HEADER)), "gated_linear_attention_liger_b200")
    for root, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(root, f)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle\b", text, flags=re.M), f
                assert "liboracle" not in text and "oracle_prefill" not in text, f


def _t(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def test_binding_checks_shapes_before_the_library_sees_pointers(lib):
    """A wrong output buffer must be an error, not an out-of-bounds write on the device."""
    q, kv = _t(2, 70, 4, 64), _t(2, 70, 2, 64)
    bad = [
        dict(k=_t(2, 70, 3, 64)),                                    # Hq % Hkv aside, k != v shape
        dict(out=_t(2, 70, 4, 32)),
        dict(out=_t(2, 70, 4, 64, dtype=torch.float32)),
        dict(final_state=_t(2, 4, 64, 64, dtype=torch.bfloat16)),
        dict(final_state=_t(1, 4, 64, 64, dtype=torch.float32)),
        dict(ring=_t(2, 2, 2, 32, 64), return_ring=True),
        dict(pos=_t(2, dtype=torch.int64), return_ring=True),
        dict(initial_state=_t(2, 4, 64, 64)),
    ]
    for kw in bad:
        args = dict(k=kv, v=kv)
        args.update(kw)
        with pytest.raises(ValueError, match="shape|must be"):
            ops.prefill(q, args.pop("k"), args.pop("v"), **args)
    qd, kd = _t(3, 8, 128), _t(3, 2, 128)
    ring, pos = _t(3, 2, 2, 64, 128), _t(3, dtype=torch.int32)
    with pytest.raises(ValueError, match="state must have shape"):
        ops.decode(qd, kd, kd, _t(3, 2, 128, 128, dtype=torch.float32), ring, pos)   # per-head needs Hq
    with pytest.raises(ValueError, match="state must have shape"):
        ops.decode_kvshared(qd, kd, kd, _t(3, 8, 128, 128, dtype=torch.float32), ring, pos)
    with pytest.raises(ValueError, match="pos must be"):
        ops.decode(qd, kd, kd, _t(3, 8, 128, 128, dtype=torch.float32), ring, _t(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="out must have shape"):
        ops.decode(qd, kd, kd, _t(3, 8, 128, 128, dtype=torch.float32), ring, pos, out=_t(3, 2, 128))


@pytest.mark.parametrize("call", [
    # the argument shapes the GPU tests, the smoke check and the benchmark pass: valid, so the
    # only complaint on a host without tensors on a device is the device check
    dict(kind="prefill", q=(2, 8192, 32, 128), kv=(2, 8192, 8, 128), out=True, fs=2, ws=True),
    dict(kind="prefill", q=(1, 270, 4, 128), kv=(1, 270, 1, 128), cu=6, ring=5, pos=5),
    dict(kind="prefill", q=(2, 0, 4, 64), kv=(2, 0, 2, 64), s0=2, ring=2, pos=2),
    dict(kind="prefill", q=(1, 150, 4, 128), kv=(1, 150, 2, 128), dtype=torch.float32, s0=1),
    dict(kind="decode", q=(3, 8, 64), kv=(3, 2, 64), state=8, w=16),
    dict(kind="decode", q=(64, 32, 128), kv=(64, 8, 128), state=32, w=64, out=True),
    dict(kind="decode_kvshared", q=(256, 32, 128), kv=(256, 8, 128), state=8, w=64, out=True),
])
def test_valid_call_shapes_reach_the_device_check(lib, call):
    dt = call.get("dtype", torch.bfloat16)
    q, kv = _t(*call["q"], dtype=dt), _t(*call["kv"], dtype=dt)
    with pytest.raises(ValueError, match="CUDA"):
        if call["kind"] == "prefill":
            B, T, Hq, d = call["q"]
            Hkv = call["kv"][2]
            n = call.get("cu", B + 1) - 1 if "cu" in call else B
            ops.prefill(
                q, kv, kv,
                out=_t(B, T, Hq, d, dtype=dt) if call.get("out") else None,
                final_state=_t(n, Hq, d, d, dtype=torch.float32) if call.get("fs") else None,
                initial_state=_t(n, Hq, d, d, dtype=torch.float32) if call.get("s0") else None,
                cu_seqlens=_t(n + 1, dtype=torch.int32) if "cu" in call else None,
                ring=_t(n, Hkv, 2, 64, d, dtype=dt) if call.get("ring") else None,
                pos=_t(n, dtype=torch.int32) if call.get("pos") else None,
                return_ring=bool(call.get("ring")),
                workspace=_t(16, dtype=torch.uint8) if call.get("ws") else None)
        else:
            B, Hq, d = call["q"]
            Hkv = call["kv"][1]
            fn = ops.decode if call["kind"] == "decode" else ops.decode_kvshared
            fn(q, kv, kv, _t(B, call["state"], d, d, dtype=torch.float32), _t(B, Hkv, 2, call["w"], d, dtype=dt),
               _t(B, dtype=torch.int32), out=_t(B, Hq, d, dtype=dt) if call.get("out") else None)
