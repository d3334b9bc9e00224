"""CUDA path vs the fp64 oracle, element by element, on seeded inputs.

Small cases and the full workload sizes alike compare every output: the full
sizes run the CUDA kernels in the same launch configuration the benchmark times,
and the oracle recomputes the whole workload (every sequence, head, token and
final-state element; for decode every sequence over all 1000 steps).
Tolerances: bf16 max-abs 2e-2 and rel-L2 5e-3, fp32 1e-4 for both; the window
ring and positions are copies and must match bit for bit.
"""
import zlib

import numpy as np
import pytest
import torch

from gated_linear_attention_liger_b200 import inputs, ops
from oracle import oracle
from tests import child_scenarios
from tests.parity_util import assert_close, np64

pytestmark = pytest.mark.gpu

SMALL = [
    # name, B, Hq, Hkv, T, d, dtype, w, alpha, seqlens, key_bias, with_s0
    ("bf16_d64_ragged", 2, 4, 2, 200, 64, torch.bfloat16, 64, 0.5, (), 0.0, False),
    ("bf16_d128_ragged", 1, 8, 2, 257, 128, torch.bfloat16, 64, 0.5, (), 0.0, False),
    ("bf16_d128_one_token", 2, 4, 1, 1, 128, torch.bfloat16, 64, 0.5, (), 0.0, False),
    ("bf16_d64_one_chunk", 1, 4, 2, 64, 64, torch.bfloat16, 64, 0.5, (), 0.0, False),
    ("bf16_d128_shorter_than_window", 1, 4, 2, 30, 128, torch.bfloat16, 64, 0.5, (), 0.0, False),
    ("bf16_d128_varlen", 1, 4, 1, 270, 128, torch.bfloat16, 64, 0.5, (5, 130, 1, 64, 70), 0.0, False),
    ("bf16_d64_varlen_empty_seq", 1, 4, 2, 150, 64, torch.bfloat16, 64, 0.5, (0, 77, 73, 0), 0.0, False),
    ("bf16_mha_w16_alpha03", 1, 3, 3, 150, 64, torch.bfloat16, 16, 0.3, (), 0.0, False),
    ("bf16_d128_grm_only", 1, 4, 2, 190, 128, torch.bfloat16, 64, 1.0, (), 0.0, False),
    ("bf16_d128_swa_only", 1, 4, 2, 190, 128, torch.bfloat16, 64, 0.0, (), 0.0, False),
    ("bf16_d128_extreme_gates", 1, 8, 4, 320, 128, torch.bfloat16, 64, 0.5, (), 4.0, False),
    ("bf16_d64_initial_state", 2, 4, 2, 150, 64, torch.bfloat16, 64, 0.5, (), 0.0, True),
    ("fp32_d128_ragged", 1, 4, 2, 150, 128, torch.float32, 64, 0.5, (), 0.0, False),
    ("fp32_d64_varlen_s0", 1, 2, 1, 160, 64, torch.float32, 64, 0.5, (60, 100), 0.0, True),
]


def run_small(case, device):
    name, B, Hq, Hkv, T, d, dtype, w, alpha, seqlens, kb, with_s0 = case
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, dtype=dtype, seed=zlib.crc32(name.encode()) % 10000,
                      seqlens=seqlens, key_bias_std=kb)
    q, k, v = inputs.prefill_inputs(wl)
    cu = wl.cu_seqlens
    n = wl.n_seqs
    s0 = inputs.random_state(n, Hq, d, seed=5, scale=0.05) if with_s0 else None
    out, fs, ring, pos = ops.prefill(
        q.to(device), k.to(device), v.to(device), alpha=alpha, w=w,
        initial_state=None if s0 is None else s0.to(device),
        cu_seqlens=None if cu is None else torch.tensor(cu, dtype=torch.int32, device=device),
        return_ring=True)
    torch.cuda.synchronize()
    ref = oracle.prefill(np64(q), np64(k), np64(v), w=w, alpha=alpha, cu_seqlens=cu,
                         initial_state=None if s0 is None else np64(s0))
    return (out, fs, ring, pos), ref, dtype


@pytest.mark.parametrize("case", SMALL, ids=[c[0] for c in SMALL])
def test_prefill_small_parity(case, cuda_device):
    (out, fs, ring, pos), (ro, rfs, rring, rpos), dtype = run_small(case, cuda_device)
    assert_close(np64(out), ro, dtype, "out")
    assert_close(np64(fs), rfs, dtype, "final_state")
    np.testing.assert_array_equal(np64(ring), rring)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)


def test_prefill_general_kernel_parity(cuda_device):
    """The general (CUDA-core) prefill kernel, forced for bf16 inputs (the first six bf16
    small cases), in a child process whose library was loaded with LIGER_PREFILL_PATH=general."""
    out = child_scenarios.run("general_parity", child_scenarios.GENERAL_ENV)
    assert out.count("general kernel ok") == 6


def test_prefill_wide_feature_spread(cuda_device):
    """Rows whose first element lies far below their maximum: the feature passes
    take their exponentials against the row's first element and must fall back
    to the row maximum (queries and keys, both heads of a tile, several chunks)."""
    wl = inputs.small("wide_spread", B=1, Hq=4, Hkv=2, T=200, d=128, dtype=torch.bfloat16, seed=77)
    q, k, v = inputs.prefill_inputs(wl)
    q[:, ::3, :, 0] = -40.0          # spread 40 (about 58 in log2) on every third token
    q[:, 1::7, :, 0] = 25.0          # first element is the maximum: no fallback
    k[:, ::5, :, 0] = -40.0
    k[:, 2::11, :, 0] = -12.0        # spread about 15 in log2: shifted pass kept
    dev = cuda_device
    out, fs = ops.prefill(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v))
    assert_close(np64(out), ro, torch.bfloat16, "out")
    assert_close(np64(fs), rfs, torch.bfloat16, "final_state")


def test_prefill_sharp_gate_drops(cuda_device):
    """Gates near 1 except one token per chunk whose gate is about e^-50, e^-70 or e^-55:
    chunk log-gate totals of about -53, -73 and -58 put chunks on both sides of the
    kernel's switch between factored and exact decay, with the in-chunk decay from keys
    before the drop to the chunk's end far below the decay between the rows and keys
    that meet in the recurrent scores."""
    wl = inputs.small("sharp_drops", B=1, Hq=4, Hkv=2, T=260, d=128, dtype=torch.bfloat16, seed=91)
    q, k, v = inputs.prefill_inputs(wl)
    k += 3.0                          # sigmoid(mean k) ~ 0.95: log gate ~ -0.05 per token
    k[:, 30] = -50.0
    k[:, 100] = -70.0
    k[:, 150] = -55.0
    dev = cuda_device
    out, fs = ops.prefill(q.to(dev), k.to(dev), v.to(dev))
    torch.cuda.synchronize()
    ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v))
    assert_close(np64(out), ro, torch.bfloat16, "out")
    assert_close(np64(fs), rfs, torch.bfloat16, "final_state")


def test_prefill_empty_batch(cuda_device):
    q = torch.zeros(2, 0, 4, 64, dtype=torch.bfloat16, device=cuda_device)
    k = torch.zeros(2, 0, 2, 64, dtype=torch.bfloat16, device=cuda_device)
    s0 = inputs.random_state(2, 4, 64, seed=3).to(cuda_device)
    out, fs, ring, pos = ops.prefill(q, k, k, initial_state=s0, return_ring=True)
    torch.cuda.synchronize()
    assert out.shape == q.shape
    torch.testing.assert_close(fs, s0, rtol=0, atol=0)
    assert int(pos.abs().sum()) == 0 and float(ring.float().abs().sum()) == 0.0


def test_prefill_is_deterministic(cuda_device):
    wl = inputs.small("det", B=2, Hq=8, Hkv=2, T=600, d=128)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    a, sa = ops.prefill(q, k, v)
    b, sb = ops.prefill(q, k, v)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(sa, sb)


# ----------------------------------------------------------------- full sizes

def _full_prefill_check(name, device):
    """The whole workload on the GPU and in the oracle; every output, final-state, ring and
    position element compared."""
    wl = inputs.WORKLOADS[name]
    q, k, v = inputs.prefill_inputs(wl)
    cu = wl.cu_seqlens
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=device)
    out, fs, ring, pos = ops.prefill(q.to(device), k.to(device), v.to(device), alpha=wl.alpha, w=wl.w,
                                     cu_seqlens=cu_t, return_ring=True)
    torch.cuda.synchronize()
    ro, rfs, rring, rpos = oracle.prefill(np64(q), np64(k), np64(v), w=wl.w, alpha=wl.alpha, cu_seqlens=cu)
    assert_close(np64(out), ro, wl.dtype, f"{name} out")
    assert_close(np64(fs), rfs, wl.dtype, f"{name} final_state")
    np.testing.assert_array_equal(np64(ring), rring)
    np.testing.assert_array_equal(pos.cpu().numpy(), rpos)
    # every sequence and head on its own as well: a wrong offset for one unit cannot hide
    # inside the whole-tensor norm
    G = wl.Hq // wl.Hkv
    n = wl.n_seqs
    bounds = cu if cu is not None else None
    for s_ in range(n):
        for kv in range(wl.Hkv):
            hs = slice(kv * G, (kv + 1) * G)
            if bounds is not None:
                got, ref = np64(out[0, bounds[s_]:bounds[s_ + 1], hs]), ro[0, bounds[s_]:bounds[s_ + 1], hs]
            else:
                got, ref = np64(out[s_, :, hs]), ro[s_, :, hs]
            if ref.size:
                assert_close(got, ref, wl.dtype, f"{name} out seq={s_} kv={kv}")
            assert_close(np64(fs[s_, hs]), rfs[s_, hs], wl.dtype, f"{name} final_state seq={s_} kv={kv}")


def test_full_llama1b_prefill(cuda_device):
    _full_prefill_check("llama1b_prefill", cuda_device)


def test_full_llama8b_prefill(cuda_device):
    _full_prefill_check("llama8b_prefill", cuda_device)


def test_full_long_varlen_prefill(cuda_device):
    _full_prefill_check("long_varlen", cuda_device)


def test_full_tiny_fp32(cuda_device):
    wl = inputs.WORKLOADS["tiny_fp32"]
    q, k, v = inputs.prefill_inputs(wl)
    out, fs = ops.prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device))
    torch.cuda.synchronize()
    ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v))
    assert_close(np64(out), ro, torch.float32, "out")
    assert_close(np64(fs), rfs, torch.float32, "final_state")


# ----------------------------------------------------------------- decode

@pytest.mark.parametrize("dtype,d,w,T0,G,B", [
    (torch.bfloat16, 128, 64, 70, 4, 3),
    (torch.bfloat16, 64, 64, 0, 2, 3),
    (torch.bfloat16, 64, 16, 5, 1, 3),
    (torch.float32, 128, 64, 100, 2, 3),
    (torch.float32, 64, 64, 3, 4, 3),
    # more (sequence, head) units than SMs, ring wrapped, w < 64: each CTA of the
    # streamed kernel takes several units and reuses its two stages
    (torch.bfloat16, 128, 40, 90, 4, 40),
    (torch.float32, 64, 64, 70, 2, 50),
    # w = 1: the window is the current token alone
    (torch.bfloat16, 128, 1, 20, 2, 7),
])
def test_decode_steps_parity(dtype, d, w, T0, G, B, cuda_device):
    """Oracle prefix -> identical state/ring/pos on both sides -> several decode steps."""
    Hkv, steps = 2, 12
    Hq = Hkv * G
    wl = inputs.small("dec", B=B, Hq=Hq, Hkv=Hkv, T=T0 + steps, d=d, dtype=dtype, seed=17)
    q, k, v = inputs.prefill_inputs(wl)
    if T0:
        _, st, rg, ps = oracle.prefill(np64(q[:, :T0]), np64(k[:, :T0]), np64(v[:, :T0]), w=w)
    else:
        st, rg, ps = np.zeros((B, Hq, d, d)), np.zeros((B, Hkv, 2, w, d)), np.zeros(B, np.int32)
    g_state = torch.tensor(st, dtype=torch.float32)
    st = np64(g_state)  # the oracle continues from the same fp32 state the GPU holds
    g_state = g_state.to(cuda_device)
    g_ring = torch.tensor(rg).to(dtype)
    rg = np64(g_ring)
    g_ring = g_ring.to(cuda_device)
    g_pos = torch.tensor(ps, dtype=torch.int32, device=cuda_device)
    for t in range(T0, T0 + steps):
        qt, kt, vt = q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()
        o = ops.decode(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device), g_state, g_ring, g_pos)
        ro, st, rg, ps = oracle.decode(np64(qt), np64(kt), np64(vt), st, rg, ps, w=w)
        torch.cuda.synchronize()
        assert_close(np64(o), ro, dtype, f"decode out step {t}")
    assert_close(np64(g_state), st, dtype, "decode state")
    np.testing.assert_array_equal(np64(g_ring), rg)
    np.testing.assert_array_equal(g_pos.cpu().numpy(), ps)
    assert ops.decode_status() == ops.LIGER_OK


def test_prefill_then_decode_matches_longer_prefill(cuda_device):
    """Cross-path: GPU prefill(T1) + T2 GPU decode steps == GPU prefill(T1 + T2)."""
    wl = inputs.small("xpath", B=2, Hq=8, Hkv=2, T=300, d=128, seed=23)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(wl))
    T1 = 260
    full, fs_full, ring_full, _ = ops.prefill(q, k, v, return_ring=True)
    _, st, rg, ps = ops.prefill(q[:, :T1].contiguous(), k[:, :T1].contiguous(), v[:, :T1].contiguous(),
                                return_ring=True)
    for t in range(T1, wl.T):
        o = ops.decode(q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), st, rg, ps)
        assert_close(np64(o), np64(full[:, t]), torch.bfloat16, f"step {t}")
    assert_close(np64(st), np64(fs_full), torch.bfloat16, "state")
    assert torch.equal(rg, ring_full)
    assert int(ps.min()) == wl.T == int(ps.max())


def test_full_llama8b_decode(cuda_device):
    """The Llama-3-8B decode workload in full: B=64 sequences whose state and ring come from a
    seeded 1024-token prefill, then 1000 steps.  The GPU prefill of the prefix is compared with
    the oracle's; both decodes then start from the oracle's prefix (state rounded to fp32, ring
    to bf16) and every output of every sequence and step is compared, then the final states,
    ring and positions."""
    wl = inputs.WORKLOADS["llama8b_decode"]
    B, Hq, Hkv, d, w = wl.B, wl.Hq, wl.Hkv, wl.d, wl.w
    steps = wl.steps
    dev = cuda_device
    pre = inputs.Workload("decode_prefix", "prefill", B, Hq, Hkv, wl.T, d, wl.dtype, seed=wl.seed)
    q, k, v = inputs.prefill_inputs(pre)
    _, g_st, g_rg, g_ps = ops.prefill(q.to(dev), k.to(dev), v.to(dev), alpha=wl.alpha, w=w, return_ring=True)
    _, rst, rrg, rps = oracle.prefill(np64(q), np64(k), np64(v), w=w, alpha=wl.alpha)
    torch.cuda.synchronize()
    assert_close(np64(g_st), rst, wl.dtype, "prefix final state")
    np.testing.assert_array_equal(np64(g_rg), rrg)
    np.testing.assert_array_equal(g_ps.cpu().numpy(), rps)
    del q, k, v, g_st, g_rg
    # the common starting point
    state = torch.tensor(rst, dtype=torch.float32)
    ring = torch.tensor(rrg).to(wl.dtype)
    o_st = np.ascontiguousarray(np64(state))
    o_rg = np.ascontiguousarray(np64(ring))
    o_ps = np.ascontiguousarray(rps.astype(np.int32))
    g_state, g_ring = state.to(dev), ring.to(dev)
    g_pos = torch.tensor(rps, dtype=torch.int32, device=dev)
    del state, ring, rst, rrg
    block = 50
    for s0 in range(0, steps, block):
        step_in = [inputs.decode_step_inputs(wl, s) for s in range(s0, min(steps, s0 + block))]
        outs = []
        for qt, kt, vt in step_in:
            outs.append(ops.decode(qt.to(dev), kt.to(dev), vt.to(dev), g_state, g_ring, g_pos, alpha=wl.alpha))
        outs = torch.stack(outs).cpu()
        for i, (qt, kt, vt) in enumerate(step_in):
            ro = oracle.decode_inplace(np64(qt), np64(kt), np64(vt), o_st, o_rg, o_ps, alpha=wl.alpha)
            assert_close(np64(outs[i]), ro, wl.dtype, f"decode step {s0 + i}")
    torch.cuda.synchronize()
    assert_close(np64(g_state), o_st, wl.dtype, "state after the steps")
    np.testing.assert_array_equal(np64(g_ring), o_rg)
    np.testing.assert_array_equal(g_pos.cpu().numpy(), o_ps)
    assert int(g_pos.min()) == wl.T + steps == int(g_pos.max())


# ----------------------------------------------------------------- shared-state decode

@pytest.mark.parametrize("dtype,d,w,T0,G,B", [
    (torch.bfloat16, 128, 64, 70, 4, 3),
    (torch.bfloat16, 64, 64, 0, 2, 3),
    (torch.bfloat16, 64, 16, 5, 1, 3),
    (torch.float32, 128, 64, 100, 4, 3),
    # more (sequence, kv head) units than SMs: each CTA of the streamed kernel takes
    # several units and reuses its two stages
    (torch.bfloat16, 64, 64, 30, 4, 170),
    # ring wrapped (prefix longer than the window), w < 64, several units per CTA
    (torch.bfloat16, 128, 32, 50, 2, 160),
    (torch.float32, 64, 48, 60, 4, 90),
    (torch.bfloat16, 64, 1, 9, 4, 5),
])
def test_decode_kvshared_parity(dtype, d, w, T0, G, B, cuda_device):
    """One state per kv head: the oracle runs with that state copied to every q head of
    the group; outputs, the (shared) state, ring and positions must match."""
    Hkv, steps = 2, 10
    Hq = Hkv * G
    wl = inputs.small("deckv", B=B, Hq=Hq, Hkv=Hkv, T=T0 + steps, d=d, dtype=dtype, seed=29)
    q, k, v = inputs.prefill_inputs(wl)
    if T0:
        _, st, rg, ps = oracle.prefill(np64(q[:, :T0]), np64(k[:, :T0]), np64(v[:, :T0]), w=w)
        kv_state = torch.tensor(st[:, ::G], dtype=torch.float32)   # heads of a group hold equal copies
    else:
        kv_state = torch.zeros(B, Hkv, d, d)
        rg, ps = np.zeros((B, Hkv, 2, w, d)), np.zeros(B, np.int32)
    st = np.repeat(np64(kv_state), G, axis=1)
    g_state = kv_state.to(cuda_device)
    g_ring = torch.tensor(rg).to(dtype)
    rg = np64(g_ring)
    g_ring = g_ring.to(cuda_device)
    g_pos = torch.tensor(ps, dtype=torch.int32, device=cuda_device)
    for t in range(T0, T0 + steps):
        qt, kt, vt = q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous()
        o = ops.decode_kvshared(qt.to(cuda_device), kt.to(cuda_device), vt.to(cuda_device), g_state, g_ring, g_pos)
        ro, st, rg, ps = oracle.decode(np64(qt), np64(kt), np64(vt), st, rg, ps, w=w)
        torch.cuda.synchronize()
        assert_close(np64(o), ro, dtype, f"kv-shared decode out step {t}")
    assert_close(np64(g_state), st[:, ::G], dtype, "kv-shared state")
    np.testing.assert_array_equal(np64(g_ring), rg)
    np.testing.assert_array_equal(g_pos.cpu().numpy(), ps)
    assert ops.decode_status() == ops.LIGER_OK


def test_decode_kvshared_matches_per_head_decode_full_shape(cuda_device):
    """B=64 at the Llama-3-8B shape after a GPU prefill: 20 steps of the shared-state decode
    track the per-head decode (same inputs, same starting point)."""
    wl = inputs.WORKLOADS["llama8b_decode"]
    G = wl.Hq // wl.Hkv
    pre = inputs.Workload("pre", "prefill", wl.B, wl.Hq, wl.Hkv, 256, wl.d, wl.dtype, seed=wl.seed)
    q, k, v = (t.to(cuda_device) for t in inputs.prefill_inputs(pre))
    _, st, rg, ps = ops.prefill(q, k, v, return_ring=True)
    st_kv = st[:, ::G].contiguous()
    rg2, ps2 = rg.clone(), ps.clone()
    for step in range(20):
        qt, kt, vt = (t.to(cuda_device) for t in inputs.decode_step_inputs(wl, step))
        o1 = ops.decode(qt, kt, vt, st, rg, ps)
        o2 = ops.decode_kvshared(qt, kt, vt, st_kv, rg2, ps2)
        assert_close(np64(o2), np64(o1), wl.dtype, f"step {step}")
    assert_close(np64(st_kv), np64(st[:, ::G]), wl.dtype, "state")
    assert torch.equal(rg, rg2) and torch.equal(ps, ps2)


# ----------------------------------------------------------------- initial states on the tensor-core path

def _group_shared_state(n, Hq, Hkv, d, seed, differ_groups=()):
    """Initial states whose G copies are equal within each group, except in the listed
    (sequence, kv head) groups, whose heads get states of their own."""
    G = Hq // Hkv
    base = inputs.random_state(n, Hkv, d, seed=seed, scale=0.05)
    s0 = base.repeat_interleave(G, dim=1).contiguous()
    if differ_groups:
        other = inputs.random_state(n, Hq, d, seed=seed + 1, scale=0.05)
        for seq, kv in differ_groups:
            s0[seq, kv * G:(kv + 1) * G] = other[seq, kv * G:(kv + 1) * G]
    return s0


@pytest.mark.parametrize("name,B,Hq,Hkv,T,d,seqlens,differ", [
    ("shared_d128", 2, 8, 2, 300, 128, (), ()),
    ("shared_d64_packed_empty", 1, 8, 4, 260, 64, (90, 0, 170), ()),
    ("mixed_groups_d128", 2, 8, 2, 200, 128, (), ((0, 1), (1, 0))),
    ("mixed_groups_d64_packed", 1, 8, 2, 210, 64, (70, 140), ((1, 1),)),
])
def test_prefill_initial_state_tensor_core(name, B, Hq, Hkv, T, d, seqlens, differ, cuda_device):
    """bf16, w = 64, even G: the tensor-core path takes the initial state.  Groups whose heads
    share a state run on it; groups whose heads differ are recomputed in the same call."""
    wl = inputs.small(name, B=B, Hq=Hq, Hkv=Hkv, T=T, d=d, seed=zlib.crc32(name.encode()) % 10000, seqlens=seqlens)
    q, k, v = inputs.prefill_inputs(wl)
    n = wl.n_seqs
    s0 = _group_shared_state(n, Hq, Hkv, d, seed=13, differ_groups=differ)
    cu = wl.cu_seqlens
    dev = cuda_device
    plan = ops.prefill_plan(B, Hq, Hkv, T, d, n, packed=cu is not None)
    assert plan["chunks_per_segment"] >= 1   # the tensor-core path takes these sizes
    out, fs = ops.prefill(q.to(dev), k.to(dev), v.to(dev), initial_state=s0.to(dev),
                          cu_seqlens=None if cu is None else torch.tensor(cu, dtype=torch.int32, device=dev))
    torch.cuda.synchronize()
    ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v), cu_seqlens=cu, initial_state=np64(s0))
    assert_close(np64(out), ro, torch.bfloat16, "out")
    assert_close(np64(fs), rfs, torch.bfloat16, "final_state")


def test_prefill_resume_llama8b_shape(cuda_device):
    """Llama-3-8B shape: prefill of the first 4096 tokens, then of the next 4096 from its final
    state, on the tensor-core path.  The second call matches the oracle run from the same
    state; with alpha = 1 (the recurrent branch alone: the window restarts with each call)
    the two calls reproduce one 8192-token prefill."""
    wl = inputs.WORKLOADS["llama8b_prefill"]
    q, k, v = inputs.prefill_inputs(wl)
    dev = cuda_device
    T1 = 4096
    halves = [(t[:, :T1].contiguous(), t[:, T1:].contiguous()) for t in (q, k, v)]
    (q1, q2), (k1, k2), (v1, v2) = halves
    for alpha in (0.5, 1.0):
        _, fs1 = ops.prefill(q1.to(dev), k1.to(dev), v1.to(dev), alpha=alpha)
        out2, fs2 = ops.prefill(q2.to(dev), k2.to(dev), v2.to(dev), alpha=alpha, initial_state=fs1)
        torch.cuda.synchronize()
        ro2, rfs2, _, _ = oracle.prefill(np64(q2), np64(k2), np64(v2), alpha=alpha, initial_state=np64(fs1))
        assert_close(np64(out2), ro2, wl.dtype, f"second call out (alpha {alpha})")
        assert_close(np64(fs2), rfs2, wl.dtype, f"second call final state (alpha {alpha})")
        if alpha == 1.0:
            ro, rfs, _, _ = oracle.prefill(np64(q), np64(k), np64(v), alpha=1.0)
            assert_close(np64(out2), ro[:, T1:], wl.dtype, "resumed recurrent branch vs one long prefill")
            assert_close(np64(fs2), rfs, wl.dtype, "resumed final state vs one long prefill")
