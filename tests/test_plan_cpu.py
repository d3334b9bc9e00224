"""The tensor-core prefill's planner (host logic), through the C ABI's plan query, against a
brute-force search of the cost model the header states.  CPU only: without a device the planner
assumes 148 SMs."""
import math

import pytest

from gated_linear_attention_liger_b200 import ops

C = 64   # tokens per chunk

SHAPES = [
    # B, Hq, Hkv, T, d, n_seqs, packed
    (2, 32, 8, 8192, 128, 2, False),     # Llama-3-8B prefill
    (4, 32, 8, 2048, 64, 4, False),      # Llama-3.2-1B prefill
    (1, 32, 8, 32768, 128, 4, True),     # long packed batch
    (3, 8, 2, 300, 128, 3, False),
    (1, 4, 2, 150, 64, 4, True),
    (8, 16, 4, 1, 128, 8, False),
    (1, 32, 8, 600_000, 128, 1, False),  # long single sequence: the length search goes past 64
]


def n_segments(L, B, T, n_seqs, packed):
    if packed:
        return math.ceil(T / (C * L)) + n_seqs
    return B * math.ceil(math.ceil(T / C) / L)


def seg_cost(L, B, Hq, T, n_seqs, packed, sms):
    return math.ceil(max(1, n_segments(L, B, T, n_seqs, packed)) * (Hq // 2) / sms) * (L + 1.5)


def sub_cost(ns, units, L, sms):
    return math.ceil(units * ns / (2 * sms)) * (math.ceil(L / ns) + 0.5)


@pytest.mark.parametrize("shape", SHAPES, ids=[f"B{s[0]}_T{s[3]}_d{s[4]}{'_packed' if s[6] else ''}" for s in SHAPES])
def test_plan_minimises_its_stated_cost(shape):
    B, Hq, Hkv, T, d, n, packed = shape
    pl = ops.prefill_plan(B, Hq, Hkv, T, d, n_seqs=n, packed=packed)
    sms = pl["sm_count"]
    assert sms == 148
    L = pl["chunks_per_segment"]
    NT = T if packed else B * T
    max_L = max(1, math.ceil(NT / C) + (n if packed else 0))
    costs = {x: seg_cost(x, B, Hq, T, n, packed, sms) for x in range(1, max_L + 1)}
    short = {x: c for x, c in costs.items() if x <= 64}
    # every length up to 64 chunks is a candidate: none of them is cheaper
    assert costs[L] <= min(short.values()) + 1e-9
    best = min(costs.values())
    if min(short.values()) == best:   # the optimum lies among them: the first one is taken
        assert L == min(x for x, c in short.items() if c == best)
    else:                             # beyond 64 chunks the search steps by an eighth
        assert costs[L] <= 1.25 * best
    nseg = max(1, n_segments(L, B, T, n, packed))
    assert pl["max_segments"] == nseg
    units = nseg * Hkv
    subs = {ns: sub_cost(ns, units, L, sms) for ns in range(1, min(L, 8) + 1)}
    assert pl["state_subsegments"] == min(ns for ns, c in subs.items() if c == min(subs.values()))
    # the workspace: header, then per (segment, sub-segment, kv head) a log gate and a d x d state
    floor = 256 + nseg * pl["state_subsegments"] * Hkv * (4 + 4 * d * d)
    assert floor <= pl["plan_bytes"] <= ops.prefill_workspace_size(B, Hq, Hkv, T, d, n)


def test_llama8b_plan_is_the_documented_one():
    pl = ops.prefill_plan(2, 32, 8, 8192, 128)
    assert (pl["chunks_per_segment"], pl["max_segments"], pl["state_subsegments"]) == (15, 18, 2)


@pytest.mark.parametrize("args,status", [
    ((2, 32, 8, 8192, 96, 2, False), ops.LIGER_ERR_UNSUPPORTED),   # head dim
    ((2, 24, 8, 8192, 128, 2, False), ops.LIGER_ERR_UNSUPPORTED),  # odd group size
    ((2, 30, 8, 8192, 128, 2, False), ops.LIGER_ERR_INVALID_ARG),  # Hq % Hkv
    ((2, 32, 8, 8192, 128, 2, True), ops.LIGER_ERR_INVALID_ARG),   # packed needs B == 1
    ((2, 32, 8, 8192, 128, 3, False), ops.LIGER_ERR_INVALID_ARG),  # n_seqs != B
    ((1, 32, 8, -1, 128, 1, False), ops.LIGER_ERR_INVALID_ARG),    # T < 0
])
def test_plan_rejects_what_the_prefill_rejects(args, status):
    B, Hq, Hkv, T, d, n, packed = args
    with pytest.raises(ops.LigerError) as e:
        ops.prefill_plan(B, Hq, Hkv, T, d, n_seqs=n, packed=packed)
    assert e.value.status == status
