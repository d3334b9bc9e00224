"""Seeded synthetic inputs for the Liger Attention forward pass.

This module only draws random tensors and describes workload shapes; it holds
none of the method's arithmetic.  Both the CUDA path and the CPU oracle are
fed from here, so the two see bit-identical inputs.

Shapes are the attention shapes of the models the Liger pages evaluate
(Llama-3.2-1B and Llama-3-8B: GQA with 32 query heads and 8 key/value heads).
There is no dataset: values are i.i.d. normal draws from a seeded CPU
generator in fp32, scaled, then rounded to the workload dtype.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional, Tuple

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "prefill" or "decode"
    B: int
    Hq: int
    Hkv: int
    T: int               # tokens per sequence (prefill) / prefix length (decode)
    d: int
    dtype: torch.dtype
    w: int = 64
    alpha: float = 0.5
    scale: float = 1.0   # multiplies the N(0, 1) draws of q, k, v
    seed: int = 0
    seqlens: Tuple[int, ...] = field(default=())   # varlen packing (B == 1)
    key_bias_std: float = 0.0                      # per kv-head constant added to k
    steps: int = 0                                 # decode steps

    @property
    def cu_seqlens(self) -> Optional[list]:
        if not self.seqlens:
            return None
        cu = [0]
        for n in self.seqlens:
            cu.append(cu[-1] + n)
        return cu

    @property
    def n_seqs(self) -> int:
        return len(self.seqlens) if self.seqlens else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T


WORKLOADS = {
    # fp32 check: B=1, Hq=Hkv=2, T=256, d=64, N(0,1), zero state
    "tiny_fp32": Workload("tiny_fp32", "prefill", 1, 2, 2, 256, 64, torch.float32, seed=1001),
    # Llama-3.2-1B attention shape; N(0,1) scaled by d^(-1/4)
    "llama1b_prefill": Workload("llama1b_prefill", "prefill", 4, 32, 8, 2048, 64, torch.bfloat16,
                                scale=64 ** -0.25, seed=1002),
    # Llama-3-8B attention shape
    "llama8b_prefill": Workload("llama8b_prefill", "prefill", 2, 32, 8, 8192, 128, torch.bfloat16,
                                seed=1003),
    # Llama-3-8B decode: 64 sequences after a 1024-token prefill, 1000 steps
    "llama8b_decode": Workload("llama8b_decode", "decode", 64, 32, 8, 1024, 128, torch.bfloat16,
                               seed=1004, steps=1000),
    # the same with one state per kv head: 256 sequences, so that the fp32 states
    # (134 MB) exceed the 126 MB L2 as the per-head states (268 MB at 64) do
    "llama8b_decode_kvshared": Workload("llama8b_decode_kvshared", "decode", 256, 32, 8, 1024, 128,
                                        torch.bfloat16, seed=1006, steps=1000),
    # 32K packed as 4 sequences, keys biased per kv head by N(0, 0.5^2)
    "long_varlen": Workload("long_varlen", "prefill", 1, 32, 8, 32768, 128, torch.bfloat16,
                            seed=1005, seqlens=(4096, 8192, 8192, 12288), key_bias_std=0.5),
}


def _randn(shape, gen, scale, dtype, device):
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if scale != 1.0:
        x = x * scale
    return x.to(dtype).to(device)


def prefill_inputs(wl: Workload, device="cpu", seed: Optional[int] = None, T: Optional[int] = None,
                   B: Optional[int] = None):
    """q [B,T,Hq,d], k and v [B,T,Hkv,d] in wl.dtype (T and B may be overridden)."""
    T = wl.T if T is None else T
    B = wl.B if B is None else B
    gen = torch.Generator().manual_seed(wl.seed if seed is None else seed)
    q = _randn((B, T, wl.Hq, wl.d), gen, wl.scale, wl.dtype, "cpu")
    k = _randn((B, T, wl.Hkv, wl.d), gen, wl.scale, torch.float32, "cpu")
    v = _randn((B, T, wl.Hkv, wl.d), gen, wl.scale, wl.dtype, "cpu")
    if wl.key_bias_std:
        bias = torch.randn(wl.Hkv, generator=gen, dtype=torch.float32) * wl.key_bias_std
        k = k + bias.view(1, 1, wl.Hkv, 1)
    k = k.to(wl.dtype)
    return q.to(device), k.to(device), v.to(device)


def decode_step_inputs(wl: Workload, step: int, device="cpu"):
    """q [B,Hq,d], k and v [B,Hkv,d] for decode step ``step`` (seed 2000 + step)."""
    gen = torch.Generator().manual_seed(2000 + step)
    q = _randn((wl.B, wl.Hq, wl.d), gen, wl.scale, wl.dtype, device)
    k = _randn((wl.B, wl.Hkv, wl.d), gen, wl.scale, wl.dtype, device)
    v = _randn((wl.B, wl.Hkv, wl.d), gen, wl.scale, wl.dtype, device)
    return q, k, v


def random_state(n: int, Hq: int, d: int, seed: int, scale: float = 0.05, device="cpu"):
    """An arbitrary fp32 recurrent state [n, Hq, d, d] (for initial-state tests)."""
    gen = torch.Generator().manual_seed(seed)
    return (torch.randn(n, Hq, d, d, generator=gen, dtype=torch.float32) * scale).to(device)


def small(name: str = "small", B=2, Hq=4, Hkv=2, T=200, d=64, dtype=torch.bfloat16, seed=7,
          seqlens=(), key_bias_std=0.0, scale=1.0, alpha=0.5) -> Workload:
    """A small workload for parity tests (several chunks and a ragged tail)."""
    return Workload(name, "prefill", B, Hq, Hkv, T, d, dtype, seed=seed, seqlens=tuple(seqlens),
                    key_bias_std=key_bias_std, scale=scale, alpha=alpha)
