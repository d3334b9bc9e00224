"""Writes the stored expected values under tests/golden/.  Calls only the oracle.

oracle_small.json: the fp64 oracle on a small seeded case (B=1, T=12, Hq=2,
Hkv=1, d=4, w=4, alpha=0.5), inputs listed in the file.  It pins the oracle
against later edits; the math pins live in tests/test_oracle_pins.py.
Hybrid per "Liger: Linearizing Large Language Models to Gated Recurrent
Structures" (Paper-Notes), sections 统一的门控线性循环框架 and Liger Attention.
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))
from oracle import oracle  # noqa: E402


def main():
    rng = np.random.default_rng(2025)
    B, T, Hq, Hkv, d, w = 1, 12, 2, 1, 4, 4
    q = np.round(rng.standard_normal((B, T, Hq, d)), 3)
    k = np.round(rng.standard_normal((B, T, Hkv, d)), 3)
    v = np.round(rng.standard_normal((B, T, Hkv, d)), 3)
    out, fs, ring, pos = oracle.prefill(q, k, v, w=w, alpha=0.5)
    doc = {
        "source": "Liger Attention forward, Paper-Notes page: recurrence (统一的门控线性循环框架), "
                  "hybrid with w (Liger Attention); readings: phi = softmax over d, "
                  "g = sigmoid(mean_d k), window t-w+1..t scaled by 1/sqrt(d)",
        "shape": {"B": B, "T": T, "Hq": Hq, "Hkv": Hkv, "d": d, "w": w, "alpha": 0.5},
        "q": q.tolist(), "k": k.tolist(), "v": v.tolist(),
        "out": out.tolist(), "final_state": fs.tolist(), "pos": pos.tolist(),
    }
    with open(os.path.join(HERE, "oracle_small.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
