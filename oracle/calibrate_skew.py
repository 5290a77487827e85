"""Choose the router scale of the load-skewed workload -- TEST INFRASTRUCTURE.

The skewed workload draws x = z + 3 u (u a random unit direction) and replaces
router row 0 by alpha * u.  This script bisects alpha, routing with the CPU
oracle only, until the fraction of tokens whose chosen set contains expert 0
is 0.40 +- 0.01, and prints it.  The value printed is stored by hand as
SKEW_ALPHA in the input-generator module.
"""
from __future__ import annotations

import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import oracle  # noqa: E402
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def frac_expert0(inp, w, alpha: float) -> float:
    Wr = inp.W_router.clone()
    Wr[0] = (alpha * inp.skew_u).to(Wr.dtype)
    r = oracle.route(inp.x, Wr, w.k, w.n_group, w.topk_group, with_scores=False)
    return float((r.idx == 0).any(axis=1).mean())


def main(target: float = 0.40) -> float:
    w = WORKLOADS["skewed"]
    inp = make_inputs(w)
    lo, hi = 0.0, 2.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        f = frac_expert0(inp, w, mid)
        print(f"alpha={mid:.5f} frac={f:.4f}")
        if abs(f - target) < 0.002:
            return mid
        lo, hi = (mid, hi) if f < target else (lo, mid)
    return 0.5 * (lo + hi)


if __name__ == "__main__":
    a = main()
    print(f"SKEW_ALPHA = {a:.4f}")
