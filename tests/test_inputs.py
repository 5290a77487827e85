"""Checks of the seeded input generators: scale, independence of the random
streams, determinism, and the skewed workload's construction."""
import math

import numpy as np
import torch

from sparse_mixture_experts_03_b200.inputs import (CHUNK, SKEW_SHIFT, WORKLOADS, Workload,
                                                   _randn, make_inputs)


def test_scales_follow_fan_in():
    w = Workload("t", T=512, d=256, E=8, k=2, n_group=2, topk_group=1, inter=128, n_shared=2,
                 dtype="f32")
    inp = make_inputs(w)
    assert abs(inp.x.std().item() - 1.0) < 0.02
    assert abs(inp.W_router.std().item() * math.sqrt(w.d) - 1.0) < 0.05
    assert abs(inp.W_gate_up.std().item() * math.sqrt(w.d) - 1.0) < 0.02
    assert abs(inp.W_down.std().item() * math.sqrt(w.inter) - 1.0) < 0.02


def test_streams_are_independent():
    """Different tensors (and chunks) must not repeat each other's draws."""
    a = _randn((CHUNK + 1000,), 0, 0)
    b = _randn((CHUNK + 1000,), 0, 1)
    c = _randn((CHUNK + 1000,), 1, 0)
    for u, v in ((a, b), (a, c), (b, c)):
        r = np.corrcoef(u[:100000].numpy(), v[:100000].numpy())[0, 1]
        assert abs(r) < 0.02
    # chunk 1 differs from chunk 0
    r = np.corrcoef(a[:1000].numpy(), a[CHUNK:CHUNK + 1000].numpy())[0, 1]
    assert abs(r) < 0.15
    # gate pre-activations x . W have unit scale (no self-correlation)
    w = Workload("t", T=256, d=256, E=4, k=1, n_group=1, topk_group=1, inter=128, n_shared=0,
                 dtype="f32")
    inp = make_inputs(w)
    g = inp.x @ inp.W_gate_up[0].T
    assert 0.9 < g.std().item() < 1.1 and g.abs().max().item() < 7


def test_deterministic():
    w = WORKLOADS["tiny"]
    a, b = make_inputs(w), make_inputs(w)
    assert torch.equal(a.x, b.x) and torch.equal(a.W_gate_up, b.W_gate_up)


def test_skew_direction():
    w = WORKLOADS["skewed"].with_tokens(256)
    inp = make_inputs(w)
    u = inp.skew_u
    assert abs(u.norm().item() - 1.0) < 1e-5
    proj = inp.x.float() @ u
    assert abs(proj.mean().item() - SKEW_SHIFT) < 0.2
    cos = torch.nn.functional.cosine_similarity(inp.W_router[0].float(), u, dim=0)
    assert cos.item() > 0.999
