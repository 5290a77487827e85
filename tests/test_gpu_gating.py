"""Parity of the gating variants (softmax over the chosen experts, and the
selection-only expert bias) and of the expert-load output, CUDA path through
the C ABI against the CPU oracle; same criteria as the main parity tests
(tests/parity.py)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_03_b200 import moe
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, Workload, make_inputs

from parity import check_output, check_routing, oracle_outputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def make_bias(E, gate, seed=0):
    """A fixed, shuffled ramp of selection biases on the scale of the keys
    (sigmoid scores in (0, 1); logits of order 1)."""
    span = 0.1 if gate == "sigmoid" else 0.5
    b = np.linspace(-span, span, E).astype(np.float32)
    return np.random.default_rng(seed).permutation(b)


CASES = [
    WORKLOADS["tiny"],
    Workload("bf16_ragged", T=300, d=256, E=8, k=2, n_group=2, topk_group=1, inter=128,
             n_shared=1, dtype="bf16"),
    Workload("bf16_multi_tile", T=777, d=512, E=32, k=6, n_group=8, topk_group=4, inter=384,
             n_shared=1, dtype="bf16"),
    WORKLOADS["decode"],
    WORKLOADS["prefill"],
]
VARIANTS = [("softmax", False), ("sigmoid", True), ("softmax", True)]


@pytest.mark.parametrize("gate,with_bias", VARIANTS, ids=[f"{g}{'_bias' if b else ''}"
                                                          for g, b in VARIANTS])
@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_gating_variant_parity(w, gate, with_bias):
    inp = make_inputs(w)
    c = lambda t: None if t is None else t.to(DEV)
    x, Wr, Wgu, Wd, Wsh = c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down), c(inp.W_shared)
    bias = make_bias(w.E, gate) if with_bias else None
    bias_dev = torch.from_numpy(bias).to(DEV) if with_bias else None
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=DEV)
    wt = torch.empty(w.T, w.k, dtype=torch.float32, device=DEV)
    load = torch.full((w.E,), -1, dtype=torch.int32, device=DEV)
    ws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype)
    y = moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                    topk_idx=idx, topk_w=wt, workspace=ws, gate=gate, expert_bias=bias_dev,
                    expert_load=load)
    torch.cuda.synchronize()
    assert moe.device_status(ws)[0] == moe.MOE_OK
    ref = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group, score_func=gate,
                       bias=bias)
    gi, gw = idx.cpu().numpy(), wt.cpu().numpy()
    check_routing(gi, gw, ref, w.n_group, w.topk_group, w.E)
    np.testing.assert_array_equal(load.cpu().numpy(), np.bincount(gi.ravel(), minlength=w.E))
    tokens = np.arange(w.T, dtype=np.int32)  # every token
    y_ref = oracle_outputs(inp, w, tokens, gi[tokens], ref, score_func=gate, bias=bias)
    check_output(y.cpu().numpy()[tokens], y_ref, w.dtype)
    # the routing entry point takes the same options
    ri, rw = moe.route(x, Wr, w.k, w.n_group, w.topk_group, gate=gate, expert_bias=bias_dev)
    torch.cuda.synchronize()
    assert torch.equal(ri, idx) and torch.equal(rw, wt)


def test_bias_moves_load_to_the_favoured_expert():
    """A large bias on one expert puts it in every token's set; the weights
    still come from the unbiased scores (checked against the oracle)."""
    w = WORKLOADS["decode"]
    inp = make_inputs(w)
    x, Wr = inp.x.to(DEV), inp.W_router.to(DEV)
    bias = np.zeros(w.E, np.float32)
    bias[37] = 5.0
    idx, wt = moe.route(x, Wr, w.k, w.n_group, w.topk_group,
                        expert_bias=torch.from_numpy(bias).to(DEV))
    torch.cuda.synchronize()
    assert (idx.cpu().numpy()[:, 0] == 37).all()
    ref = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group, bias=bias)
    check_routing(idx.cpu().numpy(), wt.cpu().numpy(), ref, w.n_group, w.topk_group, w.E)


def test_invalid_gate_and_host_bias_rejected():
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    x, Wr = inp.x.to(DEV), inp.W_router.to(DEV)
    with pytest.raises(KeyError):
        moe.route(x, Wr, w.k, w.n_group, w.topk_group, gate="relu")
    with pytest.raises(moe.MoeError) as e:
        moe.route(x, Wr, w.k, w.n_group, w.topk_group, expert_bias=torch.zeros(w.E))
    assert e.value.status == moe.MOE_ERR_INVALID_ARG
