"""Pins of the FLOP / byte accounting and of the workload shapes."""
import json
import os

import pytest

from sparse_mixture_experts_03_b200 import accounting
from sparse_mixture_experts_03_b200.inputs import WORKLOADS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_ffn_accounting_matches_worked_70b_example():
    g = load("ffn_accounting_70b.json")
    p = accounting.ffn_params(g["d_model"], g["d_ffn"])
    f = accounting.ffn_flops_per_token(g["d_model"], g["d_ffn"])
    assert abs(p - g["ffn_params_per_layer"]) / g["ffn_params_per_layer"] < g["ffn_params_rel_tol"]
    assert abs(f - g["ffn_flops_per_token"]) / g["ffn_flops_per_token"] < g["ffn_flops_rel_tol"]


def test_workloads_match_fusionllm_config():
    g = load("fusionllm_moe_config.json")
    for name in ("prefill", "train", "decode", "skewed"):
        w = WORKLOADS[name]
        assert (w.d, w.E, w.k, w.n_shared, w.inter) == (
            g["dim"], g["n_routed_experts"], g["n_activated_experts"], g["n_shared_experts"],
            g["moe_inter_dim"])
    assert WORKLOADS["prefill"].T == g["max_seq_len"]
    assert WORKLOADS["train"].T == 8 * g["max_seq_len"]


@pytest.mark.parametrize("d,E,k,I,S", [(2048, 64, 6, 1536, 4), (128, 8, 2, 256, 0),
                                       (64, 16, 3, 32, 2)])
def test_flop_counter_equals_gemm_enumeration(d, E, k, I, S):
    """p8: the closed form equals 2*M*N*K summed over every GEMM the layer
    performs on one token (router, k x (gate, up, down), S x (gate, up, down))."""
    gemms = [(1, E, d)]
    for _ in range(k + S):
        gemms += [(1, I, d), (1, I, d), (1, d, I)]
    total = sum(2 * m * n * kk for m, n, kk in gemms)
    assert accounting.flops_per_token(d, E, k, I, S) == total
    # FusionLLM layer: 189.0 MFLOP per token
    if (d, E, k, I, S) == (2048, 64, 6, 1536, 4):
        assert abs(total / 1e6 - 189.0) < 0.1


@pytest.mark.parametrize("d,E,k,I,S", [(2048, 64, 6, 1536, 4), (256, 8, 2, 256, 1)])
def test_training_step_flops_equal_gemm_enumeration(d, E, k, I, S):
    """The training step's FLOPs per token: the forward's GEMMs plus, per
    chosen and shared expert, the input-gradient GEMMs (dh = W_down^T dy,
    dx = W_gate^T dg + W_up^T du) and the weight-gradient GEMMs (dW_down,
    dW_gate, dW_up), each with the shape of the forward GEMM it mirrors; and
    for the router the gradient of the k chosen logits only (dx and
    dW_router: 2*d*k each)."""
    fwd = [(1, E, d)]
    bwd = []
    for _ in range(k + S):
        fwd += [(1, I, d), (1, I, d), (1, d, I)]
        bwd += [(1, I, d), (1, d, I), (1, d, I)]          # dh; dx from dg and du
        bwd += [(d, I, 1), (I, d, 1), (I, d, 1)]          # dW_down, dW_gate, dW_up
    bwd += [(1, d, k), (k, d, 1)]                         # router: dx, dW_router
    per_token = sum(2 * m * n * kk for m, n, kk in fwd + bwd)
    T = 1000
    assert accounting.train_step_flops(T, d, E, k, I, S) == T * per_token
    # forward + backward of the FusionLLM layer ≈ 3x the forward's expert work
    if (d, E, k, I, S) == (2048, 64, 6, 1536, 4):
        assert abs(per_token / accounting.flops_per_token(d, E, k, I, S) - 3.0) < 0.01


def test_training_step_bytes():
    T, d, E, k, I, S = 4096, 2048, 64, 6, 1536, 4
    w = (E + S) * 3 * d * I + E * d        # every expert touched, plus shared and router
    saved = 2 * I * (T * k + T * S) * 2    # bf16 gate | up per routed slot and shared row
    want = 2 * w * 2 + w * 4 + 2 * T * d * 2 + 2 * T * d * 4 + 2 * saved
    assert accounting.train_step_bytes(T, d, E, k, I, S, E) == want
