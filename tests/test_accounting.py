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
