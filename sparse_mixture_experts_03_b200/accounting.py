"""Algorithmic work of the MoE layer forward: FLOPs and bytes.

Counts follow the FFN accounting of the worked LLaMA-3-70B example in
"大模型工程（一）：Transformer 到 MoE", section "实战示例" (a SwiGLU FFN has
3*d*d_ffn weights and costs 2*3*d*d_ffn FLOPs per token), applied per chosen
expert, per shared expert, plus the 2*d*E router GEMM.
"""
from __future__ import annotations

import numpy as np


def ffn_params(d: int, inter: int) -> int:
    """Weights of one SwiGLU FFN (gate, up and down projections)."""
    return 3 * d * inter


def ffn_flops_per_token(d: int, inter: int) -> int:
    """FLOPs of one SwiGLU FFN on one token (one multiply-add per weight)."""
    return 2 * ffn_params(d, inter)


def flops_per_token(d: int, E: int, k: int, inter: int, n_shared: int) -> int:
    """Router GEMM + k routed experts + n_shared shared experts."""
    return 2 * d * E + (k + n_shared) * ffn_flops_per_token(d, inter)


def layer_flops(T: int, d: int, E: int, k: int, inter: int, n_shared: int) -> int:
    return T * flops_per_token(d, E, k, inter, n_shared)


def gate_up_flops(rows: int, d: int, inter: int) -> int:
    """Gate + up projections of `rows` (token, expert) rows."""
    return 2 * rows * d * 2 * inter


def down_flops(rows: int, d: int, inter: int) -> int:
    return 2 * rows * inter * d


def touched_experts(topk_idx: np.ndarray, E: int) -> int:
    return int(np.unique(np.asarray(topk_idx).ravel()).size) if np.asarray(topk_idx).size else 0


def layer_bytes(T: int, d: int, E: int, inter: int, n_shared: int, n_touched: int,
                in_bytes: int = 2, out_bytes: int = 4) -> int:
    """Algorithmic HBM bytes: each touched expert's weights once, the shared
    and router weights, x in and y out.  Permuted copies and intermediates
    are implementation traffic and are not counted."""
    w = (n_touched + n_shared) * ffn_params(d, inter) + E * d
    return w * in_bytes + T * d * in_bytes + T * d * out_bytes


# ---- training step (forward + backward of the layer)

def backward_flops_per_token(d: int, k: int, inter: int, n_shared: int) -> int:
    """FLOPs of the chain rule per token: for every chosen and shared expert
    the input-gradient GEMMs (W_down^T dy, W_gate_up^T [dg|du]) and the
    weight-gradient GEMMs, each with the FLOPs of the forward GEMM it mirrors
    (2x the expert's forward); the router gets gradients on the k chosen
    logits only: 2*d*k for dx and 2*d*k for dW_router."""
    return 2 * (k + n_shared) * ffn_flops_per_token(d, inter) + 4 * d * k


def train_step_flops(T: int, d: int, E: int, k: int, inter: int, n_shared: int) -> int:
    return T * (flops_per_token(d, E, k, inter, n_shared)
                + backward_flops_per_token(d, k, inter, n_shared))


def train_step_bytes(T: int, d: int, E: int, k: int, inter: int, n_shared: int,
                     n_touched: int) -> int:
    """Algorithmic HBM bytes of forward + backward: the touched experts',
    shared and router weights read twice (bf16), their gradients written once
    (fp32), x and dy read (bf16), y and dx written (fp32), and the saved gate /
    up pre-activations written and read back (bf16)."""
    w = (n_touched + n_shared) * ffn_params(d, inter) + E * d
    saved = 2 * inter * (T * k + T * n_shared) * 2
    return 2 * w * 2 + w * 4 + 2 * T * d * 2 + 2 * T * d * 4 + 2 * saved
