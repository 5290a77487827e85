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
