"""Dense-mask formulation of the MoE layer forward -- TEST INFRASTRUCTURE ONLY.

A second, independent way of writing the same layer, used only on small shapes
to cross-check the per-token sparse oracle in moe_oracle.c: every expert is
evaluated on every token and the results are combined through a [T, E] gate
matrix that is zero outside each token's chosen experts.  This is the
boolean-mask view of the MoEBlock listing in "大模型工程（一）：Transformer 到
MoE", section "混合专家：更多参数，相同 FLOPs", with the gate changed to the
bias-free sigmoid and group-limited routing of "FusionLLM：融合 MLA、GDN 与
MoE 的高效混合架构大模型训练框架", section "混合专家（MoE）".

Selection here is by stable sorting (numpy argsort, kind="stable"), not by the
repeated argmax of moe_oracle.c; ties still go to the lower index.
numpy fp64 throughout.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch


def _f64(t: Optional[torch.Tensor]) -> Optional[np.ndarray]:
    return None if t is None else t.to(torch.float64).numpy()


def _silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def gate_matrix(x64: np.ndarray, Wr64: np.ndarray, k: int, n_group: int, topk_group: int):
    """[T,E] matrix: normalised sigmoid weight on each token's chosen experts, 0 elsewhere."""
    T = x64.shape[0]
    E = Wr64.shape[0]
    s = 1.0 / (1.0 + np.exp(-(x64 @ Wr64.T)))                       # [T,E]
    gs = s.reshape(T, n_group, E // n_group).max(axis=2)            # [T,G]
    g_order = np.argsort(-gs, axis=1, kind="stable")[:, :topk_group]
    gmask = np.zeros((T, n_group), bool)
    np.put_along_axis(gmask, g_order, True, axis=1)
    emask = np.repeat(gmask, E // n_group, axis=1)                  # [T,E]
    masked = np.where(emask, s, -np.inf)
    e_order = np.argsort(-masked, axis=1, kind="stable")[:, :k]
    sel = np.zeros((T, E), bool)
    np.put_along_axis(sel, e_order, True, axis=1)
    gm = np.where(sel, s, 0.0)
    gm = gm / gm.sum(axis=1, keepdims=True)
    return gm, e_order


def forward_dense(x, W_router, W_gate_up, W_down, W_shared, k, n_group, topk_group, inter,
                  n_shared):
    """y [T,d] fp64 via every expert on every token and the [T,E] gate matrix."""
    x64, Wr, Wgu, Wd = _f64(x), _f64(W_router), _f64(W_gate_up), _f64(W_down)
    T, d = x64.shape
    E = Wr.shape[0]
    I = inter
    gm, _ = gate_matrix(x64, Wr, k, n_group, topk_group)
    y = np.zeros((T, d))
    for e in range(E):
        hid = _silu(x64 @ Wgu[e, :I].T) * (x64 @ Wgu[e, I:].T)     # [T,I]
        y += gm[:, e:e + 1] * (hid @ Wd[e].T)
    if n_shared:
        Wsh = _f64(W_shared)
        SI = n_shared * I
        gu = Wsh[: 2 * SI * d].reshape(2 * SI, d)
        dn = Wsh[2 * SI * d:].reshape(d, SI)
        hid = _silu(x64 @ gu[:SI].T) * (x64 @ gu[SI:].T)           # [T,SI]
        y += hid @ dn.T
    return y
