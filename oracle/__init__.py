"""CPU oracle for the fine-grained MoE layer (forward and backward) -- TEST
INFRASTRUCTURE ONLY.

Only tests/, the smoke check in __graft_entry__ and the benchmark's CPU-baseline
leg may import this package.  It never imports the CUDA package and the CUDA
package never imports it.

Two independent formulations live here:
  * moe_oracle.c (loaded through ctypes): the per-token sparse form, fp64,
    steps in the order the pages give them -- router, sigmoid, group limit,
    top-k, normalise, chosen SwiGLU experts, unweighted shared experts.
  * dense.py: the dense-mask form (every expert evaluated for every token and
    multiplied by a zero/weight gate matrix), numpy fp64, used on small shapes
    to cross-check the sparse form.

Inputs are torch CPU tensors in float32 or bfloat16 (the exact values given to
the GPU), or float64 (the finite-difference checks of the backward); outputs
are numpy float64 / int32 arrays.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

from . import build as _build

_LIB = None
OR_F32, OR_BF16, OR_F64 = 0, 1, 2


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        vp, i32, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p
        L.oracle_route.argtypes = [vp, vp, i32, i32, i32, i32, i32, i32, i32, i32, dp, dp, dp, dp,
                                   dp, dp, i32]
        L.oracle_route.restype = i32
        L.oracle_forward.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                     i32, i32, dp, dp, i32, dp, dp, dp, dp, i32]
        L.oracle_forward.restype = i32
        L.oracle_backward.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32, i32,
                                      i32, i32, dp, dp, vp, dp, dp, dp, dp, dp, dp, dp, i32]
        L.oracle_backward.restype = i32
        L.oracle_backward_rows.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, i32,
                                           i32, i32, i32, dp, dp, vp, dp, i32, dp, dp, i32, dp,
                                           i32, i32]
        L.oracle_backward_rows.restype = i32
        L.oracle_max_threads.restype = i32
        L.oracle_check_args.argtypes = [i32] * 6
        L.oracle_check_args.restype = i32
        _LIB = L
    return _LIB


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return OR_F32
    if t.dtype == torch.bfloat16:
        return OR_BF16
    if t.dtype == torch.float64:
        return OR_F64
    raise TypeError(f"oracle takes float32, bfloat16 or float64 tensors, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    assert t.device.type == "cpu" and t.is_contiguous()
    return ctypes.c_void_p(t.data_ptr())


def _np_ptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


SCORE_FUNCS = {"sigmoid": 0, "softmax": 1}


def _bias(bias, E):
    """Selection bias as a contiguous fp64 array (the exact fp32 values given to
    the GPU), or None."""
    if bias is None:
        return None
    b = np.ascontiguousarray(np.asarray(bias, dtype=np.float32).astype(np.float64))
    assert b.shape == (E,)
    return b


class Routing:
    """Oracle routing of T tokens: idx [T,k] int32 (descending key, ties to
    the lower index), w [T,k] fp64, scores [T,E] fp64 (selection keys: the
    gate score -- sigmoid, or the logit for softmax gating -- plus the
    selection bias), gap_e / gap_g [T] fp64 (key gap at the k-th expert
    boundary inside the kept groups, and at the topk_group-th group boundary)."""

    def __init__(self, idx, w, scores, gap_e, gap_g):
        self.idx, self.w, self.scores, self.gap_e, self.gap_g = idx, w, scores, gap_e, gap_g

    def near_tie(self, eps: float = 1e-4) -> np.ndarray:
        return (self.gap_e < eps) | (self.gap_g < eps)


def route(x: torch.Tensor, W_router: torch.Tensor, k: int, n_group: int, topk_group: int,
          with_scores: bool = True, nthreads: int = 0, score_func: str = "sigmoid",
          bias=None) -> Routing:
    """Steps 1-5 (router, gate, group limit, top-k, weights) for every token."""
    T, d = x.shape
    E = W_router.shape[0]
    assert W_router.shape[1] == d and W_router.dtype == x.dtype
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float64)
    scores = np.zeros((T, E), np.float64) if with_scores else None
    ge = np.zeros(T, np.float64)
    gg = np.zeros(T, np.float64)
    b = _bias(bias, E)
    rc = lib().oracle_route(_ptr(x), _ptr(W_router), _dt(x), T, d, E, k, n_group, topk_group,
                            SCORE_FUNCS[score_func], _np_ptr(b), _np_ptr(idx), _np_ptr(w),
                            _np_ptr(scores), _np_ptr(ge), _np_ptr(gg), nthreads)
    if rc != 0:
        raise ValueError("oracle_route: invalid arguments")
    return Routing(idx, w, scores, ge, gg)


def forward(x: torch.Tensor, W_router: torch.Tensor, W_gate_up: torch.Tensor,
            W_down: torch.Tensor, W_shared: Optional[torch.Tensor], k: int, n_group: int,
            topk_group: int, inter: int, n_shared: int, tokens=None, forced_idx=None,
            nthreads: int = 0, score_func: str = "sigmoid", bias=None):
    """Full layer forward (steps 1-7) for the listed tokens (default: all).

    Returns (y [n,d] fp64, idx [n,k] int32, w [n,k] fp64).  With forced_idx
    [n,k], that expert set is used in place of the oracle's own top-k.
    """
    T, d = x.shape
    E = W_router.shape[0]
    dt = _dt(x)
    for t in (W_router, W_gate_up, W_down) + ((W_shared,) if W_shared is not None else ()):
        assert t.dtype == x.dtype and t.is_contiguous()
    assert W_gate_up.numel() == E * 2 * inter * d and W_down.numel() == E * d * inter
    if n_shared:
        assert W_shared is not None and W_shared.numel() == 3 * n_shared * inter * d
    if tokens is None:
        tokens = np.arange(T, dtype=np.int32)
    tokens = np.ascontiguousarray(np.asarray(tokens, dtype=np.int32))
    n = len(tokens)
    y = np.zeros((n, d), np.float64)
    idx = np.zeros((n, k), np.int32)
    w = np.zeros((n, k), np.float64)
    fi = None
    if forced_idx is not None:
        fi = np.ascontiguousarray(np.asarray(forced_idx, dtype=np.int32))
        assert fi.shape == (n, k)
    b = _bias(bias, E)
    rc = lib().oracle_forward(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                              _ptr(W_shared), dt, T, d, E, k, n_group, topk_group, inter,
                              n_shared, SCORE_FUNCS[score_func], _np_ptr(b), _np_ptr(tokens), n,
                              _np_ptr(fi), _np_ptr(y), _np_ptr(idx), _np_ptr(w), nthreads)
    if rc != 0:
        raise ValueError("oracle_forward: invalid arguments")
    return y, idx, w


def check_args(T, d, E, k, n_group, topk_group) -> bool:
    return lib().oracle_check_args(T, d, E, k, n_group, topk_group) == 0


def _check_layer(x, W_router, W_gate_up, W_down, W_shared, inter, n_shared):
    E = W_router.shape[0]
    d = x.shape[1]
    for t in (W_router, W_gate_up, W_down) + ((W_shared,) if W_shared is not None else ()):
        assert t.dtype == x.dtype and t.is_contiguous()
    assert W_gate_up.numel() == E * 2 * inter * d and W_down.numel() == E * d * inter
    if n_shared:
        assert W_shared is not None and W_shared.numel() == 3 * n_shared * inter * d
    return E, d


def _forced(forced_idx, T, k):
    if forced_idx is None:
        return None
    fi = np.ascontiguousarray(np.asarray(forced_idx, dtype=np.int32))
    assert fi.shape == (T, k)
    return fi


class Grads:
    """Gradients of the layer, fp64, in the layouts of the forward's tensors:
    dx [T,d], dW_router [E,d], dW_gate_up [E,2I,d], dW_down [E,d,I],
    dW_shared [3*SI*d] (gate_up block then down block) or None; idx [T,k] the
    expert sets used and dl [T,k] = dL/dlogit of the chosen experts."""

    def __init__(self, **kw):
        self.__dict__.update(kw)


def backward(x, W_router, W_gate_up, W_down, W_shared, dy, k, n_group, topk_group, inter,
             n_shared, forced_idx=None, nthreads: int = 0, score_func: str = "sigmoid",
             bias=None) -> Grads:
    """Gradients of L = sum(dy * y) with respect to x and every weight (the
    chain rule through steps 1-7, written out in moe_oracle.c).  dy has the
    dtype of x.  forced_idx [T,k]: expert sets used in place of the oracle's
    own top-k."""
    T = x.shape[0]
    E, d = _check_layer(x, W_router, W_gate_up, W_down, W_shared, inter, n_shared)
    assert dy.shape == x.shape and dy.dtype == x.dtype and dy.is_contiguous()
    I, SI = inter, n_shared * inter
    dx = np.zeros((T, d))
    dWr = np.zeros((E, d))
    dWgu = np.zeros((E, 2 * I, d))
    dWd = np.zeros((E, d, I))
    dWsh = np.zeros(3 * SI * d) if n_shared else None
    idx = np.zeros((T, k), np.int32)
    dl = np.zeros((T, k))
    rc = lib().oracle_backward(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                               _ptr(W_shared), _dt(x), T, d, E, k, n_group, topk_group, I,
                               n_shared, SCORE_FUNCS[score_func], _np_ptr(_bias(bias, E)),
                               _np_ptr(_forced(forced_idx, T, k)), _ptr(dy), _np_ptr(dx),
                               _np_ptr(dWr), _np_ptr(dWgu), _np_ptr(dWd), _np_ptr(dWsh),
                               _np_ptr(idx), _np_ptr(dl), nthreads)
    if rc != 0:
        raise ValueError("oracle_backward: invalid arguments")
    return Grads(dx=dx, dW_router=dWr, dW_gate_up=dWgu, dW_down=dWd, dW_shared=dWsh, idx=idx,
                 dl=dl)


# tensor ids of backward_rows
ROW_DWR, ROW_DWGU, ROW_DWD, ROW_DWSH_GU, ROW_DWSH_DN = 0, 1, 2, 3, 4


def backward_rows(x, W_router, W_gate_up, W_down, W_shared, dy, k, n_group, topk_group, inter,
                  n_shared, dx_tokens=(), wsel=(), forced_idx=None, nthreads: int = 0,
                  score_func: str = "sigmoid", bias=None):
    """Selected entries of the backward at any size, each computed on its own:
    dx rows of dx_tokens, and weight-gradient rows wsel = [(tensor id, row)]
    (ROW_* ids; rows in the flattened [rows, cols] view of each gradient).
    Returns (dx_rows [n, d], [row arrays])."""
    T = x.shape[0]
    E, d = _check_layer(x, W_router, W_gate_up, W_down, W_shared, inter, n_shared)
    assert dy.shape == x.shape and dy.dtype == x.dtype and dy.is_contiguous()
    I, SI = inter, n_shared * inter
    toks = np.ascontiguousarray(np.asarray(dx_tokens, dtype=np.int32).reshape(-1))
    ws = np.ascontiguousarray(np.asarray(wsel, dtype=np.int32).reshape(-1, 2))
    ld = max(d, I, SI)
    dxr = np.zeros((len(toks), d))
    wr = np.zeros((len(ws), ld))
    rc = lib().oracle_backward_rows(_ptr(x), _ptr(W_router), _ptr(W_gate_up), _ptr(W_down),
                                    _ptr(W_shared), _dt(x), T, d, E, k, n_group, topk_group, I,
                                    n_shared, SCORE_FUNCS[score_func], _np_ptr(_bias(bias, E)),
                                    _np_ptr(_forced(forced_idx, T, k)), _ptr(dy),
                                    _np_ptr(toks), len(toks), _np_ptr(dxr), _np_ptr(ws), len(ws),
                                    _np_ptr(wr), ld, nthreads)
    if rc != 0:
        raise ValueError("oracle_backward_rows: invalid arguments")
    lens = {ROW_DWR: d, ROW_DWGU: d, ROW_DWD: I, ROW_DWSH_GU: d, ROW_DWSH_DN: SI}
    return dxr, [wr[i, :lens[int(t)]].copy() for i, (t, _) in enumerate(ws)]
