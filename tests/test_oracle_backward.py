"""Pins of the oracle's backward (CPU only).

The backward in oracle/moe_oracle.c is the chain rule written out by hand.  It
is pinned here against things that do not share that derivation:

* central finite differences of the oracle's *forward* (fp64 inputs), for the
  scalar loss L = sum(dy * y), along a random direction in every input tensor;
* torch autograd through a separate torch fp64 expression of the layer, given
  the same expert sets (the library differentiates; nothing is re-derived);
* closed-form invariants of the gate normalisation: the sigmoid weights
  s_j / sum s are unchanged by scaling every chosen s_j, so
  sum_j dL/ds_j * s_j = 0, i.e. sum_j dl_j / (1 - s_j) = 0; the softmax weights
  are unchanged by shifting every chosen logit, so sum_j dl_j = 0;
* the sampled-rows variant (used at full sizes) against the full backward.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

SHAPE = dict(T=24, d=64, E=8, k=2, n_group=2, topk_group=1, inter=32, n_shared=2)


def make(seed=0, dtype=torch.float64, T=None, **over):
    p = dict(SHAPE, **over)
    if T is not None:
        p["T"] = T
    g = torch.Generator().manual_seed(seed)
    T, d, E, I, S = p["T"], p["d"], p["E"], p["inter"], p["n_shared"]
    r = lambda *s, sc=1.0: (torch.randn(*s, generator=g, dtype=torch.float64) * sc).to(dtype)
    t = dict(x=r(T, d), W_router=r(E, d, sc=d ** -0.5), W_gate_up=r(E, 2 * I, d, sc=d ** -0.5),
             W_down=r(E, d, I, sc=I ** -0.5),
             W_shared=r(3 * S * I * d, sc=d ** -0.5) if S else None, dy=r(T, d))
    return p, t


def loss(p, t, score_func="sigmoid", bias=None, forced=None):
    y, idx, _ = oracle.forward(t["x"], t["W_router"], t["W_gate_up"], t["W_down"], t["W_shared"],
                               p["k"], p["n_group"], p["topk_group"], p["inter"], p["n_shared"],
                               score_func=score_func, bias=bias, forced_idx=forced)
    return float((t["dy"].numpy() * y).sum()), idx


def grads(p, t, **kw):
    return oracle.backward(t["x"], t["W_router"], t["W_gate_up"], t["W_down"], t["W_shared"],
                           t["dy"], p["k"], p["n_group"], p["topk_group"], p["inter"],
                           p["n_shared"], **kw)


GRAD_OF = {"x": "dx", "W_router": "dW_router", "W_gate_up": "dW_gate_up", "W_down": "dW_down",
           "W_shared": "dW_shared"}


@pytest.mark.parametrize("score_func,with_bias", [("sigmoid", False), ("softmax", False),
                                                  ("sigmoid", True)])
def test_backward_matches_central_differences_of_forward(score_func, with_bias):
    p, t = make(seed=1)
    bias = np.linspace(-0.05, 0.05, p["E"]).astype(np.float32) if with_bias else None
    G = grads(p, t, score_func=score_func, bias=bias)
    _, idx0 = loss(p, t, score_func, bias)
    np.testing.assert_array_equal(idx0, G.idx)
    gen = torch.Generator().manual_seed(7)
    eps = 1e-5
    for name, gname in GRAD_OF.items():
        V = torch.randn(t[name].shape, generator=gen, dtype=torch.float64)
        tp, tm = dict(t), dict(t)
        tp[name] = (t[name] + eps * V).contiguous()
        tm[name] = (t[name] - eps * V).contiguous()
        Lp, ip = loss(p, tp, score_func, bias)
        Lm, im = loss(p, tm, score_func, bias)
        # the selection must not move inside +-eps (it passes no gradient)
        np.testing.assert_array_equal(ip, idx0)
        np.testing.assert_array_equal(im, idx0)
        fd = (Lp - Lm) / (2 * eps)
        an = float((getattr(G, gname) * V.numpy().reshape(getattr(G, gname).shape)).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def torch_layer(t, idx, p, score_func):
    """The layer forward as plain torch fp64 ops with the expert sets fixed to
    idx, for autograd."""
    x, Wr, Wgu, Wd, Wsh = t["x"], t["W_router"], t["W_gate_up"], t["W_down"], t["W_shared"]
    T, d = x.shape
    I, S = p["inter"], p["n_shared"]
    idx = torch.as_tensor(idx, dtype=torch.int64)
    logits = x @ Wr.T
    if score_func == "sigmoid":
        chosen = torch.gather(torch.sigmoid(logits), 1, idx)
        w = chosen / chosen.sum(dim=1, keepdim=True)
    else:
        w = torch.softmax(torch.gather(logits, 1, idx), dim=1)
    y = torch.zeros(T, d, dtype=torch.float64)
    for e in range(Wr.shape[0]):
        tok, slot = torch.nonzero(idx == e, as_tuple=True)
        if len(tok) == 0:
            continue
        xe = x[tok]
        hid = F.silu(xe @ Wgu[e, :I].T) * (xe @ Wgu[e, I:].T)
        y = y.index_add(0, tok, w[tok, slot].unsqueeze(1) * (hid @ Wd[e].T))
    if S:
        SI = S * I
        gu = Wsh[: 2 * SI * d].reshape(2 * SI, d)
        dn = Wsh[2 * SI * d:].reshape(d, SI)
        y = y + (F.silu(x @ gu[:SI].T) * (x @ gu[SI:].T)) @ dn.T
    return y


@pytest.mark.parametrize("score_func,forced", [("sigmoid", False), ("softmax", False),
                                               ("sigmoid", True)])
def test_backward_matches_torch_autograd(score_func, forced):
    p, t = make(seed=2, T=40)
    fi = None
    if forced:
        # arbitrary distinct sets (not the top-k): the forced-set path
        g = np.random.default_rng(3)
        fi = np.stack([g.choice(p["E"], p["k"], replace=False) for _ in range(p["T"])]).astype(
            np.int32)
    G = grads(p, t, score_func=score_func, forced_idx=fi)
    leaves = {n: t[n].clone().requires_grad_(True) for n in GRAD_OF}
    y = torch_layer(leaves, G.idx, p, score_func)
    L = (t["dy"] * y).sum()
    auto = torch.autograd.grad(L, [leaves[n] for n in GRAD_OF])
    for (name, gname), ref in zip(GRAD_OF.items(), auto):
        got = getattr(G, gname)
        np.testing.assert_allclose(got, ref.numpy().reshape(got.shape), rtol=1e-9,
                                   atol=1e-11 * max(1.0, float(ref.abs().max())), err_msg=name)


@pytest.mark.parametrize("score_func", ["sigmoid", "softmax"])
def test_gate_normalisation_invariants(score_func):
    p, t = make(seed=4, T=64, E=16, k=4, n_group=4, topk_group=2)
    G = grads(p, t, score_func=score_func)
    if score_func == "sigmoid":
        s = 1 / (1 + np.exp(-(t["x"].numpy() @ t["W_router"].numpy().T)))
        s_sel = np.take_along_axis(s, G.idx.astype(np.int64), axis=1)
        resid = (G.dl / (1 - s_sel)).sum(axis=1)
        scale = np.abs(G.dl / (1 - s_sel)).sum(axis=1)
    else:
        resid = G.dl.sum(axis=1)
        scale = np.abs(G.dl).sum(axis=1)
    assert np.all(np.abs(resid) <= 1e-12 * np.maximum(scale, 1e-300) + 1e-300)
    assert np.abs(G.dl).max() > 0  # not trivially zero


def test_no_router_gradient_with_one_expert_per_token():
    # k = 1: the single weight is 1 whatever the score, so dL/dl = 0 and the
    # router gets no gradient; dx is then the chosen experts' and shared part
    p, t = make(seed=5, k=1, n_group=1, topk_group=1)
    G = grads(p, t)
    assert np.all(G.dl == 0) and np.all(G.dW_router == 0)


def test_sampled_rows_match_full_backward():
    p, t = make(seed=6, T=30)
    G = grads(p, t)
    E, I, d, SI = p["E"], p["inter"], p["d"], p["n_shared"] * p["inter"]
    wsel = [(oracle.ROW_DWR, 3), (oracle.ROW_DWGU, 5 * 2 * I + 7),
            (oracle.ROW_DWGU, 1 * 2 * I + I + 4), (oracle.ROW_DWD, 2 * d + 11),
            (oracle.ROW_DWSH_GU, 9), (oracle.ROW_DWSH_GU, SI + 3), (oracle.ROW_DWSH_DN, 17)]
    toks = [0, 13, 29]
    dxr, rows = oracle.backward_rows(t["x"], t["W_router"], t["W_gate_up"], t["W_down"],
                                     t["W_shared"], t["dy"], p["k"], p["n_group"],
                                     p["topk_group"], I, p["n_shared"], dx_tokens=toks,
                                     wsel=wsel)
    np.testing.assert_allclose(dxr, G.dx[toks], rtol=1e-12, atol=1e-13)
    gu = G.dW_gate_up.reshape(E * 2 * I, d)
    dn = G.dW_down.reshape(E * d, I)
    sh_gu = G.dW_shared[: 2 * SI * d].reshape(2 * SI, d)
    sh_dn = G.dW_shared[2 * SI * d:].reshape(d, SI)
    full = {oracle.ROW_DWR: G.dW_router, oracle.ROW_DWGU: gu, oracle.ROW_DWD: dn,
            oracle.ROW_DWSH_GU: sh_gu, oracle.ROW_DWSH_DN: sh_dn}
    for (ten, r), row in zip(wsel, rows):
        np.testing.assert_allclose(row, full[ten][r], rtol=1e-12, atol=1e-13)


def test_bf16_inputs_read_exactly():
    # bf16 inputs are read as their exact values: same gradients as the fp64
    # copies of those values
    p, t = make(seed=8, dtype=torch.bfloat16)
    t64 = {n: (v.to(torch.float64) if v is not None else None) for n, v in t.items()}
    a, b = grads(p, t), grads(p, t64)
    for gname in GRAD_OF.values():
        np.testing.assert_array_equal(getattr(a, gname), getattr(b, gname))
