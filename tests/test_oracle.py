"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these compare the oracle with itself: every expected value comes from
brute force, a closed form worked by hand, a special case that reduces to a
library routine (torch fp64 matmul / sigmoid / silu), an invariant, or the
independent dense-mask formulation.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import dense


def rand_case(T, d, E, I, S, dtype=torch.float32, seed=0, router_scale=1.0):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(T, d, generator=g)
    Wr = torch.randn(E, d, generator=g) * router_scale / math.sqrt(d)
    Wgu = torch.randn(E, 2 * I, d, generator=g) / math.sqrt(d)
    Wd = torch.randn(E, d, I, generator=g) / math.sqrt(I)
    Wsh = None
    if S:
        Wsh = torch.cat([(torch.randn(2 * S * I, d, generator=g) / math.sqrt(d)).reshape(-1),
                         (torch.randn(d, S * I, generator=g) / math.sqrt(I)).reshape(-1)])
    cast = lambda t: None if t is None else t.to(dtype).contiguous()
    return cast(x), cast(Wr), cast(Wgu), cast(Wd), cast(Wsh)


def swiglu_lib(x64, Wg, Wu, Wdn):
    """Dense SwiGLU FFN written with torch library routines (fp64)."""
    return (F.silu(x64 @ Wg.T) * (x64 @ Wu.T)) @ Wdn.T


def brute_force_select(s, G, TG, k):
    """Best (group subset, expert subset) by exhaustive enumeration.

    Group-limited routing keeps the TG groups of largest max-score and then
    the k largest scores inside them.  As an optimisation: the kept group
    subset is the one of largest total group score, and the chosen expert
    subset is the one of largest total score among the kept groups' experts.
    Exact ties in the total fall back to the lower indices.  Returns the
    chosen experts in descending score order (ties: lower index first).
    """
    E = len(s)
    gsz = E // G
    gs = [max(s[g * gsz:(g + 1) * gsz]) for g in range(G)]

    def key(vals, comb):
        return (sum(vals[i] for i in comb), sorted(((vals[i], -i) for i in comb), reverse=True))

    best_groups = max(itertools.combinations(range(G), TG), key=lambda c: key(gs, c))
    cand = [e for e in range(E) if e // gsz in set(best_groups)]
    best = max(itertools.combinations(cand, k), key=lambda c: key(s, c))
    return sorted(best, key=lambda e: (-s[e], e))


@pytest.mark.parametrize("E,G,TG,k", [(8, 1, 1, 2), (8, 2, 1, 3), (8, 2, 2, 5), (8, 4, 2, 3),
                                      (8, 4, 3, 4), (6, 3, 2, 2), (4, 4, 4, 4), (8, 8, 3, 3)])
def test_routing_brute_force(E, G, TG, k):
    """p1/p6: the oracle's choice is the exhaustive optimum, scores from torch."""
    T, d = 40, 16
    x, Wr, *_ = rand_case(T, d, E, 8, 0, seed=E * 100 + G * 10 + k, router_scale=3.0)
    r = oracle.route(x, Wr, k, G, TG)
    s = torch.sigmoid(x.double() @ Wr.double().T).numpy()
    np.testing.assert_allclose(r.scores, s, rtol=0, atol=1e-15)
    logits = (x.double() @ Wr.double().T).numpy()
    for t in range(T):
        want = brute_force_select(list(s[t]), G, TG, k)
        assert list(r.idx[t]) == want, (t, r.idx[t], want)
        # selecting on logits picks the same ordered set (sigmoid is monotone)
        assert brute_force_select(list(logits[t]), G, TG, k) == want
        np.testing.assert_allclose(r.w[t], s[t, want] / s[t, want].sum(), rtol=1e-14)


def test_routing_ties_go_to_lower_index():
    """o7: exact ties are broken toward the lower expert / group index."""
    E, G, TG, k, d = 8, 4, 2, 3, 8
    x = torch.zeros(3, d)
    x[:, 0] = 1.0
    Wr = torch.zeros(E, d)
    # token logits are Wr[:, 0]; all groups tie at the group level for token 0
    Wr[:, 0] = torch.tensor([1.0, 0.5, 1.0, 0.5, 1.0, 0.5, 1.0, 0.5])
    r = oracle.route(x[:1].contiguous(), Wr, k, G, TG)
    # groups 0 and 1 kept (lower index wins the group tie), experts 0,2 (score
    # s(1)) then 1 (lower index among the two s(0.5))
    assert list(r.idx[0]) == [0, 2, 1]
    assert r.gap_g[0] == 0.0
    s = brute_force_select([float(torch.sigmoid(v)) for v in Wr[:, 0].double()], G, TG, k)
    assert s == [0, 2, 1]


def test_routing_handworked_closed_form():
    """Hand-derived two-token example, exact logits chosen so the sigmoid
    values are rationals: sigma(ln a) = a / (1 + a)."""
    d, E, G, TG, k, I = 2, 4, 2, 1, 2, 1
    ln = math.log
    # token 0 = e_0 sees logits column 0, token 1 = e_1 sees column 1
    Wr = torch.tensor([[ln(3), ln(9)],
                       [0.0, ln(4)],
                       [ln(7), 0.0],
                       [-ln(7), -ln(3)]], dtype=torch.float64)
    x = torch.eye(2, dtype=torch.float64)
    # the oracle reads fp32; keep the exact fp32 values for the closed form
    x32, Wr32 = x.float().contiguous(), Wr.float().contiguous()
    r = oracle.route(x32, Wr32, k, G, TG)
    sig = lambda z: 1.0 / (1.0 + math.exp(-z))
    l = Wr32.double()
    # token 0: scores (3/4, 1/2, 7/8, 1/8); group maxima 3/4 vs 7/8 -> group 1;
    # experts 2 then 3; weights 7/8 and 1/8 (they already sum to 1).  Plain
    # top-2 without the group limit would have picked experts 2 and 0.
    assert list(r.idx[0]) == [2, 3]
    s2, s3 = sig(float(l[2, 0])), sig(float(l[3, 0]))
    np.testing.assert_allclose(r.w[0], [s2 / (s2 + s3), s3 / (s2 + s3)], rtol=1e-15)
    np.testing.assert_allclose(r.w[0], [7 / 8, 1 / 8], rtol=1e-6)
    # token 1: scores (9/10, 4/5, 1/2, 1/4); group 0 kept; weights 9/17, 8/17
    assert list(r.idx[1]) == [0, 1]
    np.testing.assert_allclose(r.w[1], [9 / 17, 8 / 17], rtol=1e-6)

    # experts with inter 1: gate row a, up row b, down column c
    Wgu = torch.zeros(E, 2, d)
    Wd = torch.zeros(E, d, 1)
    Wgu[2, 0] = torch.tensor([ln(3), 0.0]); Wgu[2, 1] = torch.tensor([2.0, 0.0])
    Wd[2, :, 0] = torch.tensor([1.0, -1.0])
    Wgu[3, 0] = torch.tensor([-ln(3), 0.0]); Wgu[3, 1] = torch.tensor([4.0, 0.0])
    Wd[3, :, 0] = torch.tensor([2.0, 0.0])
    Wgu[0, 0] = torch.tensor([0.0, ln(9)]); Wgu[0, 1] = torch.tensor([0.0, 1.0])
    Wd[0, :, 0] = torch.tensor([1.0, 1.0])
    Wgu[1, 0] = torch.tensor([0.0, 0.0]); Wgu[1, 1] = torch.tensor([0.0, 5.0])
    Wd[1, :, 0] = torch.tensor([3.0, 3.0])
    y, idx, w = oracle.forward(x32, Wr32, Wgu.contiguous(), Wd.contiguous(), None, k, G, TG,
                               I, 0)
    # token 0: expert 2: silu(ln3) = ln3 * 3/4, times up 2 -> h = 1.5 ln3,
    # down (1,-1); expert 3: silu(-ln3) = -ln3 / 4, times up 4 -> h = -ln3,
    # down (2, 0).  y = 7/8 (1.5ln3, -1.5ln3) + 1/8 (-2ln3, 0)
    L3 = ln(3)
    np.testing.assert_allclose(y[0], [L3 * (7 / 8 * 1.5 - 2 / 8), -L3 * 7 / 8 * 1.5],
                               rtol=2e-6)
    # token 1: expert 0: silu(ln9) * 1 = 0.9 ln9, down (1,1), weight 9/17;
    # expert 1: silu(0) = 0 contributes nothing
    np.testing.assert_allclose(y[1], [9 / 17 * 0.9 * ln(9)] * 2, rtol=2e-6)


def test_weights_sum_to_one():
    """p3: normalised gate weights sum to 1 for every token."""
    x, Wr, *_ = rand_case(200, 32, 16, 8, 0, seed=3, router_scale=2.0)
    r = oracle.route(x, Wr, 5, 4, 2)
    np.testing.assert_allclose(r.w.sum(axis=1), 1.0, atol=1e-12)
    assert (r.w > 0).all()
    # descending score order
    sel = np.take_along_axis(r.scores, r.idx.astype(np.int64), axis=1)
    assert (np.diff(sel, axis=1) <= 0).all()


def test_k_equals_E_uniform_is_dense_mean():
    """p2: k = E, one group, zero router -> every score 1/2, every weight 1/E,
    so y is the plain mean of all experts' SwiGLU outputs."""
    T, d, E, I = 6, 24, 4, 12
    x, _, Wgu, Wd, _ = rand_case(T, d, E, I, 0, seed=5)
    Wr = torch.zeros(E, d)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, None, E, 1, 1, I, 0)
    np.testing.assert_allclose(w, 1.0 / E, rtol=0, atol=1e-15)
    x64 = x.double()
    want = sum(swiglu_lib(x64, Wgu[e, :I].double(), Wgu[e, I:].double(), Wd[e].double())
               for e in range(E)) / E
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_single_expert_is_dense_swiglu(dtype):
    """p4: E = 1, k = 1, no shared experts -> the layer is one dense SwiGLU FFN."""
    T, d, I = 9, 40, 24
    x, Wr, Wgu, Wd, _ = rand_case(T, d, 1, I, 0, dtype=dtype, seed=7)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, None, 1, 1, 1, I, 0)
    assert (idx == 0).all() and np.allclose(w, 1.0)
    want = swiglu_lib(x.double(), Wgu[0, :I].double(), Wgu[0, I:].double(), Wd[0].double())
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-12)


def test_forward_matches_library_composition():
    """The layer output is sum_j w_j * SwiGLU_{e_j}(x) + sum_s SwiGLU_s(x):
    routing by brute force, experts by torch library routines."""
    T, d, E, I, S, G, TG, k = 12, 32, 8, 16, 2, 4, 2, 3
    x, Wr, Wgu, Wd, Wsh = rand_case(T, d, E, I, S, seed=11, router_scale=2.0)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, Wsh, k, G, TG, I, S)
    x64 = x.double()
    s = torch.sigmoid(x64 @ Wr.double().T)
    SI = S * I
    gu = Wsh[: 2 * SI * d].view(2 * SI, d).double()
    dn = Wsh[2 * SI * d:].view(d, SI).double()
    for t in range(T):
        sel = brute_force_select(list(s[t].numpy()), G, TG, k)
        ws = s[t, sel] / s[t, sel].sum()
        xt = x64[t:t + 1]
        want = sum(ws[j] * swiglu_lib(xt, Wgu[e, :I].double(), Wgu[e, I:].double(),
                                      Wd[e].double()) for j, e in enumerate(sel))
        for sh in range(S):
            want = want + swiglu_lib(xt, gu[sh * I:(sh + 1) * I], gu[SI + sh * I:SI + (sh + 1) * I],
                                     dn[:, sh * I:(sh + 1) * I])
        np.testing.assert_allclose(y[t], want[0].numpy(), rtol=1e-11, atol=1e-12)


def test_shared_experts_add_unweighted():
    """p5: adding shared experts adds exactly the sum of their dense SwiGLU
    outputs (routed part unchanged), and S experts of inter I equal one of
    inter S*I with concatenated gate/up rows and down columns."""
    T, d, E, I, S = 10, 32, 4, 8, 4
    x, Wr, Wgu, Wd, Wsh = rand_case(T, d, E, I, S, seed=13)
    y_sh, *_ = oracle.forward(x, Wr, Wgu, Wd, Wsh, 2, 2, 1, I, S)
    y_no, *_ = oracle.forward(x, Wr, Wgu, Wd, None, 2, 2, 1, I, 0)
    SI = S * I
    gu = Wsh[: 2 * SI * d].view(2 * SI, d).double()
    dn = Wsh[2 * SI * d:].view(d, SI).double()
    want = swiglu_lib(x.double(), gu[:SI], gu[SI:], dn)
    np.testing.assert_allclose(y_sh - y_no, want.numpy(), rtol=1e-11, atol=1e-12)
    per = sum(swiglu_lib(x.double(), gu[s * I:(s + 1) * I], gu[SI + s * I:SI + (s + 1) * I],
                         dn[:, s * I:(s + 1) * I]) for s in range(S))
    np.testing.assert_allclose(per.numpy(), want.numpy(), rtol=1e-11, atol=1e-12)


def test_token_permutation_equivariance():
    """p7: permuting tokens permutes the outputs and the routing."""
    T, d, E, I, S = 16, 24, 8, 8, 1
    x, Wr, Wgu, Wd, Wsh = rand_case(T, d, E, I, S, seed=17, router_scale=2.0)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, Wsh, 3, 2, 1, I, S)
    perm = torch.randperm(T, generator=torch.Generator().manual_seed(1))
    yp, idxp, wp = oracle.forward(x[perm].contiguous(), Wr, Wgu, Wd, Wsh, 3, 2, 1, I, S)
    np.testing.assert_array_equal(idxp, idx[perm.numpy()])
    np.testing.assert_allclose(yp, y[perm.numpy()], rtol=0, atol=1e-13)


def test_expert_relabel_within_group():
    """p7: swapping two experts of the same group (router rows and weights)
    swaps their labels in the routing and leaves y unchanged."""
    T, d, E, I = 20, 24, 8, 8
    x, Wr, Wgu, Wd, _ = rand_case(T, d, E, I, 0, seed=19, router_scale=2.0)
    a, b = 4, 6  # both in group 1 of 2 groups of 4
    sw = torch.arange(E)
    sw[a], sw[b] = b, a
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, None, 3, 2, 1, I, 0)
    y2, idx2, w2 = oracle.forward(x, Wr[sw].contiguous(), Wgu[sw].contiguous(),
                                  Wd[sw].contiguous(), None, 3, 2, 1, I, 0)
    relabel = sw.numpy()[idx]
    # same set (order can differ only on exact ties, which random data lacks)
    np.testing.assert_array_equal(np.sort(relabel, axis=1), np.sort(idx2, axis=1))
    np.testing.assert_allclose(y2, y, rtol=0, atol=1e-13)


@pytest.mark.parametrize("T,d,E,k,G,TG,I,S,dtype", [
    (64, 128, 8, 2, 1, 1, 256, 0, torch.float32),
    (33, 64, 16, 4, 4, 2, 32, 2, torch.bfloat16),
    (20, 32, 8, 8, 2, 2, 16, 1, torch.float32),
])
def test_sparse_equals_dense_mask(T, d, E, k, G, TG, I, S, dtype):
    """p9: per-token sparse oracle == dense-mask formulation."""
    x, Wr, Wgu, Wd, Wsh = rand_case(T, d, E, I, S, dtype=dtype, seed=T)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, Wsh, k, G, TG, I, S)
    yd = dense.forward_dense(x, Wr, Wgu, Wd, Wsh, k, G, TG, I, S)
    np.testing.assert_allclose(y, yd, rtol=1e-11, atol=1e-12)
    gm, order = dense.gate_matrix(x.double().numpy(), Wr.double().numpy(), k, G, TG)
    np.testing.assert_array_equal(order, idx)


def test_forced_set_uses_own_scores():
    """With a forced expert set the weights are the oracle's normalised scores
    of that set, and the output is the composition of those experts."""
    T, d, E, I = 5, 16, 8, 8
    x, Wr, Wgu, Wd, _ = rand_case(T, d, E, I, 0, seed=23)
    forced = np.array([[7, 0], [1, 2], [3, 4], [5, 6], [6, 5]], np.int32)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, None, 2, 1, 1, I, 0, forced_idx=forced)
    np.testing.assert_array_equal(idx, forced)
    s = torch.sigmoid(x.double() @ Wr.double().T)
    for t in range(T):
        ws = s[t, forced[t]] / s[t, forced[t]].sum()
        np.testing.assert_allclose(w[t], ws.numpy(), rtol=1e-14)
        want = sum(ws[j] * swiglu_lib(x.double()[t:t + 1], Wgu[e, :I].double(),
                                      Wgu[e, I:].double(), Wd[e].double())
                   for j, e in enumerate(forced[t]))
        np.testing.assert_allclose(y[t], want[0].numpy(), rtol=1e-11, atol=1e-12)


def test_invalid_arguments_rejected():
    assert oracle.check_args(4, 8, 8, 2, 2, 1)
    assert not oracle.check_args(4, 8, 8, 2, 3, 1)      # E % n_group
    assert not oracle.check_args(4, 8, 8, 2, 2, 3)      # topk_group > n_group
    assert not oracle.check_args(4, 8, 8, 5, 2, 1)      # k > topk_group * E/G
    assert not oracle.check_args(4, 8, 8, 9, 1, 1)      # k > E
    x, Wr, *_ = rand_case(4, 8, 8, 4, 0)
    with pytest.raises(ValueError):
        oracle.route(x, Wr, 5, 2, 1)


def test_empty_token_batch():
    x, Wr, Wgu, Wd, _ = rand_case(3, 8, 4, 4, 0)
    r = oracle.route(x[:0].contiguous(), Wr, 2, 1, 1)
    assert r.idx.shape == (0, 2)
    y, idx, w = oracle.forward(x, Wr, Wgu, Wd, None, 2, 1, 1, 4, 0, tokens=[])
    assert y.shape == (0, 8)


# ---------------------------------------------------------------- gating variants
# softmax over the chosen experts (Mixtral-style gate) and the selection-only
# expert bias (aux-loss-free balancing), both from "大模型工程（一）：Transformer
# 到 MoE", section "MoE 数学：路由、容量与平衡详解"


@pytest.mark.parametrize("E,G,TG,k", [(8, 1, 1, 2), (8, 2, 1, 3), (8, 4, 2, 3), (6, 3, 2, 2)])
def test_softmax_gate_brute_force(E, G, TG, k):
    """Softmax gating: the chosen set is the exhaustive optimum of the logits,
    the weights are torch.softmax over the chosen logits."""
    T, d = 30, 16
    x, Wr, *_ = rand_case(T, d, E, 8, 0, seed=7 + E * 10 + k, router_scale=3.0)
    r = oracle.route(x, Wr, k, G, TG, score_func="softmax")
    logits = x.double() @ Wr.double().T
    np.testing.assert_allclose(r.scores, logits.numpy(), rtol=0, atol=1e-15)
    for t in range(T):
        want = brute_force_select(list(logits[t].numpy()), G, TG, k)
        assert list(r.idx[t]) == want
        w = torch.softmax(logits[t, want], dim=0).numpy()
        np.testing.assert_allclose(r.w[t], w, rtol=1e-13)


def test_softmax_gate_all_experts_is_full_softmax():
    """k = E, one group: the weights are the softmax of every logit."""
    T, d, E = 12, 8, 6
    x, Wr, *_ = rand_case(T, d, E, 4, 0, seed=3)
    r = oracle.route(x, Wr, E, 1, 1, score_func="softmax")
    full = torch.softmax(x.double() @ Wr.double().T, dim=1).numpy()
    for t in range(T):
        np.testing.assert_allclose(r.w[t], full[t, r.idx[t]], rtol=1e-13)
    np.testing.assert_allclose(r.w.sum(axis=1), 1.0, rtol=0, atol=1e-14)


@pytest.mark.parametrize("score_func", ["sigmoid", "softmax"])
def test_selection_bias_brute_force(score_func):
    """Selection bias: groups and experts are chosen on gate score + bias
    (exhaustive optimum), the weights use the unbiased gate scores."""
    E, G, TG, k, T, d = 8, 4, 2, 3, 30, 16
    x, Wr, *_ = rand_case(T, d, E, 8, 0, seed=11, router_scale=3.0)
    bias = np.linspace(-0.3, 0.4, E).astype(np.float32)
    r = oracle.route(x, Wr, k, G, TG, score_func=score_func, bias=bias)
    logits = x.double() @ Wr.double().T
    gate = torch.sigmoid(logits) if score_func == "sigmoid" else logits
    keys = gate.numpy() + bias.astype(np.float64)
    np.testing.assert_allclose(r.scores, keys, rtol=0, atol=1e-15)
    for t in range(T):
        want = brute_force_select(list(keys[t]), G, TG, k)
        assert list(r.idx[t]) == want
        g = gate[t, want]
        w = (g / g.sum()) if score_func == "sigmoid" else torch.softmax(g, dim=0)
        np.testing.assert_allclose(r.w[t], w.numpy(), rtol=1e-13)


def test_zero_bias_is_no_bias_and_large_bias_forces_an_expert():
    E, G, TG, k, T, d = 8, 2, 1, 2, 20, 16
    x, Wr, *_ = rand_case(T, d, E, 8, 0, seed=5)
    r0 = oracle.route(x, Wr, k, G, TG)
    rz = oracle.route(x, Wr, k, G, TG, bias=np.zeros(E, np.float32))
    assert (r0.idx == rz.idx).all() and (r0.w == rz.w).all()
    bias = np.zeros(E, np.float32)
    bias[5] = 10.0  # sigmoid scores are < 1: expert 5 (group 1) always wins
    rb = oracle.route(x, Wr, k, G, TG, bias=bias)
    assert (rb.idx[:, 0] == 5).all() and (rb.idx // (E // G) == 1).all()
    s = torch.sigmoid(x.double() @ Wr.double().T).numpy()
    for t in range(T):
        np.testing.assert_allclose(rb.w[t], s[t, rb.idx[t]] / s[t, rb.idx[t]].sum(), rtol=1e-14)


def test_forward_gating_variants_match_library_composition():
    """Whole layer with softmax gating and a bias: the torch fp64 composition
    of the stated steps on the oracle's own routing."""
    T, d, E, k, G, TG, I, S = 10, 16, 8, 2, 2, 1, 8, 1
    x, Wr, Wgu, Wd, Wsh = rand_case(T, d, E, I, S, seed=21, router_scale=2.0)
    bias = np.linspace(0.2, -0.2, E).astype(np.float32)
    for sf in ("sigmoid", "softmax"):
        y, idx, w = oracle.forward(x, Wr, Wgu, Wd, Wsh, k, G, TG, I, S, score_func=sf, bias=bias)
        r = oracle.route(x, Wr, k, G, TG, score_func=sf, bias=bias)
        assert (idx == r.idx).all()
        np.testing.assert_allclose(w, r.w, rtol=1e-15)
        x64 = x.double()
        ref = np.zeros((T, d))
        for t in range(T):
            for j in range(k):
                e = idx[t, j]
                ref[t] += w[t, j] * swiglu_lib(x64[t:t + 1], Wgu[e, :I].double(),
                                               Wgu[e, I:].double(), Wd[e].double()).numpy()[0]
        sh = Wsh.double()
        Wg_s = sh[:S * I * d].reshape(S * I, d)
        Wu_s = sh[S * I * d:2 * S * I * d].reshape(S * I, d)
        Wd_s = sh[2 * S * I * d:].reshape(d, S * I)
        ref += swiglu_lib(x64, Wg_s, Wu_s, Wd_s).numpy()
        np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
