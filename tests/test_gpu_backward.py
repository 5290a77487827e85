"""Backward of the layer on the GPU (moe_forward_train + moe_backward) against
the oracle's backward, element by element.

Routing: the GPU forward's expert sets must match the oracle's except on
near-tie tokens (the criterion of parity.py); on those the oracle's backward
is evaluated on the GPU's set after checking that the set is within 1e-4 of
optimal (a gradient is defined per expert set).

Tolerance, from the arithmetic: the GPU keeps bf16 copies of the
pre-activations g, u, of dg|du, of w*h and of the chosen experts' dx rows,
each with a relative rounding error <= 2^-9; every gradient entry is a sum of
products of such values with fp32 accumulation.  The errors are independent
with random signs, so a gradient's error relative to its own magnitude stays
near a few 2^-9 (2^-9 = 1.95e-3): rel-Frobenius <= 1e-2 and max |diff| <=
3e-2 * max |ref| per gradient tensor.  Measured on B200 over the small cases
below: rel-Frobenius 2.3e-3 .. 3.1e-3, max 2.2e-3 .. 6.3e-3 of max |ref|.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import check_routing
from sparse_mixture_experts_03_b200 import moe
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, Workload, make_dy, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"
TOL = {"dx": (1e-2, 3e-2), "dW_router": (1e-2, 3e-2), "dW_gate_up": (1e-2, 3e-2),
       "dW_down": (1e-2, 3e-2), "dW_shared": (1e-2, 3e-2)}


def assert_close(got, ref, name):
    got = np.asarray(got, np.float64)
    assert np.isfinite(got).all(), f"{name}: non-finite"
    diff = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    mx = np.abs(ref).max() if ref.size else 0.0
    max_rel = np.abs(diff).max() / mx if mx > 0 else np.abs(diff).max()
    tr, tm = TOL[name]
    assert rel <= tr and max_rel <= tm, f"{name}: rel_fro {rel:.3e} (tol {tr}), max {max_rel:.3e} (tol {tm})"
    return rel, max_rel


def run_gpu(w: Workload, inp, dy, gate="sigmoid"):
    c = lambda t: None if t is None else t.to(DEV)
    x, Wr, Wgu, Wd, Wsh, dyd = (c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down),
                                c(inp.W_shared), c(dy))
    y, idx, tw, saved = moe.forward_train(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group,
                                          w.inter, w.n_shared, gate=gate)
    ws = torch.empty(moe.backward_workspace_bytes(w.T, w.d, w.E, w.k, w.inter, w.n_shared),
                     dtype=torch.uint8, device=DEV)
    g = moe.backward(x, Wr, Wgu, Wd, Wsh, dyd, idx, tw, saved, w.k, w.inter, w.n_shared,
                     gate=gate, workspace=ws)
    torch.cuda.synchronize()
    st, site = moe.device_status(ws)
    assert st == moe.MOE_OK, (st, site)
    return dict(x=x, Wr=Wr, Wgu=Wgu, Wd=Wd, Wsh=Wsh, dy=dyd, y=y, idx=idx, tw=tw, saved=saved,
                g=g, ws=ws)


def forced_sets(w, inp, gpu_idx, gpu_w, score_func):
    """The oracle's sets with the GPU's set on near-tie tokens where they
    differ (checked near-optimal), or None when they agree everywhere."""
    ref = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group, score_func=score_func)
    rep = check_routing(gpu_idx, gpu_w, ref, w.n_group, w.topk_group, w.E)
    if rep.n_set_mismatch_near_tie == 0:
        return None
    f = ref.idx.copy()
    f[rep.mismatched_tokens] = gpu_idx[rep.mismatched_tokens]
    return f


SMALL = [
    Workload("bwd_small", T=300, d=256, E=8, k=2, n_group=2, topk_group=1, inter=256,
             n_shared=1, dtype="bf16"),
    Workload("bwd_mid", T=520, d=512, E=16, k=4, n_group=4, topk_group=2, inter=512,
             n_shared=2, dtype="bf16", seed=1),
    Workload("bwd_no_shared", T=260, d=256, E=8, k=2, n_group=1, topk_group=1, inter=256,
             n_shared=0, dtype="bf16", seed=2),
    Workload("bwd_one_token", T=1, d=256, E=16, k=4, n_group=4, topk_group=2, inter=256,
             n_shared=1, dtype="bf16", seed=3),
    # 5 tokens x 2 of 32 experts: most experts get no token (zero gradients)
    Workload("bwd_empty_experts", T=5, d=256, E=32, k=2, n_group=1, topk_group=1, inter=256,
             n_shared=1, dtype="bf16", seed=4),
    # several 256-token tiles per expert and a ragged tail
    Workload("bwd_many_tokens", T=1100, d=256, E=4, k=2, n_group=1, topk_group=1, inter=256,
             n_shared=1, dtype="bf16", seed=5),
]


@pytest.mark.parametrize("w", SMALL, ids=[c.name for c in SMALL])
@pytest.mark.parametrize("gate", ["sigmoid", "softmax"])
def test_backward_matches_oracle(w, gate):
    inp, dy = make_inputs(w), make_dy(w)
    r = run_gpu(w, inp, dy, gate)
    gpu_idx, gpu_w = r["idx"].cpu().numpy(), r["tw"].cpu().numpy()
    forced = forced_sets(w, inp, gpu_idx, gpu_w, gate)
    ref = oracle.backward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, dy, w.k,
                          w.n_group, w.topk_group, w.inter, w.n_shared, forced_idx=forced,
                          score_func=gate)
    g = r["g"]
    assert_close(g.dx.cpu().numpy(), ref.dx, "dx")
    assert_close(g.dW_router.cpu().numpy(), ref.dW_router, "dW_router")
    assert_close(g.dW_gate_up.cpu().numpy(), ref.dW_gate_up, "dW_gate_up")
    assert_close(g.dW_down.cpu().numpy(), ref.dW_down, "dW_down")
    if w.n_shared:
        assert_close(g.dW_shared.cpu().numpy(), ref.dW_shared, "dW_shared")
    # experts no token chose: exactly zero gradients
    unused = np.setdiff1d(np.arange(w.E), np.unique(gpu_idx))
    for e in unused:
        assert (g.dW_gate_up[e] == 0).all() and (g.dW_down[e] == 0).all()
        assert (g.dW_router[e] == 0).all()


def test_forward_train_output_equals_forward():
    w = SMALL[1]
    inp = make_inputs(w)
    c = lambda t: None if t is None else t.to(DEV)
    args = (c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down), c(inp.W_shared), w.k,
            w.n_group, w.topk_group, w.inter, w.n_shared)
    y0 = moe.forward(*args)
    y1, idx, tw, saved = moe.forward_train(*args)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    # the saved pre-activations are the bf16 gate / up projections of the
    # chosen experts' rows, in the documented layout: blocks of 16 features,
    # [I/16][T*k][16 gate | 16 up], rows expert by expert in token order
    I, Tk = w.inter, w.T * w.k
    sv = saved[: Tk * 2 * I * 2].view(torch.bfloat16).view(I // 16, Tk, 32).float().cpu()
    x32, Wgu32 = inp.x.float(), inp.W_gate_up.float()
    idx_c = idx.cpu().numpy()
    start = np.concatenate([[0], np.cumsum(np.bincount(idx_c.ravel(), minlength=w.E))])
    for t in (0, w.T // 2, w.T - 1):
        for j in range(w.k):
            e = int(idx_c[t, j])
            row = start[e] + int((idx_c[:t] == e).any(axis=1).sum())  # earlier tokens on e
            ref = (Wgu32[e] @ x32[t]).numpy()
            got_g = sv[:, row, :16].reshape(-1).numpy()
            got_u = sv[:, row, 16:].reshape(-1).numpy()
            np.testing.assert_allclose(got_g, ref[:I], rtol=1e-2, atol=2e-2)
            np.testing.assert_allclose(got_u, ref[I:], rtol=1e-2, atol=2e-2)


def test_backward_is_deterministic():
    w = SMALL[1]
    inp, dy = make_inputs(w), make_dy(w)
    r = run_gpu(w, inp, dy)
    g2 = moe.backward(r["x"], r["Wr"], r["Wgu"], r["Wd"], r["Wsh"], r["dy"], r["idx"], r["tw"],
                      r["saved"], w.k, w.inter, w.n_shared, workspace=r["ws"])
    torch.cuda.synchronize()
    for name in ("dx", "dW_router", "dW_gate_up", "dW_down", "dW_shared"):
        assert torch.equal(getattr(r["g"], name), getattr(g2, name)), name


def test_zero_tokens_zero_weight_gradients():
    w = SMALL[0]
    inp = make_inputs(w.with_tokens(1))
    c = lambda t: None if t is None else t.to(DEV)
    x = torch.empty(0, w.d, dtype=torch.bfloat16, device=DEV)
    g = moe.alloc_grads(0, w.d, w.E, w.inter, w.n_shared, DEV)
    for t in (g.dW_router, g.dW_gate_up, g.dW_down, g.dW_shared):
        t.fill_(7.0)
    idx = torch.empty(0, w.k, dtype=torch.int32, device=DEV)
    tw = torch.empty(0, w.k, dtype=torch.float32, device=DEV)
    moe.backward(x, c(inp.W_router), c(inp.W_gate_up), c(inp.W_down), c(inp.W_shared), x, idx, tw,
                 torch.empty(16, dtype=torch.uint8, device=DEV), w.k, w.inter, w.n_shared,
                 grads=g)
    torch.cuda.synchronize()
    for t in (g.dW_router, g.dW_gate_up, g.dW_down, g.dW_shared):
        assert (t == 0).all()


def test_unsupported_shapes_rejected():
    assert moe.lib().moe_backward_workspace_bytes(64, 2048, 64, 6, 1664, 4) == 0  # inter % 256
    w = SMALL[0]
    inp = make_inputs(w)
    x = inp.x.float().to(DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.backward(x, inp.W_router.float().to(DEV), inp.W_gate_up.float().to(DEV),
                     inp.W_down.float().to(DEV), inp.W_shared.float().to(DEV), x,
                     torch.zeros(w.T, w.k, dtype=torch.int32, device=DEV),
                     torch.zeros(w.T, w.k, device=DEV), torch.zeros(16, dtype=torch.uint8,
                                                                    device=DEV),
                     w.k, w.inter, w.n_shared, workspace=torch.empty(1 << 20, dtype=torch.uint8,
                                                                     device=DEV))
    assert e.value.status == moe.MOE_ERR_UNSUPPORTED


def sampled_check(w: Workload, dx_tokens, wsel):
    inp, dy = make_inputs(w), make_dy(w)
    r = run_gpu(w, inp, dy)
    gpu_idx, gpu_w = r["idx"].cpu().numpy(), r["tw"].cpu().numpy()
    forced = forced_sets(w, inp, gpu_idx, gpu_w, "sigmoid")
    dxr, rows = oracle.backward_rows(inp.x, inp.W_router, inp.W_gate_up, inp.W_down,
                                     inp.W_shared, dy, w.k, w.n_group, w.topk_group, w.inter,
                                     w.n_shared, dx_tokens=dx_tokens, wsel=wsel,
                                     forced_idx=forced)
    g = r["g"]
    E, I, d, SI = w.E, w.inter, w.d, w.n_shared * w.inter
    views = {oracle.ROW_DWR: g.dW_router, oracle.ROW_DWGU: g.dW_gate_up.view(E * 2 * I, d),
             oracle.ROW_DWD: g.dW_down.view(E * d, I),
             oracle.ROW_DWSH_GU: g.dW_shared[: 2 * SI * d].view(2 * SI, d),
             oracle.ROW_DWSH_DN: g.dW_shared[2 * SI * d:].view(d, SI)}
    names = {oracle.ROW_DWR: "dW_router", oracle.ROW_DWGU: "dW_gate_up",
             oracle.ROW_DWD: "dW_down", oracle.ROW_DWSH_GU: "dW_shared",
             oracle.ROW_DWSH_DN: "dW_shared"}
    assert_close(g.dx[torch.as_tensor(dx_tokens, device=DEV).long()].cpu().numpy(), dxr, "dx")
    for (ten, row), ref in zip(wsel, rows):
        assert_close(views[ten][row].cpu().numpy(), ref, names[ten])


def test_full_size_sampled_prefill_batch():
    """FusionLLM shapes at T = 4096: sampled rows of every gradient."""
    w = WORKLOADS["prefill"]
    E, I, d, SI = w.E, w.inter, w.d, w.n_shared * w.inter
    rng = np.random.default_rng(11)
    wsel = [(oracle.ROW_DWR, int(rng.integers(E))),
            (oracle.ROW_DWGU, int(rng.integers(E * 2 * I))),
            (oracle.ROW_DWGU, 63 * 2 * I + I + 5),
            (oracle.ROW_DWD, int(rng.integers(E * d))),
            (oracle.ROW_DWSH_GU, int(rng.integers(2 * SI))),
            (oracle.ROW_DWSH_DN, int(rng.integers(d)))]
    sampled_check(w, [0, 1, 2047, 4095], wsel)


def test_full_size_sampled_train_batch():
    """The train batch (T = 32768, the size the training step is timed on):
    dx rows and rows of the expert and shared gate/up gradients and of the
    expert down gradients."""
    w = WORKLOADS["train"]
    E, I, d, SI = w.E, w.inter, w.d, w.n_shared * w.inter
    rng = np.random.default_rng(12)
    wsel = [(oracle.ROW_DWGU, int(rng.integers(E * 2 * I))),
            (oracle.ROW_DWGU, int(rng.integers(E * 2 * I))),
            (oracle.ROW_DWD, int(rng.integers(E * d))),
            (oracle.ROW_DWSH_GU, int(rng.integers(2 * SI)))]
    sampled_check(w, [0, 16383, 32767], wsel)


def test_training_step_in_a_cuda_graph_matches_eager():
    """forward_train + backward captured once and replayed: the same bits as
    the eager calls (the backward clears its status word and tile counters
    inside every replay)."""
    w = SMALL[1]
    inp, dy = make_inputs(w), make_dy(w)
    r = run_gpu(w, inp, dy)
    c = lambda t: None if t is None else t.to(DEV)
    y = torch.empty_like(r["y"])
    idx, tw, saved = torch.empty_like(r["idx"]), torch.empty_like(r["tw"]), torch.empty_like(
        r["saved"])
    fws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, torch.bfloat16)
    bws = torch.empty_like(r["ws"])
    g = moe.alloc_grads(w.T, w.d, w.E, w.inter, w.n_shared, DEV)

    def step(stream):
        moe.forward_train(r["x"], r["Wr"], r["Wgu"], r["Wd"], r["Wsh"], w.k, w.n_group,
                          w.topk_group, w.inter, w.n_shared, y=y, topk_idx=idx, topk_w=tw,
                          saved=saved, workspace=fws, stream=stream)
        moe.backward(r["x"], r["Wr"], r["Wgu"], r["Wd"], r["Wsh"], r["dy"], idx, tw, saved, w.k,
                     w.inter, w.n_shared, grads=g, workspace=bws, stream=stream)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step(s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step(torch.cuda.current_stream())
    for _ in range(2):
        for t in (g.dx, g.dW_router, g.dW_gate_up, g.dW_down, g.dW_shared):
            t.zero_()
        graph.replay()
        torch.cuda.synchronize()
        assert moe.device_status(bws)[0] == moe.MOE_OK
        assert torch.equal(y, r["y"])
        for name in ("dx", "dW_router", "dW_gate_up", "dW_down", "dW_shared"):
            assert torch.equal(getattr(g, name), getattr(r["g"], name)), name
    del graph


def test_backward_with_selection_bias():
    """A selection-only bias moves the expert sets; the gradients follow the
    sets chosen and the unbiased weights (the oracle with the same bias)."""
    w = SMALL[1]
    inp, dy = make_inputs(w), make_dy(w)
    bias = np.random.default_rng(9).permutation(np.linspace(-0.1, 0.1, w.E)).astype(np.float32)
    c = lambda t: None if t is None else t.to(DEV)
    x, Wr, Wgu, Wd, Wsh, dyd = (c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down),
                                c(inp.W_shared), c(dy))
    b = torch.from_numpy(bias).to(DEV)
    y, idx, tw, saved = moe.forward_train(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group,
                                          w.inter, w.n_shared, expert_bias=b)
    g = moe.backward(x, Wr, Wgu, Wd, Wsh, dyd, idx, tw, saved, w.k, w.inter, w.n_shared)
    torch.cuda.synchronize()
    gpu_idx, gpu_w = idx.cpu().numpy(), tw.cpu().numpy()
    ref_r = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group, bias=bias)
    rep = check_routing(gpu_idx, gpu_w, ref_r, w.n_group, w.topk_group, w.E)
    forced = None
    if rep.n_set_mismatch_near_tie:
        forced = ref_r.idx.copy()
        forced[rep.mismatched_tokens] = gpu_idx[rep.mismatched_tokens]
    ref = oracle.backward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, dy, w.k,
                          w.n_group, w.topk_group, w.inter, w.n_shared, forced_idx=forced,
                          bias=bias)
    # the bias changed some sets relative to the unbiased routing
    plain = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group)
    assert (np.sort(plain.idx, 1) != np.sort(ref.idx, 1)).any(1).sum() > 0
    assert_close(g.dx.cpu().numpy(), ref.dx, "dx")
    assert_close(g.dW_router.cpu().numpy(), ref.dW_router, "dW_router")
    assert_close(g.dW_gate_up.cpu().numpy(), ref.dW_gate_up, "dW_gate_up")
    assert_close(g.dW_down.cpu().numpy(), ref.dW_down, "dW_down")
    assert_close(g.dW_shared.cpu().numpy(), ref.dW_shared, "dW_shared")


def test_full_size_sampled_skewed_batch():
    """The load-skewed workload (40% of tokens on expert 0, T = 16384): rows
    of the overloaded expert's gradients and of a light one, and dx rows."""
    w = WORKLOADS["skewed"]
    E, I, d, SI = w.E, w.inter, w.d, w.n_shared * w.inter
    wsel = [(oracle.ROW_DWGU, 0 * 2 * I + 17), (oracle.ROW_DWGU, 0 * 2 * I + I + 900),
            (oracle.ROW_DWD, 0 * d + 1234), (oracle.ROW_DWGU, 37 * 2 * I + 5),
            (oracle.ROW_DWR, 0), (oracle.ROW_DWSH_GU, 333)]
    sampled_check(w, [0, 8191, 16383], wsel)
