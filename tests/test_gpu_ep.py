"""Expert-parallel layer on the GPU, through the C ABI: N ranks emulated one
after another on one device.

Each emulated rank owns E/N experts and a slice of the tokens; its dispatch,
local experts, shared experts and final sum are the library's kernels
(moe_dispatch, moe_experts_forward, moe_shared_forward, moe_combine).  The
two all-to-all exchanges between them are done here by plain tensor copies
in the order NCCL's all_to_all_single would deliver (source rank order), so
no kernel ever waits for another rank's.  The result is compared with the
oracle on every token, and with the single-GPU moe_forward of the same
tokens."""
import numpy as np
import pytest
import torch

import oracle
from sparse_mixture_experts_03_b200 import moe
from sparse_mixture_experts_03_b200.ep import ExpertParallelMoE, rank_rows
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, Workload, make_inputs

from parity import check_output, check_routing, oracle_outputs, write_record

pytestmark = pytest.mark.gpu

DEV = "cuda"


def emulate(w: Workload, inp, T_per_rank):
    """y [T, d] of the expert-parallel layer over len(T_per_rank) emulated ranks."""
    N = len(T_per_rank)
    E_l = w.E // N
    c = lambda t: None if t is None else t.to(DEV)
    x = c(inp.x)
    Wr, Wsh = c(inp.W_router), c(inp.W_shared)
    layers, xs, bounds = [], [], []
    lo = 0
    for r in range(N):
        sl = slice(r * E_l, (r + 1) * E_l)
        layers.append(ExpertParallelMoE(Wr, c(inp.W_gate_up[sl].contiguous()),
                                        c(inp.W_down[sl].contiguous()), Wsh, w.k, w.n_group,
                                        w.topk_group, w.inter, w.n_shared, r, N))
        xs.append(x[lo:lo + T_per_rank[r]].contiguous())
        bounds.append((lo, lo + T_per_rank[r]))
        lo += T_per_rank[r]
    disp = [layers[r].dispatch(xs[r]) for r in range(N)]
    shared = [layers[r].shared(xs[r]) for r in range(N)]
    counts = [d.counts.cpu().tolist() for d in disp]
    send = [rank_rows(cn, N) for cn in counts]  # send[src][dst]
    # first exchange: rank q receives, in source order, each source's block for q
    y_recv = []
    for q in range(N):
        xq, wq = [], []
        for src in range(N):
            off = sum(send[src][:q])
            xq.append(disp[src].x_perm[off:off + send[src][q]])
            wq.append(disp[src].w_perm[off:off + send[src][q]])
        rc = torch.tensor([counts[src][q * E_l:(q + 1) * E_l] for src in range(N)],
                          dtype=torch.int32, device=DEV)
        y_recv.append(layers[q].experts(torch.cat(xq).contiguous(), torch.cat(wq).contiguous(),
                                        rc))
    # return exchange: source r gets, in destination order, its rows back
    ys = []
    for r in range(N):
        back = []
        for q in range(N):
            off = sum(send[src][q] for src in range(r))
            back.append(y_recv[q][off:off + send[r][q]])
        rows_back = torch.cat(back).contiguous()
        ys.append(layers[r].combine(rows_back, disp[r], shared[r], T_per_rank[r]))
    torch.cuda.synchronize()
    return torch.cat(ys), torch.cat([d.topk_idx for d in disp]), torch.cat(
        [d.topk_w for d in disp])


CASES = [
    # the FusionLLM layer at prefill over 8 ranks of 512 tokens (8 experts each)
    ("prefill_8_ranks", WORKLOADS["prefill"], [512] * 8),
    # 2 ranks of 2048 tokens: the dispatch's grid-wide permutation (T > 1024)
    ("prefill_2_ranks", WORKLOADS["prefill"], [2048, 2048]),
    # decode over 4 ranks, ragged
    ("decode_4_ranks", WORKLOADS["decode"], [20, 1, 31, 12]),
    # small layer, 2 ranks, one rank with a single token, no shared experts
    ("small_2_ranks", Workload("ep_small", T=301, d=256, E=16, k=4, n_group=4, topk_group=2,
                               inter=256, n_shared=0, dtype="bf16"), [1, 300]),
]


@pytest.mark.parametrize("name,w,T_per_rank", CASES, ids=[c[0] for c in CASES])
def test_expert_parallel_matches_oracle_and_single_gpu(name, w, T_per_rank):
    assert sum(T_per_rank) == w.T
    inp = make_inputs(w)
    y, idx, wt = emulate(w, inp, T_per_rank)
    ref = oracle.route(inp.x, inp.W_router, w.k, w.n_group, w.topk_group)
    gi = idx.cpu().numpy()
    check_routing(gi, wt.cpu().numpy(), ref, w.n_group, w.topk_group, w.E)
    tokens = np.arange(w.T, dtype=np.int32)
    y_ref = oracle_outputs(inp, w, tokens, gi, ref)
    check_output(y.cpu().numpy(), y_ref, w.dtype)
    # the single-GPU layer on the same tokens: the same expert arithmetic; the
    # router may run another kernel at another batch size (fp32 logits summed
    # in another order), so gate weights can differ in their last bits and a
    # slot's bf16 rounding with them
    c = lambda t: None if t is None else t.to(DEV)
    idx1 = torch.empty(w.T, w.k, dtype=torch.int32, device=DEV)
    y1 = moe.forward(c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down),
                     c(inp.W_shared), w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                     topk_idx=idx1)
    torch.cuda.synchronize()
    same = (idx.cpu() == idx1.cpu()).all(dim=1).numpy()
    assert (same | ref.near_tie(1e-4)).all()
    d = (y - y1)[torch.from_numpy(same).to(DEV)]
    assert float(d.abs().max()) <= 1.6e-2
    assert float(d.norm()) <= 1e-4 * float(y1.norm())
    write_record("test_expert_parallel_matches_oracle_and_single_gpu",
                 {"case": name, "ranks": len(T_per_rank),
                  "bitwise_equal_single_gpu": bool(torch.equal(y, y1))})


def test_experts_forward_reports_count_overflow():
    """recv_counts summing to more than R rows: MOE_ERR_DEVICE in the status
    word and nothing computed (the output rows keep their contents)."""
    d, E_l, I, R = 256, 2, 128, 40
    x = torch.randn(R, d, device=DEV).to(torch.bfloat16)
    wr = torch.ones(R, device=DEV)
    Wgu = (torch.randn(E_l, 2 * I, d, device=DEV) * 0.05).to(torch.bfloat16)
    Wd = (torch.randn(E_l, d, I, device=DEV) * 0.05).to(torch.bfloat16)
    rc = torch.tensor([[30, 20]], dtype=torch.int32, device=DEV)  # 50 > 40
    ws = torch.empty(moe.lib().moe_experts_workspace_bytes(R, d, E_l, I), dtype=torch.uint8,
                     device=DEV)
    y = torch.zeros(R, d, dtype=torch.bfloat16, device=DEV)
    moe.experts_forward(x, wr, rc, Wgu, Wd, I, y_rows=y, workspace=ws)
    st, _ = moe.device_status(ws)
    assert st == moe.MOE_ERR_DEVICE
    assert (y.float() == 0).all()
