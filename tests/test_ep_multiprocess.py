"""Expert-parallel layer (sparse_mixture_experts_03_b200/ep.py): the exchange
logic run as 2 and 4 gloo ranks on the CPU.

The four computing steps (routing + permutation, the local experts, the shared
experts, the final sum) are restated here on the CPU in fp64 -- routing from
the oracle, the expert FFNs written out per row -- and handed to the layer as
`ops`; what runs for real is the layer's own split sizing, the count and row
all-to-alls, the receive layout and the return path.  Every rank's output
must equal the oracle's forward of its tokens.  The CUDA kernels of the same
steps are tested on the GPU in test_gpu_ep.py."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _silu(v):
    return v / (1.0 + np.exp(-v))


class CpuOps:
    """fp64 CPU restatement of the four computing steps (test only)."""

    @staticmethod
    def dispatch(x, W_router, k, n_group, topk_group, gate="sigmoid", expert_bias=None):
        import oracle
        from sparse_mixture_experts_03_b200 import moe
        E = W_router.shape[0]
        r = oracle.route(x, W_router, k, n_group, topk_group, score_func=gate,
                         bias=None if expert_bias is None else expert_bias.numpy())
        flat = torch.from_numpy(r.idx).reshape(-1).long()
        order = torch.sort(flat, stable=True).indices  # by expert, then slot order
        slot_row = torch.empty_like(order)
        slot_row[order] = torch.arange(order.numel())
        return moe.Dispatched(torch.from_numpy(r.idx), torch.from_numpy(r.w),
                              torch.bincount(flat, minlength=E).to(torch.int32),
                              x[order // k].contiguous(),
                              torch.from_numpy(r.w).reshape(-1)[order].contiguous(),
                              slot_row.to(torch.int32))

    @staticmethod
    def _ffn(xr, Wgu, Wd, inter):
        g = Wgu[:inter] @ xr
        u = Wgu[inter:] @ xr
        return Wd @ (_silu(g) * u)

    @staticmethod
    def experts_forward(x_rows, w_rows, recv_counts, W_gate_up, W_down, inter):
        xr = x_rows.double().numpy()
        w = w_rows.double().numpy()
        Wgu = W_gate_up.double().numpy()
        Wd = W_down.double().numpy()
        out = np.zeros((x_rows.shape[0], x_rows.shape[1]))
        row = 0
        for src in range(recv_counts.shape[0]):
            for e in range(recv_counts.shape[1]):
                for _ in range(int(recv_counts[src, e])):
                    out[row] = w[row] * CpuOps._ffn(xr[row], Wgu[e], Wd[e], inter)
                    row += 1
        assert row == x_rows.shape[0]
        return torch.from_numpy(out)

    @staticmethod
    def shared_forward(x, W_shared, inter, n_shared):
        from sparse_mixture_experts_03_b200.inputs import shared_views
        d = x.shape[1]
        SI = n_shared * inter
        gu, dn = shared_views(W_shared, d, inter, n_shared)
        xd = x.double().numpy()
        g = xd @ gu[:SI].double().numpy().T
        u = xd @ gu[SI:].double().numpy().T
        return torch.from_numpy((_silu(g) * u) @ dn.double().numpy().T)

    @staticmethod
    def combine(rows, slot_row, shared, T, k, out_dtype):
        y = torch.zeros(T, rows.shape[1], dtype=torch.float64) if shared is None else shared.clone()
        for j in range(k):
            y += rows[slot_row.view(T, k)[:, j].long()]
        return y


class BadCountsOps(CpuOps):
    """CpuOps whose dispatch reports counts that do not add up to T*k, as a
    device error in moe_dispatch would leave them (fault injected on the host)."""

    @staticmethod
    def dispatch(*args, **kw):
        d = CpuOps.dispatch(*args, **kw)
        d.counts[0] += 5
        return d


def layer_for_rank(w, inp, rank, world, ops):
    from sparse_mixture_experts_03_b200.ep import ExpertParallelMoE
    E_l = w.E // world
    sl = slice(rank * E_l, (rank + 1) * E_l)
    return ExpertParallelMoE(inp.W_router, inp.W_gate_up[sl].contiguous(),
                             inp.W_down[sl].contiguous(), inp.W_shared, w.k, w.n_group,
                             w.topk_group, w.inter, w.n_shared, rank, world, ops=ops)


def rank_tokens(T_per_rank, rank):
    lo = sum(T_per_rank[:rank])
    return lo, lo + T_per_rank[rank]


def _rank_main(rank, world, port, case, q, bad_ranks=()):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import datetime
    import torch.distributed as dist
    import oracle
    from sparse_mixture_experts_03_b200.inputs import make_inputs

    try:
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=90))
        w, T_per_rank, one_expert = case
        inp = make_inputs(w)
        if one_expert:  # every token on expert E-1 first: other ranks receive nothing
            Wr = torch.zeros(w.E, w.d)
            Wr[w.E - 1] = 1e-2
            inp.W_router = Wr.to(inp.x.dtype)
            inp.x = inp.x.float().abs().add(0.1).to(inp.x.dtype)
        lo, hi = rank_tokens(T_per_rank, rank)
        x = inp.x[lo:hi].contiguous()
        ops = BadCountsOps() if rank in bad_ranks else CpuOps()
        layer = layer_for_rank(w, inp, rank, world, ops)
        try:
            y = layer(x)
        except RuntimeError as err:  # the injected device error, raised after the exchanges
            q.put({"rank": rank, "raised": str(err)})
            dist.destroy_process_group()
            return
        y_ref, _, _ = oracle.forward(x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared,
                                     w.k, w.n_group, w.topk_group, w.inter, w.n_shared)
        err = float(np.abs(y.numpy() - y_ref).max()) if y.numel() else 0.0
        q.put({"rank": rank, "err": err, "scale": float(np.abs(y_ref).max()) if y.numel() else 0,
               "T": hi - lo})
        dist.destroy_process_group()
    except Exception as e:  # report, never hang the other ranks
        import traceback
        q.put({"rank": rank, "error": repr(e) + traceback.format_exc()})


def _cases():
    from sparse_mixture_experts_03_b200.inputs import Workload
    w = Workload("ep", T=120, d=64, E=8, k=2, n_group=2, topk_group=1, inter=32, n_shared=1,
                 dtype="bf16")
    w4 = Workload("ep4", T=96, d=64, E=16, k=3, n_group=4, topk_group=2, inter=32, n_shared=0,
                  dtype="bf16")
    return {
        "two_ranks": (2, (w, [70, 50], False)),
        "two_ranks_one_token": (2, (w, [1, 37], False)),
        "two_ranks_all_on_one_expert": (2, (w, [40, 40], True)),
        "four_ranks_no_shared": (4, (w4, [30, 20, 40, 6], False)),
    }


CASES = ["two_ranks", "two_ranks_one_token", "two_ranks_all_on_one_expert",
         "four_ranks_no_shared"]


@pytest.mark.parametrize("name", CASES)
def test_expert_parallel_exchange_on_gloo_ranks(name):
    sys.path.insert(0, ROOT)
    world, case = _cases()[name]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in sorted(res, key=lambda r: r["rank"]):
        assert "error" not in r, r["error"]
        assert r["err"] <= 1e-9 * max(1.0, r["scale"]), r


def test_dispatch_error_on_one_rank_raises_there_and_others_finish():
    """Rank 1's dispatch reports inconsistent counts: it announces no rows,
    takes every exchange step the other rank takes (no collective is left
    waiting) and raises at the end; rank 0's tokens, computed on both ranks'
    experts, still match the oracle."""
    sys.path.insert(0, ROOT)
    world, case = _cases()["two_ranks"]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, case, q, (1,)))
             for r in range(world)]
    for p in procs:
        p.start()
    res = {r["rank"]: r for r in (q.get(timeout=240) for _ in range(world))}
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert "error" not in res[0], res[0].get("error")
    assert res[0]["err"] <= 1e-9 * max(1.0, res[0]["scale"]), res[0]
    assert "do not add up" in res[1].get("raised", ""), res[1]


def test_rank_rows_splits_expert_blocks():
    sys.path.insert(0, ROOT)
    from sparse_mixture_experts_03_b200.ep import rank_rows
    assert rank_rows([1, 2, 3, 4, 5, 6, 7, 8], 4) == [3, 7, 11, 15]
    assert rank_rows([0] * 8, 2) == [0, 0]
    with pytest.raises(ValueError):
        rank_rows([1, 2, 3], 2)
