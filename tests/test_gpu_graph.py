"""The forward captured in a CUDA graph and replayed: same output bits as the
eager call (the tile ticket counters and the status word are reset by the
routing kernel inside every replay), for a decode-sized and a prefill-sized
batch."""
import pytest
import torch

from sparse_mixture_experts_03_b200 import moe
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_graph_replay_matches_eager(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    c = lambda t: None if t is None else t.to(DEV)
    x, Wr, Wgu, Wd, Wsh = c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down), c(inp.W_shared)
    ws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype)
    y_eager = moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                          workspace=ws)
    torch.cuda.synchronize()
    y = torch.empty_like(y_eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up on the capture stream
        moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared, y=y,
                    workspace=ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared, y=y,
                    workspace=ws, stream=torch.cuda.current_stream())
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert moe.device_status(ws)[0] == moe.MOE_OK
        assert torch.equal(y, y_eager)
    # new input values in the same buffers are picked up by the replay
    x2 = (x.float() * 0.5).to(x.dtype)
    x.copy_(x2)
    g.replay()
    y2 = moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                     workspace=moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared,
                                                   x.dtype))
    torch.cuda.synchronize()
    assert torch.equal(y, y2)
    del g
