"""moe_expert_counts_noalloc (scratch in a fixed device array, no allocation)
against the forward's own permutation stage, which computes the same counts
and unpadded offsets (bf16 layers) in the caller's workspace.  Integer
results: compared exactly, on two calls in a row."""
import numpy as np
import pytest
import torch

from sparse_mixture_experts_03_b200 import moe
from sparse_mixture_experts_03_b200.inputs import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

DEV = "cuda"


def forward_counts(w: Workload):
    """topk_idx, counts, offsets from moe_forward (the existing entry point)."""
    inp = make_inputs(w)
    c = lambda t: None if t is None else t.to(DEV)
    x, Wr, Wgu, Wd, Wsh = c(inp.x), c(inp.W_router), c(inp.W_gate_up), c(inp.W_down), c(inp.W_shared)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=DEV)
    ws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype)
    moe.forward(x, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                topk_idx=idx, workspace=ws)
    torch.cuda.synchronize()
    lay = moe.workspace_layout(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype)
    wsc = ws.cpu()
    counts = wsc[lay["counts"]:lay["counts"] + 4 * w.E].view(torch.int32).clone()
    offsets = wsc[lay["offsets"]:lay["offsets"] + 4 * (w.E + 1)].view(torch.int32).clone()
    return idx, counts, offsets


CASES = [
    WORKLOADS["prefill"],
    Workload("ragged", T=300, d=256, E=8, k=2, n_group=2, topk_group=1, inter=128, n_shared=1,
             dtype="bf16"),
    Workload("one_token", T=1, d=256, E=16, k=4, n_group=4, topk_group=2, inter=256, n_shared=2,
             dtype="bf16"),
]


@pytest.mark.parametrize("w", CASES, ids=[c.name for c in CASES])
def test_matches_forward_permutation_two_calls(w):
    idx, ref_counts, ref_offsets = forward_counts(w)
    np.testing.assert_array_equal(ref_counts.numpy(),
                                  np.bincount(idx.cpu().numpy().ravel(), minlength=w.E))
    for _ in range(2):  # two calls in a row share the fixed scratch
        counts = torch.full((w.E,), -7, dtype=torch.int32, device=DEV)
        offsets = torch.full((w.E + 1,), -7, dtype=torch.int32, device=DEV)
        moe.expert_counts_noalloc(idx, w.E, counts, offsets)
        torch.cuda.synchronize()
        assert torch.equal(counts.cpu(), ref_counts)
        assert torch.equal(offsets.cpu(), ref_offsets)


def test_empty_routing_gives_zeros():
    idx = torch.empty(0, 6, dtype=torch.int32, device=DEV)
    counts = torch.full((64,), -1, dtype=torch.int32, device=DEV)
    offsets = torch.full((65,), -1, dtype=torch.int32, device=DEV)
    moe.expert_counts_noalloc(idx, 64, counts, offsets)
    torch.cuda.synchronize()
    assert (counts.cpu() == 0).all() and (offsets.cpu() == 0).all()


def test_sizes_beyond_the_fixed_scratch_are_rejected():
    # ceil(65537 / 256) * 256 experts = 65792 words > 65536
    idx = torch.zeros(65537, 1, dtype=torch.int32, device=DEV)
    counts = torch.empty(256, dtype=torch.int32, device=DEV)
    offsets = torch.empty(257, dtype=torch.int32, device=DEV)
    with pytest.raises(moe.MoeError) as e:
        moe.expert_counts_noalloc(idx, 256, counts, offsets)
    assert e.value.status == moe.MOE_ERR_WORKSPACE
    # the largest size that fits still runs
    idx = torch.randint(0, 256, (65536, 1), dtype=torch.int32, device=DEV)
    moe.expert_counts_noalloc(idx, 256, counts, offsets)
    torch.cuda.synchronize()
    ref = np.bincount(idx.cpu().numpy().ravel(), minlength=256)
    np.testing.assert_array_equal(counts.cpu().numpy(), ref)
    np.testing.assert_array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(ref)]))


def test_repeated_and_out_of_range_ids_count_per_occurrence():
    """Rows given by the caller may repeat an id ([3, 3] counts expert 3
    twice) and may hold ids outside [0, E), which are skipped: the counts are
    np.bincount of the in-range ids, on two calls in a row."""
    E, k, T = 16, 4, 1000
    g = torch.Generator().manual_seed(5)
    idx = torch.randint(0, E, (T, k), generator=g, dtype=torch.int32)
    idx[::3, 1] = idx[::3, 0]             # repeats inside a row
    idx[7] = torch.tensor([3, 3, 3, 3])
    idx[11, 2] = E                        # out of range: skipped
    idx[13, 0] = -1
    ids = idx.numpy().ravel()
    ref = np.bincount(ids[(ids >= 0) & (ids < E)], minlength=E)
    idx_d = idx.to(DEV)
    for _ in range(2):
        counts = torch.full((E,), -7, dtype=torch.int32, device=DEV)
        offsets = torch.full((E + 1,), -7, dtype=torch.int32, device=DEV)
        moe.expert_counts_noalloc(idx_d, E, counts, offsets)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(counts.cpu().numpy(), ref)
        np.testing.assert_array_equal(offsets.cpu().numpy(),
                                      np.concatenate([[0], np.cumsum(ref)]))
