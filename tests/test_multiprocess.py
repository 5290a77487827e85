"""Host-side multi-rank logic of the benchmark (token-parallel replicas), run as
two gloo ranks on the CPU: rank setup from the launcher's environment,
per-rank token batches (and upstream gradients) with shared weights, barrier
and max-over-ranks of the timings.  The data path has no collective, so nothing else crosses ranks."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    sys.path.insert(0, ROOT)
    import bench
    import torch.distributed as dist
    from sparse_mixture_experts_03_b200.inputs import Workload, make_inputs

    try:
        got_world, got_rank, got_local = bench.dist_setup(backend="gloo", timeout_s=60)
        w = Workload("mp", T=16, d=128, E=8, k=2, n_group=2, topk_group=1, inter=128,
                     n_shared=1, dtype="bf16")
        inp = make_inputs(w)
        x = bench.rank_batch(w, inp, got_rank)
        # every rank sees the others' batches and weights through all_gather
        xs = [torch.empty_like(x.float()) for _ in range(world)]
        dist.all_gather(xs, x.float())
        ws = [torch.empty_like(inp.W_gate_up.float()) for _ in range(world)]
        dist.all_gather(ws, inp.W_gate_up.float())
        # the training step's upstream gradient: each rank its own
        dy = bench.dy_batch(w, got_rank).float()
        dys = [torch.empty_like(dy) for _ in range(world)]
        dist.all_gather(dys, dy)
        bench.barrier(got_world, cuda=False)
        mx = bench.max_over_ranks(float(10 + got_rank), got_world, device="cpu")
        q.put({"rank": got_rank, "world": got_world, "local": got_local, "max": mx,
               "x_differ": not torch.equal(xs[0], xs[1]),
               "dy_differ": not torch.equal(dys[0], dys[1]),
               "w_same": torch.equal(ws[0], ws[1]),
               "cfg": bench.run_config(w, got_world)})
        dist.destroy_process_group()
    except Exception as e:  # report, never hang the other rank
        q.put({"rank": rank, "error": repr(e)})


def test_two_gloo_ranks_replicas():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda r: r["rank"])
    for r in res:
        assert "error" not in r, r
        assert r["world"] == world and r["local"] == r["rank"]
        assert r["max"] == 10 + world - 1  # max over ranks, seen by every rank
        assert r["x_differ"] and r["w_same"] and r["dy_differ"]
        assert r["cfg"]["global_batch"] == world * 16
        assert r["cfg"]["parallelism"] == "token-parallel x2 (replicas)"


@pytest.mark.parametrize("step", ["forward", "train"])
def test_reference_arm_other_ranks_exit_quietly(step):
    """Under a launcher, the reference arm runs on rank 0 only; rank 1 prints
    nothing and exits 0 (no GPU, no oracle work), for the forward and for the
    training step."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--step", step, "--steps", "1", "--warmup", "3"], env=env,
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""
