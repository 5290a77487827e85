"""Benchmark of the MoE layer on B200 (one process per GPU).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload prefill]
    python bench.py --step train --workload train ...   # forward + backward
    python bench.py --impl reference ...        # the CPU oracle, timed on host cores

One step = one full layer forward (routing, permutation, routed and shared
expert GEMMs, combine) over one batch of T tokens already resident in HBM;
with --step train, one forward with saved pre-activations plus the layer
backward (all gradients) over that batch.
Under torchrun every rank runs its own batch with a full weight replica
(token-parallel, no collective on the data path): weak scaling, value = all
ranks' tokens / max-over-ranks time.  Prints one JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sparse_mixture_experts_03_b200 import accounting, moe  # noqa: E402
from sparse_mixture_experts_03_b200.inputs import (  # noqa: E402
    SKEW_SHIFT, WORKLOADS, _randn, make_inputs)

METRIC = "MoE layer tokens/sec and TFLOP/s at 1 B200; % of roofline (TC or HBM)"
L2_FLUSH_BYTES = 512 << 20  # > 126 MB L2


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons of one GPU through NVML (read only)."""

    def __init__(self, device_index: int, period_s: float = 0.02):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            bus = torch.cuda.get_device_properties(device_index)
            handle = None
            try:
                pci = "%08X:%02X:%02X.0" % (bus.pci_domain_id, bus.pci_bus_id, bus.pci_device_id)
                handle = pynvml.nvmlDeviceGetHandleByPciBusId(pci.encode())
            except Exception:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._nv, self._h = pynvml, handle
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception as e:  # no NVML: report it, do not guess
            self.error = str(e)

    def _run(self):
        nv = self._nv
        names = {
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for n, bit in names.items():
                    if r & bit:
                        self.reasons.add(n)
            except Exception:
                pass
            self._stop.wait(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": getattr(self, "error", "no samples")}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def dist_setup(backend: str = "nccl", timeout_s: float = 120.0):
    """One process per GPU: rank, world size and local rank from the launcher's
    environment.  The process group (NCCL on GPUs, gloo for host-side tests)
    carries only barriers and the max-over-ranks of the timings."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if backend == "nccl":
        torch.cuda.set_device(local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        kw = {"device_id": torch.device("cuda", local)} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, cuda: bool = True):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    if cuda:
        torch.cuda.synchronize()


def rank_batch(w, inp, rank: int) -> torch.Tensor:
    """Token batch of one rank (host tensor): rank 0 takes the workload's x,
    rank r > 0 its own draw (seed + r), shifted along the same skew direction
    as rank 0's for the load-skewed workload; the weights are the same on
    every rank."""
    if rank == 0:
        return inp.x
    x = _randn((w.T, w.d), w.seed + rank, 0)
    if w.skew:
        x.add_(inp.skew_u, alpha=SKEW_SHIFT)
    return x.to(inp.x.dtype)


def profiled_traffic(w):
    """DRAM bytes per launch of the gate/up GEMM from the committed ncu summary,
    or None when the workload differs or the kernel source changed since."""
    import hashlib
    if w.name != "prefill":
        return None
    csrc = os.path.join(ROOT, "sparse_mixture_experts_03_b200", "csrc")
    try:
        with open(os.path.join(csrc, "gemm_pair.cu"), "rb") as f:
            src = f.read()
        with open(os.path.join(csrc, "moe_device.cuh"), "rb") as f:
            src += f.read()
        with open(os.path.join(ROOT, "profiles", "pair_gemm_prefill_T4096.md")) as f:
            fields = dict(l.strip().split(": ", 1) for l in f if ": " in l and l.startswith("    "))
        if fields.get("kernel_source_sha256") != hashlib.sha256(src).hexdigest():
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


def bias_ramp(w, gate: str) -> np.ndarray:
    """The selection bias used with --expert-bias: a fixed, shuffled ramp on
    the scale of the gate scores (sigmoid scores in (0, 1); logits of order 1)."""
    span = 0.1 if gate == "sigmoid" else 0.5
    return np.random.default_rng(0).permutation(np.linspace(-span, span, w.E)).astype(np.float32)


def oracle_gating(args, w) -> dict:
    """The oracle's gating keyword arguments for the bench options."""
    return {"score_func": getattr(args, "gate", "sigmoid"),
            "bias": bias_ramp(w, args.gate) if getattr(args, "expert_bias", False) else None}


def run_config(w, world: int, args=None) -> dict:
    """The `config` object of the JSON line (both arms)."""
    gating = ""
    if args is not None and (getattr(args, "gate", "sigmoid") != "sigmoid" or
                             getattr(args, "expert_bias", False)):
        gating = f" gate={args.gate}" + (" expert_bias=on" if args.expert_bias else "")
    return {"workload": f"{w.name}: {w.describe()}{gating}", "global_batch": world * w.T,
            "tokens_per_gpu": w.T, "parallelism": f"token-parallel x{world} (replicas)",
            "l2": ("flushed between timed steps (512 MB write); weights 1.28 GB > L2"
                   if getattr(args, "l2", "flush") == "flush" else
                   "not flushed: each step streams 1.28 GB of weights (> 126 MB L2)"),
            "out_dtype": "f32"}


def cpu_baseline(w, inp, args, budget_s: float = 15.0):
    """Time the CPU oracle (as it stands) on a bounded sample of the workload's tokens."""
    import oracle
    nthreads = os.cpu_count() or 1
    probe = np.arange(min(w.T, max(8, nthreads)), dtype=np.int32)
    t0 = time.perf_counter()
    oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, w.k,
                   w.n_group, w.topk_group, w.inter, w.n_shared, tokens=probe, nthreads=nthreads,
                   **oracle_gating(args, w))
    per_tok = (time.perf_counter() - t0) / len(probe)
    n = int(min(w.T, max(len(probe), budget_s / max(per_tok, 1e-9))))
    n = max(nthreads, n // nthreads * nthreads) if n >= nthreads else n
    toks = np.linspace(0, w.T - 1, n).astype(np.int32)
    t0 = time.perf_counter()
    oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, w.k,
                   w.n_group, w.topk_group, w.inter, w.n_shared, tokens=toks, nthreads=nthreads,
                   **oracle_gating(args, w))
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"{n} of {w.T} tokens of the {w.name} workload (full layer per token, "
                      f"fp64), {dt:.1f} s wall"}


def run_reference(args, w):
    """--impl reference: the CPU oracle timed on the host cores, same metric/config."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    inp = make_inputs(w)
    nthreads = os.cpu_count() or 1
    # bounded sample per step, sized so warmup+steps finish in a few minutes
    probe = np.arange(min(w.T, max(4, nthreads)), dtype=np.int32)
    t0 = time.perf_counter()
    oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, w.k,
                   w.n_group, w.topk_group, w.inter, w.n_shared, tokens=probe, nthreads=nthreads,
                   **oracle_gating(args, w))
    per_tok = (time.perf_counter() - t0) / len(probe)
    total_steps = args.steps + args.warmup
    per_step_budget = 150.0 / max(total_steps, 1)
    n = int(max(1, min(w.T, per_step_budget / max(per_tok, 1e-9))))
    rng = np.random.default_rng(0)
    times = []
    for s in range(total_steps):
        toks = np.sort(rng.choice(w.T, size=n, replace=False)).astype(np.int32)
        t0 = time.perf_counter()
        oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, w.k,
                       w.n_group, w.topk_group, w.inter, w.n_shared, tokens=toks,
                       nthreads=nthreads, **oracle_gating(args, w))
        if s >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = n / sec
    flops = accounting.flops_per_token(w.d, w.E, w.k, w.inter, w.n_shared) * n
    out = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": run_config(w, world, args),
        "tflops": flops / sec / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{n} random tokens of {w.T} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


TRAIN_METRIC = ("MoE layer training step (forward + backward) tokens/sec and TFLOP/s at 1 B200; "
                "% of roofline (TC or HBM)")


def dy_batch(w, rank: int) -> torch.Tensor:
    """Upstream gradient of rank `rank` (stream 7, seed offset by the rank)."""
    return _randn((w.T, w.d), w.seed + rank, 7).to(torch.bfloat16)


def oracle_train_sample(w, inp, dy, toks, nthreads, args):
    """The oracle's forward + backward of the sub-batch `toks` (its own batch)."""
    import oracle
    xs, dys = inp.x[toks].contiguous(), dy[toks].contiguous()
    kw = oracle_gating(args, w)
    oracle.forward(xs, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, w.k, w.n_group,
                   w.topk_group, w.inter, w.n_shared, nthreads=nthreads, **kw)
    oracle.backward(xs, inp.W_router, inp.W_gate_up, inp.W_down, inp.W_shared, dys, w.k,
                    w.n_group, w.topk_group, w.inter, w.n_shared, nthreads=nthreads, **kw)


def train_sample_size(w, inp, dy, args, budget_s: float, nthreads: int) -> int:
    probe = np.arange(min(w.T, max(8, nthreads)), dtype=np.int64)
    t0 = time.perf_counter()
    oracle_train_sample(w, inp, dy, probe, nthreads, args)
    per_tok = (time.perf_counter() - t0) / len(probe)
    return int(max(1, min(w.T, budget_s / max(per_tok, 1e-9))))


def cpu_baseline_train(w, inp, dy, args, budget_s: float = 15.0):
    """The oracle's forward + backward (as it stands) on a sub-batch of the
    workload's tokens, sized to about budget_s of host time."""
    nthreads = os.cpu_count() or 1
    n = train_sample_size(w, inp, dy, args, budget_s, nthreads)
    toks = np.linspace(0, w.T - 1, n).astype(np.int64)
    t0 = time.perf_counter()
    oracle_train_sample(w, inp, dy, toks, nthreads, args)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
            "sample": f"forward + backward of a sub-batch of {n} of the {w.T} tokens of the "
                      f"{w.name} workload (fp64, all gradients of that sub-batch), {dt:.1f} s wall"}


def run_reference_train(args, w):
    """--impl reference --step train: the oracle's forward + backward on a
    bounded sub-batch per step, rank 0 only."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if int(os.environ.get("RANK", "0")) != 0:
        return
    inp = make_inputs(w)
    dy = dy_batch(w, 0)
    nthreads = os.cpu_count() or 1
    total_steps = args.steps + args.warmup
    n = train_sample_size(w, inp, dy, args, 150.0 / max(total_steps, 1), nthreads)
    rng = np.random.default_rng(0)
    times = []
    for s_ in range(total_steps):
        toks = np.sort(rng.choice(w.T, size=n, replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        oracle_train_sample(w, inp, dy, toks, nthreads, args)
        if s_ >= args.warmup:
            times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = n / sec
    flops = accounting.train_step_flops(n, w.d, w.E, w.k, w.inter, w.n_shared)
    cfg = run_config(w, world, args)
    cfg["step"] = "forward + backward"
    out = {
        "impl": "reference", "metric": TRAIN_METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": cfg, "tflops": flops / sec / 1e12,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"forward + backward of {n} random tokens of {w.T} per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def run_train(args, w):
    """--step train: one step = moe_forward_train + moe_backward over one batch
    resident in HBM (all gradients: dx, dW_router, dW_gate_up, dW_down,
    dW_shared)."""
    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    inp = make_inputs(w)
    inp.x = rank_batch(w, inp, rank)
    dy_host = dy_batch(w, rank)
    x, dy = inp.x.to(dev), dy_host.to(dev)
    Wr, Wgu, Wd = inp.W_router.to(dev), inp.W_gate_up.to(dev), inp.W_down.to(dev)
    Wsh = inp.W_shared.to(dev) if inp.W_shared is not None else None
    f32 = dict(dtype=torch.float32, device=dev)
    y = torch.empty(w.T, w.d, **f32)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wt = torch.empty(w.T, w.k, **f32)
    saved = torch.empty(moe.saved_bytes(w.T, w.k, w.inter, w.n_shared), dtype=torch.uint8,
                        device=dev)
    ws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype, dev)
    bws = torch.empty(moe.backward_workspace_bytes(w.T, w.d, w.E, w.k, w.inter, w.n_shared),
                      dtype=torch.uint8, device=dev)
    grads = moe.alloc_grads(w.T, w.d, w.E, w.inter, w.n_shared, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, **f32)
    stream = torch.cuda.current_stream()
    bias = torch.from_numpy(bias_ramp(w, args.gate)).to(dev) if args.expert_bias else None
    load = torch.empty(w.E, dtype=torch.int32, device=dev) if args.expert_bias else None

    def step(xin=x, dyin=dy, yout=y, dxout=None):
        moe.forward_train(xin, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter,
                          w.n_shared, y=yout, topk_idx=idx, topk_w=wt, saved=saved,
                          workspace=ws, gate=args.gate, expert_bias=bias, expert_load=load)
        g = grads if dxout is None else moe.Grads(dxout, grads.dW_router, grads.dW_gate_up,
                                                  grads.dW_down, grads.dW_shared)
        moe.backward(xin, Wr, Wgu, Wd, Wsh, dyin, idx, wt, saved, w.k, w.inter, w.n_shared,
                     gate=args.gate, grads=g, workspace=bws)

    def check(where):
        for buf in (ws, bws):
            st, site = moe.device_status(buf)
            if st != moe.MOE_OK:
                raise SystemExit(f"device status {where}: {moe.status_string(st)} (site {site})")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    check("after warm-up")

    # ---- per-stage breakdown of forward and backward (instrumented pass,
    # before the timed region: it also decides which GEMM launch dominates)
    nf, nb = moe.N_STAGE_EVENTS, moe.N_BWD_STAGE_EVENTS
    n_stage = min(args.steps, 20)
    f_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nf)] for _ in range(n_stage)]
    b_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nb)] for _ in range(n_stage)]
    for evs in f_ev + b_ev:  # create the CUDA handles the library records into
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(n_stage):
        if args.l2 == "flush":
            flush.fill_(float(i))
        moe.set_stage_events(f_ev[i])
        moe.set_backward_stage_events(b_ev[i])
        step()
    moe.set_stage_events(None)
    moe.set_backward_stage_events(None)
    torch.cuda.synchronize()
    fst = np.mean([[e[j].elapsed_time(e[j + 1]) for j in range(nf - 1)] for e in f_ev], 0)
    bst = np.mean([[e[j].elapsed_time(e[j + 1]) for j in range(nb - 1)] for e in b_ev], 0)
    # the GEMM launches: (forward or backward events, boundary index, FLOPs, name)
    rows = w.T * w.k
    SI = w.n_shared * w.inter
    f_gu = accounting.gate_up_flops(rows, w.d, w.inter) + accounting.gate_up_flops(w.T, w.d, SI)
    f_dn = accounting.down_flops(rows, w.d, w.inter) + accounting.down_flops(w.T, w.d, SI)
    gemms = {
        "forward gate/up + SwiGLU, saving pre-activations": ("f", 2, f_gu,
            "pair_gemm_kernel<SWIGLU_SAVE,SWIGLU_SAVE,KIND_FWD>"),
        "forward down + weighted scatter": ("f", 3, f_dn,
            "pair_gemm_kernel<STORE_F32,SCATTER,KIND_FWD>"),
        "dh = W_down^T dy + SwiGLU backward": ("b", 1, f_dn,
            "pair_gemm_kernel<DSWIGLU,DSWIGLU,KIND_DGRAD>"),
        "dx parts = W_gate_up^T [dg|du]": ("b", 3, f_gu,
            "pair_gemm_kernel<STORE_F32,SCATTER,KIND_DGRAD>"),
        "dW_down": ("b", 5, f_dn, "pair_gemm_kernel<STORE_ROWS,STORE_ROWS,KIND_WGRAD>"),
        "dW_gate_up": ("b", 6, f_gu, "pair_gemm_kernel<STORE_ROWS,STORE_ROWS,KIND_WGRAD>"),
    }
    stage_of = lambda g: (fst if g[0] == "f" else bst)[g[1]]
    dom_name = max(gemms, key=lambda n: stage_of(gemms[n]))
    dom = gemms[dom_name]

    def dom_events(evs):
        """Stage-event lists that record only the dominant launch's two boundaries."""
        n = nf if dom[0] == "f" else nb
        lst = [None] * n
        lst[dom[1]], lst[dom[1] + 1] = evs
        return lst

    # ---- timed region (as for the forward): per-step events, L2 flushed
    # between steps; the dominant GEMM launch is bracketed by stage events on
    # every 8th step only.
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dom_steps = [i for i in range(args.steps) if i % 8 == 0] or [0]
    dom_ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(2)] for i in dom_steps}
    for evs in dom_ev.values():
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    set_dom = moe.set_stage_events if dom[0] == "f" else moe.set_backward_stage_events
    barrier(world)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            if args.l2 == "flush":
                flush.fill_(float(i))
            set_dom(dom_events(dom_ev[i]) if i in dom_ev else None)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        set_dom(None)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(sum(s_.elapsed_time(e) for s_, e in zip(starts, ends)) / args.steps, world)
    dom_ms = sum(a.elapsed_time(b) for a, b in dom_ev.values()) / len(dom_ev)
    check("after timing")

    # ---- end to end through the public calls: every step copies x and dy
    # from pinned host memory and reads y and dx back (what the layer hands
    # the rest of the model); copies on two streams, double-buffered.
    x_host, dy_host = inp.x.pin_memory(), dy_host.pin_memory()
    y_host = [torch.empty(w.T, w.d).pin_memory() for _ in range(2)]
    dx_host = [torch.empty(w.T, w.d).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    dy_dev = [torch.empty_like(dy) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    dx_dev = [torch.empty_like(grads.dx) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_run(n_steps, e_start=None, e_stop=None):
        h2d_done = [torch.cuda.Event() for _ in range(n_steps)]
        comp_done = [torch.cuda.Event() for _ in range(n_steps)]
        d2h_done = [torch.cuda.Event() for _ in range(n_steps)]
        if e_start is not None:
            e_start.record(s_h2d)
        for i in range(n_steps):
            b = i & 1
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(comp_done[i - 2])
                x_dev[b].copy_(x_host, non_blocking=True)
                dy_dev[b].copy_(dy_host, non_blocking=True)
                h2d_done[i].record(s_h2d)
            stream.wait_event(h2d_done[i])
            if i >= 2:
                stream.wait_event(d2h_done[i - 2])
            step(x_dev[b], dy_dev[b], y_dev[b], dx_dev[b])
            comp_done[i].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(comp_done[i])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                dx_host[b].copy_(dx_dev[b], non_blocking=True)
                d2h_done[i].record(s_d2h)
        if e_stop is not None:
            e_stop.record(s_d2h)
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(3)
    barrier(world)
    e2e_steps = max(5, args.steps // 4)
    e2e_run(e2e_steps, e0, e1)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)

    # ---- accounting
    n_touched = accounting.touched_experts(idx.cpu().numpy(), w.E)
    flops = accounting.train_step_flops(w.T, w.d, w.E, w.k, w.inter, w.n_shared)
    bytes_alg = accounting.train_step_bytes(w.T, w.d, w.E, w.k, w.inter, w.n_shared, n_touched)
    pk = peaks()
    t_tensor = flops / (pk["bf16_tflops"] * 1e12)
    t_hbm = bytes_alg / (pk["hbm_gbs"] * 1e9)
    roof_ms = max(t_tensor, t_hbm) * 1e3
    dom_flops = dom[2]
    dom_ach = dom_flops / (dom_ms * 1e-3) / 1e12
    # forward: route, permutation with the row gather, 2 GEMMs, final sum; backward:
    # permutation, gather, dgrad GEMM, dL/dlogit, dgrad GEMM, dx sum, 2
    # weight-gradient GEMMs, dW_router (2)
    launches = (1 + 1 + 2 + 1) + (1 + 9)
    cfg = run_config(w, world, args)
    cfg["step"] = "forward (saving pre-activations) + backward (dx and all weight gradients, fp32)"
    out = {
        "metric": TRAIN_METRIC, "value": world * w.T / (ms * 1e-3), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations and upstream gradient, N(0,1/fan_in) "
                "weights; no dataset)",
        "config": cfg, "tflops": flops / (ms * 1e-3) / 1e12,
        "roofline_layer": {"bound": "tensor" if t_tensor >= t_hbm else "hbm",
                           "roofline_ms": roof_ms, "frac": roof_ms / ms,
                           "peak_tflops": pk["bf16_tflops"], "hbm_gbs": pk["hbm_gbs"],
                           "alg_flops": flops, "alg_bytes": bytes_alg,
                           "touched_experts": n_touched, "peak_source": pk["source"]},
        "roofline": {"bound": "tensor",
                     "kernel": f"{dom[3]} ({dom_name}; shared and routed experts, one launch)",
                     "achieved": dom_ach, "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": dom_ach / pk["bf16_tflops"], "traffic": None,
                     "flops_per_launch": dom_flops, "avg_launch_ms": dom_ms,
                     "timed_launches": len(dom_ev),
                     "peak_kind": f"bf16 burst ({pk['source']})",
                     **({"frac_of_sustained_peak": dom_ach / pk["bf16_tflops_sustained"]}
                        if pk.get("bf16_tflops_sustained") else {})},
        "stage_ms": {"forward": {n: float(v) for n, v in zip(moe.STAGES, fst)},
                     "backward": {n: float(v) for n, v in zip(moe.BWD_STAGES, bst)}},
        "stage_ms_note": f"separate pass of {n_stage} steps with an event at every stage "
                         "boundary (before the timed steps; it picks the dominant launch)",
        "gpu_launches": launches * args.steps,
        "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": 2 * x.numel() * x.element_size(),
                "d2h_bytes_per_step": 2 * y.numel() * y.element_size(), "ms_per_step": e2e_ms,
                "copies": "x and dy in, y and dx out; pinned host buffers, two copy streams, "
                          "double-buffered, overlapping neighbouring steps"},
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_train(w, inp, dy_host, args)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="prefill", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--l2", default="flush", choices=["flush", "stream"],
                    help="flush: write 512 MB between timed steps; stream: rely on the "
                         "step's inputs (1.28 GB of expert weights) being larger than L2")
    ap.add_argument("--gate", default="sigmoid", choices=["sigmoid", "softmax"],
                    help="routing gate (the FusionLLM sigmoid gate is the headline)")
    ap.add_argument("--expert-bias", action="store_true",
                    help="add a selection-only expert bias (and read back the expert loads)")
    ap.add_argument("--step", default="forward", choices=["forward", "train"],
                    help="forward: the layer forward (headline); train: forward with saved "
                         "pre-activations + backward")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = WORKLOADS[args.workload]
    if args.impl == "reference":
        if args.step == "train":
            run_reference_train(args, w)
        else:
            run_reference(args, w)
        return
    if args.step == "train":
        run_train(args, w)
        return

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    inp = make_inputs(w)
    inp.x = rank_batch(w, inp, rank)  # each rank its own batch of tokens, same weights
    x = inp.x.to(dev)
    Wr, Wgu, Wd = inp.W_router.to(dev), inp.W_gate_up.to(dev), inp.W_down.to(dev)
    Wsh = inp.W_shared.to(dev) if inp.W_shared is not None else None
    y = torch.empty(w.T, w.d, dtype=torch.float32, device=dev)
    idx = torch.empty(w.T, w.k, dtype=torch.int32, device=dev)
    wt = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
    ws = moe.alloc_workspace(w.T, w.d, w.E, w.k, w.inter, w.n_shared, x.dtype, dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    bias = None
    load = None
    if args.expert_bias:
        bias = torch.from_numpy(bias_ramp(w, args.gate)).to(dev)
        load = torch.empty(w.E, dtype=torch.int32, device=dev)

    def step(xin=x, yout=y):
        moe.forward(xin, Wr, Wgu, Wd, Wsh, w.k, w.n_group, w.topk_group, w.inter, w.n_shared,
                    gate=args.gate, expert_bias=bias, expert_load=load,
                    y=yout, topk_idx=idx, topk_w=wt, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, site = moe.device_status(ws)
    if st != moe.MOE_OK:
        raise SystemExit(f"device status after warm-up: {moe.status_string(st)} (site {site})")

    # ---- timed region: per-step events around the forward, L2 flushed between
    # steps.  Inside the forward only the two boundaries of the dominant kernel
    # (the gate/up GEMM) are recorded, and only on every 8th step: an event
    # between two kernels keeps the second from being launched early (a few
    # microseconds per step), so the other stage boundaries are timed in a
    # separate instrumented pass below.
    n_ev = moe.N_STAGE_EVENTS
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    dom_steps = [i for i in range(args.steps) if i % 8 == 0] or [0]
    dom_ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(2)] for i in dom_steps}
    n_stage_steps = min(args.steps, 50)
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
                for _ in range(n_stage_steps)]
    for evs in stage_ev + list(dom_ev.values()):  # create the CUDA handles
        for e in evs:
            e.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            if args.l2 == "flush":
                flush.fill_(float(i))
            if i in dom_ev:
                moe.set_stage_events([None, None, dom_ev[i][0], dom_ev[i][1], None, None])
            else:
                moe.set_stage_events(None)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        moe.set_stage_events(None)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)
    ms = max_over_ranks(ms, world)
    dom_ms = sum(a.elapsed_time(b) for a, b in dom_ev.values()) / len(dom_ev)
    # ---- per-stage breakdown (instrumented pass, not the headline)
    for i in range(n_stage_steps):
        if args.l2 == "flush":
            flush.fill_(float(i))
        moe.set_stage_events(stage_ev[i])
        step()
    moe.set_stage_events(None)
    torch.cuda.synchronize()
    stage_ms = np.zeros(n_ev - 1)
    for evs in stage_ev:
        stage_ms += np.array([evs[j].elapsed_time(evs[j + 1]) for j in range(n_ev - 1)])
    stage_ms /= n_stage_steps
    st, site = moe.device_status(ws)
    if st != moe.MOE_OK:
        raise SystemExit(f"device status after timing: {moe.status_string(st)} (site {site})")

    # ---- end to end through the public call: every step copies its x from
    # pinned host memory and reads its y back.  Copies run on their own
    # streams, double-buffered, so step i's copies overlap the forwards of its
    # neighbours (the way a serving loop feeds the layer); the clock runs from
    # the first host-to-device copy to the last device-to-host copy.
    x_host = inp.x.pin_memory()
    y_host = [torch.empty(w.T, w.d, dtype=torch.float32).pin_memory() for _ in range(2)]
    x_dev = [torch.empty_like(x) for _ in range(2)]
    y_dev = [torch.empty_like(y) for _ in range(2)]
    s_h2d, s_d2h = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def e2e_run(n_steps, e_start=None, e_stop=None):
        h2d_done = [torch.cuda.Event() for _ in range(n_steps)]
        comp_done = [torch.cuda.Event() for _ in range(n_steps)]
        d2h_done = [torch.cuda.Event() for _ in range(n_steps)]
        if e_start is not None:
            e_start.record(s_h2d)
        for i in range(n_steps):
            b = i & 1
            with torch.cuda.stream(s_h2d):
                if i >= 2:  # buffer b is free once step i-2's forward has read it
                    s_h2d.wait_event(comp_done[i - 2])
                x_dev[b].copy_(x_host, non_blocking=True)
                h2d_done[i].record(s_h2d)
            stream.wait_event(h2d_done[i])
            if i >= 2:  # y buffer b is free once step i-2's result is on the host
                stream.wait_event(d2h_done[i - 2])
            step(x_dev[b], y_dev[b])
            comp_done[i].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(comp_done[i])
                y_host[b].copy_(y_dev[b], non_blocking=True)
                d2h_done[i].record(s_d2h)
        if e_stop is not None:
            e_stop.record(s_d2h)
        torch.cuda.synchronize()

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(3)
    barrier(world)
    e2e_steps = max(10, args.steps // 4)
    e2e_run(e2e_steps, e0, e1)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)

    # ---- accounting
    gi = idx.cpu().numpy()
    rows = w.T * w.k
    flops = accounting.layer_flops(w.T, w.d, w.E, w.k, w.inter, w.n_shared)
    n_touched = accounting.touched_experts(gi, w.E)
    bytes_alg = accounting.layer_bytes(w.T, w.d, w.E, w.inter, w.n_shared, n_touched)
    pk = peaks()
    tflops = flops / (ms * 1e-3) / 1e12
    t_tensor = flops / (pk["bf16_tflops"] * 1e12)
    t_hbm = bytes_alg / (pk["hbm_gbs"] * 1e9)
    roof_ms = max(t_tensor, t_hbm) * 1e3
    layer_bound = "tensor" if t_tensor >= t_hbm else "hbm"
    names = moe.STAGES
    stage = {n: float(v) for n, v in zip(names, stage_ms)}
    # dominant kernel: the gate/up grouped GEMM (routed + shared tiles, one
    # launch).  Tensor-bound batches: its FLOPs; HBM-bound (decode): its
    # algorithmic bytes -- the touched experts' and the shared gate/up weights,
    # the token rows read and the SwiGLU outputs written.
    g1_flops = (accounting.gate_up_flops(rows, w.d, w.inter)
                + accounting.gate_up_flops(w.T, w.d, w.n_shared * w.inter))
    esz = 2 if w.dtype == "bf16" else 4
    SI = w.n_shared * w.inter
    g1_bytes = esz * (n_touched * 2 * w.inter * w.d + 2 * SI * w.d + rows * w.d + w.T * w.d
                      + rows * w.inter + w.T * SI)
    if layer_bound == "tensor":
        dom = {"bound": "tensor", "achieved": g1_flops / (dom_ms * 1e-3) / 1e12,
               "peak": pk["bf16_tflops"], "unit": "TFLOP/s", "flops_per_launch": g1_flops,
               "peak_kind": f"bf16 burst ({pk['source']})"}
        if pk.get("bf16_tflops_sustained"):
            dom["frac_of_sustained_peak"] = dom["achieved"] / pk["bf16_tflops_sustained"]
    else:
        dom = {"bound": "hbm", "achieved": g1_bytes / (dom_ms * 1e-3) / 1e9,
               "peak": pk["hbm_gbs"], "unit": "GB/s", "bytes_per_launch": g1_bytes,
               "peak_kind": f"HBM copy ({pk['source']})"}
    dom["frac"] = dom["achieved"] / dom["peak"]
    # route, permutation with the row gather (one launch), the two GEMM
    # launches, final sum
    launches_per_step = (1 + 1 + 2 + 1) if w.dtype == "bf16" else None
    value = world * w.T / (ms * 1e-3)
    out = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) activations, N(0,1/fan_in) weights; no dataset)",
        "config": run_config(w, world, args),
        "tflops": tflops,
        "roofline_layer": {"bound": layer_bound, "roofline_ms": roof_ms,
                           "frac": roof_ms / ms, "peak_tflops": pk["bf16_tflops"],
                           "hbm_gbs": pk["hbm_gbs"], "alg_bytes": bytes_alg,
                           "touched_experts": n_touched, "peak_source": pk["source"]},
        "roofline": {**{"bound": dom["bound"],
                        "kernel": "pair_gemm_kernel<SWIGLU,SWIGLU> (gate/up + SwiGLU, "
                                  "shared and routed experts)",
                        "achieved": dom["achieved"], "peak": dom["peak"], "unit": dom["unit"],
                        "frac": dom["frac"], "traffic": profiled_traffic(w)},
                     **{k: v for k, v in dom.items()
                        if k not in ("bound", "achieved", "peak", "unit", "frac")},
                     "avg_launch_ms": dom_ms, "timed_launches": len(dom_ev)},
        "stage_ms": stage,
        "stage_ms_note": f"separate pass of {n_stage_steps} steps with an event at every stage "
                         "boundary (the headline steps record only the gate/up boundaries)",
        "gpu_launches": launches_per_step * args.steps if launches_per_step else None,
        "e2e": {"value": world * w.T / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": x.numel() * x.element_size(),
                "d2h_bytes_per_step": y.numel() * y.element_size(), "ms_per_step": e2e_ms,
                "copies": "pinned host buffers; copies on two streams, double-buffered, "
                          "overlapping neighbouring steps' forwards"},
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, inp, args)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
