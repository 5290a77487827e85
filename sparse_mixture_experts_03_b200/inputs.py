"""Seeded synthetic inputs for the fine-grained MoE layer forward.

This module only draws random tensors and names the workloads.  It holds none
of the layer's arithmetic (no routing, no expert math), so both the CUDA path
and the CPU oracle can take their inputs from it without sharing any code that
decides a result.

Workload shapes follow the FusionLLM configuration (FusionLLM page, section
"模型配置与规模": dim 2048, 64 routed experts, 6 activated, 4 shared, moe_inter_dim
1536) plus a small fp32 case.  Initialisation: x ~ N(0, 1), router weight
~ N(0, 1/d), every expert weight ~ N(0, 1/d_in) where d_in is the fan-in of
that projection (d for gate/up, inter for down; each shared expert is its own
expert of inter I, so its down projection uses 1/I).

Random streams: each tensor has a fixed stream id (x 0, W_router 1, W_gate_up
2, W_down 3, shared gate_up 4, shared down 5, skew direction u 6, upstream
gradient dy of the backward 7) and is filled
in chunks of 2**24 elements; chunk c of stream i is drawn by torch.randn from a
CPU torch.Generator seeded with the 32-bit value (seed << 24) | (i << 16) | c
(the CPU generator keeps only 32 bits of a seed, so the fields are packed into
32 bits: seed < 256, stream < 256, chunk < 65536).  The values do not depend
on how many threads fill the chunks.  Everything is drawn in fp32
and cast to bf16 with round-to-nearest-even where the workload is bf16.

Layouts (all row-major, contiguous):
  x          [T, d]
  W_router   [E, d]
  W_gate_up  [E, 2*inter, d]   rows 0..inter-1 are the gate projection,
                               rows inter..2*inter-1 the up projection
  W_down     [E, d, inter]
  W_shared   one flat buffer: gate_up [2*S*inter, d] (all S gate blocks, then
             all S up blocks) followed by down [d, S*inter]; None when S == 0
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Optional

import torch

# Router scale for the load-skewed workload: W_router[0] is replaced by
# SKEW_ALPHA * u, where x = z + SKEW_SHIFT * u.  SKEW_ALPHA was chosen by
# oracle/calibrate_skew.py so that about 40% of tokens route to expert 0.
SKEW_SHIFT = 3.0
SKEW_ALPHA = 0.4111


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d: int
    E: int
    k: int
    n_group: int
    topk_group: int
    inter: int
    n_shared: int
    dtype: str  # "f32" or "bf16"
    skew: bool = False
    seed: int = 0

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T)

    def describe(self) -> str:
        s = (f"T={self.T} d={self.d} E={self.E} k={self.k} n_group={self.n_group} "
             f"topk_group={self.topk_group} inter={self.inter} n_shared={self.n_shared} "
             f"{self.dtype}")
        return s + (" skewed" if self.skew else "")


WORKLOADS = {
    "tiny": Workload("tiny", T=64, d=128, E=8, k=2, n_group=1, topk_group=1,
                     inter=256, n_shared=0, dtype="f32"),
    "prefill": Workload("prefill", T=4096, d=2048, E=64, k=6, n_group=8, topk_group=4,
                        inter=1536, n_shared=4, dtype="bf16"),
    "train": Workload("train", T=32768, d=2048, E=64, k=6, n_group=8, topk_group=4,
                      inter=1536, n_shared=4, dtype="bf16"),
    "decode": Workload("decode", T=64, d=2048, E=64, k=6, n_group=8, topk_group=4,
                       inter=1536, n_shared=4, dtype="bf16"),
    "skewed": Workload("skewed", T=16384, d=2048, E=64, k=6, n_group=8, topk_group=4,
                       inter=1536, n_shared=4, dtype="bf16", skew=True),
}


@dataclasses.dataclass
class Inputs:
    """CPU tensors of one workload (dtype float32 or bfloat16)."""
    x: torch.Tensor
    W_router: torch.Tensor
    W_gate_up: torch.Tensor
    W_down: torch.Tensor
    W_shared: Optional[torch.Tensor]
    skew_u: Optional[torch.Tensor] = None


def torch_dtype(name: str) -> torch.dtype:
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


CHUNK = 1 << 24


def _randn(shape, seed: int, stream: int, scale: float = 1.0) -> torch.Tensor:
    """N(0, scale^2) fp32 tensor of `shape` from stream `stream` of `seed`."""
    n = math.prod(shape)
    out = torch.empty(n, dtype=torch.float32)
    n_chunks = (n + CHUNK - 1) // CHUNK
    if not (0 <= seed < 256 and 0 <= stream < 256 and n_chunks <= 65536):
        raise ValueError("seed, stream or size outside the packed 32-bit seed fields")

    def fill(c: int) -> None:
        g = torch.Generator(device="cpu").manual_seed((seed << 24) | (stream << 16) | c)
        lo, hi = c * CHUNK, min(n, (c + 1) * CHUNK)
        out[lo:hi] = torch.randn(hi - lo, generator=g)
        if scale != 1.0:
            out[lo:hi].mul_(scale)

    if n_chunks <= 1:
        for c in range(n_chunks):
            fill(c)
    else:
        workers = max(1, min(n_chunks, os.cpu_count() or 1, 32))
        with concurrent.futures.ThreadPoolExecutor(workers) as ex:
            list(ex.map(fill, range(n_chunks)))
    return out.view(*shape)


def make_inputs(w: Workload, skew_alpha: Optional[float] = None) -> Inputs:
    """Draw the seeded inputs of workload `w` on the CPU."""
    T, d, E, I, S, sd = w.T, w.d, w.E, w.inter, w.n_shared, w.seed
    x = _randn((T, d), sd, 0)
    W_router = _randn((E, d), sd, 1, 1.0 / math.sqrt(d))
    W_gate_up = _randn((E, 2 * I, d), sd, 2, 1.0 / math.sqrt(d))
    W_down = _randn((E, d, I), sd, 3, 1.0 / math.sqrt(I))
    W_shared = None
    if S > 0:
        sh_gu = _randn((2 * S * I, d), sd, 4, 1.0 / math.sqrt(d))
        sh_d = _randn((d, S * I), sd, 5, 1.0 / math.sqrt(I))
        W_shared = torch.cat([sh_gu.reshape(-1), sh_d.reshape(-1)])
    u = None
    if w.skew:
        u = _randn((d,), sd, 6)
        u = u / u.norm()
        x.add_(u, alpha=SKEW_SHIFT)
        W_router[0] = (SKEW_ALPHA if skew_alpha is None else skew_alpha) * u
    dt = torch_dtype(w.dtype)

    def cast(t: torch.Tensor) -> torch.Tensor:
        return t.to(dt).contiguous() if dt != torch.float32 else t.contiguous()

    return Inputs(x=cast(x), W_router=cast(W_router), W_gate_up=cast(W_gate_up),
                  W_down=cast(W_down), W_shared=None if W_shared is None else cast(W_shared),
                  skew_u=u)


def shared_views(W_shared: torch.Tensor, d: int, inter: int, n_shared: int):
    """Split the flat shared-expert buffer into its gate_up [2*S*I, d] and down [d, S*I] views."""
    SI = n_shared * inter
    gu = W_shared[: 2 * SI * d].view(2 * SI, d)
    dn = W_shared[2 * SI * d: 2 * SI * d + d * SI].view(d, SI)
    return gu, dn


def make_dy(w: Workload) -> torch.Tensor:
    """Upstream gradient dL/dy [T, d] for the backward: N(0, 1), in the
    workload's dtype (stream 7 of the workload's seed)."""
    return _randn((w.T, w.d), w.seed, 7).to(torch_dtype(w.dtype)).contiguous()
