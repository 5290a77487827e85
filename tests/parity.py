"""Helpers that compare the CUDA path with the CPU oracle (test infrastructure).

Routing criterion: chosen expert sets must be identical (bit-exact indices)
for every token whose oracle decision gaps are both >= 1e-4 -- the gap
between the k-th chosen and best unchosen score inside the kept groups, and
the gap between the last kept and best dropped group score.  Near-tie tokens
are counted; where the GPU picked another set, that set must be within 1e-4
of optimal in the oracle's own scores, and the output of those tokens is then
checked against the oracle evaluated on the GPU's set.  The ordered list
(descending key) must equal the oracle's position by position wherever the
oracle's adjacent chosen keys differ by more than 1e-4.

Output criterion (bf16 inputs, fp32 accumulation): max |y - y_ref| <= 2e-2
and ||y - y_ref||_F / ||y_ref||_F <= 5e-3.  fp32 inputs: 1e-4 and 1e-5.
"""
from __future__ import annotations

import dataclasses
import json
import os

import numpy as np

import oracle

NEAR_TIE = 1e-4
TOL = {"bf16": (2e-2, 5e-3), "f32": (1e-4, 1e-5)}


@dataclasses.dataclass
class RoutingReport:
    n_tokens: int
    n_near_tie: int
    n_set_mismatch_near_tie: int
    n_order_exact: int  # tokens whose ordered list was required to equal the oracle's
    n_order_tied: int   # same set, some adjacent chosen keys within the tie threshold
    mismatched_tokens: np.ndarray  # near-tie tokens whose GPU set differs

    def record(self) -> dict:
        return {"tokens": self.n_tokens, "near_tie": self.n_near_tie,
                "near_tie_set_differs": self.n_set_mismatch_near_tie,
                "order_exact": self.n_order_exact, "order_tied": self.n_order_tied}


def check_routing(gpu_idx: np.ndarray, gpu_w: np.ndarray, ref: "oracle.Routing",
                  n_group: int, topk_group: int, E: int) -> RoutingReport:
    """Routing of every token against the oracle.

    * the chosen set equals the oracle's on every token that is not near-tie;
    * the ordered list equals the oracle's exactly (position by position)
      wherever the set is the same and the oracle's adjacent chosen keys
      differ by more than the tie threshold; where some adjacent keys are
      closer than that, every position holds a key within the threshold of
      the oracle's key at that position;
    * weights match the oracle's per expert (2e-5) and sum to 1 (1e-5);
    * near-tie tokens with another set: that set is within the threshold of
      optimal, expert- and group-wise.
    """
    T, k = gpu_idx.shape
    assert ((gpu_idx >= 0) & (gpu_idx < E)).all(), "expert index out of range"
    # no expert twice in one token
    srt = np.sort(gpu_idx, axis=1)
    assert (np.diff(srt, axis=1) > 0).all(), "an expert chosen twice"
    same = (srt == np.sort(ref.idx, axis=1)).all(axis=1)
    near = ref.near_tie(NEAR_TIE)
    bad = np.nonzero(~same & ~near)[0]
    assert bad.size == 0, f"routing differs on {bad.size} non-near-tie tokens, e.g. {bad[:8]}"
    # weights: same set -> same weights per expert (fp32 gate vs fp64)
    og = np.argsort(gpu_idx, axis=1)
    orf = np.argsort(ref.idx, axis=1)
    wg = np.take_along_axis(gpu_w, og, axis=1)[same]
    wr = np.take_along_axis(ref.w, orf, axis=1)[same]
    np.testing.assert_allclose(wg, wr, rtol=0, atol=2e-5)
    np.testing.assert_allclose(gpu_w.sum(axis=1), 1.0, atol=1e-5)
    # order
    key_ref = np.take_along_axis(ref.scores, ref.idx.astype(np.int64), axis=1)
    key_gpu = np.take_along_axis(ref.scores, gpu_idx.astype(np.int64), axis=1)
    assert (np.diff(key_ref, axis=1) <= 0).all(), "oracle list not in descending order"
    distinct = (-np.diff(key_ref, axis=1) > NEAR_TIE).all(axis=1)
    exact = same & distinct
    wrong = np.nonzero(exact & ~(gpu_idx == ref.idx).all(axis=1))[0]
    assert wrong.size == 0, (f"ordered top-k differs on {wrong.size} tokens with distinct "
                             f"keys, e.g. {wrong[:8]}")
    tied = same & ~distinct
    assert (np.abs(key_gpu - key_ref)[tied] <= NEAR_TIE).all(), "tied positions out of order"
    # near-tie tokens with another set: that set must be within 1e-4 of optimal
    mism = np.nonzero(~same)[0]
    gsz = E // n_group
    for t in mism:
        s = ref.scores[t]
        s_k = np.sort(s[ref.idx[t]])[0]
        assert s[gpu_idx[t]].min() >= s_k - NEAR_TIE, f"token {t}: GPU set not near-optimal"
        gs = s.reshape(n_group, gsz).max(axis=1)
        gs_tg = np.sort(gs)[::-1][topk_group - 1]
        groups = np.unique(gpu_idx[t] // gsz)
        assert groups.size <= topk_group
        assert gs[groups].min() >= gs_tg - NEAR_TIE, f"token {t}: GPU groups not near-optimal"
    return RoutingReport(T, int(near.sum()), int(mism.size), int(exact.sum()), int(tied.sum()),
                         mism)


def output_errors(y: np.ndarray, y_ref: np.ndarray):
    diff = y.astype(np.float64) - y_ref
    max_abs = float(np.abs(diff).max()) if diff.size else 0.0
    den = float(np.linalg.norm(y_ref))
    rel = float(np.linalg.norm(diff) / den) if den > 0 else float(np.linalg.norm(diff))
    return max_abs, rel


def check_output(y: np.ndarray, y_ref: np.ndarray, dtype: str):
    max_abs, rel = output_errors(y, y_ref)
    tol_abs, tol_rel = TOL[dtype]
    assert np.isfinite(y).all(), "non-finite output"
    assert max_abs <= tol_abs and rel <= tol_rel, (
        f"output mismatch: max_abs={max_abs:.3e} (tol {tol_abs}), rel_fro={rel:.3e} (tol {tol_rel})")
    return max_abs, rel


def oracle_outputs(inp, w, tokens, gpu_idx_rows, ref_routing, nthreads=0, score_func="sigmoid",
                   bias=None):
    """Oracle y for `tokens`; near-tie tokens whose GPU set differs are
    evaluated on the GPU's set (forced), the rest on the oracle's own."""
    tokens = np.asarray(tokens, dtype=np.int32)
    same = (np.sort(gpu_idx_rows, 1) == np.sort(ref_routing.idx[tokens], 1)).all(1)
    y_ref = np.zeros((len(tokens), w.d))
    if same.any():
        y_ref[same], _, _ = oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down,
                                           inp.W_shared, w.k, w.n_group, w.topk_group, w.inter,
                                           w.n_shared, tokens=tokens[same], nthreads=nthreads,
                                           score_func=score_func, bias=bias)
    if (~same).any():
        y_ref[~same], _, _ = oracle.forward(inp.x, inp.W_router, inp.W_gate_up, inp.W_down,
                                            inp.W_shared, w.k, w.n_group, w.topk_group,
                                            w.inter, w.n_shared, tokens=tokens[~same],
                                            forced_idx=gpu_idx_rows[~same], nthreads=nthreads,
                                            score_func=score_func, bias=bias)
    return y_ref


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    """First, last, tile-boundary and random tokens (sorted, unique)."""
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, T // 2, T - 2, T - 1]
    extra = rng.choice(T, size=min(T, max(0, n - len(fixed))), replace=False)
    s = np.unique(np.clip(np.concatenate([fixed, extra]), 0, T - 1))
    return s.astype(np.int32)


def write_record(test: str, fields: dict) -> None:
    """Append one JSON line describing a parity result to the file named by
    MOE_PARITY_RECORD (nothing when it is unset).  The fields are the values
    the test has already asserted on."""
    path = os.environ.get("MOE_PARITY_RECORD")
    if not path:
        return
    with open(path, "a") as f:
        f.write(json.dumps({"test": test, **fields}) + "\n")
