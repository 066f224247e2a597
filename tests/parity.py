"""Helpers shared by the GPU parity tests: run the C-ABI path on seeded inputs and
compare it with the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation on the GPU, fp64 oracle):
* block indices: identical, except near-tie rows, whose oracle gap between the
  last kept and the first dropped fp32-rounded score is below
  TIE_EPS * max(1, |largest kept past score|); there the GPU set must still be a valid
  top-k (current block kept, right size, strictly ascending, every kept past
  block within that margin of every dropped one).  The margin is the stated
  1e-5 for scores up to 1 and 1e-5 relative above: an fp32 score of magnitude
  |s| is itself only resolved to |s| * 2^-23 (at |s| = 68, two scores 1e-5
  apart are one ulp apart), so an absolute 1e-5 would ask two fp32
  computations of a large score to agree to the last bit;
* outputs: max |gpu - oracle| <= OUT_MAX_ABS and mean |gpu - oracle| <= OUT_MEAN_ABS;
* pooled keys (fp32): <= 1e-5 absolute; compressed tokens (bf16): one bf16
  rounding of the fp64 mean (relative 2^-8) plus 1e-6.
"""
from __future__ import annotations

import numpy as np
import torch

from dynamic_block_sparse_scoring_b200 import abi
from dynamic_block_sparse_scoring_b200.workloads import Workload, make_inputs
from oracle import nsa_oracle as O

TIE_EPS = 1e-5
OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
SCORE_ATOL = 1e-4
SCORE_RTOL = 1e-5


def f64(x: torch.Tensor) -> np.ndarray:
    return x.detach().to("cpu", torch.float64).numpy()


def oracle_cfg(wl: Workload) -> dict:
    return dict(h_q=wl.h_q, h_kv=wl.h_kv, d_qk=wl.d_qk, d_v=wl.d_v, sel_block=wl.sel_block,
                top_k=wl.top_k, window=wl.window, cmp_block=wl.cmp_block,
                cmp_stride=wl.cmp_stride, scale=wl.scale, branches=wl.branches,
                per_head_select=wl.per_head_select, gated=wl.gated, score_mode=wl.score_mode,
                sink_blocks=wl.sink_blocks)


def oracle_selection(wl: Workload, q: np.ndarray, pos: np.ndarray, K: np.ndarray, V=None):
    """(scores, idx, gap) of the oracle's selection for query rows q [R, Hq, d] at `pos`."""
    nb_all = -(-wl.seqlen_kv // wl.sel_block)
    pooled = {"Kbar": O.pool_block_keys(K, wl.sel_block)}
    if wl.score_mode == "cmp":
        pooled["Kc"] = O.compress(K, wl.cmp_block, wl.cmp_stride)
    s = O.selection_scores(oracle_cfg(wl), q, pos, pooled, nb_all)
    idx, gap = O.select_blocks(s, pos, wl.sel_block, wl.top_k, wl.sink_blocks)
    return s, idx, gap


class GpuCase:
    """Inputs for a workload on cuda:0 and the library's outputs for them."""

    def __init__(self, wl: Workload, seed=None):
        self.wl = wl
        self.cfg = abi.config(wl)
        self.x = make_inputs(wl, device="cuda", seed=seed)
        self.pooled = abi.alloc_pooled(self.cfg, "cuda")
        abi.nsa_pool_kv(self.cfg, self.x["k"], self.x["v"], self.pooled["kbar"],
                        self.pooled["kcmp"], self.pooled["vcmp"])
        self.idx = None
        if wl.branches & abi.NSA_BR_SEL:
            self.idx = torch.empty(wl.batch, wl.h_sel, wl.seqlen_q, wl.top_k, dtype=torch.int32,
                                   device="cuda")
            abi.nsa_topk_select_ex(self.cfg, self.x["q"], self.pooled["kbar"], self.pooled["kcmp"],
                                   None, self.idx)
        # the forward with the selection inside the call; it leaves its selected ids at
        # the start of the workspace
        ws = torch.empty(max(abi.nsa_workspace_size(self.cfg), 1), dtype=torch.uint8, device="cuda")
        self.out, _ = abi.forward(self.cfg, self.x["q"], self.x["k"], self.x["v"],
                                  self.x["gates"], pooled=self.pooled, workspace=ws)
        self.idx_fwd = None
        if self.idx is not None:
            n = self.idx.numel()
            self.idx_fwd = ws[:4 * n].view(torch.int32).view(self.idx.shape).clone()
        torch.cuda.synchronize()
        assert abi.nsa_get_device_status() == 0, "a kernel's bounded wait timed out"

    def oracle_rows(self, b: int, rows, idx=None):
        """Oracle (out, idx, gap) for sequence b and the given query rows."""
        wl, x = self.wl, self.x
        rows = np.asarray(rows)
        rows_t = torch.as_tensor(rows, device=x["q"].device)
        q = f64(x["q"][b].index_select(0, rows_t))
        K, V = f64(x["k"][b]), f64(x["v"][b])
        g = None if x["gates"] is None else f64(x["gates"][b].index_select(0, rows_t))
        pos = rows + wl.q_pos0
        return O.nsa_rows(oracle_cfg(wl), q, pos, K, V, g, idx=idx)


def tie_margin(ora_idx: np.ndarray, scores: np.ndarray, rows=None) -> np.ndarray:
    """TIE_EPS * max(1, |s|) per row, s = the largest |score| among the oracle's kept
    past blocks (computed for the (unit, row) pairs in `rows`, TIE_EPS elsewhere)."""
    U, R, _ = ora_idx.shape
    out = np.full((U, R), TIE_EPS)
    pairs = zip(*np.nonzero(np.ones((U, R), bool))) if rows is None else zip(*rows)
    for u, r in pairs:
        kept = [int(b) for b in ora_idx[u, r] if b >= 0 and np.isfinite(scores[u, r, b])]
        if kept:
            out[u, r] = TIE_EPS * max(1.0, float(np.abs(scores[u, r, kept]).max()))
    return out


def check_idx(gpu_idx: np.ndarray, ora_idx: np.ndarray, gap: np.ndarray, scores: np.ndarray,
              positions: np.ndarray, sel_block: int, top_k: int, n_sink: int = 0):
    """gpu_idx/ora_idx [U, R, k], gap [U, R], scores [U, R, nb] (oracle, -inf non-candidates)."""
    differ = (gpu_idx != ora_idx).any(axis=-1)
    margin = tie_margin(ora_idx, scores, np.nonzero(differ))
    bad = differ & ~(gap < margin)
    if bad.any():
        lines = []
        for u, r in list(zip(*np.nonzero(bad)))[:6]:
            g_set = {int(b) for b in gpu_idx[u, r] if b >= 0}
            o_set = {int(b) for b in ora_idx[u, r] if b >= 0}
            only_g, only_o = sorted(g_set - o_set), sorted(o_set - g_set)
            sg = [f"{scores[u, r, b]:.9g}" for b in only_g]
            so = [f"{scores[u, r, b]:.9g}" for b in only_o]
            lines.append(f"unit {u} row {r} pos {positions[r]} gap {gap[u, r]:.3g}: gpu-only "
                         f"{only_g} oracle s {sg}; oracle-only {only_o} oracle s {so}")
        raise AssertionError(f"{int(bad.sum())} rows select different blocks without a near-tie:\n"
                             + "\n".join(lines))
    for u, r in zip(*np.nonzero(differ)):
        c = int(positions[r]) // sel_block
        got = [int(b) for b in gpu_idx[u, r] if b >= 0]
        # strictly ascending (no repeated id), own block kept, right size
        assert got == sorted(set(got)) and c in got and len(got) == min(top_k, c + 1)
        # forced leading blocks are kept; the scored places compare like a plain top-k
        forced = list(range(min(n_sink, c)))
        assert all(b in got for b in forced)
        past = [b for b in got if b != c and b not in forced]
        dropped = [b for b in range(c) if b not in past and b not in forced]
        if past and dropped:
            s = scores[u, r]
            assert min(s[past]) >= max(s[dropped]) - margin[u, r]
    return int(differ.sum())


def check_out(gpu: np.ndarray, ora: np.ndarray, what=""):
    err = np.abs(gpu - ora)
    assert np.isfinite(gpu).all(), f"{what}: non-finite output"
    assert err.max() <= OUT_MAX_ABS, f"{what}: max abs err {err.max():.3e}"
    assert err.mean() <= OUT_MEAN_ABS, f"{what}: mean abs err {err.mean():.3e}"
    return float(err.max()), float(err.mean())


def check_selection_all_rows(run: "GpuCase", chunk: int = 2048):
    """Both GPU selections (stand-alone and inside the forward call) against the
    oracle's selection on every query row of every sequence, in row chunks.

    Returns the number of rows (per unit) resolved differently at a near-tie."""
    wl = run.wl
    ties = 0
    for b in range(wl.batch):
        K = f64(run.x["k"][b])
        for r0 in range(0, wl.seqlen_q, chunk):
            rows = np.arange(r0, min(wl.seqlen_q, r0 + chunk))
            pos = rows + wl.q_pos0
            rows_t = torch.as_tensor(rows, device=run.x["q"].device)
            q = f64(run.x["q"][b].index_select(0, rows_t))
            s, ora_idx, gap = oracle_selection(wl, q, pos, K, None)
            for got in (run.idx, run.idx_fwd):
                gpu_idx = got[b].index_select(1, rows_t).cpu().numpy()
                ties += check_idx(gpu_idx, ora_idx, gap, s, pos, wl.sel_block, wl.top_k,
                                  wl.sink_blocks)
    return ties
