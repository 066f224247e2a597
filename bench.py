"""Benchmark of the block-sparse attention forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload nsa64k] [--no-decode] [--no-e2e] [--no-cpu-baseline]

One step = the whole hot path over one batch of synthetic input already in
HBM: pool K/V (block keys + compressed tokens), fused block scoring + top-k,
and the gated three-branch attention.  Each step is preceded by an L2 flush
(a 256 MB write) outside the timed events.  Under torchrun every rank runs its
own independent sequence (seed = rank; weak scaling, no data-path
collective); the reported time is the max over ranks and ``value`` is the
aggregate algorithmic TFLOP/s of all ranks.  Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only, a
bounded sample of query rows per step).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, Workload, make_inputs  # noqa

METRIC = "64k-prefill sparse-attn TFLOP/s & tokens/s; decode KV GB/s (fraction of roofline)"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 FFMA peak: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz (max SM clock)
ALU_FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
CSRC = os.path.join(ROOT, "dynamic_block_sparse_scoring_b200", "csrc")
# stage name reported by nsa_timing_read -> (kernel, source file) for the ncu traffic record
STAGE_KERNELS = {
    "attn_tc": ("attn_tc_kernel", os.path.join(CSRC, "attn_tc.cu")),
    "sel_bm": ("sel_bm_kernel", os.path.join(CSRC, "attn_sel_bm.cu")),
    "sel_merge": ("sel_merge_kernel", os.path.join(CSRC, "sel_merge.cu")),
    "index": ("sel_index", os.path.join(CSRC, "sel_index.cu")),
    "expand": ("expand_kernel", os.path.join(CSRC, "sel_index.cu")),
    "split_merge": ("split_merge_kernel", os.path.join(CSRC, "attn_tc.cu")),
    "rowwise": ("attn_rowwise_kernel", os.path.join(CSRC, "attn_rowwise.cu")),
    "attn_dec": ("dec_kernel", os.path.join(CSRC, "attn_decode.cu")),
    "dec_merge": ("dec_merge_kernel", os.path.join(CSRC, "attn_decode.cu")),
    "select": ("score_tc_kernel", os.path.join(CSRC, "score_tc.cu")),
}


# ---------------------------------------------------------------------------
# Algorithmic work (only causally visible keys count)
# ---------------------------------------------------------------------------

def visible_key_counts(wl: Workload):
    t = np.arange(wl.seqlen_q, dtype=np.int64) + wl.q_pos0
    c = t // wl.sel_block
    out = {}
    if wl.branches & 2:
        out["sel"] = np.minimum(wl.top_k - 1, c) * wl.sel_block + (t - c * wl.sel_block + 1)
    if wl.branches & 4:
        out["win"] = np.minimum(wl.window, t + 1)
    if wl.branches & 1:
        n_cmp = (wl.seqlen_kv - wl.cmp_block) // wl.cmp_stride + 1 if wl.seqlen_kv >= wl.cmp_block else 0
        nv = np.where(t >= wl.cmp_block - 1, (t - wl.cmp_block + 1) // wl.cmp_stride + 1, 0)
        out["cmp"] = np.minimum(nv, n_cmp)
    return out


def algorithmic_flops(wl: Workload, rows=None) -> dict:
    """FLOPs of the branches (2*(d_qk+d_v) per query, head and visible key) and the scoring
    (2*d_qk per query row, selection unit and candidate block), per sequence."""
    keys = visible_key_counts(wl)
    sel = slice(None) if rows is None else np.asarray(rows)
    per_key = 2 * (wl.d_qk + wl.d_v) * wl.h_q
    f = {name: float(v[sel].sum()) * per_key for name, v in keys.items()}
    t = np.arange(wl.seqlen_q, dtype=np.int64) + wl.q_pos0
    cand = np.minimum(t // wl.sel_block, wl.seqlen_kv // wl.sel_block)
    f["score"] = float(cand[sel].sum()) * 2 * wl.d_qk * wl.h_sel if wl.branches & 2 else 0.0
    f["total"] = sum(f.values())
    return f


def decode_bytes(wl: Workload, idx: torch.Tensor) -> float:
    """Bytes a decode step must read/write: pooled keys, compressed K/V, the union of
    window and selected tokens per (sequence, KV head), q, gates and out."""
    B, Hkv = wl.batch, wl.h_kv
    nb_full = wl.seqlen_kv // wl.sel_block
    n_cmp = (wl.seqlen_kv - wl.cmp_block) // wl.cmp_stride + 1
    t = wl.q_pos0
    kbar = B * Hkv * min(t // wl.sel_block, nb_full) * wl.d_qk * 4
    cmpb = B * Hkv * n_cmp * (wl.d_qk + wl.d_v) * 2
    win_lo = max(0, t - wl.window + 1)
    tok = 0
    idx_c = idx.cpu().numpy()
    for b in range(B):
        for g in range(Hkv):
            keys = set(range(win_lo, t + 1))
            for blk in idx_c[b, g, 0]:
                if blk >= 0:
                    keys.update(range(blk * wl.sel_block, min((blk + 1) * wl.sel_block, t + 1)))
            tok += len(keys)
    kv = tok * (wl.d_qk + wl.d_v) * 2
    small = B * wl.h_q * (wl.d_qk * 2 + 3 * 4 + wl.d_v * 2)
    return float(kbar + cmpb + kv + small)


# ---------------------------------------------------------------------------
# Clocks sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index=0):
        self.proc = None
        self.path = None
        self.dev = self._device_id(device_index)

    @staticmethod
    def _device_id(i):
        try:
            u = str(torch.cuda.get_device_properties(i).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            return str(i)

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", self.dev], stdout=open(self.path, "w"),
                stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) >= 9 and p[1].replace(".", "").isdigit():
                rows.append(p)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows]
        mx = float(rows[0][2])
        loaded = [r for r in rows if float(r[1]) > 0.5 * mx] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(float(r[1]) for r in loaded), "sm_max_mhz": mx,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())
                if any(r[3].replace(".", "").isdigit() for r in rows) else None,
                "sm_mhz_min": min(sm)}


# ---------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------

def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return FALLBACK, "fallback"


def traffic_for(kernel: str, source: str):
    """DRAM bytes per launch recorded by ncu for `kernel`, if its source is unchanged."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        rec = json.load(f).get(kernel)
    if not rec:
        return None
    sha = hashlib.sha256(open(source, "rb").read()).hexdigest()
    return rec["bytes_per_launch"] if rec.get("src_sha256") == sha else None


class Prefill:
    """Device buffers and one timed step of the prefill hot path."""

    def __init__(self, wl: Workload, seed: int):
        from dynamic_block_sparse_scoring_b200 import abi
        self.abi, self.wl = abi, wl
        self.cfg = abi.config(wl)
        self.x = make_inputs(wl, device="cuda", seed=seed)
        self.pooled = abi.alloc_pooled(self.cfg, "cuda")
        self.idx = torch.empty(wl.batch, wl.h_sel, wl.seqlen_q, wl.top_k, dtype=torch.int32,
                               device="cuda")
        self.out = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, wl.d_v, dtype=torch.bfloat16,
                               device="cuda")
        self.ws_bytes = abi.nsa_workspace_size(self.cfg)
        self.ws = torch.empty(max(self.ws_bytes, 1), dtype=torch.uint8, device="cuda")
        self.launches_per_step = 0
        self.append = None

    def enable_append(self, seed: int):
        """Decode: each step first appends the query's own token to the cache
        (nsa_append_kv at the query position, refreshing the pooled tokens it completes)
        instead of pooling the whole cache."""
        wl = self.wl
        g = torch.Generator(device="cuda")
        g.manual_seed(seed)
        self.append = {
            "cfg": self.abi.config(wl, seqlen_q=1, q_pos0=wl.q_pos0),
            "side": torch.cuda.Stream(),
            "k": torch.randn(wl.batch, wl.h_kv, 1, wl.d_qk, generator=g, device="cuda").to(torch.bfloat16),
            "v": torch.randn(wl.batch, wl.h_kv, 1, wl.d_v, generator=g, device="cuda").to(torch.bfloat16)}

    def append_bytes(self) -> float:
        """Bytes one append moves: the new rows, the keys of the selection block and the
        K/V window of the compressed token it completes (if any), and their pooled tokens."""
        wl, t = self.wl, self.wl.q_pos0
        rows = wl.batch * wl.h_kv
        n = rows * (wl.d_qk + wl.d_v) * 2                              # new K/V rows written
        if (t + 1) % wl.sel_block == 0:
            n += rows * (wl.sel_block * wl.d_qk * 2 + wl.d_qk * 4)     # block keys read, mean written
        if t + 1 >= wl.cmp_block and (t + 1 - wl.cmp_block) % wl.cmp_stride == 0:
            n += rows * (wl.cmp_block + 1) * (wl.d_qk + wl.d_v) * 2    # window read, token written
        return float(n)

    def append_launches(self) -> int:
        wl, t = self.wl, self.wl.q_pos0
        return 1 + int((t + 1) % wl.sel_block == 0) + \
            int(t + 1 >= wl.cmp_block and (t + 1 - wl.cmp_block) % wl.cmp_stride == 0)

    def attn_launches(self) -> int:
        """Kernels nsa_sparse_attn_fwd launches with the selection inside (the library
        reports its own plan: the selection, block-major adds the index build, its
        attention kernel and the partial merge; split-K and decode add a merge)."""
        self.path, n = self.abi.nsa_attn_plan(self.cfg, bool(self.wl.branches & 2), self.ws_bytes)
        return n

    def step(self, ev=None, pool=True):
        a, x, p = self.abi, self.x, self.pooled
        n = 0
        if ev:
            ev[0].record()
        if pool and self.append is not None:
            # decode: the cache append and the block selection are independent (a new
            # token completes at most its own block, which is never a scored candidate),
            # so the append runs on a side stream next to the selection; the attention
            # waits for both
            ap, cur = self.append, torch.cuda.current_stream()
            ap["side"].wait_stream(cur)
            with torch.cuda.stream(ap["side"]):
                a.nsa_append_kv(ap["cfg"], x["k"], x["v"], ap["k"], ap["v"], p["kbar"], p["kcmp"],
                                p["vcmp"])
            if ev:
                ev[1].record()
            a.nsa_topk_select(self.cfg, x["q"], p["kbar"], None, self.idx)
            cur.wait_stream(ap["side"])
            if ev:
                ev[2].record()
            a.nsa_sparse_attn_fwd(self.cfg, x["q"], x["k"], x["v"], p["kbar"], p["kcmp"], p["vcmp"],
                                  x["gates"], self.idx, self.out, self.ws, self.ws_bytes)
            if ev:
                ev[3].record()
            self.path, k_attn = self.abi.nsa_attn_plan(self.cfg, False, self.ws_bytes)
            self.launches_per_step = self.append_launches() + 1 + k_attn
            return
        if pool:
            a.nsa_pool_kv(self.cfg, x["k"], x["v"], p["kbar"], p["kcmp"], p["vcmp"])
            n += int(self.wl.branches & 2 > 0 and self.cfg.seqlen_kv >= self.cfg.sel_block) + \
                int(self.wl.branches & 1 > 0)
        if ev:
            ev[1].record()
            ev[2].record()
        # selection inside the call (idx NULL): it leaves the selected ids at the start
        # of the workspace, read back into self.idx after the timed steps
        a.nsa_sparse_attn_fwd(self.cfg, x["q"], x["k"], x["v"], p["kbar"], p["kcmp"], p["vcmp"],
                              x["gates"], None, self.out, self.ws, self.ws_bytes)
        n += self.attn_launches()
        if ev:
            ev[3].record()
        self.launches_per_step = n

    def selected_ids(self):
        if self.append is not None:
            return self.idx                   # decode steps select into idx directly
        if self.wl.branches & 2:
            self.idx.copy_(self.ws[:4 * self.idx.numel()].view(torch.int32).view(self.idx.shape))
        return self.idx


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The largest of every rank's `v` (the slowest rank's time).  Every rank must
    call it the same number of times in the same order."""
    if world == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput (units per second): every rank processes the same
    number of units (weak scaling), and the job takes as long as its slowest rank."""
    return units_per_rank * world / (ms_max / 1e3)


def rank_seed(rank: int, decode: bool = False) -> int:
    """Each rank draws its own independent problem."""
    return (1000 if decode else 0) + rank


def timed_steps(pf: Prefill, steps: int, warmup: int, world: int, pool=True):
    """Per-step device times (pool, select, attention) and the mean time of every stage
    inside the attention call (the library's stage events on the launching stream; the
    host reads them between steps, outside the steps' own events)."""
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    for _ in range(warmup):
        flush.fill_(1.0)
        pf.step(pool=pool)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    stages = {}
    barrier(world)
    torch.cuda.synchronize()
    pf.abi.nsa_timing_enable(True)
    wall0 = time.perf_counter()
    for s in range(steps):
        flush.fill_(float(s))
        pf.step(evs[s], pool=pool)
        for name, ms in pf.abi.nsa_timing_read():
            stages.setdefault(name, []).append(ms)
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    pf.abi.nsa_timing_enable(False)
    barrier(world)
    per = np.array([[e[0].elapsed_time(e[1]), e[1].elapsed_time(e[2]), e[2].elapsed_time(e[3])]
                    for e in evs])                                     # ms: pool, select, attn
    return per, wall, {k: float(np.mean(v)) for k, v in stages.items()}


def stage_rooflines(wl: Workload, path: str, stage_ms: dict, idx: torch.Tensor, pk: dict) -> dict:
    """Algorithmic work of every attention stage over its measured mean duration.

    Tensor-core stages count the branch FLOPs they compute (block-major: the selected
    branch in sel_bm, window + compressed in attn_tc; otherwise attn_tc does all three).
    The index and merge stages are HBM-bound: they count the bytes they must move."""
    fl = algorithmic_flops(wl)
    B = wl.batch
    idx_bytes = idx.numel() * 4
    n_valid = int((idx >= 0).sum().item()) if wl.branches & 2 else 0
    hpt = wl.h_q // wl.h_sel
    # the selected branch alone with one head per unit runs over 64-key sub-blocks: a kept
    # block is one partial per sub-block that starts at or before the query
    spb = wl.sel_block // 64 if (wl.branches == 2 and hpt == 1 and wl.sel_block % 64 == 0) else 1
    n_parts = n_valid
    if spb > 1 and n_valid:
        ic = idx.cpu().numpy()
        t = (np.arange(wl.seqlen_q) + wl.q_pos0)[None, None, :, None]
        n_parts = int(np.where(ic >= 0, np.clip((t - ic * wl.sel_block) // 64 + 1, 0, spb), 0).sum())
    out = {}
    for name, ms in stage_ms.items():
        if ms <= 0:
            continue
        if name == "select":
            if wl.seqlen_q > 16:         # tensor cores, tf32 (3 products per pair; 1 counted)
                work = fl["score"] * B
                peak = pk["bf16_tflops"] * 1.1 / 2.25
                ach = work / (ms / 1e3) / 1e12
                out[name] = {"ms": ms, "bound": "tensor", "unit": "TFLOP/s", "work": work,
                             "achieved": ach, "peak": peak, "frac": ach / peak,
                             "peak_note": "tf32 = measured bf16 x 1.1/2.25 (nominal ratio)"}
            else:                        # few rows: streams the pooled keys
                t = np.arange(wl.seqlen_q) + wl.q_pos0
                cand = np.minimum(t // wl.sel_block, wl.seqlen_kv // wl.sel_block)
                work = float(cand.sum()) * wl.d_qk * 4 * B * wl.h_sel / max(1, wl.h_sel // wl.h_kv)
                ach = work / (ms / 1e3) / 1e9
                out[name] = {"ms": ms, "bound": "hbm", "unit": "GB/s", "work": work,
                             "achieved": ach, "peak": pk["hbm_gbs"], "frac": ach / pk["hbm_gbs"]}
            continue
        if name in ("attn_tc", "sel_bm", "rowwise"):
            if name == "sel_bm":
                work = fl.get("sel", 0.0) * B
            elif path == "block-major":
                work = (fl.get("win", 0.0) + fl.get("cmp", 0.0)) * B
            else:
                work = (fl["total"] - fl["score"]) * B
            ach = work / (ms / 1e3) / 1e12
            out[name] = {"ms": ms, "bound": "tensor", "unit": "TFLOP/s", "work": work,
                         "achieved": ach, "peak": pk["bf16_tflops"], "frac": ach / pk["bf16_tflops"]}
        else:
            if name == "sel_merge":      # read every valid partial (o bf16 + lse), write o_sel
                work = n_parts * hpt * (2 * wl.d_v + 4) + B * wl.seqlen_q * wl.h_q * wl.d_v * 2 + idx_bytes * spb
            elif name == "index":        # read idx twice, write the pair lists
                work = 2 * idx_bytes * spb + n_parts * 4
            elif name == "expand":       # read the kept blocks, write their sub-blocks
                work = idx_bytes * (1 + spb)
            else:                        # split merge: fp32 (o, l, m) per split, branch and row
                work = 0.0
            ach = work / (ms / 1e3) / 1e9
            out[name] = {"ms": ms, "bound": "hbm", "unit": "GB/s", "work": work,
                         "achieved": ach, "peak": pk["hbm_gbs"], "frac": ach / pk["hbm_gbs"]}
    return out


SELECTED_STAGES = ("index", "sel_bm", "sel_merge", "expand")


def selected_roofline(wl: Workload, path: str, stage_ms: dict, pk: dict):
    """The selected branch's algorithmic FLOPs over the time of every stage that serves
    only that branch (block-major plans: the inverted index, the block-major attention
    and the partial merge; the selection itself is counted separately, as "select").
    None when the plan computes the selected branch inside another kernel."""
    if not wl.branches & 2 or path != "block-major":
        return None
    parts = {k: v for k, v in stage_ms.items() if k in SELECTED_STAGES}
    if "sel_bm" not in parts:
        return None
    ms = sum(parts.values())
    work = algorithmic_flops(wl)["sel"] * wl.batch
    ach = work / (ms / 1e3) / 1e12
    return {"stages": sorted(parts), "ms": ms, "bound": "tensor", "unit": "TFLOP/s",
            "flops_per_step": work, "achieved": ach, "peak": pk["bf16_tflops"],
            "frac": ach / pk["bf16_tflops"],
            "peak_source": "measured dense bf16 (burst, cuBLAS)"}


def e2e_steps(pf: Prefill, steps: int, warmup: int, world: int):
    """Same step through the public API with pinned host inputs: every step copies its
    own inputs host->device, runs the forward (pool + select + attention) and reads its
    output back device->host.  The three run on their own streams with two sets of
    device buffers, so that step i's copies overlap the compute of steps i - 1 and
    i + 1 (PCIe is full duplex); the timed region runs from the first input copy to the
    last output copy."""
    a, wl = pf.abi, pf.wl
    host = {k: v.cpu().pin_memory() for k, v in pf.x.items() if v is not None}
    out_h = [torch.empty(pf.out.shape, dtype=pf.out.dtype).pin_memory() for _ in range(2)]
    dev = [{k: torch.empty_like(v, device="cuda") for k, v in host.items()} for _ in range(2)]
    outs = [pf.out, torch.empty_like(pf.out)]
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = out_h[0].numel() * out_h[0].element_size()
    ws = pf.ws_bytes
    work = pf.ws
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    s_comp = torch.cuda.current_stream()
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_done = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def one(i):
        b = i % 2
        if used[b]:
            s_in.wait_event(comp_done[b])          # the inputs of step i - 2 are consumed
            s_comp.wait_event(out_done[b])         # its output has been read back
        with torch.cuda.stream(s_in):
            for k in host:
                dev[b][k].copy_(host[k], non_blocking=True)
            in_ready[b].record(s_in)
        s_comp.wait_event(in_ready[b])
        d = dev[b]
        a.nsa_pool_kv(pf.cfg, d["k"], d["v"], pf.pooled["kbar"], pf.pooled["kcmp"], pf.pooled["vcmp"],
                      stream=s_comp)
        a.nsa_sparse_attn_fwd(pf.cfg, d["q"], d["k"], d["v"], pf.pooled["kbar"], pf.pooled["kcmp"],
                              pf.pooled["vcmp"], d.get("gates"), None, outs[b], work, ws, stream=s_comp)
        comp_done[b].record(s_comp)
        s_out.wait_event(comp_done[b])
        with torch.cuda.stream(s_out):
            out_h[b].copy_(outs[b], non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        one(warmup + i)
    e1.record(s_out)
    torch.cuda.synchronize()
    barrier(world)
    return e0.elapsed_time(e1) / steps, h2d, d2h


def cpu_baseline(wl: Workload, x, budget_s: float = 15.0, rows_per_step=None):
    """Time the fp64 oracle on an evenly strided sample of query rows (sequence 0)."""
    from oracle import nsa_oracle as O

    def f64(t):
        return t.detach().to("cpu", torch.float64).numpy()

    ocfg = dict(h_q=wl.h_q, h_kv=wl.h_kv, d_qk=wl.d_qk, d_v=wl.d_v, sel_block=wl.sel_block,
                top_k=wl.top_k, window=wl.window, cmp_block=wl.cmp_block,
                cmp_stride=wl.cmp_stride, scale=wl.scale, branches=wl.branches,
                per_head_select=wl.per_head_select)
    # One Python process walks the rows; only numpy's BLAS products inside a row may
    # run on more threads.  Report the process as one core and the BLAS pool beside it.
    try:
        from threadpoolctl import threadpool_info
        blas_threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        blas_threads = 1
    cores = 1
    K, V = f64(x["k"][0]), f64(x["v"][0])
    T = wl.seqlen_q
    t0 = time.perf_counter()
    pooled = O.pooled_inputs(K, V, wl.sel_block, wl.cmp_block if wl.branches & 1 else 0,
                             wl.cmp_stride if wl.branches & 1 else 1)
    t_pool = time.perf_counter() - t0
    n = 8 if rows_per_step is None else rows_per_step
    spent, done_rows, flops = 0.0, 0, 0.0
    rng_rows = np.linspace(0, T - 1, num=max(n, 1)).astype(np.int64)
    while True:
        rows = rng_rows
        rows_t = torch.as_tensor(rows, device=x["q"].device)
        q = f64(x["q"][0].index_select(0, rows_t))
        g = None if x["gates"] is None else f64(x["gates"][0].index_select(0, rows_t))
        t0 = time.perf_counter()
        O.nsa_rows(ocfg, q, rows + wl.q_pos0, K, V, g, pooled=pooled)
        spent += time.perf_counter() - t0
        done_rows += len(rows)
        flops += algorithmic_flops(wl, rows)["total"]
        if rows_per_step is not None or spent > budget_s:
            break
        rng_rows = np.linspace(done_rows % 7, T - 1, num=n).astype(np.int64)
    total = spent + t_pool
    return {"value": flops / total / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "parallelism": f"one Python process (row loop single-threaded; numpy BLAS products "
                           f"may use up to {blas_threads} threads of the {os.cpu_count()} host "
                           f"cores)",
            "sample": f"{done_rows} evenly strided query rows of {wl.name} sequence 0 "
                      f"(all selection units, all branches, K/V pooling included: "
                      f"{t_pool:.1f} s pooling + {spent:.1f} s rows)",
            "seconds": total, "rows": done_rows}


def graph_steps(pf: Prefill, steps: int, warmup: int, world: int) -> float:
    """Mean device time of one decode step (the cache append when enabled, selection,
    attention), captured once as a CUDA graph and replayed, so that host launch gaps
    between the few short kernels of a decode step are not counted.  The 256 MB L2 flush
    runs before every replay, outside the timed events."""
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    pool = pf.append is not None                      # decode: the append is part of the step
    with torch.cuda.stream(side):                    # warm-up (and lazy set-up) outside capture
        pf.step(pool=pool)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pf.step(pool=pool)
    for _ in range(warmup):
        flush.fill_(1.0)
        g.replay()
    torch.cuda.synchronize()
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for k in range(steps):
        flush.fill_(float(k))
        evs[k][0].record()
        g.replay()
        evs[k][1].record()
    torch.cuda.synchronize()
    barrier(world)
    ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    del g
    return ms


def run_decode(world: int, steps: int, warmup: int):
    wl = WORKLOADS["decode64x64k"]
    seed = rank_seed(torch.distributed.get_rank() if world > 1 else 0, decode=True)
    pf = Prefill(wl, seed=seed)
    pf.step()                        # the prefilled cache pooled once (before decoding, not timed)
    torch.cuda.synchronize()
    # a decode step: append the query's own token (pooled tokens refreshed incrementally),
    # select, attend
    pf.enable_append(seed + 500)
    per, _, dec_stages = timed_steps(pf, steps, warmup, world, pool=True)
    pf.attn_launches()
    path = pf.path
    ms_stream = float(per.sum(axis=1).mean())
    ms_sel_append = float(per[:, 1].mean())       # selection, with the append beside it
    ms = max_over_ranks(graph_steps(pf, steps, warmup, world), world)
    nbytes = decode_bytes(wl, pf.selected_ids()) + pf.append_bytes()
    pk, _ = peaks()
    gbs = job_rate(nbytes, world, ms) / 1e9
    pf_append_bytes = pf.append_bytes()
    del pf
    torch.cuda.empty_cache()
    return {"workload": wl.name, "ms_per_step": ms, "value": gbs, "unit": "GB/s",
            "bytes_per_step": nbytes, "frac": gbs / world / pk["hbm_gbs"],
            "peak_gbs": pk["hbm_gbs"], "path": path, "timing": "CUDA graph replay",
            "ms_per_step_stream": ms_stream, "select_with_append_ms_stream": ms_sel_append,
            "append_bytes": pf_append_bytes,
            "frac_stream": job_rate(nbytes, world, ms_stream) / 1e9 / world / pk["hbm_gbs"],
            "frac_note": "frac: the step replayed as one CUDA graph; frac_stream: the same "
                         "kernels launched one by one on the stream (host launch gaps included)",
            "stage_ms": dec_stages}


def config_of(wl: Workload, world: int) -> dict:
    """The workload description both arms print."""
    return {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seqlen_q,
            "h_q": wl.h_q, "h_kv": wl.h_kv, "d_qk": wl.d_qk, "d_v": wl.d_v,
            "sel_block": wl.sel_block, "top_k": wl.top_k, "window": wl.window,
            "cmp": [wl.cmp_block, wl.cmp_stride],
            "parallelism": f"independent sequences x{world}",
            "l2": "256 MB flush before every step; inputs > L2"}


def run_config(name: str, steps: int, warmup: int, world: int, rank: int):
    """One prefill workload through the same step as the headline: mean step time,
    tokens/s, algorithmic TFLOP/s and the stage rooflines."""
    wl = WORKLOADS[name]
    pf = Prefill(wl, seed=rank_seed(rank))
    per, _, stage_ms = timed_steps(pf, steps, warmup, world)
    ms = max_over_ranks(float(per.sum(axis=1).mean()), world)
    fl = algorithmic_flops(wl)
    pk, _ = peaks()
    pf.attn_launches()
    stages = stage_rooflines(wl, pf.path, stage_ms, pf.selected_ids(), pk)
    launches = pf.launches_per_step
    status = pf.abi.nsa_get_device_status()
    res = {"workload": name, "batch": wl.batch, "seq_len": wl.seqlen_q, "h_q": wl.h_q,
           "h_kv": wl.h_kv, "d_qk": wl.d_qk, "d_v": wl.d_v, "sel_block": wl.sel_block,
           "top_k": wl.top_k, "per_head_select": wl.per_head_select, "steps": steps,
           "ms_per_step": ms, "tokens_per_s": job_rate(wl.seqlen_q * wl.batch, world, ms),
           "value": job_rate(fl["total"] * wl.batch, world, ms) / 1e12, "unit": "TFLOP/s",
           "algorithmic_flops_per_step": fl["total"] * wl.batch, "path": pf.path,
           "kernels_per_step": launches,
           "stages": {k: {"ms": v["ms"], "achieved": v["achieved"], "unit": v["unit"],
                          "frac": v["frac"], "bound": v["bound"]} for k, v in stages.items()},
           "roofline_selected": selected_roofline(wl, pf.path, stage_ms, pk)}
    del pf
    torch.cuda.empty_cache()
    if status != 0:
        raise SystemExit(f"device status {status} on {name}: a kernel's bounded wait timed out")
    return res


def _event_ms(fn, steps: int, warmup: int) -> float:
    """Mean device time of fn() over `steps` calls after `warmup`, each call preceded by a
    256 MB L2 flush; CUDA events on the current stream."""
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    for _ in range(warmup):
        flush.fill_(1.0)
        fn()
    torch.cuda.synchronize()
    tot = 0.0
    for s in range(steps):
        flush.fill_(float(s))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        tot += e0.elapsed_time(e1)
    return tot / steps


def run_backward(steps: int, warmup: int, seqlen: int = 8192):
    """The backward pass (nsa_sparse_attn_bwd) on the 64k prefill's shapes at `seqlen`
    queries, for the blocks the forward selected.  Algorithmic work: per visible (query,
    head, key) 2*(3*d_qk + 2*d_v) FLOP (S recomputed, dP, dV, dQ, dK); the kernel runs on
    the FP32 FFMA units, so the roofline is their peak."""
    from dynamic_block_sparse_scoring_b200 import abi
    wl = WORKLOADS["nsa64k"].with_(name=f"nsa64k_bwd_{seqlen}", seqlen_q=seqlen, seqlen_kv=seqlen)
    cfg = abi.config(wl)
    x = make_inputs(wl, device="cuda", seed=0)
    idx = torch.empty(wl.batch, wl.h_sel, wl.seqlen_q, wl.top_k, dtype=torch.int32, device="cuda")
    pooled = abi.alloc_pooled(cfg, "cuda")
    abi.nsa_pool_kv(cfg, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
    abi.nsa_topk_select(cfg, x["q"], pooled["kbar"], None, idx)
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    d_out = torch.randn(wl.batch, wl.seqlen_q, wl.h_q, wl.d_v, generator=g, device="cuda").to(torch.bfloat16)
    dq = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, wl.d_qk, device="cuda")
    dk = torch.empty(wl.batch, wl.h_kv, wl.seqlen_kv, wl.d_qk, device="cuda")
    dv = torch.empty(wl.batch, wl.h_kv, wl.seqlen_kv, wl.d_v, device="cuda")
    dg = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, 3, device="cuda")
    ws = torch.empty(max(abi.nsa_bwd_workspace_size(cfg), 1), dtype=torch.uint8, device="cuda")

    def call():
        abi.nsa_sparse_attn_bwd(cfg, x["q"], x["k"], x["v"], pooled["kcmp"], pooled["vcmp"], x["gates"],
                                idx, d_out, dq, dk, dv, dg, ws, ws.numel())
    ms = _event_ms(call, steps, warmup)
    keys = sum(float(v.sum()) for v in visible_key_counts(wl).values())
    flops = keys * wl.h_q * 2 * (3 * wl.d_qk + 2 * wl.d_v) * wl.batch
    status = abi.nsa_get_device_status()
    if status != 0:
        raise SystemExit(f"device status {status} in the backward: a kernel's bounded wait timed out")
    return {"workload": wl.name, "seq_len": seqlen, "steps": steps, "ms_per_step": ms,
            "algorithmic_flops_per_step": flops, "value": flops / ms / 1e9, "unit": "TFLOP/s",
            "bound": "alu", "peak": ALU_FP32_TFLOPS, "frac": flops / ms / 1e9 / ALU_FP32_TFLOPS,
            "peak_source": "FP32 FFMA: 148 SMs x 128 lanes x 2 FLOP x 1.965 GHz"}


def run_selection_variants(steps: int, warmup: int, seqlen: int = 16384):
    """The block selection alone (nsa_topk_select_ex) on the 64k prefill's shapes at `seqlen`
    queries, for each score definition: summed scaled dot products (the default, on the
    tensor cores inside the forward; here the stand-alone FFMA kernel), summed per-head
    probabilities, compressed-branch weights, and the default with two forced sink blocks.
    Reported as ms per call and (query, selection unit) rows per second."""
    from dynamic_block_sparse_scoring_b200 import abi
    from dynamic_block_sparse_scoring_b200.workloads import SCORE_CMP, SCORE_PROB, SINK_SHIFT
    wl = WORKLOADS["nsa64k"].with_(seqlen_q=seqlen, seqlen_kv=seqlen)
    x = make_inputs(wl, device="cuda", seed=0)
    base = abi.config(wl)
    pooled = abi.alloc_pooled(base, "cuda")
    abi.nsa_pool_kv(base, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
    idx = torch.empty(wl.batch, wl.h_sel, wl.seqlen_q, wl.top_k, dtype=torch.int32, device="cuda")
    out = {}
    for name, extra in (("dot", 0), ("prob", SCORE_PROB), ("cmp", SCORE_CMP), ("dot_2_sinks", 2 << SINK_SHIFT)):
        cfg = abi.config(wl, flags=wl.flags | extra)
        ms = _event_ms(lambda: abi.nsa_topk_select_ex(cfg, x["q"], pooled["kbar"], pooled["kcmp"], None, idx),
                       steps, warmup)
        out[name] = {"ms": ms, "rows_per_s": wl.batch * wl.h_sel * wl.seqlen_q / ms * 1e3}
    status = abi.nsa_get_device_status()
    if status != 0:
        raise SystemExit(f"device status {status} in the selection variants")
    return {"workload": f"nsa64k shapes at {seqlen} queries", "steps": steps, "variants": out}


def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if world > 1:
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    wl = WORKLOADS[args.workload]
    if args.seqlen:
        wl = wl.with_(seqlen_q=args.seqlen, seqlen_kv=args.seqlen)
    if args.batch:
        wl = wl.with_(batch=args.batch)
    pf = Prefill(wl, seed=rank_seed(rank))
    clocks = ClockSampler(torch.cuda.current_device())
    # warm-up and timed region (clocks sampled during it)
    clocks.start()
    per, wall, stage_ms = timed_steps(pf, args.steps, args.warmup, world)
    clk = clocks.stop()
    step_ms = per.sum(axis=1)
    ms = max_over_ranks(float(step_ms.mean()), world)
    fl = algorithmic_flops(wl)
    fl_all = fl["total"] * wl.batch * world
    value = job_rate(fl["total"] * wl.batch, world, ms) / 1e12
    tokens = job_rate(wl.seqlen_q * wl.batch, world, ms)
    pk, src = peaks()
    pf.attn_launches()
    stages = stage_rooflines(wl, pf.path, stage_ms, pf.selected_ids(), pk)
    stage_ms_all = {k: max_over_ranks(v["ms"], world) for k, v in stages.items()}
    dom = max(stages, key=lambda k: stages[k]["ms"])
    d = dict(stages[dom])
    d["achieved"] *= d["ms"] / stage_ms_all[dom]       # slowest rank
    d["frac"] = d["achieved"] / d["peak"]
    kernel, source = STAGE_KERNELS[dom]
    roof = {"what": "dominant stage: the longest stage of the step",
            "kernel": kernel, "stage": dom, "bound": d["bound"], "achieved": d["achieved"],
            "peak": d["peak"], "unit": d["unit"], "frac": d["frac"],
            "traffic": traffic_for(kernel, source),
            "peak_source": f"{src} " + ("dense bf16 (burst, cuBLAS)" if d["bound"] == "tensor"
                                        else "HBM copy"),
            ("flops_per_launch" if d["bound"] == "tensor" else "bytes_per_launch"): d["work"],
            "launch_ms": stage_ms_all[dom],
            "share_of_step": float(stage_ms[dom] / step_ms.mean()),
            "path": pf.path,
            "stages": {k: {"ms": v["ms"], "achieved": v["achieved"], "unit": v["unit"],
                           "frac": v["frac"], "bound": v["bound"]} for k, v in stages.items()}}
    sel_roof = selected_roofline(wl, pf.path, {k: stage_ms_all[k] for k in stage_ms_all}, pk)
    e2e = None
    if not args.no_e2e:
        e2e_ms, h2d, d2h = e2e_steps(pf, max(4, args.steps), 2, world)
        e2e_ms = max_over_ranks(e2e_ms, world)
        e2e = {"value": job_rate(fl["total"] * wl.batch, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e2e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    x_cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        x_cpu = {k: (v[:1].cpu() if v is not None else None) for k, v in pf.x.items()}
    launches = pf.launches_per_step * args.steps
    dev_status = pf.abi.nsa_get_device_status()
    if dev_status != 0:
        raise SystemExit(f"device status {dev_status}: a kernel's bounded wait timed out")
    del pf
    torch.cuda.empty_cache()
    decode = None if args.no_decode else run_decode(world, args.steps, args.warmup)
    others = {}
    if not args.no_configs:
        for name in ("tiny", "moba32k", "moba32k_full", "nsa128k_planted"):
            if name != wl.name:
                others[name] = run_config(name, min(args.steps, 5), args.warmup, world, rank)
    extras = {}
    if not args.no_configs:
        extras["backward"] = run_backward(min(args.steps, 3), 1)
        extras["selection_variants"] = run_selection_variants(min(args.steps, 5), 2)
        torch.cuda.empty_cache()
    cpu = cpu_baseline(wl, x_cpu) if x_cpu is not None else None
    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16, sigmoid gates)",
                "config": config_of(wl, world),
                "tokens_per_s": tokens, "algorithmic_flops_per_step": fl_all,
                "stage_ms": {"pool": float(per[:, 0].mean()), "select": stage_ms.get("select", 0.0),
                             "attn": float(per[:, 2].mean()) - stage_ms.get("select", 0.0)},
                "roofline": roof, "roofline_selected": sel_roof, "peaks": src,
                "cpu_baseline": cpu, "e2e": e2e,
                "decode": decode, "configs": others, "extras": extras, "gpu_launches": launches,
                "clocks": clk,
                "wall_s_timed_region": wall}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[args.workload]
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    x = make_inputs(wl, device=gen_dev, seed=0)
    x = {k: (v[:1].cpu() if v is not None else None) for k, v in x.items()}
    times, flops = [], []
    res = None
    for s in range(args.warmup + args.steps):
        res = cpu_baseline(wl, x, rows_per_step=4)
        if s >= args.warmup:
            times.append(res["seconds"])
            flops.append(res["value"] * res["seconds"])
    value = sum(flops) / sum(times)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_of(wl, world),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": res["cores"],
                             "kind": "oracle", "parallelism": res["parallelism"],
                             "sample": res["sample"] + " per step"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="nsa64k", choices=sorted(WORKLOADS))
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other prefill workloads (tiny, moba32k, moba32k_full, "
                         "nsa128k_planted)")
    ap.add_argument("--seqlen", type=int, default=0, help="override the prefill length (profiling)")
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        print("note: fewer than 3 warm-up steps", file=sys.stderr)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
