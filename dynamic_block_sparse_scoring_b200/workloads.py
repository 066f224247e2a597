"""Named workloads and their seeded synthetic inputs.

This module holds shapes and random-number recipes only: no step of the
sparse-attention method is computed here.  Both the CUDA path (through the
tests and ``bench.py``) and the fp64 oracle draw their inputs from it, so the
two sides always see the same tensors.

Workload shapes follow the model settings discussed in the Zhang Xiaojun #94
transcript (bidclub.ai): §4 "Inside Native Sparse Attention" (GQA groups),
§5 "Hardware Makes Sparsity Work" (64 query heads, d_q = 192, 4 groups) and
§7 "Kimi Simplifies The Sparse Route" (MoBA: block 512 / top-3, NSA: block
64 / top-16).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, asdict, replace
from typing import Optional

import torch

BR_CMP = 1
BR_SEL = 2
BR_WIN = 4
PER_HEAD_SELECT = 8
SCORE_PROB = 16
SCORE_CMP = 32
SINK_SHIFT = 16


@dataclass(frozen=True)
class Workload:
    """Problem shape of one sparse-attention forward call.

    Query ``i`` of a sequence sits at KV position ``q_pos0 + i``; prefill uses
    ``q_pos0 = 0`` and ``seqlen_q = seqlen_kv``, decode uses one query at
    ``q_pos0 = seqlen_kv - 1``.
    """
    name: str
    batch: int
    seqlen_q: int
    seqlen_kv: int
    q_pos0: int
    h_q: int
    h_kv: int
    d_qk: int
    d_v: int
    sel_block: int
    top_k: int
    window: int
    cmp_block: int
    cmp_stride: int
    branches: int               # bit set of BR_CMP | BR_SEL | BR_WIN
    per_head_select: bool       # MoBA: every query head picks its own blocks
    gated: bool                 # False: enabled branches are summed with weight 1
    planted: bool = False       # keys from a block-run Gaussian mixture
    seed: int = 0
    score_mode: str = "dot"     # block scores: "dot" (summed scaled dot products), "prob"
                                # (summed per-head probabilities), "cmp" (from the compressed branch)
    sink_blocks: int = 0        # leading blocks always kept

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_qk)

    @property
    def group(self) -> int:
        return self.h_q // self.h_kv

    @property
    def h_sel(self) -> int:
        return self.h_q if self.per_head_select else self.h_kv

    @property
    def flags(self) -> int:
        mode = {"dot": 0, "prob": SCORE_PROB, "cmp": SCORE_CMP}[self.score_mode]
        return (self.branches | (PER_HEAD_SELECT if self.per_head_select else 0) | mode |
                (self.sink_blocks << SINK_SHIFT))

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


def _prefill(name, T, **kw):
    return Workload(name=name, batch=kw.pop("batch", 1), seqlen_q=T, seqlen_kv=T, q_pos0=0, **kw)


# The five workloads.  Sizes are the ones the method is discussed at: a tiny
# single-group case, MoBA-style per-head selection, NSA prefill at 64k, NSA
# decode against 64 caches of 64k tokens, and a 128k prefill whose keys carry
# planted block structure so that the top-k is far from uniform; plus the
# full-attention layers of MoBA's hybrid at the MoBA shapes.
WORKLOADS = {
    "tiny": _prefill("tiny", 1024, h_q=4, h_kv=1, d_qk=64, d_v=64, sel_block=64, top_k=4,
                     window=128, cmp_block=32, cmp_stride=32,
                     branches=BR_CMP | BR_SEL | BR_WIN, per_head_select=False, gated=True),
    "moba32k": _prefill("moba32k", 32768, h_q=16, h_kv=16, d_qk=128, d_v=128, sel_block=512,
                        top_k=3, window=0, cmp_block=0, cmp_stride=0, branches=BR_SEL,
                        per_head_select=True, gated=False),
    "nsa64k": _prefill("nsa64k", 65536, h_q=64, h_kv=4, d_qk=192, d_v=128, sel_block=64,
                       top_k=16, window=512, cmp_block=32, cmp_stride=16,
                       branches=BR_CMP | BR_SEL | BR_WIN, per_head_select=False, gated=True),
    "decode64x64k": Workload(name="decode64x64k", batch=64, seqlen_q=1, seqlen_kv=65536,
                             q_pos0=65535, h_q=64, h_kv=4, d_qk=192, d_v=128, sel_block=64,
                             top_k=16, window=512, cmp_block=32, cmp_stride=16,
                             branches=BR_CMP | BR_SEL | BR_WIN, per_head_select=False,
                             gated=True),
    # MoBA's hybrid: the layers that switch back to full attention (same shapes as
    # moba32k), i.e. dense causal attention, run as a window covering the whole cache
    "moba32k_full": _prefill("moba32k_full", 32768, h_q=16, h_kv=16, d_qk=128, d_v=128,
                             sel_block=512, top_k=3, window=32768, cmp_block=0, cmp_stride=0,
                             branches=BR_WIN, per_head_select=False, gated=False),
    "nsa128k_planted": _prefill("nsa128k_planted", 131072, h_q=64, h_kv=4, d_qk=192, d_v=128,
                                sel_block=64, top_k=16, window=512, cmp_block=32, cmp_stride=16,
                                branches=BR_CMP | BR_SEL | BR_WIN, per_head_select=False,
                                gated=True, planted=True),
}


def _generator(device: torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_inputs(wl: Workload, device="cpu", seed: Optional[int] = None):
    """Seeded inputs for ``wl`` on ``device``.

    Layouts: q [B, Tq, Hq, d_qk] bf16; k [B, Hkv, Tkv, d_qk] bf16;
    v [B, Hkv, Tkv, d_v] bf16; gates [B, Tq, Hq, 3] fp32 in the order
    (compressed, selected, window), or None for an ungated workload.

    Recipe: one generator seeded with ``seed``; fp32 standard normals drawn in
    the order q, k, v, gate logits; q/k/v rounded to bf16 (round to nearest
    even); gates = sigmoid(logits) in fp32.  Planted workloads draw keys from
    a 64-component Gaussian mixture laid over contiguous runs of 1..16 blocks
    and build every (token, group) query from 1..4 of those component means
    plus N(0, 0.5^2) noise.
    """
    device = torch.device(device)
    seed = wl.seed if seed is None else seed
    g = _generator(device, seed)
    B, Tq, Tk = wl.batch, wl.seqlen_q, wl.seqlen_kv
    if wl.planted:
        q, k = _planted_qk(wl, g, device)
    else:
        q = torch.randn(B, Tq, wl.h_q, wl.d_qk, generator=g, device=device).to(torch.bfloat16)
        k = torch.randn(B, wl.h_kv, Tk, wl.d_qk, generator=g, device=device).to(torch.bfloat16)
    v = torch.randn(B, wl.h_kv, Tk, wl.d_v, generator=g, device=device).to(torch.bfloat16)
    gates = None
    if wl.gated:
        gates = torch.sigmoid(torch.randn(B, Tq, wl.h_q, 3, generator=g, device=device))
    return {"q": q, "k": k, "v": v, "gates": gates}


def _planted_qk(wl: Workload, g: torch.Generator, device):
    """Keys from a block-run Gaussian mixture and queries mixing 1..4 of its means."""
    B, Tq, Tk, Hkv, d = wl.batch, wl.seqlen_q, wl.seqlen_kv, wl.h_kv, wl.d_qk
    n_comp = 64
    nb = -(-Tk // wl.sel_block)
    mu = torch.randn(B, Hkv, n_comp, d, generator=g, device=device)
    # contiguous runs of U{1..16} blocks, each run one uniformly drawn component
    run_len = torch.randint(1, 17, (B, Hkv, nb), generator=g, device=device)
    run_comp = torch.randint(0, n_comp, (B, Hkv, nb), generator=g, device=device)
    block_comp = torch.empty(B, Hkv, nb, dtype=torch.long, device=device)
    rl, rc = run_len.cpu(), run_comp.cpu()
    bc = torch.empty(B, Hkv, nb, dtype=torch.long)
    for b in range(B):
        for h in range(Hkv):
            pos, r = 0, 0
            while pos < nb:
                n = int(rl[b, h, r])
                bc[b, h, pos:pos + n] = int(rc[b, h, r])
                pos += n
                r += 1
    block_comp.copy_(bc)
    tok_comp = block_comp.repeat_interleave(wl.sel_block, dim=2)[:, :, :Tk]      # [B,Hkv,Tk]
    k = torch.gather(mu, 2, tok_comp.unsqueeze(-1).expand(B, Hkv, Tk, d))
    k = (k + torch.randn(B, Hkv, Tk, d, generator=g, device=device)).to(torch.bfloat16)
    # per (token, group): m ~ U{1..4} distinct components, mean of their centres
    m = torch.randint(1, 5, (B, Tq, Hkv), generator=g, device=device)
    pick = torch.rand(B, Tq, Hkv, n_comp, generator=g, device=device).argsort(dim=-1)[..., :4]
    use = (torch.arange(4, device=device).view(1, 1, 1, 4) < m.unsqueeze(-1)).float()
    centre = torch.zeros(B, Tq, Hkv, d, device=device)
    for j in range(4):
        cj = torch.gather(mu, 2, pick[..., j].permute(0, 2, 1).unsqueeze(-1).expand(B, Hkv, Tq, d))
        centre += cj.permute(0, 2, 1, 3) * use[..., j:j + 1]
    centre /= m.unsqueeze(-1).float()
    G = wl.group
    q = centre.repeat_interleave(G, dim=2)                                         # [B,Tq,Hq,d]
    q = (q + 0.5 * torch.randn(B, Tq, wl.h_q, d, generator=g, device=device)).to(torch.bfloat16)
    return q, k


def row_sample(T: int, stride: int = 16, head: int = 1024, extra=()):
    """Evenly strided query rows plus the first ``head`` rows and the last row."""
    rows = set(range(min(head, T)))
    rows.update(range(0, T, stride))
    rows.add(T - 1)
    rows.update(r for r in extra if 0 <= r < T)
    return sorted(rows)


__all__ = ["Workload", "WORKLOADS", "make_inputs", "row_sample", "BR_CMP", "BR_SEL", "BR_WIN",
           "PER_HEAD_SELECT", "asdict"]
