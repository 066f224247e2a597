"""Backward pass (nsa_sparse_attn_bwd) against the fp64 oracle's gradients.

The loss is sum(d_out * out) for a seeded bf16 d_out; the blocks are the ones
the forward selected (the top-k choice passes no gradient).  Gradients are
compared element by element: max |gpu - oracle| <= 1e-3 * max |oracle| and
mean <= 1e-4 * max |oracle| (fp32 sums of bf16 products against fp64).
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_scoring_b200 import abi
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, BR_CMP, BR_SEL, BR_WIN
from oracle import nsa_oracle as O
from tests.parity import GpuCase, f64, oracle_cfg

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny"]
CASES = {
    "tiny": TINY,
    "gqa_cmp16": TINY.with_(name="gqa_cmp16", seqlen_q=300, seqlen_kv=300, h_q=8, h_kv=2,
                            cmp_block=32, cmp_stride=16, window=64),
    "per_head": TINY.with_(name="per_head", seqlen_q=260, seqlen_kv=260, h_q=4, h_kv=2,
                           per_head_select=True),
    "chunk_ungated": TINY.with_(name="chunk_ungated", seqlen_q=120, seqlen_kv=500, q_pos0=380,
                                gated=False, d_qk=128, d_v=128),
    "sel_only_d192": TINY.with_(name="sel_only_d192", seqlen_q=200, seqlen_kv=200, h_q=16,
                                h_kv=1, d_qk=192, d_v=128, branches=BR_SEL, top_k=3),
}


def _close(got, ref, what):
    scale = max(float(np.abs(ref).max()), 1e-6)
    err = np.abs(got - ref)
    assert np.isfinite(got).all(), what
    assert err.max() <= 1e-3 * scale and err.mean() <= 1e-4 * scale, \
        f"{what}: max {err.max():.3e} mean {err.mean():.3e} scale {scale:.3e}"


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_oracle(name):
    wl = CASES[name]
    run = GpuCase(wl)
    cfg = run.cfg
    g = torch.Generator(device="cuda")
    g.manual_seed(77)
    d_out = torch.randn(run.out.shape, generator=g, device="cuda").to(torch.bfloat16)
    dq = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, wl.d_qk, device="cuda")
    dk = torch.empty(wl.batch, wl.h_kv, wl.seqlen_kv, wl.d_qk, device="cuda")
    dv = torch.empty(wl.batch, wl.h_kv, wl.seqlen_kv, wl.d_v, device="cuda")
    dg = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, 3, device="cuda") if wl.gated else None
    ws = torch.empty(max(abi.nsa_bwd_workspace_size(cfg), 1), dtype=torch.uint8, device="cuda")
    abi.nsa_sparse_attn_bwd(cfg, run.x["q"], run.x["k"], run.x["v"], run.pooled["kcmp"],
                            run.pooled["vcmp"], run.x["gates"], run.idx_fwd, d_out, dq, dk, dv, dg,
                            ws, ws.numel())
    torch.cuda.synchronize()
    assert abi.nsa_get_device_status() == 0
    for b in range(wl.batch):
        rows = np.arange(wl.seqlen_q)
        gates = None if run.x["gates"] is None else f64(run.x["gates"][b])
        idx = run.idx_fwd[b].cpu().numpy() if wl.branches & BR_SEL else None
        rq, rK, rV, rg = O.nsa_rows_backward(oracle_cfg(wl), f64(run.x["q"][b]), rows + wl.q_pos0,
                                             f64(run.x["k"][b]), f64(run.x["v"][b]), gates, idx,
                                             f64(d_out[b]))
        _close(f64(dq[b]), rq, f"{name} dq")
        _close(f64(dk[b]), rK, f"{name} dK")
        _close(f64(dv[b]), rV, f"{name} dV")
        if dg is not None:
            _close(f64(dg[b]), rg, f"{name} dgates")
