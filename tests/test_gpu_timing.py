"""Stage timing through the C-ABI: names follow the launch plan, durations are positive."""
import pytest
import torch

from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu


STAGES = {"rowwise": ["rowwise"], "query-major": ["attn_tc"], "split-k": ["attn_tc", "split_merge"],
          "block-major": ["index", "sel_bm", "sel_merge", "attn_tc"],
          # the selected branch alone, one head per unit: 64-key sub-blocks, merged into out
          "block-major-sub": ["expand", "index", "sel_bm", "sel_merge"]}


@pytest.mark.parametrize("name,seqlen,want_path,stage_key", [
    ("tiny", None, "split-k", "split-k"),
    ("nsa64k", 1024, "block-major", "block-major"),
    ("moba32k", 1024, "block-major", "block-major-sub"),
])
def test_stage_timing_follows_the_plan(name, seqlen, want_path, stage_key):
    from dynamic_block_sparse_scoring_b200 import abi as a
    wl = WORKLOADS[name]
    if seqlen:
        wl = wl.with_(seqlen_q=seqlen, seqlen_kv=seqlen)
    cfg = a.config(wl)
    x = make_inputs(wl, "cuda", seed=3)
    pooled = a.alloc_pooled(cfg, "cuda")
    a.nsa_pool_kv(cfg, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
    ws = torch.empty(a.nsa_workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, wl.d_v, dtype=torch.bfloat16, device="cuda")
    path, kernels = a.nsa_attn_plan(cfg, True, ws.numel())
    a.nsa_timing_enable(True)
    try:
        a.nsa_sparse_attn_fwd(cfg, x["q"], x["k"], x["v"], pooled["kbar"], pooled["kcmp"],
                              pooled["vcmp"], x["gates"], None, out, ws, ws.numel())
        stages = a.nsa_timing_read()
    finally:
        a.nsa_timing_enable(False)
    assert path == want_path
    assert [n for n, _ in stages] == ["select"] + STAGES[stage_key], stages
    assert all(ms > 0 for _, ms in stages)
    # after disabling, a call records nothing new; the last timed call stays readable
    a.nsa_sparse_attn_fwd(cfg, x["q"], x["k"], x["v"], pooled["kbar"], pooled["kcmp"],
                          pooled["vcmp"], x["gates"], None, out, ws, ws.numel())
    torch.cuda.synchronize()
    assert a.nsa_get_device_status() == 0
