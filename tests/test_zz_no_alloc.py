"""The allocation-free forward, nsa_sparse_attn_fwd_noalloc, against the regular
entry point.

Some callers may not allocate device memory at all (plugin hosts whose execute
call must not allocate, latency-critical code that cannot afford cudaMalloc's
device synchronisation), so they cannot provide the workspace that
nsa_sparse_attn_fwd needs when it selects blocks itself.  The no-alloc variant
keeps that scratch in a fixed array inside the library.  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

from dynamic_block_sparse_scoring_b200 import abi
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

OUT_MAX_ABS = 2e-2
OUT_MEAN_ABS = 2e-3
NOALLOC_BYTES = 32 << 20     # size of the library's scratch array


def _forward_pair(wl, seed):
    cfg = abi.config(wl)
    x = make_inputs(wl, device="cuda", seed=seed)
    pooled = abi.alloc_pooled(cfg, "cuda")
    abi.nsa_pool_kv(cfg, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
    ref, _ = abi.forward(cfg, x["q"], x["k"], x["v"], x["gates"], pooled=pooled)
    got = torch.full_like(ref, float("nan"))
    status = abi.lib.nsa_sparse_attn_fwd_noalloc(
        ctypes.byref(cfg), x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
        pooled["kbar"].data_ptr(), pooled["kcmp"].data_ptr(), pooled["vcmp"].data_ptr(),
        None if x["gates"] is None else x["gates"].data_ptr(), got.data_ptr(),
        torch.cuda.current_stream().cuda_stream)
    assert status == 0, abi.nsa_status_string(status)
    torch.cuda.synchronize()
    return ref.double().cpu().numpy(), got.double().cpu().numpy()


# The regular entry point uses the same kernels as the no-alloc one on these
# problems (16 heads per group over 192 queries of a 2048-token cache, and the
# tiny single-group problem), so the two results are compared directly.
@pytest.mark.parametrize("name", ["tiny", "nsa_chunk"])
def test_noalloc_matches_regular_entry_point_twice_in_a_row(name):
    wl = WORKLOADS["tiny"] if name == "tiny" else WORKLOADS["nsa64k"].with_(
        name="nsa_chunk", seqlen_q=192, seqlen_kv=2048, q_pos0=2048 - 192, h_q=16, h_kv=1)
    for seed in (0, 1):                  # two calls in a row on the shared scratch array
        ref, got = _forward_pair(wl, seed)
        assert np.isfinite(got).all()
        err = np.abs(got - ref)
        assert err.max() <= OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS


def test_noalloc_takes_the_small_workspace_plan_when_the_full_one_does_not_fit():
    """Selected ids fit the 32 MiB array but the fastest plan's lists and partials
    do not: the no-alloc call runs the plan a workspace of that size gets, which is
    the plan of the minimal workspace, and matches the regular call given exactly
    nsa_workspace_size_min() bytes."""
    wl = WORKLOADS["nsa64k"].with_(name="nsa_tail4k", seqlen_q=4096, seqlen_kv=16384,
                                   q_pos0=16384 - 4096)
    cfg = abi.config(wl)
    wmin, wfull = abi.nsa_workspace_size_min(cfg), abi.nsa_workspace_size(cfg)
    assert wmin <= NOALLOC_BYTES < wfull
    assert abi.nsa_attn_plan(cfg, True, NOALLOC_BYTES) == abi.nsa_attn_plan(cfg, True, wmin)
    x = make_inputs(wl, device="cuda")
    pooled = abi.alloc_pooled(cfg, "cuda")
    abi.nsa_pool_kv(cfg, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
    ws = torch.empty(wmin, dtype=torch.uint8, device="cuda")
    ref = torch.empty(wl.batch, wl.seqlen_q, wl.h_q, wl.d_v, dtype=torch.bfloat16, device="cuda")
    abi.nsa_sparse_attn_fwd(cfg, x["q"], x["k"], x["v"], pooled["kbar"], pooled["kcmp"],
                            pooled["vcmp"], x["gates"], None, ref, ws, wmin)
    for _ in range(2):
        got = torch.full_like(ref, float("nan"))
        status = abi.lib.nsa_sparse_attn_fwd_noalloc(
            ctypes.byref(cfg), x["q"].data_ptr(), x["k"].data_ptr(), x["v"].data_ptr(),
            pooled["kbar"].data_ptr(), pooled["kcmp"].data_ptr(), pooled["vcmp"].data_ptr(),
            x["gates"].data_ptr(), got.data_ptr(), torch.cuda.current_stream().cuda_stream)
        assert status == 0, abi.nsa_status_string(status)
        torch.cuda.synchronize()
        # same plan, same kernels, same inputs: the same bits
        assert torch.equal(got, ref)


def test_noalloc_rejects_problems_beyond_its_scratch():
    # 131072 queries x 64 heads (per-head selection) x top-32 x 4 B = 1 GiB > 32 MiB
    wl = WORKLOADS["nsa128k_planted"].with_(per_head_select=True, top_k=32)
    cfg = abi.config(wl)
    status = abi.lib.nsa_sparse_attn_fwd_noalloc(ctypes.byref(cfg), 1 << 20, 1 << 20, 1 << 20,
                                                 1 << 20, 1 << 20, 1 << 20, 1 << 20, 1 << 20,
                                                 None)
    assert status == 3                   # NSA_ERR_WORKSPACE, before anything is launched
