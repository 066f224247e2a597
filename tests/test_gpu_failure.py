"""Failure detection on the GPU without a GPU fault.

* The bounded wait that every tensor-core kernel uses gives up on a barrier
  that nothing completes, records NSA_ERR_TIMEOUT in the device status word,
  and leaves the context usable (a forward right after is still correct).
* The tensor-core attention kernel itself, with its wait limit cut to 1 ns so
  that its waits on copies and MMAs give up, unwinds every role (the warps
  that share rows leave their barriers together), reports NSA_ERR_TIMEOUT,
  and the same calls with the default limit are correct afterwards.
* NSA_DEBUG_CHECKS: a caller-supplied idx that breaks the id rules is refused
  with NSA_ERR_INVALID_ARG before any attention kernel runs; out is untouched.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_scoring_b200 import abi
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, make_inputs
from tests.parity import GpuCase, check_out, f64

pytestmark = pytest.mark.gpu

TINY = WORKLOADS["tiny"]


def test_bounded_wait_times_out_and_the_context_stays_usable():
    assert abi.nsa_get_device_status() == 0
    abi.nsa_check_bounded_wait(2_000_000)            # 2 ms on a barrier nothing completes
    torch.cuda.synchronize()
    assert abi.nsa_get_device_status() == 5          # NSA_ERR_TIMEOUT ...
    assert abi.nsa_get_device_status() == 0          # ... read once, then cleared
    run = GpuCase(TINY)                               # a full forward afterwards
    rows = np.arange(TINY.seqlen_q)
    ora, _, _ = run.oracle_rows(0, rows, idx=run.idx_fwd[0].cpu().numpy())
    check_out(f64(run.out[0]), ora, "forward after a timed-out wait")


def _forward(cfg, run, idx, out):
    return abi.lib.nsa_sparse_attn_fwd(
        abi.ctypes.byref(cfg), run.x["q"].data_ptr(), run.x["k"].data_ptr(), run.x["v"].data_ptr(),
        run.pooled["kbar"].data_ptr(), run.pooled["kcmp"].data_ptr(), run.pooled["vcmp"].data_ptr(),
        run.x["gates"].data_ptr(), idx.data_ptr(), out.data_ptr(), None, 0,
        torch.cuda.current_stream().cuda_stream)


def test_debug_checks_refuse_bad_ids_before_any_attention_kernel():
    run = GpuCase(TINY)
    checked = abi.config(TINY, flags=TINY.flags | abi.NSA_DEBUG_CHECKS)
    good = run.idx.clone()
    # valid ids pass and give the same bits as the unchecked call
    ref = torch.empty_like(run.out)
    got = torch.empty_like(run.out)
    assert _forward(run.cfg, run, good, ref) == 0
    assert _forward(checked, run, good, got) == 0
    torch.cuda.synchronize()
    assert torch.equal(ref, got)
    nb_all = -(-TINY.seqlen_kv // TINY.sel_block)
    row = 900                                       # position 900: own block 14, four kept blocks
    bad_rows = {
        "beyond the cache": lambda r: r.__setitem__(0, nb_all + 5),
        "a future block": lambda r: r.__setitem__(1, 15),
        "not ascending": lambda r: r.__setitem__(slice(0, 2), r[0:2].flip(0).clone()),
        "own block missing": lambda r: r.__setitem__(3, -1),
        "an id after the padding": lambda r: (r.__setitem__(2, -1), r.__setitem__(3, 14)),
        "a negative id": lambda r: r.__setitem__(0, -7),
    }
    for name, spoil in bad_rows.items():
        idx = good.clone()
        spoil(idx[0, 0, row])
        out = torch.full_like(run.out, 7.0)
        assert _forward(checked, run, idx, out) == 1, name          # NSA_ERR_INVALID_ARG
        torch.cuda.synchronize()
        assert bool((out == 7.0).all()), f"{name}: out was written"
    assert abi.nsa_get_device_status() == 0


def test_attention_kernel_waits_run_out_and_the_next_calls_are_correct():
    run = GpuCase(TINY)
    assert abi.nsa_get_device_status() == 0
    out = torch.empty_like(run.out)
    ws = torch.empty(abi.nsa_workspace_size(run.cfg), dtype=torch.uint8, device="cuda")
    abi.nsa_set_wait_limit_ns(1)
    try:
        # the query-major plan (ids given, no workspace) and the split-K plan (workspace)
        st = _forward(run.cfg, run, run.idx, out)
        torch.cuda.synchronize()
        status_qm = abi.nsa_get_device_status()
        abi.forward(run.cfg, run.x["q"], run.x["k"], run.x["v"], run.x["gates"], idx=run.idx,
                    pooled=run.pooled, workspace=ws, out=out)
        torch.cuda.synchronize()
        status_split = abi.nsa_get_device_status()
    finally:
        abi.nsa_set_wait_limit_ns(0)
    assert st == 0
    assert status_qm == 5 and status_split == 5        # NSA_ERR_TIMEOUT from both launches
    rows = np.arange(TINY.seqlen_q)
    ora, _, _ = run.oracle_rows(0, rows, idx=run.idx[0].cpu().numpy())
    assert _forward(run.cfg, run, run.idx, out) == 0
    torch.cuda.synchronize()
    assert abi.nsa_get_device_status() == 0
    check_out(f64(out[0]), ora, "query-major forward after timed-out launches")
    out2, _ = abi.forward(run.cfg, run.x["q"], run.x["k"], run.x["v"], run.x["gates"], idx=run.idx,
                          pooled=run.pooled, workspace=ws)
    torch.cuda.synchronize()
    assert abi.nsa_get_device_status() == 0
    check_out(f64(out2[0]), ora, "split-K forward after timed-out launches")
