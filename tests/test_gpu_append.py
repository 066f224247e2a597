"""Decode with an incremental cache update (nsa_append_kv) against full pooling and
the fp64 oracle.

A decode loop appends each new token's K/V to a cache of fixed capacity and
refreshes only the pooled tokens that the token completes (transcript #94 §6:
decoding costs the KV bytes it reads, so a step must not re-pool the whole
cache).  After any sequence of appends the pooled tensors must equal
nsa_pool_kv of the filled cache bit for bit, and a decode step run on the
capacity-sized cache with the query at the newest position must match the
oracle run on the filled prefix.
"""
import numpy as np
import pytest
import torch

from dynamic_block_sparse_scoring_b200 import abi
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, make_inputs
from oracle import nsa_oracle as O
from tests.parity import check_idx, check_out, f64, oracle_cfg

pytestmark = pytest.mark.gpu

DEC = WORKLOADS["decode64x64k"]


def _filled_inputs(wl, seed):
    """Seeded K/V of the whole capacity; the test feeds them to the cache piece by piece."""
    return make_inputs(wl.with_(seqlen_q=wl.seqlen_kv, q_pos0=0), device="cuda", seed=seed)


def _append(wl, k, v, pooled, src_k, src_v, t0, n):
    """Append rows [t0, t0 + n) of the seeded K/V to the cache."""
    cfg = abi.config(wl, seqlen_q=n, q_pos0=t0)
    abi.nsa_append_kv(cfg, k, v, src_k[:, :, t0:t0 + n].contiguous(),
                      src_v[:, :, t0:t0 + n].contiguous(), pooled["kbar"], pooled["kcmp"],
                      pooled["vcmp"])


@pytest.mark.parametrize("shape", ["decode", "small_blocks"])
def test_appends_equal_full_pooling_bit_for_bit(shape):
    wl = DEC.with_(batch=2, seqlen_kv=2600, q_pos0=2599, h_q=16, h_kv=2)
    if shape == "small_blocks":       # 16-key blocks, compression 16/8, head dim 64
        wl = wl.with_(sel_block=16, cmp_block=16, cmp_stride=8, d_qk=64, d_v=64)
    cfg = abi.config(wl)
    x = _filled_inputs(wl, seed=5)
    C = wl.seqlen_kv
    k = torch.zeros_like(x["k"])
    v = torch.zeros_like(x["v"])
    pooled = abi.alloc_pooled(cfg, "cuda")
    for t in pooled.values():
        t.fill_(float("nan"))
    # a prefill of 1000 tokens, then single-token steps across block and compression
    # boundaries, a ragged multi-token append, and single tokens to the end of a block
    plan = [(0, 1000)] + [(t, 1) for t in range(1000, 1090)] + [(1090, 37)] + \
           [(t, 1) for t in range(1127, 1152)]
    for t0, n in plan:
        _append(wl, k, v, pooled, x["k"], x["v"], t0, n)
    L = 1152
    torch.cuda.synchronize()
    assert torch.equal(k[:, :, :L], x["k"][:, :, :L]) and torch.equal(v[:, :, :L], x["v"][:, :, :L])
    assert not k[:, :, L:].any() and not v[:, :, L:].any()
    full = abi.alloc_pooled(cfg, "cuda")
    abi.nsa_pool_kv(cfg, k, v, full["kbar"], full["kcmp"], full["vcmp"])
    torch.cuda.synchronize()
    nb = L // wl.sel_block
    nc = (L - wl.cmp_block) // wl.cmp_stride + 1
    assert torch.equal(pooled["kbar"][:, :, :nb], full["kbar"][:, :, :nb])
    assert torch.equal(pooled["kcmp"][:, :, :nc], full["kcmp"][:, :, :nc])
    assert torch.equal(pooled["vcmp"][:, :, :nc], full["vcmp"][:, :, :nc])
    # tokens not yet complete were not touched
    assert torch.isnan(pooled["kbar"][:, :, nb:]).all()
    assert torch.isnan(pooled["kcmp"][:, :, nc:].float()).all()
    # and the pooled tokens agree with the oracle's pooling of the filled prefix
    for b in range(wl.batch):
        K, V = f64(x["k"][b, :, :L]), f64(x["v"][b, :, :L])
        np.testing.assert_allclose(f64(pooled["kbar"][b, :, :nb]),
                                   O.pool_block_keys(K, wl.sel_block), rtol=0, atol=1e-5)
        for got, X in [(pooled["kcmp"], K), (pooled["vcmp"], V)]:
            ref = O.compress(X, wl.cmp_block, wl.cmp_stride)
            assert (np.abs(f64(got[b, :, :nc]) - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6).all()


def test_decode_steps_on_the_growing_cache_match_the_oracle():
    """Append + selection + attention per step, with the cache's unfilled rows zero."""
    wl = DEC.with_(batch=2, seqlen_kv=3000, q_pos0=2999)
    cfg = abi.config(wl)
    x = _filled_inputs(wl, seed=6)
    g = torch.Generator(device="cuda")
    g.manual_seed(60)
    k = torch.zeros_like(x["k"])
    v = torch.zeros_like(x["v"])
    # a new cache: its rows and its pooled tokens start at zero (finite), since masked
    # keys still enter the value products with weight 0
    pooled = {name: t.zero_() for name, t in abi.alloc_pooled(cfg, "cuda").items()}
    _append(wl, k, v, pooled, x["k"], x["v"], 0, 2000)
    filled = 2000
    for t in [2000, 2001, 2047, 2048, 2063, 2100]:
        if t > filled:                    # the tokens between two checked steps
            _append(wl, k, v, pooled, x["k"], x["v"], filled, t - filled)
        _append(wl, k, v, pooled, x["k"], x["v"], t, 1)
        filled = t + 1
        step = abi.config(wl, seqlen_q=1, q_pos0=t)
        q = torch.randn(wl.batch, 1, wl.h_q, wl.d_qk, generator=g, device="cuda").to(torch.bfloat16)
        gates = torch.sigmoid(torch.randn(wl.batch, 1, wl.h_q, 3, generator=g, device="cuda"))
        idx = torch.empty(wl.batch, wl.h_kv, 1, wl.top_k, dtype=torch.int32, device="cuda")
        abi.nsa_topk_select(step, q, pooled["kbar"], None, idx)
        out = torch.empty(wl.batch, 1, wl.h_q, wl.d_v, dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(abi.nsa_workspace_size(step), dtype=torch.uint8, device="cuda")
        assert abi.nsa_attn_plan(step, False, ws.numel())[0] == "decode"
        abi.nsa_sparse_attn_fwd(step, q, k, v, pooled["kbar"], pooled["kcmp"], pooled["vcmp"],
                                gates, idx, out, ws, ws.numel())
        torch.cuda.synchronize()
        assert abi.nsa_get_device_status() == 0
        for b in range(wl.batch):
            K, V = f64(x["k"][b, :, :t + 1]), f64(x["v"][b, :, :t + 1])
            pos = np.array([t])
            Kbar = O.pool_block_keys(K, wl.sel_block)
            s = O.block_scores(f64(q[b]), pos, Kbar, wl.h_q, wl.h_kv, wl.sel_block, wl.scale,
                               False, -(-(t + 1) // wl.sel_block))
            ora_idx, gap = O.select_blocks(s, pos, wl.sel_block, wl.top_k)
            gi = idx[b].cpu().numpy()
            check_idx(gi, ora_idx, gap, s, pos, wl.sel_block, wl.top_k)
            ora, _, _ = O.nsa_rows(oracle_cfg(wl), f64(q[b]), pos, K, V, f64(gates[b]), idx=gi)
            check_out(f64(out[b]), ora, f"decode step at {t} seq {b}")
