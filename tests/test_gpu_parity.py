"""GPU parity: the C-ABI CUDA path against the fp64 oracle, element by element.

Small problems are compared on every row.  The full-size prefills have their
selected block ids compared on every row, and their outputs on sampled rows
(first rows, evenly strided rows, block boundaries, the last row); the decode
batch is compared on every sequence.  Tolerances are stated in tests/parity.py.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS, BR_CMP, BR_SEL, BR_WIN, row_sample
from oracle import nsa_oracle as O

pytestmark = pytest.mark.gpu

from dynamic_block_sparse_scoring_b200 import abi
from tests.parity import (GpuCase, check_idx, check_out, check_selection_all_rows, f64,
                          oracle_cfg, oracle_selection, OUT_MAX_ABS, OUT_MEAN_ABS, SCORE_ATOL,
                          SCORE_RTOL)

TINY = WORKLOADS["tiny"]

# Edge cases around the tiny workload: ragged lengths, degenerate branch sizes,
# every block kept, per-head selection under GQA, chunked prefill, batch > 1,
# other head dimensions, and scaled-down versions of the big workloads.
EDGE = {
    "tiny": TINY,
    "ragged_1000": TINY.with_(name="ragged_1000", seqlen_q=1000, seqlen_kv=1000),
    "ragged_77": TINY.with_(name="ragged_77", seqlen_q=77, seqlen_kv=77, sel_block=16, top_k=3,
                            window=20, cmp_block=16, cmp_stride=8),
    "every_block": TINY.with_(name="every_block", seqlen_q=512, seqlen_kv=512, top_k=32,
                              branches=BR_SEL, gated=False),
    "gqa_per_head": TINY.with_(name="gqa_per_head", seqlen_q=700, seqlen_kv=700, h_q=8, h_kv=2,
                               d_qk=128, d_v=128, per_head_select=True),
    "window_1": TINY.with_(name="window_1", seqlen_q=300, seqlen_kv=300, window=1),
    "shorter_than_cmp_block": TINY.with_(name="short", seqlen_q=20, seqlen_kv=20),
    "single_query": TINY.with_(name="single_query", seqlen_q=1, seqlen_kv=1),
    "top1": TINY.with_(name="top1", seqlen_q=400, seqlen_kv=400, top_k=1),
    "chunked_prefill": TINY.with_(name="chunked", seqlen_q=300, seqlen_kv=1000, q_pos0=700),
    "batch3": TINY.with_(name="batch3", batch=3, seqlen_q=256, seqlen_kv=256),
    "d256": TINY.with_(name="d256", seqlen_q=333, seqlen_kv=333, h_q=4, h_kv=2, d_qk=256,
                       d_v=256),
    "moba_small": WORKLOADS["moba32k"].with_(name="moba_small", seqlen_q=4096, seqlen_kv=4096,
                                             h_q=4, h_kv=4),
    "nsa_small": WORKLOADS["nsa64k"].with_(name="nsa_small", seqlen_q=2048, seqlen_kv=2048,
                                           h_q=16, h_kv=1),
    "cmp_identity": TINY.with_(name="cmp_identity", seqlen_q=200, seqlen_kv=200, cmp_block=1,
                               cmp_stride=1),
    # a few queries at the end of a cache (the few-row selection kernel; split-K)
    "few_queries": TINY.with_(name="few_queries", seqlen_q=5, seqlen_kv=900, q_pos0=895),
    "few_d256": TINY.with_(name="few_d256", seqlen_q=4, seqlen_kv=2000, q_pos0=1996, h_q=4, h_kv=2,
                           d_qk=256, d_v=256),
    "decode_small": WORKLOADS["decode64x64k"].with_(name="decode_small", batch=3, seqlen_kv=3000,
                                                     q_pos0=2999),
    # few-query kernel (keys as the MMA M dimension): groups of 8 and 16 heads, up to 4 queries,
    # caches shorter than the window / a compressed block, ragged blocks, 128-key blocks,
    # selected-only ungated
    "dec_g8_tq3": WORKLOADS["decode64x64k"].with_(name="dec_g8_tq3", batch=2, seqlen_q=3,
                                                   seqlen_kv=2500, q_pos0=2497, h_q=16, h_kv=2,
                                                   d_qk=128),
    "dec_short": WORKLOADS["decode64x64k"].with_(name="dec_short", batch=2, seqlen_kv=100,
                                                  q_pos0=99),
    "dec_tiny_cache": WORKLOADS["decode64x64k"].with_(name="dec_tiny_cache", batch=2, seqlen_kv=20,
                                                       q_pos0=19),
    "dec_ragged": WORKLOADS["decode64x64k"].with_(name="dec_ragged", batch=2, seqlen_kv=1000,
                                                   q_pos0=999, d_qk=64),
    "dec_bs128": WORKLOADS["decode64x64k"].with_(name="dec_bs128", batch=2, seqlen_kv=3000,
                                                  q_pos0=2999, sel_block=128, top_k=8),
    "dec_sel_only": WORKLOADS["decode64x64k"].with_(name="dec_sel_only", batch=2, seqlen_kv=1500,
                                                     q_pos0=1499, branches=BR_SEL, gated=False),
    # more work items per (sequence, group) than the in-kernel merge stages: separate merge
    "dec_long_cache": WORKLOADS["decode64x64k"].with_(name="dec_long_cache", batch=1,
                                                       seqlen_kv=110000, q_pos0=109999, h_q=32,
                                                       h_kv=2),
    # selected branch alone with one head per unit: block-major over 64-key sub-blocks
    # (128-key blocks under GQA with a ragged cache; 256-key blocks filling all 32 slots)
    "sub_gqa_bs128": TINY.with_(name="sub_gqa_bs128", seqlen_q=700, seqlen_kv=1000, q_pos0=300,
                                h_q=4, h_kv=2, d_qk=128, d_v=128, sel_block=128, top_k=4,
                                branches=BR_SEL, per_head_select=True),
    "sub_slots32": TINY.with_(name="sub_slots32", seqlen_q=300, seqlen_kv=2500, q_pos0=2200,
                              h_q=2, h_kv=2, sel_block=256, top_k=8, branches=BR_SEL, gated=False),
    # block-major selected branch (groups of 8 and 16 heads, sel_block 64, >= 256 queries)
    "bm_g8_ragged": WORKLOADS["nsa64k"].with_(name="bm_g8_ragged", seqlen_q=1000, seqlen_kv=1000,
                                              h_q=16, h_kv=2, d_qk=128, d_v=128),
    "bm_chunked": WORKLOADS["nsa64k"].with_(name="bm_chunked", seqlen_q=300, seqlen_kv=2000,
                                            q_pos0=1700, h_q=16, h_kv=1),
    "bm_batch2": WORKLOADS["nsa64k"].with_(name="bm_batch2", batch=2, seqlen_q=700, seqlen_kv=700,
                                           h_q=32, h_kv=2, d_qk=64, d_v=64),
    # selection-score variants and forced leading blocks, on every selection kernel:
    # the variant kernel (prefill, decode, block-major), the FFMA / tensor-core / few-row
    # fused selections with sinks, per-head selection with sinks
    "prob_tiny": TINY.with_(name="prob_tiny", score_mode="prob"),
    "cmp_tiny": TINY.with_(name="cmp_tiny", score_mode="cmp", cmp_block=32, cmp_stride=16),
    "sinks_tiny": TINY.with_(name="sinks_tiny", sink_blocks=2),
    "prob_sinks_nsa_small": WORKLOADS["nsa64k"].with_(name="prob_sinks_nsa_small", seqlen_q=2048,
                                                      seqlen_kv=2048, h_q=16, h_kv=1,
                                                      score_mode="prob", sink_blocks=1),
    "cmp_nsa_small": WORKLOADS["nsa64k"].with_(name="cmp_nsa_small", seqlen_q=2048, seqlen_kv=2048,
                                               h_q=16, h_kv=1, score_mode="cmp"),
    "sinks_nsa_small": WORKLOADS["nsa64k"].with_(name="sinks_nsa_small", seqlen_q=2048,
                                                 seqlen_kv=2048, h_q=16, h_kv=1, sink_blocks=3),
    "dec_sinks": WORKLOADS["decode64x64k"].with_(name="dec_sinks", batch=2, seqlen_kv=3000,
                                                 q_pos0=2999, sink_blocks=2),
    "dec_prob": WORKLOADS["decode64x64k"].with_(name="dec_prob", batch=2, seqlen_kv=3000,
                                                q_pos0=2999, score_mode="prob"),
    "dec_cmp": WORKLOADS["decode64x64k"].with_(name="dec_cmp", batch=2, seqlen_kv=3000,
                                               q_pos0=2999, score_mode="cmp"),
    "moba_small_sinks": WORKLOADS["moba32k"].with_(name="moba_small_sinks", seqlen_q=4096,
                                                   seqlen_kv=4096, h_q=4, h_kv=4, sink_blocks=1),
    # per-head selection on the sub-block path with up to 64 sub-blocks per query
    # (1024-key blocks; 512-key blocks x top-8; 256-key blocks x top-16)
    "sub_bs1024": WORKLOADS["moba32k"].with_(name="sub_bs1024", seqlen_q=3000, seqlen_kv=3000,
                                             h_q=2, h_kv=2, sel_block=1024, top_k=3),
    "sub_bs512_top8": WORKLOADS["moba32k"].with_(name="sub_bs512_top8", seqlen_q=2000,
                                                 seqlen_kv=5000, q_pos0=3000, h_q=2, h_kv=2,
                                                 top_k=8),
    "sub_bs256_top16": WORKLOADS["moba32k"].with_(name="sub_bs256_top16", seqlen_q=4200,
                                                  seqlen_kv=4200, h_q=2, h_kv=1, sel_block=256,
                                                  top_k=16),
    # full causal attention (MoBA's hybrid layers) on the tensor cores with one head per
    # unit, and window + compressed branches with two heads per unit
    "full_attn_mha": WORKLOADS["moba32k_full"].with_(name="full_attn_mha", seqlen_q=2000,
                                                     seqlen_kv=2000, window=2000, h_q=4, h_kv=4),
    "win_cmp_g2": TINY.with_(name="win_cmp_g2", seqlen_q=900, seqlen_kv=900, h_q=4, h_kv=2,
                             branches=BR_CMP | BR_WIN),
}


def compare_run(run: GpuCase, rows_per_seq, seqs=None):
    wl = run.wl
    seqs = range(wl.batch) if seqs is None else seqs
    for b in seqs:
        rows = np.asarray(rows_per_seq)
        pos = rows + wl.q_pos0
        # selection against the oracle's own selection
        if wl.branches & BR_SEL:
            K = f64(run.x["k"][b])
            rows_t = torch.as_tensor(rows, device="cuda")
            q = f64(run.x["q"][b].index_select(0, rows_t))
            s, ora_idx, gap = oracle_selection(wl, q, pos, K)
            # the stand-alone selection and the one inside the forward call
            gpu_idx = run.idx[b].index_select(1, rows_t).cpu().numpy()
            check_idx(gpu_idx, ora_idx, gap, s, pos, wl.sel_block, wl.top_k, wl.sink_blocks)
            fwd_idx = run.idx_fwd[b].index_select(1, rows_t).cpu().numpy()
            check_idx(fwd_idx, ora_idx, gap, s, pos, wl.sel_block, wl.top_k, wl.sink_blocks)
            idx_for_out = fwd_idx
        else:
            idx_for_out = None
        # outputs, with the oracle attending over the blocks the GPU kept
        ora_out, _, _ = run.oracle_rows(b, rows, idx=idx_for_out)
        gpu_out = f64(run.out[b].index_select(0, torch.as_tensor(rows, device="cuda")))
        check_out(gpu_out, ora_out, f"{wl.name} seq {b}")


@pytest.mark.parametrize("name", sorted(EDGE))
def test_small_problem_all_rows(name):
    wl = EDGE[name]
    run = GpuCase(wl)
    compare_run(run, np.arange(wl.seqlen_q))


def test_pool_kv_matches_oracle():
    for wl in [TINY, EDGE["ragged_77"], WORKLOADS["nsa64k"], WORKLOADS["moba32k"]]:
        run = GpuCase(wl) if wl.seqlen_q <= 4096 else None
        if run is None:
            cfg = abi.config(wl)
            from dynamic_block_sparse_scoring_b200.workloads import make_inputs
            x = make_inputs(wl, device="cuda")
            pooled = abi.alloc_pooled(cfg, "cuda")
            abi.nsa_pool_kv(cfg, x["k"], x["v"], pooled["kbar"], pooled["kcmp"], pooled["vcmp"])
            torch.cuda.synchronize()
        else:
            x, pooled = run.x, run.pooled
        K, V = f64(x["k"][0]), f64(x["v"][0])
        if wl.branches & BR_SEL:
            np.testing.assert_allclose(f64(pooled["kbar"][0]), O.pool_block_keys(K, wl.sel_block),
                                       rtol=0, atol=1e-5)
        if wl.branches & BR_CMP:
            for got, X, d in [(pooled["kcmp"], K, wl.d_qk), (pooled["vcmp"], V, wl.d_v)]:
                ref = O.compress(X, wl.cmp_block, wl.cmp_stride)
                err = np.abs(f64(got[0]) - ref)
                assert (err <= np.abs(ref) * 2.0 ** -8 + 1e-6).all()


@pytest.mark.parametrize("name", ["tiny", "ragged_77", "gqa_per_head", "chunked_prefill",
                                  "nsa_small", "prob_tiny", "cmp_tiny", "sinks_tiny",
                                  "prob_sinks_nsa_small"])
def test_materialised_scores_and_select_from_scores(name):
    wl = EDGE[name]
    run = GpuCase(wl)
    cfg = run.cfg
    nb_all = -(-wl.seqlen_kv // wl.sel_block)
    scores = torch.empty(wl.batch, wl.h_sel, wl.seqlen_q, nb_all, device="cuda")
    abi.nsa_score_blocks_ex(cfg, run.x["q"], run.pooled["kbar"], run.pooled["kcmp"], scores)
    idx2 = torch.empty_like(run.idx)
    abi.nsa_topk_select(cfg, None, None, scores, idx2)
    torch.cuda.synchronize()
    # selecting from the materialised scores gives the fused selection exactly
    assert torch.equal(idx2, run.idx)
    pos = np.arange(wl.seqlen_q) + wl.q_pos0
    for b in range(wl.batch):
        q = f64(run.x["q"][b])
        s, _, _ = oracle_selection(wl, q, pos, f64(run.x["k"][b]))
        got = scores[b].cpu().double().numpy()
        cur = pos // wl.sel_block
        for r in range(wl.seqlen_q):
            c = cur[r]
            ns = min(wl.sink_blocks, c)
            assert np.all(got[:, r, :ns] == np.inf)          # forced leading blocks
            np.testing.assert_allclose(got[:, r, ns:c], s[:, r, ns:c], rtol=SCORE_RTOL,
                                       atol=SCORE_ATOL)
            assert np.all(got[:, r, c] == np.inf)
            assert np.all(got[:, r, c + 1:] == -np.inf)


def test_full_attention_layer_is_dense_causal_attention():
    """MoBA's full-attention layers (a window covering the cache) against library SDPA (fp32)."""
    wl = EDGE["full_attn_mha"]
    run = GpuCase(wl)
    assert abi.nsa_attn_plan(run.cfg, False, abi.nsa_workspace_size(run.cfg))[0] in ("query-major", "split-k")
    q = run.x["q"][0].float().permute(1, 0, 2)
    ref = F.scaled_dot_product_attention(q, run.x["k"][0].float(), run.x["v"][0].float(),
                                         is_causal=True, scale=wl.scale).permute(1, 0, 2)
    check_out(run.out[0].double().cpu().numpy(), ref.double().cpu().numpy(), "full attention")


def test_every_block_kept_is_dense_causal_attention():
    """Library SDPA (fp32) as an independent check of the special case."""
    wl = EDGE["every_block"].with_(h_q=8, h_kv=2)
    run = GpuCase(wl)
    q = run.x["q"][0].float().permute(1, 0, 2)
    k = run.x["k"][0].float().repeat_interleave(4, dim=0)
    v = run.x["v"][0].float().repeat_interleave(4, dim=0)
    ref = F.scaled_dot_product_attention(q, k, v, is_causal=True, scale=wl.scale).permute(1, 0, 2)
    check_out(run.out[0].double().cpu().numpy(), ref.double().cpu().numpy(), "dense causal")


SAMPLED = {name: WORKLOADS[name] for name in ["moba32k", "nsa64k", "nsa128k_planted", "moba32k_full"]}
# block-major work items cross the 8192-query chunk boundary (ragged second chunk)
SAMPLED["bm_two_chunks"] = WORKLOADS["nsa64k"].with_(name="bm_two_chunks", seqlen_q=9000,
                                                     seqlen_kv=9000, h_q=16, h_kv=1)


@pytest.mark.parametrize("name", sorted(SAMPLED))
def test_full_size_prefill_sampled_rows(name):
    """Selected ids on every row against the oracle; outputs on sampled rows."""
    wl = SAMPLED[name]
    run = GpuCase(wl)
    if wl.branches & BR_SEL:
        check_selection_all_rows(run)
    T = wl.seqlen_q
    extra = [wl.sel_block - 1, wl.sel_block, wl.sel_block + 1, 511, 512, 513, T // 2, T - 2]
    extra += [r for r in (8190, 8191, 8192, 8193) if r < T]
    rows = row_sample(T, stride=max(1, T // 384), head=128, extra=extra)
    compare_run(run, rows)
    if not wl.branches & BR_SEL:
        return
    # every row of both selections: structural invariants
    for idx in (run.idx[0], run.idx_fwd[0]):
        t = torch.arange(T, device="cuda") + wl.q_pos0
        c = (t // wl.sel_block).view(1, T, 1)
        valid = idx >= 0
        n = valid.sum(-1)
        assert torch.equal(n, torch.clamp(c.view(1, T) + 1, max=wl.top_k).expand_as(n))
        assert bool(((idx == c) & valid).any(-1).all())               # current block kept
        assert bool((idx < c + 1).all())                               # causal blocks only
        srt = torch.where(valid, idx, torch.full_like(idx, 1 << 30))
        ascending = (srt[..., 1:] > srt[..., :-1]) | ~valid[..., 1:]
        assert bool(ascending.all())                                   # ascending, no repeats


def test_decode_every_sequence():
    wl = WORKLOADS["decode64x64k"]
    run = GpuCase(wl)
    compare_run(run, [0], seqs=range(wl.batch))


@pytest.mark.parametrize("name", ["nsa_small", "bm_g8_ragged"])
def test_minimal_workspace_path_matches_oracle(name):
    """With only nsa_workspace_size_min() bytes the selected branch runs query-major."""
    wl = EDGE[name]
    run = GpuCase(wl)
    cfg = run.cfg
    wmin = abi.nsa_workspace_size_min(cfg)
    assert wmin < abi.nsa_workspace_size(cfg)
    ws = torch.empty(wmin, dtype=torch.uint8, device="cuda")
    out = torch.empty_like(run.out)
    abi.nsa_sparse_attn_fwd(cfg, run.x["q"], run.x["k"], run.x["v"], run.pooled["kbar"],
                            run.pooled["kcmp"], run.pooled["vcmp"], run.x["gates"], None, out, ws,
                            wmin)
    torch.cuda.synchronize()
    assert abi.nsa_get_device_status() == 0
    rows = np.arange(wl.seqlen_q)
    ora, _, _ = run.oracle_rows(0, rows, idx=run.idx[0].cpu().numpy())
    check_out(f64(out[0]), ora, f"{name} minimal workspace")
    # the two selected-branch organisations agree with each other as well; each is
    # within the output tolerance of the oracle, so they are within twice it of
    # each other (a bf16 output of magnitude 2-4 can round one ulp = 0.0156 apart).
    # Rows whose two selections differ (a near-tie resolved differently by the
    # stand-alone and the in-call selection) are compared with the oracle only.
    same = (run.idx[0] == run.idx_fwd[0]).all(dim=0).all(dim=-1).cpu().numpy()
    err = np.abs(f64(out[0]) - f64(run.out[0]))[same]
    assert err.max() <= 2 * OUT_MAX_ABS and err.mean() <= OUT_MEAN_ABS


@pytest.mark.parametrize("name", ["nsa_small", "bm_g8_ragged"])
def test_block_major_rounding_budget(name):
    """The block-major plan rounds each kept block's partial result and the merged
    selected branch to bf16 before the final rounding (include/nsa.h).  Bound the extra
    error per (row, head): against the fp64 oracle within half a bf16 ulp of the output
    plus 2 * 2^-9 * g_sel * max|o_sel| plus 1e-3 (mean <= 1e-3, half the general
    tolerance), and against the query-major plan (one rounding) within the extra term
    plus one bf16 ulp (2^-7 relative) of the output."""
    wl = EDGE[name]
    run = GpuCase(wl)
    assert abi.nsa_attn_plan(run.cfg, True, abi.nsa_workspace_size(run.cfg))[0] == "block-major"
    rows = np.arange(wl.seqlen_q)
    ora, _, _ = run.oracle_rows(0, rows, idx=run.idx_fwd[0].cpu().numpy())
    got = f64(run.out[0])
    err = np.abs(got - ora)
    # the selected branch alone (oracle, fp64) bounds what the extra roundings can move
    sel_only = dict(oracle_cfg(wl), branches=BR_SEL, gated=False)
    q = f64(run.x["q"][0])
    o_sel, _, _ = O.nsa_rows(sel_only, q, rows + wl.q_pos0, f64(run.x["k"][0]), f64(run.x["v"][0]),
                             None, idx=run.idx_fwd[0].cpu().numpy())
    g_sel = f64(run.x["gates"][0])[..., 1]
    extra = 2 * 2.0 ** -9 * g_sel * np.abs(o_sel).max(axis=-1)
    # against the oracle: the final rounding (half a bf16 ulp, 2^-8 relative), the two
    # extra roundings, and fp32 accumulation
    ora_bound = 2.0 ** -8 * np.abs(ora).max(axis=-1) + extra + 1e-3
    assert (err.max(axis=-1) <= ora_bound).all(), float((err.max(axis=-1) - ora_bound).max())
    assert err.mean() <= 1e-3, err.mean()
    bound = extra + 2.0 ** -7 * np.abs(ora).max(axis=-1)
    ws = torch.empty(abi.nsa_workspace_size_min(run.cfg), dtype=torch.uint8, device="cuda")
    qm = torch.empty_like(run.out)
    abi.nsa_sparse_attn_fwd(run.cfg, run.x["q"], run.x["k"], run.x["v"], run.pooled["kbar"],
                            run.pooled["kcmp"], run.pooled["vcmp"], run.x["gates"], run.idx_fwd,
                            qm, ws, ws.numel())
    torch.cuda.synchronize()
    diff = np.abs(got - f64(qm)).max(axis=-1)
    assert (diff <= bound + 1e-6).all(), float((diff - bound).max())
    print(f"{name}: block-major vs oracle max {err.max():.3e} mean {err.mean():.3e}")
