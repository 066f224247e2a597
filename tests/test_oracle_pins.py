"""Pins for the fp64 oracle: each test ties it to something other than itself.

Kinds of pin used here: a library routine (avg_pool1d, scaled_dot_product_attention
in float64), a closed form (constant blocks, dense causal attention as the
special case that keeps every block, identity compression), brute-force
enumeration (rank counting for the top-k), hand-derived worked examples under
tests/golden/, and invariants (causality, gate linearity, decode = last prefill
row).  ``test_planted_mistakes_are_caught`` plants plausible mistakes in the
oracle and checks that one of these pins fails for each.
"""
import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import nsa_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def cfg_of(**kw):
    base = dict(h_q=4, h_kv=1, d_qk=16, d_v=8, sel_block=8, top_k=3, window=12, cmp_block=8,
                cmp_stride=4, branches=7, per_head_select=False, gated=True)
    base.update(kw)
    base.setdefault("scale", 1.0 / math.sqrt(base["d_qk"]))
    return base


def rand_problem(cfg, T, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, cfg["h_q"], cfg["d_qk"]))
    K = rng.standard_normal((cfg["h_kv"], T, cfg["d_qk"]))
    V = rng.standard_normal((cfg["h_kv"], T, cfg["d_v"]))
    gates = 1 / (1 + np.exp(-rng.standard_normal((T, cfg["h_q"], 3))))
    return q, K, V, gates


def run(cfg, q, K, V, gates, rows=None, idx=None):
    T = q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    return O.nsa_rows(cfg, q[rows], rows, K, V, None if gates is None else gates[rows], idx=idx)


def sdpa(q, k, v, scale, mask):
    """Library softmax attention in float64: q [n,d], k [m,d], v [m,dv], mask [n,m] bool."""
    out = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None],
                                         attn_mask=torch.from_numpy(mask)[None], scale=scale)
    return out[0].numpy()


# ---------------------------------------------------------------------------
# Block representations
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T,b", [(64, 8), (67, 8), (512, 64), (40, 16)])
def test_pool_block_keys_is_avg_pool(T, b):
    rng = np.random.default_rng(1)
    K = rng.standard_normal((3, T, 5))
    got = O.pool_block_keys(K, b)
    ref = F.avg_pool1d(torch.from_numpy(K).permute(0, 2, 1), kernel_size=b, stride=b)
    np.testing.assert_allclose(got, ref.permute(0, 2, 1).numpy(), rtol=0, atol=1e-14)
    assert got.shape[1] == T // b


@pytest.mark.parametrize("T,l,s", [(64, 32, 16), (1024, 32, 32), (100, 32, 16), (31, 32, 16),
                                   (50, 4, 2)])
def test_compress_is_avg_pool(T, l, s):
    rng = np.random.default_rng(2)
    X = rng.standard_normal((2, T, 3))
    got = O.compress(X, l, s)
    if T < l:
        assert got.shape[1] == 0
        return
    ref = F.avg_pool1d(torch.from_numpy(X).permute(0, 2, 1), kernel_size=l, stride=s)
    np.testing.assert_allclose(got, ref.permute(0, 2, 1).numpy(), rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# Block scores
# ---------------------------------------------------------------------------

def test_scores_closed_form_constant_blocks():
    """Blocks of constant keys: Kbar_b = c_b, q_h = e_i for all heads -> score = scale*G*c_b[i]."""
    G, d, b_s, nb = 4, 8, 8, 6
    c = np.arange(nb * d, dtype=np.float64).reshape(nb, d) / 10 - 2
    K = np.repeat(c, b_s, axis=0)[None]                       # [1, T, d]
    T = nb * b_s
    i = 3
    q = np.zeros((1, G, d))
    q[0, :, i] = 1.0
    pos = np.array([T - 1])
    s = O.block_scores(q, pos, O.pool_block_keys(K, b_s), G, 1, b_s, 0.25, False, nb)
    c_last = (T - 1) // b_s
    np.testing.assert_allclose(s[0, 0, :c_last], 0.25 * G * c[:c_last, i], atol=1e-12)
    assert np.all(np.isneginf(s[0, 0, c_last:]))


def test_group_score_equals_score_of_summed_query():
    """Linearity: sum_h scale*q_h.Kbar = scale*(sum_h q_h).Kbar (a different formula)."""
    cfg = cfg_of(h_q=8, h_kv=2)
    q, K, V, _ = rand_problem(cfg, 96)
    pos = np.arange(96)
    Kbar = O.pool_block_keys(K, cfg["sel_block"])
    s = O.block_scores(q, pos, Kbar, 8, 2, 8, cfg["scale"], False, 12)
    for g in range(2):
        qt = q[:, 4 * g:4 * g + 4].sum(axis=1)
        ref = cfg["scale"] * qt @ Kbar[g].T
        for t in range(96):
            c = t // 8
            np.testing.assert_allclose(s[g, t, :c], ref[t, :c], rtol=1e-12, atol=1e-12)


def test_golden_group_sum_selection():
    gd = golden("group_sum_selection.json")
    K = np.repeat(np.array([1.0, -2.0, 0.5, 0.0]), 4)[None, :, None]      # [1, 16, 1]
    q = np.array([[[3.0], [-1.0]]])                                          # [1, 2, 1]
    pos = np.array([15])
    Kbar = O.pool_block_keys(K, 4)
    s = O.block_scores(q, pos, Kbar, 2, 1, 4, 1.0, False, 4)
    np.testing.assert_allclose(s[0, 0, :3], gd["expected_group_scores"], atol=1e-15)
    idx, _ = O.select_blocks(s, pos, 4, 2)
    assert idx[0, 0].tolist() == gd["expected_group_blocks"]
    s_h = O.block_scores(q, pos, Kbar, 2, 1, 4, 1.0, True, 4)
    idx_h, _ = O.select_blocks(s_h, pos, 4, 2)
    assert [idx_h[h, 0].tolist() for h in range(2)] == gd["expected_per_head_blocks"]


def test_golden_figure2_selection():
    gd = golden("figure2_selection.json")
    T, b_s, d = gd["T"], gd["sel_block"], gd["d_qk"]
    K = np.zeros((1, T, d))
    K[0, b_s:2 * b_s, 0] = 1.0
    q = np.zeros((1, 1, d))
    q[0, 0, 0] = 1.0
    pos = np.array([gd["query_position"]])
    s = O.block_scores(q, pos, O.pool_block_keys(K, b_s), 1, 1, b_s, 1 / math.sqrt(d), False, 4)
    np.testing.assert_allclose(s[0, 0, :3], gd["expected_scores"], atol=1e-15)
    idx, _ = O.select_blocks(s, pos, b_s, gd["top_k"])
    assert idx[0, 0].tolist() == gd["expected_blocks"]


def test_golden_selection_gap():
    """The near-tie measure: last kept minus first dropped past score, in fp32."""
    gd = golden("selection_gap.json")
    b_s = gd["sel_block"]
    for row in gd["rows"]:
        s = np.array(row["scores"], dtype=np.float64)
        c = row["position"] // b_s
        scores = np.full((1, 1, c + 1), -np.inf)
        scores[0, 0, :len(s)] = s
        idx, gap = O.select_blocks(scores, np.array([row["position"]]), b_s, row["top_k"])
        got = [int(x) for x in idx[0, 0] if x >= 0]
        assert got == row["expected_blocks"]
        want = np.inf if row["expected_gap"] == "inf" else float(row["expected_gap"])
        assert gap[0, 0] == want, (gap[0, 0], want)


# ---------------------------------------------------------------------------
# Top-k selection
# ---------------------------------------------------------------------------

def brute_force_selection(s, c, k):
    """Rank counting: past block b is kept iff fewer than k-1 candidates beat it."""
    kept = []
    for b in range(c):
        beaten_by = sum(1 for b2 in range(c) if s[b2] > s[b] or (s[b2] == s[b] and b2 < b))
        if beaten_by < k - 1:
            kept.append(b)
    return sorted(kept + [c])


@pytest.mark.parametrize("seed", range(4))
def test_selection_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    T, b_s, k = 200, 8, 4
    # coarse integer scores force many exact ties
    scores = np.full((2, T, 25), -np.inf)
    for r in range(T):
        c = r // b_s
        scores[:, r, :c] = rng.integers(0, 4, size=(2, c))
    idx, gap = O.select_blocks(scores, np.arange(T), b_s, k)
    for u in range(2):
        for r in range(T):
            c = r // b_s
            want = brute_force_selection(scores[u, r], c, k)
            got = [x for x in idx[u, r].tolist() if x >= 0]
            assert got == want
            assert len(got) == min(k, c + 1)
            assert all(x == -1 for x in idx[u, r, len(got):])


def test_selection_ties_go_to_lower_index():
    scores = np.zeros((1, 1, 10))
    idx, gap = O.select_blocks(scores, np.array([10 * 4 + 1]), 4, 4)
    assert idx[0, 0].tolist() == [0, 1, 2, 10]
    assert gap[0, 0] == 0.0


def test_group_sum_changes_the_selection_somewhere():
    """On the tiny workload's shapes the shared (summed) set differs from some head's own set."""
    cfg = cfg_of(h_q=4, h_kv=1, d_qk=64, d_v=64, sel_block=64, top_k=4)
    q, K, V, _ = rand_problem(cfg, 1024, seed=3)
    pos = np.arange(1024)
    Kbar = O.pool_block_keys(K, 64)
    sg = O.block_scores(q, pos, Kbar, 4, 1, 64, cfg["scale"], False, 16)
    sh = O.block_scores(q, pos, Kbar, 4, 1, 64, cfg["scale"], True, 16)
    ig, _ = O.select_blocks(sg, pos, 64, 4)
    ih, _ = O.select_blocks(sh, pos, 64, 4)
    assert any((ih[h] != ig[0]).any() for h in range(4))


# ---------------------------------------------------------------------------
# Attention
# ---------------------------------------------------------------------------

def test_golden_softmax_two_keys():
    gd = golden("softmax_two_keys.json")
    out = O.softmax_attention(np.array([[1.0]]), np.array([[0.0], [math.log(3)]]),
                              np.array([[0.0], [4.0]]), 1.0)
    assert abs(out[0, 0] - gd["expected"]) < 1e-13


def test_softmax_attention_is_sdpa():
    rng = np.random.default_rng(4)
    q, k, v = rng.standard_normal((5, 7)), rng.standard_normal((9, 7)), rng.standard_normal((9, 3))
    np.testing.assert_allclose(O.softmax_attention(q, k, v, 0.3),
                               sdpa(q, k, v, 0.3, np.ones((5, 9), bool)), atol=1e-13)
    # weights sum to one: values of ones give ones
    np.testing.assert_allclose(O.softmax_attention(q, k, np.ones((9, 2)), 0.3), 1.0, atol=1e-14)


def test_golden_uniform_query_outputs():
    gd = golden("uniform_query_outputs.json")
    cfg = dict(h_q=1, h_kv=1, d_qk=2, d_v=1, sel_block=2, top_k=2, window=3, cmp_block=4,
               cmp_stride=2, scale=1 / math.sqrt(2), branches=7, per_head_select=False)
    T = 8
    q = np.zeros((T, 1, 2))
    K = np.random.default_rng(5).standard_normal((1, T, 2))
    V = np.arange(1, 9, dtype=np.float64).reshape(1, T, 1)
    gates = np.tile(np.array([0.5, 0.25, 0.125]), (T, 1, 1))
    rows = np.array(gd["rows"])
    out, _, _ = O.nsa_rows(cfg, q[rows], rows, K, V, gates[rows])
    np.testing.assert_allclose(out[:, 0, 0], gd["expected"], atol=1e-13)


def dense_causal(q, K, V, scale, G):
    """Dense causal GQA attention with the library routine: K/V repeated G times."""
    T, H, d = q.shape
    qq = torch.from_numpy(q).permute(1, 0, 2)                       # [H, T, d]
    kk = torch.from_numpy(K).repeat_interleave(G, dim=0)
    vv = torch.from_numpy(V).repeat_interleave(G, dim=0)
    out = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True, scale=scale)
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("T", [64, 77])
def test_selected_branch_keeping_every_block_is_dense_causal(T):
    cfg = cfg_of(h_q=4, h_kv=2, top_k=64, branches=2)
    q, K, V, _ = rand_problem(cfg, T, seed=6)
    gates = np.zeros((T, 4, 3))
    gates[..., 1] = 1.0
    out, idx, _ = run(cfg, q, K, V, gates)
    np.testing.assert_allclose(out, dense_causal(q, K, V, cfg["scale"], 2), atol=1e-12)


def test_window_covering_everything_is_dense_causal():
    T = 70
    cfg = cfg_of(h_q=6, h_kv=3, window=T, branches=4)
    q, K, V, _ = rand_problem(cfg, T, seed=7)
    out, _, _ = run(cfg, q, K, V, None)
    np.testing.assert_allclose(out, dense_causal(q, K, V, cfg["scale"], 2), atol=1e-12)


def test_window_of_one_returns_own_value():
    T = 40
    cfg = cfg_of(window=1, branches=4)
    q, K, V, _ = rand_problem(cfg, T, seed=8)
    out, _, _ = run(cfg, q, K, V, None)
    for t in range(T):
        np.testing.assert_allclose(out[t], np.repeat(V[0, t][None], 4, axis=0), atol=1e-14)


def test_identity_compression_is_dense_causal():
    T = 50
    cfg = cfg_of(h_q=4, h_kv=2, cmp_block=1, cmp_stride=1, branches=1)
    q, K, V, _ = rand_problem(cfg, T, seed=9)
    out, _, _ = run(cfg, q, K, V, None)
    np.testing.assert_allclose(out, dense_causal(q, K, V, cfg["scale"], 2), atol=1e-12)


def test_compressed_branch_is_empty_before_first_window_ends():
    cfg = cfg_of(cmp_block=8, cmp_stride=4, branches=1)
    q, K, V, _ = rand_problem(cfg, 40, seed=10)
    out, _, _ = run(cfg, q, K, V, None)
    assert np.all(out[:7] == 0)
    assert np.all(np.abs(out[7:]).sum(axis=-1) > 0)


def test_compressed_branch_matches_sdpa_on_pooled_tokens():
    """Compressed branch = library attention over avg-pooled K/V, visible once the window ends."""
    T = 64
    cfg = cfg_of(h_q=2, h_kv=1, cmp_block=8, cmp_stride=4, branches=1)
    q, K, V, _ = rand_problem(cfg, T, seed=11)
    out, _, _ = run(cfg, q, K, V, None)
    Kc = F.avg_pool1d(torch.from_numpy(K).permute(0, 2, 1), 8, 4).permute(0, 2, 1).numpy()[0]
    Vc = F.avg_pool1d(torch.from_numpy(V).permute(0, 2, 1), 8, 4).permute(0, 2, 1).numpy()[0]
    ends = np.arange(Kc.shape[0]) * 4 + 7
    for t in range(7, T):
        mask = np.broadcast_to(ends <= t, (2, Kc.shape[0]))
        np.testing.assert_allclose(out[t], sdpa(q[t], Kc, Vc, cfg["scale"], mask.copy()),
                                   atol=1e-12)


def test_selected_branch_matches_sdpa_with_block_mask():
    """Given the kept blocks, the branch is library attention over their visible tokens."""
    T = 96
    cfg = cfg_of(h_q=4, h_kv=1, sel_block=8, top_k=3, branches=2)
    q, K, V, _ = rand_problem(cfg, T, seed=12)
    out, idx, _ = run(cfg, q, K, V, None)
    for t in range(T):
        mask = np.zeros(T, bool)
        for b in idx[0, t]:
            if b >= 0:
                mask[b * 8:(b + 1) * 8] = True
        mask[t + 1:] = False
        m = np.broadcast_to(mask, (4, T)).copy()
        np.testing.assert_allclose(out[t], sdpa(q[t], K[0], V[0], cfg["scale"], m), atol=1e-12)


def test_selected_branch_over_sub_blocks_is_the_same_softmax():
    """The selected branch is one softmax over every key of the kept blocks up to the
    query, so cutting each kept block into sub-blocks and keeping those that start at or
    before the query changes neither the key set nor the output (the restatement the
    per-head block-major path runs: 512-key blocks as 64-key sub-blocks; 32 as 8 here)."""
    T, bs, sub = 200, 32, 8
    spb = bs // sub
    cfg = cfg_of(h_q=4, h_kv=2, sel_block=bs, top_k=3, branches=2, per_head_select=True)
    q, K, V, _ = rand_problem(cfg, T, seed=21)
    out, idx, _ = run(cfg, q, K, V, None)
    n_units = idx.shape[0]
    idx_sub = np.full((n_units, T, cfg["top_k"] * spb), -1, np.int64)
    for u in range(n_units):
        for t in range(T):
            subs = [b * spb + k for b in idx[u, t] if b >= 0 for k in range(spb) if b * bs + k * sub <= t]
            assert sorted(O.selected_keys(idx[u, t], t, bs)) == sorted(O.selected_keys(subs, t, sub))
            idx_sub[u, t, :len(subs)] = subs
    cfg_sub = dict(cfg, sel_block=sub, top_k=cfg["top_k"] * spb)
    out_sub, _, _ = run(cfg_sub, q, K, V, None, idx=idx_sub)
    np.testing.assert_allclose(out_sub, out, atol=1e-12)


def test_top1_keeps_only_the_own_block():
    T = 48
    cfg = cfg_of(h_q=2, h_kv=1, sel_block=8, top_k=1, branches=2)
    q, K, V, _ = rand_problem(cfg, T, seed=13)
    out, idx, _ = run(cfg, q, K, V, None)
    for t in range(T):
        assert idx[0, t].tolist() == [t // 8]
        lo = (t // 8) * 8
        m = np.zeros((2, T), bool)
        m[:, lo:t + 1] = True
        np.testing.assert_allclose(out[t], sdpa(q[t], K[0], V[0], cfg["scale"], m), atol=1e-12)


def test_causality_future_keys_do_not_matter():
    T = 90
    cfg = cfg_of(h_q=4, h_kv=2, top_k=3)
    q, K, V, gates = rand_problem(cfg, T, seed=14)
    out, idx, _ = run(cfg, q, K, V, gates)
    t0 = 50
    K2, V2 = K.copy(), V.copy()
    K2[:, t0 + 1:] = np.random.default_rng(0).standard_normal(K2[:, t0 + 1:].shape) * 5
    V2[:, t0 + 1:] = -V2[:, t0 + 1:]
    out2, idx2, _ = run(cfg, q, K2, V2, gates)
    assert np.array_equal(out[:t0 + 1], out2[:t0 + 1])
    assert np.array_equal(idx[:, :t0 + 1], idx2[:, :t0 + 1])


def test_gates_are_linear():
    T = 60
    cfg = cfg_of(h_q=4, h_kv=1)
    q, K, V, gates = rand_problem(cfg, T, seed=15)
    out, _, _ = run(cfg, q, K, V, gates)
    acc = np.zeros_like(out)
    for br in range(3):
        e = np.zeros_like(gates)
        e[..., br] = 1.0
        o_br, _, _ = run(cfg, q, K, V, e)
        acc += gates[..., br:br + 1] * o_br
    np.testing.assert_allclose(out, acc, atol=1e-13)


def test_ungated_sums_branches():
    T = 40
    cfg = cfg_of(h_q=2, h_kv=1)
    q, K, V, _ = rand_problem(cfg, T, seed=16)
    out, _, _ = run(cfg, q, K, V, None)
    out1, _, _ = run(cfg, q, K, V, np.ones((T, 2, 3)))
    np.testing.assert_allclose(out, out1, atol=1e-14)


def test_decode_row_equals_last_prefill_row():
    T = 130
    cfg = cfg_of(h_q=4, h_kv=2, top_k=4)
    q, K, V, gates = rand_problem(cfg, T, seed=17)
    out, idx, _ = run(cfg, q, K, V, gates)
    out_d, idx_d, _ = O.nsa_rows(cfg, q[T - 1:], np.array([T - 1]), K, V, gates[T - 1:])
    assert np.array_equal(out_d[0], out[T - 1])
    assert np.array_equal(idx_d[:, 0], idx[:, T - 1])


def test_per_head_selection_is_group_of_one():
    """MoBA mode on an MHA problem equals NSA mode on the same problem (groups of one head)."""
    T = 80
    cfg = cfg_of(h_q=3, h_kv=3, top_k=3)
    q, K, V, gates = rand_problem(cfg, T, seed=18)
    a, ia, _ = run(cfg, q, K, V, gates)
    b, ib, _ = run(dict(cfg, per_head_select=True), q, K, V, gates)
    assert np.array_equal(a, b) and np.array_equal(ia, ib)


def test_external_idx_is_used():
    T = 64
    cfg = cfg_of(h_q=2, h_kv=1, top_k=2, branches=2)
    q, K, V, _ = rand_problem(cfg, T, seed=19)
    idx = np.full((1, T, 2), -1, np.int32)
    idx[0, :, 0] = np.arange(T) // 8                     # own block only
    out, _, _ = run(cfg, q, K, V, None, idx=idx)
    cfg1 = dict(cfg, top_k=1)
    ref, _, _ = run(cfg1, q, K, V, None)
    np.testing.assert_allclose(out, ref, atol=1e-14)


# ---------------------------------------------------------------------------
# Planted mistakes: each must make at least one pin above fail.
# ---------------------------------------------------------------------------

# ---------------------------------------------------------------------------
# Selection-score variants and forced leading blocks
# ---------------------------------------------------------------------------

def test_golden_prob_selection():
    """Probability-sum scores on a hand-computed 2-head example; the raw sum picks otherwise."""
    gd = golden("prob_selection.json")
    Kbar = np.array(gd["Kbar"])[None]                  # [1, nb_full, d]
    q = np.array(gd["q"])[None]                        # [1 row, heads, d]
    pos = np.array([gd["position"]])
    args = (q, pos, Kbar, gd["h_q"], gd["h_kv"], gd["sel_block"], gd["scale"], False, 4)
    s = O.block_scores_prob(*args)
    np.testing.assert_allclose(s[0, 0, :3], gd["expected_scores"], atol=1e-7)
    idx, _ = O.select_blocks(s, pos, gd["sel_block"], gd["top_k"])
    assert idx[0, 0].tolist() == gd["expected_blocks"]
    idx_raw, _ = O.select_blocks(O.block_scores(*args), pos, gd["sel_block"], gd["top_k"])
    assert idx_raw[0, 0].tolist() == gd["expected_blocks_raw_sum"]


def test_prob_scores_sum_to_the_number_of_heads():
    """Each head's probabilities over the candidates sum to 1."""
    cfg = cfg_of(h_q=8, h_kv=2, d_qk=32, d_v=16, sel_block=16, top_k=4)
    q, K, V, _ = rand_problem(cfg, 200, seed=11)
    pos = np.arange(200)
    Kbar = O.pool_block_keys(K, 16)
    s = O.block_scores_prob(q, pos, Kbar, 8, 2, 16, cfg["scale"], False, 13)
    for r in range(200):
        c = r // 16
        if c:
            np.testing.assert_allclose(s[:, r, :c].sum(axis=-1), 4.0, rtol=1e-12)


def test_prob_selection_equals_raw_selection_for_single_head_units():
    """Softmax is strictly increasing, so one head's probabilities rank blocks like its scores."""
    cfg = cfg_of(h_q=4, h_kv=4, d_qk=32, d_v=16, sel_block=16, top_k=5)
    q, K, V, _ = rand_problem(cfg, 300, seed=12)
    pos = np.arange(300)
    Kbar = O.pool_block_keys(K, 16)
    args = (q, pos, Kbar, 4, 4, 16, cfg["scale"], True, 19)
    a, _ = O.select_blocks(O.block_scores_prob(*args), pos, 16, 5)
    b, _ = O.select_blocks(O.block_scores(*args), pos, 16, 5)
    assert np.array_equal(a, b)


def test_golden_compressed_aggregation():
    """Uniform compressed probabilities spread over the overlapped blocks, by hand."""
    gd = golden("cmp_aggregation.json")
    rng = np.random.default_rng(13)
    T = gd["position"] + 1
    Kc = rng.standard_normal((1, O.n_compressed(T, gd["cmp_block"], gd["cmp_stride"]), 8))
    q = np.zeros((1, gd["h_q"], 8))
    pos = np.array([gd["position"]])
    s = O.block_scores_from_compressed(q, pos, Kc, gd["h_q"], gd["h_kv"], gd["sel_block"],
                                       gd["cmp_block"], gd["cmp_stride"], 1.0, False, 4)
    np.testing.assert_allclose(s[0, 0, :3], gd["expected_scores"], rtol=1e-12)
    idx, _ = O.select_blocks(s, pos, gd["sel_block"], gd["top_k"])
    assert idx[0, 0].tolist() == gd["expected_blocks"]


def test_compressed_aggregation_by_source_tokens():
    """Brute force at the token level: every compressed token's probability is spread
    evenly over its source tokens, and a block's score sums its tokens' shares."""
    rng = np.random.default_rng(14)
    h_q, h_kv, d, bs, lc, sc, T = 4, 2, 16, 16, 8, 4, 150
    K = rng.standard_normal((h_kv, T, d))
    Kc = O.compress(K, lc, sc)
    q = rng.standard_normal((T, h_q, d))
    pos = np.arange(T)
    nb = -(-T // bs)
    s = O.block_scores_from_compressed(q, pos, Kc, h_q, h_kv, bs, lc, sc, 0.3, False, nb)
    G = h_q // h_kv
    for r in range(0, T, 7):
        c = r // bs
        vis = [j for j in range(Kc.shape[1]) if j * sc + lc - 1 <= r]
        for g in range(h_kv):
            share = np.zeros(T + lc)
            for h in range(g * G, (g + 1) * G):
                if not vis:
                    continue
                lg = np.array([0.3 * float(q[r, h] @ Kc[g, j]) for j in vis])
                w = np.exp(lg - lg.max())
                w /= w.sum()
                for wj, j in zip(w, vis):
                    share[j * sc:j * sc + lc] += wj / lc
            want = [share[b * bs:(b + 1) * bs].sum() for b in range(c)]
            np.testing.assert_allclose(s[g, r, :c], want, rtol=1e-10, atol=1e-14)


def test_compressed_aggregation_with_aligned_blocks_is_the_compressed_probability():
    """cmp_block = cmp_stride = sel_block: token j is block j, so a block's score is the
    unit's summed compressed-branch weight of that token."""
    rng = np.random.default_rng(15)
    h_q, h_kv, d, bs, T = 2, 1, 8, 8, 80
    K = rng.standard_normal((h_kv, T, d))
    Kc = O.compress(K, bs, bs)
    q = rng.standard_normal((T, h_q, d))
    pos = np.arange(T)
    s = O.block_scores_from_compressed(q, pos, Kc, h_q, h_kv, bs, bs, bs, 1.0, False, T // bs)
    for r in range(bs, T):
        c = r // bs
        vis = np.arange((r - bs + 1) // bs + 1)
        want = np.zeros(c)
        for h in range(h_q):
            lg = Kc[0, vis] @ q[r, h]
            w = np.exp(lg - lg.max())
            want += (w / w.sum())[:c]
        np.testing.assert_allclose(s[0, r, :c], want, rtol=1e-12)


def brute_force_selection_with_sinks(s, c, k, n_sink):
    forced = list(range(min(n_sink, c)))
    rest = [b for b in range(len(forced), c)]
    kept = []
    for b in rest:
        beaten_by = sum(1 for b2 in rest if s[b2] > s[b] or (s[b2] == s[b] and b2 < b))
        if beaten_by < k - 1 - len(forced):
            kept.append(b)
    return sorted(forced + kept + [c])


@pytest.mark.parametrize("n_sink", [1, 2, 3])
def test_sink_blocks_match_brute_force(n_sink):
    rng = np.random.default_rng(20 + n_sink)
    T, b_s, k = 400, 16, 4
    scores = np.full((2, T, 25), -np.inf)
    for r in range(T):
        c = r // b_s
        scores[:, r, :c] = rng.integers(0, 4, size=(2, c))
    idx, _ = O.select_blocks(scores, np.arange(T), b_s, k, n_sink)
    for u in range(2):
        for r in range(T):
            c = r // b_s
            got = [x for x in idx[u, r].tolist() if x >= 0]
            assert got == brute_force_selection_with_sinks(scores[u, r], c, k, n_sink)
            assert len(got) == min(k, c + 1)
            assert all(b in got for b in range(min(n_sink, c)))


def test_sinks_filling_every_free_place_keep_the_leading_blocks():
    scores = np.random.default_rng(30).standard_normal((1, 1, 20))
    idx, gap = O.select_blocks(scores, np.array([19 * 4]), 4, 5, n_sink=4)
    assert idx[0, 0].tolist() == [0, 1, 2, 3, 19]
    assert gap[0, 0] == np.inf


def test_golden_bf16_rounding():
    """Round to nearest, ties to even, on hand-derived cases; and torch's bf16 cast."""
    gd = golden("bf16_rounding.json")
    for c in gd["cases"]:
        assert O.round_bf16(np.array([c["x"]]))[0] == c["expected"], c
    x = np.random.default_rng(40).standard_normal(10000) * 30
    want = torch.tensor(x, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_bf16(x), want)


# ---------------------------------------------------------------------------
# Backward pass
# ---------------------------------------------------------------------------

def _bwd_problem(seed=0, T=40):
    rng = np.random.default_rng(seed)
    cfg = dict(h_q=4, h_kv=2, d_qk=8, d_v=4, sel_block=8, top_k=3, window=10, cmp_block=8,
               cmp_stride=4, scale=8 ** -0.5, branches=7, per_head_select=False)
    q = rng.standard_normal((T, 4, 8))
    K = rng.standard_normal((2, T, 8))
    V = rng.standard_normal((2, T, 4))
    g = rng.uniform(0.2, 1.0, (T, 4, 3))
    return rng, cfg, q, K, V, g


def test_backward_matches_finite_differences():
    """Central differences of the loss sum(d_out * out) in fp64, blocks held fixed."""
    rng, cfg, q, K, V, g = _bwd_problem()
    pos = np.arange(q.shape[0])
    out, idx, _ = O.nsa_rows(cfg, q, pos, K, V, g)
    d_out = rng.standard_normal(out.shape)
    grads = O.nsa_rows_backward(cfg, q, pos, K, V, g, idx, d_out)

    def loss():
        return float((O.nsa_rows(cfg, q, pos, K, V, g, idx=idx)[0] * d_out).sum())

    h = 1e-6
    for arr, grad in zip((q, K, V, g), grads):
        flat, gflat = arr.reshape(-1), grad.reshape(-1)
        for i in rng.choice(flat.size, 24, replace=False):
            old = flat[i]
            flat[i] = old + h
            lp = loss()
            flat[i] = old - h
            lm = loss()
            flat[i] = old
            fd = (lp - lm) / (2 * h)
            assert abs(fd - gflat[i]) <= 1e-7 + 1e-6 * abs(fd), (fd, gflat[i])


def test_backward_of_dense_causal_attention_is_autograd():
    """Window covering the sequence, gates (0, 0, 1): the gradients are those of dense
    causal softmax attention, computed by torch autograd in float64 (K/V shared by each
    group of two heads, so their gradients sum over the group)."""
    rng, cfg, q, K, V, _ = _bwd_problem(seed=1, T=30)
    cfg = dict(cfg, window=30, branches=4)
    T = q.shape[0]
    pos = np.arange(T)
    d_out = rng.standard_normal((T, 4, 4))
    dq, dK, dV, _ = O.nsa_rows_backward(cfg, q, pos, K, V, None, None, d_out)
    qt = torch.tensor(q, requires_grad=True)
    Kt = torch.tensor(K, requires_grad=True)
    Vt = torch.tensor(V, requires_grad=True)
    o = F.scaled_dot_product_attention(qt.permute(1, 0, 2), Kt.repeat_interleave(2, 0),
                                       Vt.repeat_interleave(2, 0), is_causal=True,
                                       scale=cfg["scale"]).permute(1, 0, 2)
    (o * torch.tensor(d_out)).sum().backward()
    np.testing.assert_allclose(dq, qt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dK, Kt.grad.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(dV, Vt.grad.numpy(), rtol=1e-10, atol=1e-12)


def _mut_window_off_by_one(t, window):
    return np.arange(max(0, t - window + 2), t + 1, dtype=np.int64)


def _mut_selected_strict_causal(blocks, t, sel_block):
    keys = []
    for b in blocks:
        if b >= 0:
            keys.extend(range(b * sel_block, min((b + 1) * sel_block, t)))
    return np.asarray(keys, dtype=np.int64)


def _mut_compressed_early(t, n_cmp, cmp_block, cmp_stride):
    j = np.arange(n_cmp, dtype=np.int64)
    return j[j * cmp_stride <= t]


def _mut_pool_drops_last(K, sel_block):
    H, T, d = K.shape
    nb = T // sel_block
    out = np.zeros((H, nb, d))
    for b in range(nb):
        out[:, b] = K[:, b * sel_block:(b + 1) * sel_block - 1].mean(axis=1)
    return out


def _mut_select_higher_index_on_tie(scores, positions, sel_block, top_k, n_sink=0):
    U, R, nb = scores.shape
    idx = np.full((U, R, top_k), -1, dtype=np.int32)
    gap = np.full((U, R), np.inf)
    for u in range(U):
        for r in range(R):
            c = int(positions[r]) // sel_block
            s = scores[u, r, :c]
            order = sorted(range(c), key=lambda b: (-s[b], -b))
            chosen = sorted(order[:min(top_k - 1, c)] + [c])
            idx[u, r, :len(chosen)] = chosen
    return idx, gap


def _mut_gap_one_place_late(scores, positions, sel_block, top_k, n_sink=0):
    """Tie gap measured between the first and second dropped scores."""
    U, R, nb = scores.shape
    idx = np.full((U, R, top_k), -1, dtype=np.int32)
    gap = np.full((U, R), np.inf)
    for u in range(U):
        for r in range(R):
            c = int(positions[r]) // sel_block
            n_cand = min(c, nb)
            s = scores[u, r, :n_cand]
            order = np.argsort(-s, kind="stable")
            chosen = sorted([int(b) for b in order[:min(top_k - 1, n_cand)]] + [c])
            idx[u, r, :len(chosen)] = chosen
            if n_cand > top_k:
                s32 = s.astype(np.float32).astype(np.float64)
                gap[u, r] = s32[order[top_k - 1]] - s32[order[top_k]]
    return idx, gap


def _mut_scores_max_not_sum(q_rows, positions, Kbar, h_q, h_kv, sel_block, scale, per_head,
                            n_blocks):
    R = q_rows.shape[0]
    units = O.selection_units(h_q, h_kv, per_head)
    out = np.full((len(units), R, n_blocks), -np.inf)
    for u, (hk, heads) in enumerate(units):
        per = np.stack([scale * (q_rows[:, h, :] @ Kbar[hk].T) for h in heads])
        total = per.max(axis=0)
        for r in range(R):
            c = min(int(positions[r]) // sel_block, Kbar.shape[1])
            out[u, r, :c] = total[r, :c]
    return out


def _mut_softmax_no_max(q, k, v, scale):
    if k.shape[0] == 0:
        return np.zeros((q.shape[0], v.shape[1]))
    p = np.exp(scale * (q @ k.T))
    return (p / p.sum(axis=1, keepdims=True).clip(min=1.0)) @ v


def _mut_prob_over_all_blocks(q_rows, positions, Kbar, h_q, h_kv, sel_block, scale, per_head,
                              n_blocks):
    """Probability-sum scores normalised over every pooled block, current and later ones too."""
    R = q_rows.shape[0]
    units = O.selection_units(h_q, h_kv, per_head)
    out = np.full((len(units), R, n_blocks), -np.inf)
    nb_full = Kbar.shape[1]
    for u, (hk, heads) in enumerate(units):
        for r in range(R):
            c = min(int(positions[r]) // sel_block, nb_full)
            if c == 0:
                continue
            total = np.zeros(nb_full)
            for h in heads:
                lg = scale * (Kbar[hk] @ q_rows[r, h])
                p = np.exp(lg - lg.max())
                total += p / p.sum()
            out[u, r, :c] = total[:c]
    return out


def _mut_cmp_weight_in_tokens(q_rows, positions, Kc, h_q, h_kv, sel_block, cmp_block, cmp_stride,
                              scale, per_head, n_blocks):
    """Compressed aggregation weighted by overlapping tokens, not by the share of the window."""
    return O_REAL_CMP(q_rows, positions, Kc, h_q, h_kv, sel_block, cmp_block, cmp_stride, scale,
                      per_head, n_blocks) * cmp_block


def _mut_sinks_outside_k(scores, positions, sel_block, top_k, n_sink=0):
    """Sink blocks added on top of k - 1 scored blocks."""
    return O_REAL_SELECT(scores, positions, sel_block, top_k + min(n_sink, 1) * n_sink, 0)


O_REAL_CMP = O.block_scores_from_compressed
O_REAL_SELECT = O.select_blocks


def _mut_softmax_grad_no_rowsum(q, k, v, scale, d_o):
    """Softmax gradient without the row-sum (normaliser) term."""
    if k.shape[0] == 0:
        return np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    lg = scale * (q @ k.T)
    p = np.exp(lg - lg.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    ds = p * (d_o @ v.T)
    return scale * (ds @ k), scale * (ds.T @ q), p.T @ d_o


def _mut_bwd_cmp_not_averaged(cfg, q_rows, positions, K, V, gates_rows, idx, d_out):
    """Compressed-token gradients added to every window token undivided."""
    dq, dK, dV, dg = O_REAL_BWD(cfg, q_rows, positions, K, V, gates_rows, idx, d_out)
    c = dict(cfg, branches=1)
    _, dK1, dV1, _ = O_REAL_BWD(c, q_rows, positions, K, V, gates_rows, idx, d_out)
    l = cfg["cmp_block"]
    return dq, dK + (l - 1) * dK1, dV + (l - 1) * dV1, dg


O_REAL_BWD = O.nsa_rows_backward


MUTATIONS = {
    "window off by one": ("window_keys", _mut_window_off_by_one),
    "selected keys exclude self": ("selected_keys", _mut_selected_strict_causal),
    "compressed token visible at its first token": ("compressed_keys", _mut_compressed_early),
    "block mean drops a key": ("pool_block_keys", _mut_pool_drops_last),
    "tie goes to higher index": ("select_blocks", _mut_select_higher_index_on_tie),
    "tie gap one place late": ("select_blocks", _mut_gap_one_place_late),
    "group max instead of sum": ("block_scores", _mut_scores_max_not_sum),
    "softmax normaliser clipped": ("softmax_attention", _mut_softmax_no_max),
    "probabilities normalised over later blocks": ("block_scores_prob", _mut_prob_over_all_blocks),
    "compressed weights in tokens": ("block_scores_from_compressed", _mut_cmp_weight_in_tokens),
    "sinks kept outside k": ("select_blocks", _mut_sinks_outside_k),
    "softmax gradient without the normaliser term": ("softmax_attention_grad", _mut_softmax_grad_no_rowsum),
    "compressed gradient not averaged over its window": ("nsa_rows_backward", _mut_bwd_cmp_not_averaged),
}

PINS = [test_golden_uniform_query_outputs, test_golden_figure2_selection,
        test_golden_selection_gap, test_golden_prob_selection, test_prob_scores_sum_to_the_number_of_heads,
        test_golden_compressed_aggregation, test_compressed_aggregation_by_source_tokens,
        lambda: test_sink_blocks_match_brute_force(2), test_backward_matches_finite_differences,
        test_golden_group_sum_selection, test_selection_ties_go_to_lower_index,
        test_window_of_one_returns_own_value, test_golden_softmax_two_keys,
        lambda: test_selected_branch_keeping_every_block_is_dense_causal(64),
        test_compressed_branch_matches_sdpa_on_pooled_tokens,
        test_group_score_equals_score_of_summed_query,
        lambda: test_pool_block_keys_is_avg_pool(64, 8)]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failures = 0
    for pin in PINS:
        try:
            pin()
        except AssertionError:
            failures += 1
    assert failures > 0, f"no pin caught the planted mistake: {name}"
