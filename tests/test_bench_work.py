"""The work counts bench.py divides by (CPU, no GPU).

visible_key_counts is checked against a brute-force enumeration of every
query's visible keys per branch (window [t - W + 1, t], compressed tokens whose
window ends at or before t, the top-k blocks' keys up to t with the current
block forced), on small shapes with ragged ends and a query offset; the 64k
totals are the figures the roofline fractions of the bench line use.
"""
import numpy as np
import pytest

import bench
from dynamic_block_sparse_scoring_b200.workloads import WORKLOADS


def brute_counts(wl):
    out = {"sel": [], "win": [], "cmp": []}
    n_cmp = (wl.seqlen_kv - wl.cmp_block) // wl.cmp_stride + 1 if wl.seqlen_kv >= wl.cmp_block else 0
    for i in range(wl.seqlen_q):
        t = wl.q_pos0 + i
        out["win"].append(sum(1 for u in range(t - wl.window + 1, t + 1) if u >= 0))
        out["cmp"].append(sum(1 for j in range(n_cmp) if j * wl.cmp_stride + wl.cmp_block - 1 <= t))
        c = t // wl.sel_block
        past = min(wl.top_k - 1, c)                 # full past blocks kept (every past block is full)
        out["sel"].append(past * wl.sel_block + sum(1 for u in range(c * wl.sel_block, t + 1)))
    return {k: np.array(v) for k, v in out.items()}


CASES = [
    WORKLOADS["tiny"],
    WORKLOADS["tiny"].with_(seqlen_q=77, seqlen_kv=500, q_pos0=423, window=100, cmp_block=32, cmp_stride=16),
    WORKLOADS["nsa64k"].with_(seqlen_q=700, seqlen_kv=700),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: f"{w.name}_{w.seqlen_q}_{w.q_pos0}")
def test_visible_key_counts_match_brute_force(wl):
    got = bench.visible_key_counts(wl)
    ref = brute_counts(wl)
    for name in got:
        assert np.array_equal(got[name], ref[name]), name


def test_64k_prefill_work():
    f = bench.algorithmic_flops(WORKLOADS["nsa64k"])
    assert f["sel"] == pytest.approx(2.64e12, rel=5e-3)
    assert f["win"] == pytest.approx(1.37e12, rel=5e-3)
    assert f["cmp"] == pytest.approx(5.49e12, rel=5e-3)
    assert f["score"] == pytest.approx(5.1e10, rel=2e-2)
    assert f["total"] == pytest.approx(f["sel"] + f["win"] + f["cmp"] + f["score"])
