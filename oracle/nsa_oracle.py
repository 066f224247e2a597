"""fp64 CPU oracle for query-dependent top-k block-sparse causal attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
baseline leg of the benchmark may import this module; the library never calls
it and shares no code with it.  Everything here is plain numpy in float64,
written to be checked by eye against the method as the pages describe it:

* Zhang Xiaojun #94 transcript (bidclub.ai), §2 "Attention From First
  Principles": a token's query is dotted with the keys of earlier tokens, the
  scalar scores go through a softmax under a causal mask, and the normalised
  weights mix the value vectors.
* same page, §4 "Inside Native Sparse Attention", Figure 2 walk-through: the
  KV sequence is cut into contiguous blocks; a compressed (coarse) branch
  attends over one pooled key/value per block under a causal mask; a
  selected branch scores the blocks, keeps the top-k and attends over every
  token of the kept blocks; a sliding-window branch attends over the nearest
  tokens; each branch output is scaled by its own gate and the three are
  summed.  Under GQA the per-head block scores of a group are summed into one
  selection score so that the whole group shares one block set.
* same page, §7 "Kimi Simplifies The Sparse Route": MoBA represents a block
  by the mean of its keys (no parameters), keeps only the selected branch and
  lets every head choose its own blocks.
* LateTalk #103 (zjai.club), §13: MoBA always selects the block that holds
  the current token.

Readings taken where the pages leave a step open (each is stated again where
it is used): block representation = mean pooling (no trained MLP exists
here); selection score = the pre-softmax scaled dot product, summed over the
group's heads; only complete past blocks are candidates and the current block
is always added, so at most ``top_k`` blocks are kept including it; equal
scores go to the lower block index; the window holds the ``window`` most
recent keys including the query's own; a compressed token is visible once its
last source token is visible; a branch with no visible key contributes zero;
gates are taken as given (no normalisation).

Parity status: every function below is pinned by a test under ``tests/``
against a closed form, a library routine, a brute-force enumeration or a
worked example (see ``tests/test_oracle_pins.py``).
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# Block representations
# ---------------------------------------------------------------------------

def pool_block_keys(K: np.ndarray, sel_block: int) -> np.ndarray:
    """Mean of the keys of every complete selection block.

    MoBA's block representation (transcript #94, §7): the mean of the block's
    keys.  K is [H_kv, T_kv, d]; returns [H_kv, T_kv // sel_block, d].
    Only complete blocks are pooled: an incomplete tail block is never a
    candidate because a query can only score blocks that end before its own.
    """
    H, T, d = K.shape
    nb = T // sel_block
    out = np.zeros((H, nb, d), dtype=np.float64)
    for b in range(nb):
        out[:, b, :] = K[:, b * sel_block:(b + 1) * sel_block, :].mean(axis=1)
    return out


def n_compressed(T_kv: int, cmp_block: int, cmp_stride: int) -> int:
    """Number of compression windows [j*stride, j*stride + block) inside T_kv."""
    if cmp_block <= 0 or T_kv < cmp_block:
        return 0
    return (T_kv - cmp_block) // cmp_stride + 1


def compress(X: np.ndarray, cmp_block: int, cmp_stride: int) -> np.ndarray:
    """Compressed tokens: mean of X over windows of ``cmp_block`` tokens every ``cmp_stride``.

    Transcript #94, §4, Figure 2: each block of keys (and of values) is
    compressed into one representation; with no trained compression MLP the
    representation is the mean (§7).  X is [H_kv, T_kv, d].
    """
    H, T, d = X.shape
    n = n_compressed(T, cmp_block, cmp_stride)
    out = np.zeros((H, n, d), dtype=np.float64)
    for j in range(n):
        out[:, j, :] = X[:, j * cmp_stride:j * cmp_stride + cmp_block, :].mean(axis=1)
    return out


# ---------------------------------------------------------------------------
# Selection
# ---------------------------------------------------------------------------

def selection_units(h_q: int, h_kv: int, per_head: bool):
    """List of (kv_head, [query heads]) that share one selected block set.

    NSA (transcript #94, §4, GQA discussion): all heads of a GQA group share
    one set.  MoBA (§7): every head has its own set.
    """
    G = h_q // h_kv
    if per_head:
        return [(h // G, [h]) for h in range(h_q)]
    return [(g, list(range(g * G, (g + 1) * G))) for g in range(h_kv)]


def block_scores(q_rows: np.ndarray, positions: np.ndarray, Kbar: np.ndarray, h_q: int,
                 h_kv: int, sel_block: int, scale: float, per_head: bool, n_blocks: int):
    """Selection score of every candidate block, per selection unit and query row.

    q_rows [R, H_q, d] (the rows' queries), positions [R] (their KV
    positions), Kbar [H_kv, nb_full, d].  Returns [n_units, R, n_blocks] with
    -inf where block b is not a candidate (b >= current block).

    Transcript #94, §4: each query has one score per block; NSA adds the
    scores of the group's heads to get one selection score per block.  The
    per-head score is the attention score of §2 (scaled q . Kbar_b, before
    the softmax).  The sum over heads is taken literally, head by head.
    """
    R = q_rows.shape[0]
    units = selection_units(h_q, h_kv, per_head)
    out = np.full((len(units), R, n_blocks), NEG_INF)
    cur = positions // sel_block
    nb_full = Kbar.shape[1]
    for u, (hk, heads) in enumerate(units):
        total = np.zeros((R, nb_full))
        for h in heads:
            total += scale * (q_rows[:, h, :] @ Kbar[hk].T)
        for r in range(R):
            c = min(int(cur[r]), nb_full)
            out[u, r, :c] = total[r, :c]
    return out


def block_scores_prob(q_rows: np.ndarray, positions: np.ndarray, Kbar: np.ndarray, h_q: int,
                      h_kv: int, sel_block: int, scale: float, per_head: bool, n_blocks: int):
    """Selection-score variant: each head's block probabilities, summed over the unit.

    Transcript #94, §4 (GQA discussion): the group's heads add up their block
    scores.  This variant reads "score" as the normalised score of §2 (after
    the softmax) instead of the raw scaled dot product: per head h, the
    softmax of scale * q_h . Kbar_b over the row's candidate blocks b < c(t),
    then the sum over the unit's heads.  Shapes and -inf marking as in
    ``block_scores``.
    """
    R = q_rows.shape[0]
    units = selection_units(h_q, h_kv, per_head)
    out = np.full((len(units), R, n_blocks), NEG_INF)
    cur = positions // sel_block
    nb_full = Kbar.shape[1]
    for u, (hk, heads) in enumerate(units):
        for r in range(R):
            c = min(int(cur[r]), nb_full)
            if c == 0:
                continue
            total = np.zeros(c)
            for h in heads:
                logits = scale * (Kbar[hk, :c] @ q_rows[r, h, :])
                p = np.exp(logits - logits.max())
                total += p / p.sum()
            out[u, r, :c] = total
    return out


def block_scores_from_compressed(q_rows: np.ndarray, positions: np.ndarray, Kc: np.ndarray,
                                 h_q: int, h_kv: int, sel_block: int, cmp_block: int,
                                 cmp_stride: int, scale: float, per_head: bool, n_blocks: int):
    """Selection-score variant: block scores taken from the compressed branch.

    Transcript #94, §4: when the selection blocks and the compressed tokens
    are cut differently, the selection score of a block has to be gathered
    from the compressed tokens that overlap it (the "corner case").  Read
    plainly: per head h, p_j = softmax over the visible compressed tokens
    (j * stride + cmp_block - 1 <= t) of scale * q_h . Kc_j (the compressed
    branch's attention weights); block b's score is sum_j p_j * w_jb with
    w_jb = |[j*stride, j*stride + cmp_block) ∩ [b*sel_block, (b+1)*sel_block)|
    / cmp_block, the share of token j's window inside block b; the unit sums
    its heads.  Candidates are the past blocks b < c(t) as in ``block_scores``.
    """
    R = q_rows.shape[0]
    units = selection_units(h_q, h_kv, per_head)
    out = np.full((len(units), R, n_blocks), NEG_INF)
    n_cmp = Kc.shape[1]
    for u, (hk, heads) in enumerate(units):
        for r in range(R):
            t = int(positions[r])
            c = t // sel_block
            if c == 0:
                continue
            js = compressed_keys(t, n_cmp, cmp_block, cmp_stride)
            total = np.zeros(c)
            if len(js):
                lo, hi = js * cmp_stride, js * cmp_stride + cmp_block
                for h in heads:
                    logits = scale * (Kc[hk, js] @ q_rows[r, h, :])
                    p = np.exp(logits - logits.max())
                    p /= p.sum()
                    for b in range(c):
                        ov = np.clip(np.minimum(hi, (b + 1) * sel_block) - np.maximum(lo, b * sel_block),
                                     0, None)
                        total[b] += float((p * ov).sum()) / cmp_block
            out[u, r, :c] = total
    return out


def select_blocks(scores: np.ndarray, positions: np.ndarray, sel_block: int, top_k: int,
                  n_sink: int = 0):
    """Top-k block sets from candidate scores.

    scores [n_units, R, n_blocks] (-inf for non-candidates).  For each row the
    current block c = pos // sel_block is always kept (LateTalk #103, §13:
    MoBA's static part), and so are the first ``n_sink`` blocks when they lie
    before it (transcript #94, §4: the attention sink at the start of the
    sequence, read as leading blocks kept like the current one); the rest of
    the top_k places go to the best remaining past blocks by score, equal
    scores going to the lower block index (transcript #94, §4, Figure 2: keep
    the k highest-scoring blocks).  Returns

    * idx [n_units, R, top_k] int32, ascending, -1 padded;
    * gap [n_units, R]: the fp32-rounded difference between the last kept and
      the first dropped scored past block (inf when every candidate is kept),
      which says how close the row's selection is to a tie.
    """
    U, R, nb = scores.shape
    idx = np.full((U, R, top_k), -1, dtype=np.int32)
    gap = np.full((U, R), np.inf)
    for u in range(U):
        for r in range(R):
            c = int(positions[r]) // sel_block
            n_cand = min(c, nb)
            forced = list(range(min(n_sink, n_cand)))
            free = top_k - 1 - len(forced)            # places left for scored blocks
            rest = np.arange(len(forced), n_cand)
            s = scores[u, r, rest]
            # stable sort on -s: equal scores keep ascending block order
            order = np.argsort(-s, kind="stable")
            keep = rest[order[:max(0, min(free, len(rest)))]]
            chosen = sorted(forced + [int(b) for b in keep] + [c])
            idx[u, r, :len(chosen)] = chosen
            if free >= 1 and len(rest) > free:
                s32 = s.astype(np.float32).astype(np.float64)
                gap[u, r] = s32[order[free - 1]] - s32[order[free]]
    return idx, gap


# ---------------------------------------------------------------------------
# Attention branches
# ---------------------------------------------------------------------------

def softmax_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(scale * q k^T) v over the given keys; zero output when there are none.

    Transcript #94, §2: inner products give scalar attention scores, a
    softmax normalises them, the weights linearly combine the value vectors.
    q [n, d], k [m, d], v [m, dv].  Two passes: max, then normalised sum.
    """
    n = q.shape[0]
    if k.shape[0] == 0:
        return np.zeros((n, v.shape[1]))
    logits = scale * (q @ k.T)
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    p /= p.sum(axis=1, keepdims=True)
    return p @ v


def selected_keys(blocks, t: int, sel_block: int) -> np.ndarray:
    """Every token of the selected blocks that the query at t may see (u <= t)."""
    keys = []
    for b in blocks:
        if b < 0:
            continue
        keys.extend(range(b * sel_block, min((b + 1) * sel_block, t + 1)))
    return np.asarray(keys, dtype=np.int64)


def window_keys(t: int, window: int) -> np.ndarray:
    """The ``window`` most recent keys, the query's own included: [t-window+1, t] ∩ [0, t]."""
    return np.arange(max(0, t - window + 1), t + 1, dtype=np.int64)


def compressed_keys(t: int, n_cmp: int, cmp_block: int, cmp_stride: int) -> np.ndarray:
    """Compressed tokens whose whole source window lies at or before t."""
    j = np.arange(n_cmp, dtype=np.int64)
    return j[j * cmp_stride + cmp_block - 1 <= t]


def pooled_inputs(K, V, sel_block, cmp_block, cmp_stride):
    """The pooled tensors a sequence needs: block keys and compressed keys/values."""
    return {"Kbar": pool_block_keys(K, sel_block),
            "Kc": compress(K, cmp_block, cmp_stride),
            "Vc": compress(V, cmp_block, cmp_stride)}


def opt(cfg, name, default):
    """Optional configuration entry (mapping or attribute)."""
    if isinstance(cfg, dict):
        return cfg.get(name, default)
    return getattr(cfg, name, default)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bfloat16 (8-bit significand), to nearest with ties to even, via
    float32 (the value is first rounded to float32, as a float32 mean would be).
    Returned as float64.  Finite inputs only."""
    f = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    lsb = (f >> 16) & 1
    r = ((f + 0x7FFF + lsb) >> 16) << 16
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def selection_scores(cfg, q_rows, positions, pooled, n_blocks):
    """Block scores of the configured kind: "dot" (the scaled dot product with the
    pooled key, summed over the unit; the default), "prob" (``block_scores_prob``)
    or "cmp" (``block_scores_from_compressed``).

    The "cmp" scores read the compressed keys as the kernel stores them, rounded
    to bfloat16: the top-k is an integer decision, taken on both sides from the
    same stored keys (the fp64 means differ from the stored ones by up to 2^-9
    relative, enough to reorder blocks whose scores are 1e-4 apart)."""
    mode = opt(cfg, "score_mode", "dot")
    h_q, h_kv, sel_block = opt(cfg, "h_q", 0), opt(cfg, "h_kv", 0), opt(cfg, "sel_block", 0)
    scale, per_head = opt(cfg, "scale", 1.0), bool(opt(cfg, "per_head_select", False))
    if mode == "prob":
        return block_scores_prob(q_rows, positions, pooled["Kbar"], h_q, h_kv, sel_block, scale,
                                 per_head, n_blocks)
    if mode == "cmp":
        return block_scores_from_compressed(q_rows, positions, round_bf16(pooled["Kc"]), h_q, h_kv,
                                            sel_block,
                                            opt(cfg, "cmp_block", 0), opt(cfg, "cmp_stride", 1),
                                            scale, per_head, n_blocks)
    return block_scores(q_rows, positions, pooled["Kbar"], h_q, h_kv, sel_block, scale, per_head,
                        n_blocks)


def nsa_rows(cfg, q_rows, positions, K, V, gates_rows=None, idx=None, pooled=None):
    """Gated NSA output for a set of query rows of one sequence.

    cfg: mapping or object with h_q, h_kv, d_qk, sel_block, top_k, window,
    cmp_block, cmp_stride, scale, branches (1 cmp | 2 sel | 4 win),
    per_head_select, gated, and optionally score_mode ("dot", "prob", "cmp")
    and sink_blocks (leading blocks always kept).
    q_rows [R, H_q, d_qk], positions [R], K [H_kv, T_kv, d_qk],
    V [H_kv, T_kv, d_v], gates_rows [R, H_q, 3] (cmp, sel, win) or None,
    idx: optional externally chosen [n_units, R, top_k] block sets,
    pooled: optional result of ``pooled_inputs`` for this K, V (saves recomputing it).

    Returns (out [R, H_q, d_v], idx [n_units, R, top_k], gap [n_units, R]).

    Transcript #94, §4, Figure 2: the three branch outputs are each multiplied
    by a per-token gate and summed; MoBA (§7) keeps the selected branch only.
    """
    get = (lambda name: cfg[name]) if isinstance(cfg, dict) else (lambda name: getattr(cfg, name))
    h_q, h_kv = get("h_q"), get("h_kv")
    sel_block, top_k, window = get("sel_block"), get("top_k"), get("window")
    cmp_block, cmp_stride = get("cmp_block"), get("cmp_stride")
    scale, branches, per_head = get("scale"), get("branches"), bool(get("per_head_select"))
    R = q_rows.shape[0]
    T_kv = K.shape[1]
    d_v = V.shape[2]
    positions = np.asarray(positions, dtype=np.int64)
    units = selection_units(h_q, h_kv, per_head)
    n_blocks = -(-T_kv // sel_block)

    if pooled is None:
        need_cmp = branches & 1 or opt(cfg, "score_mode", "dot") == "cmp"
        pooled = pooled_inputs(K, V, sel_block, cmp_block if need_cmp else 0,
                               cmp_stride if need_cmp else 1)
    gap = np.full((len(units), R), np.inf)
    if branches & 2:
        if idx is None:
            s = selection_scores(cfg, q_rows, positions, pooled, n_blocks)
            idx, gap = select_blocks(s, positions, sel_block, top_k, opt(cfg, "sink_blocks", 0))
    if branches & 1:
        Kc, Vc = pooled["Kc"], pooled["Vc"]
        n_cmp = Kc.shape[1]

    out = np.zeros((R, h_q, d_v))
    for r in range(R):
        t = int(positions[r])
        for u, (hk, heads) in enumerate(units):
            q = q_rows[r, heads, :]
            weight = (lambda br: gates_rows[r, heads, br][:, None]) if gates_rows is not None \
                else (lambda br: 1.0)
            if branches & 1:
                js = compressed_keys(t, n_cmp, cmp_block, cmp_stride)
                out[r, heads] += weight(0) * softmax_attention(q, Kc[hk, js], Vc[hk, js], scale)
            if branches & 2:
                ks = selected_keys(idx[u, r], t, sel_block)
                out[r, heads] += weight(1) * softmax_attention(q, K[hk, ks], V[hk, ks], scale)
            if branches & 4:
                ks = window_keys(t, window)
                out[r, heads] += weight(2) * softmax_attention(q, K[hk, ks], V[hk, ks], scale)
    return out, idx, gap


# ---------------------------------------------------------------------------
# Backward pass
# ---------------------------------------------------------------------------

def softmax_attention_grad(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                           d_o: np.ndarray):
    """Gradients of o = softmax(scale * q k^T) v with respect to q, k and v.

    Transcript #94, §2: the output is the softmax-weighted sum of the values.
    The chain rule through it, with P the weights and dO the output gradient:
    dV = P^T dO; dP = dO V^T; dS = P * (dP - rowsum(dP * P)) (the softmax
    Jacobian); dq = scale * dS k; dk = scale * dS^T q.  q [n, d], k [m, d],
    v [m, dv], d_o [n, dv]; no keys: zero gradients.
    """
    if k.shape[0] == 0:
        return np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    logits = scale * (q @ k.T)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    dv = p.T @ d_o
    dp = d_o @ v.T
    ds = p * (dp - (dp * p).sum(axis=1, keepdims=True))
    return scale * (ds @ k), scale * (ds.T @ q), dv


def nsa_rows_backward(cfg, q_rows, positions, K, V, gates_rows, idx, d_out):
    """Gradients of the gated output of ``nsa_rows`` for fixed selected blocks.

    The top-k choice is discrete and passes no gradient (transcript #94, §6:
    the compressed branch is what carries gradient to the block
    representations), so ``idx`` [n_units, R, top_k] is an input.  The
    compressed tokens are means of K/V windows (§4, Figure 2; mean pooling,
    §7), so their gradients reach every token of the window with weight
    1 / cmp_block.  Returns (dq [R, H_q, d_qk], dK [H_kv, T_kv, d_qk],
    dV [H_kv, T_kv, d_v], dg [R, H_q, 3] or None) for the loss
    sum(d_out * out), d_out [R, H_q, d_v].
    """
    get = (lambda name: cfg[name]) if isinstance(cfg, dict) else (lambda name: getattr(cfg, name))
    h_q, h_kv = get("h_q"), get("h_kv")
    sel_block, window = get("sel_block"), get("window")
    cmp_block, cmp_stride = get("cmp_block"), get("cmp_stride")
    scale, branches, per_head = get("scale"), get("branches"), bool(get("per_head_select"))
    positions = np.asarray(positions, dtype=np.int64)
    units = selection_units(h_q, h_kv, per_head)
    R = q_rows.shape[0]
    dq = np.zeros_like(q_rows)
    dK = np.zeros_like(K)
    dV = np.zeros_like(V)
    dg = None if gates_rows is None else np.zeros((R, h_q, 3))
    if branches & 1:
        Kc, Vc = compress(K, cmp_block, cmp_stride), compress(V, cmp_block, cmp_stride)
        dKc, dVc = np.zeros_like(Kc), np.zeros_like(Vc)
        n_cmp = Kc.shape[1]
    for r in range(R):
        t = int(positions[r])
        for u, (hk, heads) in enumerate(units):
            q = q_rows[r, heads, :]
            for br in (0, 1, 2):
                if not branches & (1 << br):
                    continue
                if br == 0:
                    js = compressed_keys(t, n_cmp, cmp_block, cmp_stride)
                    kk, vv = Kc[hk, js], Vc[hk, js]
                else:
                    ks = selected_keys(idx[u, r], t, sel_block) if br == 1 else window_keys(t, window)
                    kk, vv = K[hk, ks], V[hk, ks]
                g = gates_rows[r, heads, br] if gates_rows is not None else np.ones(len(heads))
                if dg is not None:
                    dg[r, heads, br] = (d_out[r, heads] * softmax_attention(q, kk, vv, scale)).sum(axis=1)
                gq, gk, gv = softmax_attention_grad(q, kk, vv, scale, g[:, None] * d_out[r, heads])
                dq[r, heads] += gq
                if br == 0:
                    dKc[hk, js] += gk
                    dVc[hk, js] += gv
                else:
                    np.add.at(dK[hk], ks, gk)
                    np.add.at(dV[hk], ks, gv)
    if branches & 1:
        for j in range(n_cmp):
            dK[:, j * cmp_stride:j * cmp_stride + cmp_block] += dKc[:, j:j + 1] / cmp_block
            dV[:, j * cmp_stride:j * cmp_stride + cmp_block] += dVc[:, j:j + 1] / cmp_block
    return dq, dK, dV, dg
