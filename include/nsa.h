/*
 * nsa.h - C ABI of libnsa_b200.so: query-dependent top-k block-sparse causal
 * attention forward (NSA-style group-shared selection, MoBA-style per-head
 * selection) for NVIDIA B200 (sm_100a).
 *
 * Method, as described in the Zhang Xiaojun #94 transcript (bidclub.ai):
 *   §2 "Attention From First Principles" - scaled dot products, causal mask,
 *      softmax, weighted sum of values;
 *   §4 "Inside Native Sparse Attention", Figure 2 - KV cut into contiguous
 *      blocks; a compressed branch over pooled block tokens, a selected branch
 *      over the top-k scoring blocks, a sliding-window branch, each multiplied
 *      by a per-token gate and summed; GQA heads add their block scores so the
 *      group shares one block set;
 *   §7 "Kimi Simplifies The Sparse Route" - MoBA: mean-pooled block keys,
 *      per-head selection, selected branch only;
 * and LateTalk #103 (zjai.club) §13 - the block holding the query is always
 * selected.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Tensors are dense, row-major, caller-owned DEVICE memory (16-byte aligned).
 *   q      [B, Tq, Hq, d_qk]        bf16   head h belongs to KV head h / (Hq/Hkv)
 *   k      [B, Hkv, Tkv, d_qk]      bf16
 *   v      [B, Hkv, Tkv, d_v]       bf16
 *   kbar   [B, Hkv, nb_full, d_qk]  fp32   nb_full = Tkv / sel_block (complete blocks)
 *   kcmp   [B, Hkv, n_cmp, d_qk]    bf16   n_cmp = (Tkv - cmp_block) / cmp_stride + 1
 *   vcmp   [B, Hkv, n_cmp, d_v]     bf16
 *   scores [B, Hsel, Tq, nb_all]    fp32   nb_all = ceil(Tkv / sel_block)
 *   idx    [B, Hsel, Tq, top_k]     int32  ascending block ids, -1 padded
 *   gates  [B, Tq, Hq, 3]           fp32   (compressed, selected, window)
 *   out    [B, Tq, Hq, d_v]         bf16
 * Hsel = Hkv (group-shared selection) or Hq (NSA_PER_HEAD_SELECT).
 * Query i of a sequence sits at KV position t = q_pos0 + i (prefill: q_pos0 = 0
 * and Tq = Tkv; decode: Tq = 1, q_pos0 = Tkv - 1).  Its current block is
 * c = t / sel_block.
 *
 * `stream` is a cudaStream_t (NULL = legacy default stream).  Every entry
 * point validates its arguments on the host before launching anything and
 * returns NSA_ERR_INVALID_ARG / NSA_ERR_UNSUPPORTED without side effects;
 * launch failures return NSA_ERR_CUDA.  Work is enqueued asynchronously on
 * `stream`: no entry point synchronises, allocates device memory or keeps a
 * pointer after it returns.  Calls are thread-safe; two calls that write the
 * same buffers must be ordered by the caller.
 *
 * GPU-path limits (NSA_ERR_UNSUPPORTED otherwise): d_qk in {64, 128, 192, 256},
 * d_v in {64, 128, 256}; sel_block a multiple of 16; 1 <= top_k <= 32;
 * cmp_block a multiple of cmp_stride; Hq a multiple of Hkv, Hq/Hkv <= 16 for
 * group-shared selection.
 */
#ifndef NSA_B200_NSA_H
#define NSA_B200_NSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NSA_OK = 0,
    NSA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer */
    NSA_ERR_UNSUPPORTED = 2,   /* valid problem outside the GPU path's limits */
    NSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than nsa_workspace_size() */
    NSA_ERR_CUDA = 4,          /* a CUDA launch or driver call failed */
    NSA_ERR_TIMEOUT = 5        /* a device-side bounded wait gave up */
} nsa_status;

/* Branch and mode bits of nsa_config.flags. */
#define NSA_BR_CMP 1u            /* compressed (coarse) branch */
#define NSA_BR_SEL 2u            /* selected-block branch */
#define NSA_BR_WIN 4u            /* sliding-window branch */
#define NSA_PER_HEAD_SELECT 8u   /* MoBA: every query head selects its own blocks */
/* Selection-score variants (default: the scaled dot product with the pooled
 * block key, summed over the unit's heads).  At most one of the two. */
#define NSA_SCORE_PROB 16u       /* per head, softmax of the block scores over the row's
                                    candidates; the unit sums its heads' probabilities */
#define NSA_SCORE_CMP 32u        /* per head, the compressed branch's softmax weights over the
                                    visible compressed tokens, gathered to each selection
                                    block by the share of the token's window inside it; the
                                    unit sums its heads (needs NSA_BR_CMP) */
/* Debug mode: nsa_sparse_attn_fwd validates a caller-supplied idx before any
 * attention kernel reads it (see there). */
#define NSA_DEBUG_CHECKS 64u
/* Forced leading blocks ("attention sink"): blocks 0 .. n-1 before the
 * query's own block are always kept, like the own block; n <= top_k - 1. */
#define NSA_SINK_SHIFT 16
#define NSA_SINK_BLOCKS(n) ((uint32_t)(n) << NSA_SINK_SHIFT)

typedef struct {
    int32_t batch;       /* B: independent sequences */
    int32_t seqlen_q;    /* Tq: queries per sequence */
    int32_t seqlen_kv;   /* Tkv: keys/values per sequence */
    int32_t q_pos0;      /* KV position of query 0; q_pos0 + Tq <= Tkv */
    int32_t h_q;         /* Hq: query heads */
    int32_t h_kv;        /* Hkv: key/value heads */
    int32_t d_qk;        /* query/key head dimension */
    int32_t d_v;         /* value head dimension */
    int32_t sel_block;   /* tokens per selection block */
    int32_t top_k;       /* blocks kept per query, the current block included */
    int32_t window;      /* sliding window: keys [t - window + 1, t] */
    int32_t cmp_block;   /* tokens per compressed token */
    int32_t cmp_stride;  /* distance between compressed tokens */
    float scale;         /* logit scale, normally 1/sqrt(d_qk) */
    uint32_t flags;      /* NSA_BR_* | NSA_PER_HEAD_SELECT | NSA_SCORE_* | NSA_SINK_BLOCKS(n) */
} nsa_config;

/*
 * Bytes of device workspace for nsa_sparse_attn_fwd's fastest path on `cfg`:
 * the selected block ids (when it selects them itself) plus, for long
 * prefills on the tensor-core path, the per-block query lists and the
 * per-(query, slot) partial outputs of the block-major selected branch
 * (about topk * heads * d_v * 2 bytes per query; with the selected branch
 * alone and one head per selection unit, a slot per 64-key sub-block of a
 * kept block, i.e. sel_block / 64 times as many).  Writes 0 when no
 * workspace is needed.  Pure host function.
 */
nsa_status nsa_workspace_size(const nsa_config* cfg, size_t* bytes);

/*
 * Smallest workspace nsa_sparse_attn_fwd accepts with idx == NULL: the
 * selected block ids only.  With a workspace smaller than
 * nsa_workspace_size() the selected branch runs inside the query-major
 * kernel instead (same result, slower for long prefills).  Pure host function.
 */
nsa_status nsa_workspace_size_min(const nsa_config* cfg, size_t* bytes);

/*
 * Block representations (transcript #94 §4 Figure 2 "compression", §7 mean
 * pooling).  kbar[b,h,j,:] = mean of k over tokens [j*sel_block, (j+1)*sel_block)
 * for every complete block (fp32).  When NSA_BR_CMP is set, kcmp/vcmp[b,h,j,:]
 * = mean of k/v over [j*cmp_stride, j*cmp_stride + cmp_block), rounded to bf16;
 * otherwise kcmp and vcmp may be NULL.  kbar may be NULL when NSA_BR_SEL is
 * clear.  Reads k and v once.
 */
nsa_status nsa_pool_kv(const nsa_config* cfg, const void* k, const void* v, float* kbar,
                       void* kcmp, void* vcmp, void* stream);

/*
 * Incremental cache update for decoding (transcript #94 §6 "Why Sparse
 * Attention Wins": decoding is memory-bound and costs the KV bytes it reads,
 * so a step must not re-read the whole cache to refresh its pooled tokens).
 *
 * The cache has room for cfg->seqlen_kv tokens per (sequence, KV head); the
 * call appends cfg->seqlen_q new tokens per sequence at KV positions
 * [q_pos0, q_pos0 + seqlen_q):
 *   k_new [B, Hkv, seqlen_q, d_qk] bf16, v_new [B, Hkv, seqlen_q, d_v] bf16
 * are copied into k and v (layouts as above), then every pooled token that the
 * new rows complete is recomputed from the cache:
 *   kbar[j] for each selection block with j*sel_block + sel_block - 1 in the
 *   new range (NSA_BR_SEL), and kcmp/vcmp[j] for each compressed token with
 *   j*cmp_stride + cmp_block - 1 in it (NSA_BR_CMP),
 * with the same arithmetic as nsa_pool_kv, so after appending tokens one call
 * at a time the pooled tensors equal nsa_pool_kv of the filled cache bit for
 * bit.  Nothing else is read or written.  A decode step then calls
 * nsa_topk_select / nsa_sparse_attn_fwd with seqlen_kv = the cache size and
 * q_pos0 = the newest position: every branch is causal, so cache rows after
 * the query are never attended, but they must hold finite values (e.g.
 * zeros), because masked keys still enter the value products with weight 0;
 * the same holds for the compressed tokens not yet complete (zero kcmp and
 * vcmp once when the cache is created).  kbar / kcmp / vcmp may be NULL when
 * the call completes none of their tokens.
 */
nsa_status nsa_append_kv(const nsa_config* cfg, void* k, void* v, const void* k_new,
                         const void* v_new, float* kbar, void* kcmp, void* vcmp, void* stream);

/*
 * Block selection scores (transcript #94 §4: one score per query and block;
 * group heads add theirs).  scores[b,u,i,j] =
 *   scale * sum_{h in unit u} q[b,i,h,:] . kbar[b,kv(u),j,:]   for j < c(t),
 *   +INFINITY for j == c(t) (always selected), -INFINITY for j > c(t).
 * Computed in fp32 as scale * (sum_h q_h) . kbar_j (the sum is linear).
 */
nsa_status nsa_score_blocks(const nsa_config* cfg, const void* q, const float* kbar,
                            float* scores, void* stream);

/*
 * nsa_score_blocks for every score kind: kcmp [B, Hkv, n_cmp, d_qk] is read
 * by NSA_SCORE_CMP (kbar may then be NULL); the other kinds read kbar (kcmp
 * may be NULL).  Variant scores (NSA_SCORE_PROB, NSA_SCORE_CMP):
 *   PROB: sum over the unit's heads h of softmax_b(scale * q_h . kbar_b),
 *         the softmax over the row's candidates b < c(t);
 *   CMP:  sum over h and visible compressed tokens j (j*cmp_stride +
 *         cmp_block - 1 <= t) of softmax_j(scale * q_h . kcmp_j) * w(j, b),
 *         w(j, b) = |[j*cmp_stride, j*cmp_stride + cmp_block) ∩ block b| / cmp_block
 * (transcript #94 §4: the normalised score of §2; the "corner case" of
 * selection blocks cut differently from the compressed tokens), computed in
 * fp32.  Forced leading blocks (NSA_SINK_BLOCKS) score +INFINITY like the
 * own block, in every kind.  Limits: <= 16 heads per unit, <= 16384 blocks
 * and compressed tokens (NSA_ERR_UNSUPPORTED otherwise).
 */
nsa_status nsa_score_blocks_ex(const nsa_config* cfg, const void* q, const float* kbar,
                               const void* kcmp, float* scores, void* stream);

/*
 * Top-k block sets (transcript #94 §4 Figure 2: keep the k best blocks;
 * LateTalk #103 §13: the current block is always kept).  For every (b, u, i):
 * idx = {c(t)} plus the (top_k - 1) best past blocks by score, equal scores
 * resolved to the lower block index; written ascending and padded with -1 to
 * top_k entries (a row keeps min(top_k, c(t) + 1) blocks).  If `scores` is
 * NULL the scores are computed on the fly from q and kbar (fused, nothing
 * materialised); otherwise they are read from `scores` (layout above) and q,
 * kbar may be NULL.
 */
nsa_status nsa_topk_select(const nsa_config* cfg, const void* q, const float* kbar,
                           const float* scores, int32_t* idx, void* stream);

/*
 * nsa_topk_select for every score kind (kcmp as in nsa_score_blocks_ex).
 * With NSA_SINK_BLOCKS(n) the first n blocks before the own block are kept
 * and the remaining top_k - 1 - n places go to the best other past blocks.
 * With `scores` given, forced blocks are kept whatever their entries hold.
 */
nsa_status nsa_topk_select_ex(const nsa_config* cfg, const void* q, const float* kbar,
                              const void* kcmp, const float* scores, int32_t* idx, void* stream);

/*
 * Gated sparse attention forward (transcript #94 §4 Figure 2).  For each
 * query row (position t) and head h:
 *   o_cmp = softmax attention over compressed tokens j with
 *           j*cmp_stride + cmp_block - 1 <= t           (NSA_BR_CMP)
 *   o_sel = softmax attention over the tokens u <= t of the blocks in idx (NSA_BR_SEL)
 *   o_win = softmax attention over keys max(0, t-window+1) .. t           (NSA_BR_WIN)
 *   out   = g0*o_cmp + g1*o_sel + g2*o_win   (gates NULL: weight 1 each)
 * A branch with no visible key contributes 0.  Precision: bf16 inputs; scores,
 * softmax and accumulation in fp32; out rounded to bf16.  On the query-major,
 * split-k and decode plans (nsa_attn_plan) that is the only rounding.  The
 * block-major plan keeps each kept block's partial result o = (P V) / l in
 * bf16 (one rounding per (query, head, block), relative error <= 2^-9),
 * merges a query's partials in fp32 and, when other branches follow, hands
 * the merged o_sel to the query-major kernel in bf16 (a second rounding of
 * the selected branch) before the gated sum is rounded once more; with the
 * selected branch alone the merge writes g_sel * o_sel to out directly.  The
 * extra roundings add at most about 2 * 2^-9 * g_sel * max|o_sel| to an
 * output element (measured on the 64k workload: see the parity tests).
 * idx may be NULL, in which case the blocks are selected as nsa_topk_select
 * does (needs q, kbar and at least nsa_workspace_size_min() bytes of
 * workspace; with nsa_workspace_size() bytes and more than 16 query rows the
 * scores run on the tensor cores, three tf32 products per pair), and the
 * selected ids are left in the first B*Hsel*Tq*top_k int32 of the workspace,
 * laid out like idx; otherwise kbar may be NULL.  A workspace of
 * nsa_workspace_size() bytes enables the block-major selected branch (each
 * selected KV block attended once for all the queries that kept it); a
 * smaller one (or NULL with an external idx) computes the same result with
 * the selected branch inside the query-major kernel.  With the selected
 * branch alone and one head per selection unit (MoBA's per-head selection,
 * transcript #94 §7), at least 256 query rows, sel_block a multiple of 64
 * and top_k * sel_block / 64 <= 32, the full workspace runs the block-major
 * kernel over the 64-key sub-blocks of the kept blocks and writes out from
 * their merge directly.
 * kcmp/vcmp are read only with NSA_BR_CMP.
 * A caller-supplied idx must hold, per row, block ids in [0, c(t)] (and
 * below nb_all), strictly ascending, then -1 padding, the own block c(t)
 * included.  These rules are trusted, not checked, unless cfg->flags has
 * NSA_DEBUG_CHECKS: then a read-only kernel checks every row first, the call
 * synchronises its stream, and a row that breaks them makes the call return
 * NSA_ERR_INVALID_ARG with nothing else launched (out untouched).
 */
nsa_status nsa_sparse_attn_fwd(const nsa_config* cfg, const void* q, const void* k,
                               const void* v, const float* kbar, const void* kcmp,
                               const void* vcmp, const float* gates, const int32_t* idx,
                               void* out, void* workspace, size_t ws_bytes, void* stream);

/*
 * Same result as nsa_sparse_attn_fwd with idx == NULL (blocks selected
 * inside), but it allocates nothing and takes no workspace: the block ids live
 * in a 32 MiB array inside the library (a file-scope __device__ array that
 * every GPU loading the library keeps until the process exits).  The pages
 * describe no counterpart; this exists for callers that may not allocate
 * device memory - plugin hosts whose execute call must not allocate because
 * the host framework owns all device buffers, and latency-critical callers for
 * which cudaMalloc/cudaFree are off limits because they can synchronise the
 * device.
 * Limit: problems with nsa_workspace_size_min() > 32 MiB return NSA_ERR_WORKSPACE
 * (e.g. 65536 queries x 4 selection units x top-16 need 16 MiB).
 * Every call looks up the array's device address on the current device (a
 * host-side lookup, nothing cached) and passes the array as a workspace of
 * 32 MiB, so it holds whatever scratch the plan for that size uses (the block
 * ids, plus the plan's lists and partials when the full workspace fits).
 * Every call uses the same array, which keeps the previous call's contents
 * (nothing in it needs to start at zero); calls whose GPU work overlaps race
 * on it, so order them (e.g. one stream).
 */
nsa_status nsa_sparse_attn_fwd_noalloc(const nsa_config* cfg, const void* q, const void* k,
                                       const void* v, const float* kbar, const void* kcmp,
                                       const void* vcmp, const float* gates, void* out,
                                       void* stream);

/*
 * Backward pass for fixed block sets (transcript #94 §6: the top-k choice is
 * discrete and passes no gradient, the compressed branch carries gradient to
 * the keys and values it pools; §2: each branch is a softmax-weighted sum).
 * For the loss sum(d_out * out), with out as nsa_sparse_attn_fwd computes it
 * from the same q, k, v, kcmp, vcmp, gates and the blocks in idx:
 *   dq     [B, Tq, Hq, d_qk]  fp32, overwritten
 *   dk, dv [B, Hkv, Tkv, d]   fp32, overwritten (every key's gradient, summed
 *                             over queries and heads; a compressed token's
 *                             gradient reaches each token of its window
 *                             divided by cmp_block)
 *   dgates [B, Tq, Hq, 3]     fp32, d_out . o_branch (NULL when gates is NULL)
 * d_out [B, Tq, Hq, d_v] bf16; idx as returned by the selection (required
 * with NSA_BR_SEL); kcmp/vcmp as nsa_pool_kv writes them (with NSA_BR_CMP).
 * Needs nsa_bwd_workspace_size() bytes of workspace (the compressed tokens'
 * gradients).  Plain fp32 CUDA-core arithmetic with atomic accumulation of
 * dk / dv (summation order varies between runs).  Limits: d_qk, d_v <= 256,
 * <= 16 heads per selection unit, top_k <= 32 (NSA_ERR_UNSUPPORTED otherwise).
 */
nsa_status nsa_bwd_workspace_size(const nsa_config* cfg, size_t* bytes);
nsa_status nsa_sparse_attn_bwd(const nsa_config* cfg, const void* q, const void* k,
                               const void* v, const void* kcmp, const void* vcmp,
                               const float* gates, const int32_t* idx, const void* d_out,
                               float* dq, float* dk, float* dv, float* dgates,
                               void* workspace, size_t ws_bytes, void* stream);

/*
 * Reads and clears the device-side status word of the tensor-core kernels:
 * NSA_OK, or NSA_ERR_TIMEOUT when a bounded wait inside a kernel gave up (the
 * kernel then unwound without finishing its output).  Synchronous: waits for
 * all work on the current device first.  Not for use inside stream capture.
 */
nsa_status nsa_get_device_status(int32_t* status);

/*
 * Self-test of the device-side failure path (the pages have no counterpart):
 * one warp runs the tensor-core kernels' bounded wait on a barrier that
 * nothing ever completes, gives up after limit_ns (1 .. 1e9 ns) and records
 * NSA_ERR_TIMEOUT in the same status word, which nsa_get_device_status then
 * returns.  The GPU context stays usable.  Asynchronous on `stream`.
 */
nsa_status nsa_check_bounded_wait(uint64_t limit_ns, void* stream);

/*
 * Test and debug knob (the pages have no counterpart): the limit, in ns, of
 * every bounded wait of the tensor-core attention kernel launched after this
 * call (the kernel behind nsa_sparse_attn_fwd's query-major, block-major and
 * split-K plans); 0 restores the default of one second, values above 1e9 are
 * refused.  With a limit shorter than the copies and MMAs take, the kernel's
 * waits give up: it raises NSA_ERR_TIMEOUT in the status word, every role
 * unwinds (the two warps that share rows leave their barriers together) and
 * the context stays usable.  The waits that drain in-flight copies and MMAs
 * before the kernel frees its tensor memory keep one second.  Synchronous;
 * not for use while another thread launches this library's kernels.
 */
nsa_status nsa_set_wait_limit_ns(uint64_t limit_ns);

/* Organisations of nsa_sparse_attn_fwd (same results, different speed). */
#define NSA_PATH_ROWWISE 0       /* shapes outside the tensor-core kernels' limits */
#define NSA_PATH_QUERY_MAJOR 1   /* tensor cores; selected branch over each tile's block union */
#define NSA_PATH_BLOCK_MAJOR 2   /* + selected branch block-major (long prefills, full workspace;
                                    the selected branch alone with one head per unit: 64-key
                                    sub-blocks, no query-major kernel) */
#define NSA_PATH_SPLIT_K 3       /* + each tile's keys split over several CTAs (few tiles) */
#define NSA_PATH_DECODE 4        /* tensor cores with the keys as the MMA M dimension: <= 4 query
                                    rows per sequence, 8 or 16 heads per group, d_v 128, full workspace */

/*
 * The organisation nsa_sparse_attn_fwd picks for `cfg` with a workspace of
 * `ws_bytes` bytes, and the number of kernels it launches (select_inside != 0:
 * idx == NULL, the selection kernel included).  Pure host function.
 */
nsa_status nsa_attn_plan(const nsa_config* cfg, int select_inside, size_t ws_bytes,
                         int32_t* path, int32_t* kernels);

/*
 * Stage timing, a measurement aid (the pages have no counterpart).
 *
 * nsa_timing_enable(1) makes the calling host thread's later
 * nsa_sparse_attn_fwd calls record a CUDA event on the call's stream before
 * each stage and one after the last.  The events (NSA_TIMING_MAX_STAGES + 1
 * per host thread) are created with cudaEventCreate on first use, on the
 * device current then; calls made while another device is current record
 * nothing.  No device memory is allocated.  nsa_timing_enable(0) stops the
 * recording (the events are kept).
 *
 * nsa_timing_read waits for the last event of the thread's most recent timed
 * call and writes up to `max_stages` stage names (static strings) and
 * durations in milliseconds; *n_stages receives the number of stages (0 if
 * no call was timed).  Stage names: "select" (score + top-k when idx is
 * NULL), "expand" (kept blocks to 64-key sub-blocks), "index" (block-major
 * inverted index), "sel_bm" (block-major selected
 * branch), "sel_merge", "attn_tc" (tensor-core branches + gated merge),
 * "split_merge", "attn_dec" (few-query kernel), "dec_merge", "rowwise".
 * Each stage's time runs from its first launch to the next stage's first
 * launch on the same stream.
 */
#define NSA_TIMING_MAX_STAGES 8
nsa_status nsa_timing_enable(int32_t on);
nsa_status nsa_timing_read(int32_t max_stages, float* ms, const char** names, int32_t* n_stages);

/* CUDA's description of the error behind the calling thread's most recent
 * NSA_ERR_CUDA (a static string; "no error" if there was none). */
const char* nsa_last_cuda_error(void);

/* Static, human-readable name of a status code. */
const char* nsa_status_string(nsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* NSA_B200_NSA_H */
