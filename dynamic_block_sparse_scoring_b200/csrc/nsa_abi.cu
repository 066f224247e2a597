// C ABI of libnsa_b200: host-side validation and kernel launches.
//
// Every entry point checks its arguments before anything is enqueued and
// returns a status code; no C++ exception crosses the boundary, nothing is
// allocated and nothing synchronises.  The operations themselves are defined
// in include/nsa.h.
#include <math.h>
#include <stdint.h>

#include <algorithm>

#include <nvtx3/nvToolsExt.h>
#include "common.cuh"
#include "sel_index.cuh"

namespace {

using nsa::Shape;

bool aligned16(const void* p) { return p == nullptr || (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool supported_dqk(int d) { return d == 64 || d == 128 || d == 192 || d == 256; }
bool supported_dv(int d) { return d == 64 || d == 128 || d == 256; }

// Validates `cfg` and fills the derived sizes.
nsa_status make_shape(const nsa_config* cfg, Shape* s) {
    if (!cfg || !s) return NSA_ERR_INVALID_ARG;
    const nsa_config& c = *cfg;
    const uint32_t known = NSA_BR_CMP | NSA_BR_SEL | NSA_BR_WIN | NSA_PER_HEAD_SELECT | NSA_SCORE_PROB |
                           NSA_SCORE_CMP | NSA_DEBUG_CHECKS | (0xFFu << NSA_SINK_SHIFT);
    if (c.flags & ~known) return NSA_ERR_INVALID_ARG;
    if ((c.flags & NSA_SCORE_PROB) && (c.flags & NSA_SCORE_CMP)) return NSA_ERR_INVALID_ARG;
    // scores from the compressed branch need its compressed tokens
    if ((c.flags & NSA_SCORE_CMP) && !(c.flags & NSA_BR_CMP)) return NSA_ERR_INVALID_ARG;
    const int n_sink = (int)((c.flags >> NSA_SINK_SHIFT) & 0xFFu);
    if (n_sink > 0 && (!(c.flags & NSA_BR_SEL) || n_sink > c.top_k - 1)) return NSA_ERR_INVALID_ARG;
    if (!(c.flags & (NSA_BR_CMP | NSA_BR_SEL | NSA_BR_WIN))) return NSA_ERR_INVALID_ARG;
    if (c.batch < 1 || c.seqlen_q < 0 || c.seqlen_kv < 1 || c.q_pos0 < 0) return NSA_ERR_INVALID_ARG;
    if ((int64_t)c.q_pos0 + c.seqlen_q > c.seqlen_kv) return NSA_ERR_INVALID_ARG;
    if (c.h_q < 1 || c.h_kv < 1 || c.h_q % c.h_kv != 0) return NSA_ERR_INVALID_ARG;
    if (c.d_qk < 1 || c.d_v < 1) return NSA_ERR_INVALID_ARG;
    if (!isfinite(c.scale)) return NSA_ERR_INVALID_ARG;
    if (c.sel_block < 1) return NSA_ERR_INVALID_ARG;
    if ((c.flags & NSA_BR_SEL) && c.top_k < 1) return NSA_ERR_INVALID_ARG;
    if ((c.flags & NSA_BR_WIN) && c.window < 1) return NSA_ERR_INVALID_ARG;
    if ((c.flags & NSA_BR_CMP) && (c.cmp_block < 1 || c.cmp_stride < 1)) return NSA_ERR_INVALID_ARG;

    if (!supported_dqk(c.d_qk) || !supported_dv(c.d_v)) return NSA_ERR_UNSUPPORTED;
    if (c.sel_block % 16 != 0) return NSA_ERR_UNSUPPORTED;
    if ((c.flags & NSA_BR_SEL) && c.top_k > 32) return NSA_ERR_UNSUPPORTED;
    if (c.flags & NSA_BR_CMP) {
        if (c.cmp_block % c.cmp_stride != 0 || c.cmp_block / c.cmp_stride > 16)
            return NSA_ERR_UNSUPPORTED;
    }
    const int G = c.h_q / c.h_kv;
    const bool per_head = (c.flags & NSA_PER_HEAD_SELECT) != 0;
    if (!per_head && G > 16) return NSA_ERR_UNSUPPORTED;

    s->B = c.batch;
    s->Tq = c.seqlen_q;
    s->Tk = c.seqlen_kv;
    s->q0 = c.q_pos0;
    s->Hq = c.h_q;
    s->Hkv = c.h_kv;
    s->G = G;
    s->dqk = c.d_qk;
    s->dv = c.d_v;
    s->bs = c.sel_block;
    s->topk = (c.flags & NSA_BR_SEL) ? c.top_k : 1;
    s->win = c.window;
    s->lc = (c.flags & NSA_BR_CMP) ? c.cmp_block : 1;
    s->sc = (c.flags & NSA_BR_CMP) ? c.cmp_stride : 1;
    s->nb_full = c.seqlen_kv / c.sel_block;
    s->nb_all = (c.seqlen_kv + c.sel_block - 1) / c.sel_block;
    s->n_cmp = (c.flags & NSA_BR_CMP) && c.seqlen_kv >= c.cmp_block
                   ? (c.seqlen_kv - c.cmp_block) / c.cmp_stride + 1
                   : 0;
    s->per_head = per_head;
    s->Hsel = per_head ? c.h_q : c.h_kv;
    s->heads_per_unit = per_head ? 1 : G;
    s->scale = c.scale;
    s->flags = c.flags;
    s->n_sink = n_sink;
    s->score_mode = (c.flags & NSA_SCORE_PROB) ? 1 : ((c.flags & NSA_SCORE_CMP) ? 2 : 0);
    if (s->score_mode != 0 && !nsa::score_variant_supported(*s)) return NSA_ERR_UNSUPPORTED;
    return NSA_OK;
}

size_t idx_bytes(const Shape& s) {
    return (size_t)s.B * s.Hsel * s.Tq * s.topk * sizeof(int32_t);
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The selected branch runs block-major (inverted index + partials) for long
// prefills on the tensor-core path; decode and short chunks keep it inside
// the query-major kernel.
bool use_block_major(const Shape& s) {
    return (s.flags & NSA_BR_SEL) && nsa::attn_tc_supported(s) && nsa::sel_bm_supported(s) &&
           s.Tq >= 256;
}

// The selected branch alone with one head per unit (MoBA's per-head
// selection, blocks of any multiple of 64 keys): every kept block is cut into
// its 64-key sub-blocks and the block-major kernel runs over those, the merge
// writing out directly.  This is the problem restated with 64-key blocks and
// top_k * (sel_block / 64) slots.
Shape sub_block_shape(const Shape& s) {
    Shape t = s;
    t.topk = s.topk * (s.bs / 64);
    t.bs = 64;
    t.nb_full = s.Tk / 64;
    t.nb_all = (s.Tk + 63) / 64;
    return t;
}

bool use_sub_block_major(const Shape& s) {
    if (!(s.flags & NSA_BR_SEL) || (s.flags & (NSA_BR_CMP | NSA_BR_WIN))) return false;
    if (s.heads_per_unit != 1 || s.bs % 64 != 0 || s.Tq < 256) return false;
    if (s.topk * (s.bs / 64) > nsa::SEL_SLOTS) return false;
    return nsa::sel_bm_supported(sub_block_shape(s));
}

// Selection inside nsa_sparse_attn_fwd on the tensor cores: prefill-sized
// problems (the few-row kernel serves <= 16 rows).
bool use_score_tc(const Shape& s) { return s.score_mode == 0 && nsa::score_tc_supported(s) && s.Tq > 16; }

// Few query rows per sequence (decode): keys as the MMA M dimension.
bool use_decode(const Shape& s) { return nsa::attn_dec_supported(s); }

// Workspace regions, each 256-byte aligned, in this order.
struct WsLayout {
    size_t idx = 0, idx_sub = 0, cnt = 0, off = 0, item_off = 0, cursor = 0, list = 0, items = 0, part_o = 0,
           part_lse = 0, o_sel = 0, split_o = 0, split_lse = 0, dec_o = 0, dec_lse = 0, sc_qh = 0,
           sc_ql = 0, sc_kh = 0, sc_kl = 0, total = 0, minimal = 0;
    bool sc = false;    // the selection inside the call runs on the tensor cores
    bool sub = false;   // block-major over 64-key sub-blocks (selected branch alone)
    int n_split = 1;
};

WsLayout ws_layout(const Shape& s) {
    WsLayout w;
    size_t at = 0;
    auto take = [&](size_t bytes) {
        const size_t o = at;
        at = round_up(at + bytes, 256);
        return o;
    };
    if (s.flags & NSA_BR_SEL) w.idx = take(idx_bytes(s));
    w.minimal = at;
    // split operands of the tensor-core selection (prefill)
    if (use_score_tc(s)) {
        w.sc = true;
        w.sc_qh = take(nsa::score_tc_q_floats(s) * 4);
        w.sc_ql = take(nsa::score_tc_q_floats(s) * 4);
        w.sc_kh = take(nsa::score_tc_k_floats(s) * 4);
        w.sc_kl = take(nsa::score_tc_k_floats(s) * 4);
    }
    // split-K partials for problems with few work tiles (decode)
    if (use_decode(s)) {
        const size_t items = nsa::attn_dec_items(s);
        w.dec_o = take(items * nsa::attn_dec_part_floats() * 4);
        w.dec_lse = take(items * 16 * 4);
    } else if (nsa::attn_tc_supported(s) && !use_block_major(s)) {
        w.n_split = nsa::attn_tc_split_count(s);
        if (w.n_split > 1) {
            const size_t rows = (size_t)s.B * s.Tq * s.Hq * 3 * w.n_split;
            w.split_o = take(rows * s.dv * 4);
            w.split_lse = take(rows * 4);
        }
    }
    if (use_block_major(s)) {
        const size_t L = nsa::sel_lists(s);
        const int tok = 128 / s.heads_per_unit;
        w.cnt = take(L * 4);
        w.off = take((L + 1) * 4);
        w.item_off = take((L + 1) * 4);
        w.cursor = take(L * 4);
        w.list = take(nsa::sel_list_alloc(s) * 4);
        w.items = take(nsa::sel_items_max(s, tok) * sizeof(int4));
        w.part_o = take(nsa::sel_pairs_max(s) * s.heads_per_unit * s.dv * 2);
        w.part_lse = take(nsa::sel_pairs_max(s) * s.heads_per_unit * 4);
        w.o_sel = take((size_t)s.B * s.Tq * s.Hq * s.dv * 2);
    } else if (use_sub_block_major(s)) {
        const Shape t = sub_block_shape(s);
        const size_t L = nsa::sel_lists(t);
        const int tok = 128;                  // one head per unit: 128 queries per item
        w.sub = true;
        w.idx_sub = take(idx_bytes(t));
        w.cnt = take(L * 4);
        w.off = take((L + 1) * 4);
        w.item_off = take((L + 1) * 4);
        w.cursor = take(L * 4);
        w.list = take(nsa::sel_list_alloc(t) * 4);
        w.items = take(nsa::sel_items_max(t, tok) * sizeof(int4));
        w.part_o = take(nsa::sel_pairs_max(t) * t.dv * 2);
        w.part_lse = take(nsa::sel_pairs_max(t) * 4);
    }
    w.total = at;
    return w;
}

thread_local const char* g_last_cuda_error = "no error";

nsa_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return NSA_OK;
    g_last_cuda_error = cudaGetErrorString(e);
    return NSA_ERR_CUDA;
}

// Per-host-thread stage events for nsa_timing_enable / nsa_timing_read.  The
// same stage boundaries open and close NVTX ranges (one per stage inside one
// per call), which a profiler attached to the process shows on its timeline;
// without one the NVTX calls return at once.
struct StageTiming {
    bool nvtx_open = false;  // a stage range is open
    bool on = false;
    bool created = false;
    int dev = -1;
    cudaEvent_t ev[NSA_TIMING_MAX_STAGES + 1];
    const char* names[NSA_TIMING_MAX_STAGES];
    int n = 0;             // stages recorded by the current / most recent call
    bool closed = false;   // the most recent call recorded its final event
    bool active = false;   // the current call records

    void begin() {
        n = 0;
        closed = false;
        active = false;
        if (!on || !created) return;
        int d = -1;
        active = cudaGetDevice(&d) == cudaSuccess && d == dev;
    }
    void mark(const char* name, cudaStream_t st) {
        if (nvtx_open) nvtxRangePop();
        nvtxRangePushA(name);
        nvtx_open = true;
        if (!active || n >= NSA_TIMING_MAX_STAGES) return;
        if (cudaEventRecord(ev[n], st) != cudaSuccess) {
            active = false;
            n = 0;
            return;
        }
        names[n++] = name;
    }
    void end(cudaStream_t st) {
        if (nvtx_open) nvtxRangePop();
        nvtx_open = false;
        if (!active) return;
        closed = n > 0 && cudaEventRecord(ev[n], st) == cudaSuccess;
        if (!closed) n = 0;
        active = false;
    }
};
thread_local StageTiming g_timing;

// Records the end of the timed call on every return path of nsa_sparse_attn_fwd.
struct TimingScope {
    cudaStream_t st;
    explicit TimingScope(cudaStream_t s) : st(s) {
        nvtxRangePushA("nsa_sparse_attn_fwd");
        g_timing.begin();
    }
    ~TimingScope() {
        g_timing.end(st);
        nvtxRangePop();
    }
};

}  // namespace

extern "C" {

const char* nsa_status_string(nsa_status status) {
    switch (status) {
        case NSA_OK: return "NSA_OK";
        case NSA_ERR_INVALID_ARG: return "NSA_ERR_INVALID_ARG: null pointer, bad shape or misaligned pointer";
        case NSA_ERR_UNSUPPORTED: return "NSA_ERR_UNSUPPORTED: problem outside the GPU path's limits";
        case NSA_ERR_WORKSPACE: return "NSA_ERR_WORKSPACE: workspace missing or too small";
        case NSA_ERR_CUDA: return "NSA_ERR_CUDA: a CUDA launch or driver call failed";
        case NSA_ERR_TIMEOUT: return "NSA_ERR_TIMEOUT: a device-side bounded wait gave up";
    }
    return "unknown nsa_status";
}

nsa_status nsa_workspace_size(const nsa_config* cfg, size_t* bytes) {
    if (!bytes) return NSA_ERR_INVALID_ARG;
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    *bytes = ws_layout(s).total;
    return NSA_OK;
}

// Which organisation nsa_sparse_attn_fwd uses for a call, and how many
// kernels it launches (shared by the dispatch below and nsa_attn_plan).
struct Plan {
    int path;       // NSA_PATH_*
    int kernels;
};

Plan make_plan(const Shape& s, bool select_inside, size_t ws_bytes, const WsLayout& wl) {
    Plan p{NSA_PATH_ROWWISE, 1};
    if (use_decode(s) && ws_bytes >= wl.total) {
        p = {NSA_PATH_DECODE, 2};
    } else if (use_sub_block_major(s) && ws_bytes >= wl.total) {
        p = {NSA_PATH_BLOCK_MAJOR, 7};    // expand, index (4), block-major, merge into out
    } else if (nsa::attn_tc_supported(s)) {
        if (use_block_major(s) && ws_bytes >= wl.total) p = {NSA_PATH_BLOCK_MAJOR, 7};
        else if (wl.n_split > 1 && ws_bytes >= wl.total) p = {NSA_PATH_SPLIT_K, 2};
        else p = {NSA_PATH_QUERY_MAJOR, 1};
    }
    // selection inside the call: the tensor-core selection (split + split + score) or one kernel
    if (select_inside) p.kernels += (wl.sc && ws_bytes >= wl.total) ? 3 : 1;
    return p;
}

nsa_status nsa_attn_plan(const nsa_config* cfg, int select_inside, size_t ws_bytes, int32_t* path,
                         int32_t* kernels) {
    if (!path || !kernels) return NSA_ERR_INVALID_ARG;
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    const Plan p = make_plan(s, select_inside && (cfg->flags & NSA_BR_SEL), ws_bytes, ws_layout(s));
    *path = p.path;
    *kernels = p.kernels;
    return NSA_OK;
}

nsa_status nsa_workspace_size_min(const nsa_config* cfg, size_t* bytes) {
    if (!bytes) return NSA_ERR_INVALID_ARG;
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    *bytes = ws_layout(s).minimal;
    return NSA_OK;
}

nsa_status nsa_pool_kv(const nsa_config* cfg, const void* k, const void* v, float* kbar,
                       void* kcmp, void* vcmp, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    // buffers of zero elements (no complete block / no compressed token) may be NULL
    const bool need_sel = (cfg->flags & NSA_BR_SEL) != 0 && s.nb_full > 0;
    const bool need_cmp = (cfg->flags & NSA_BR_CMP) != 0 && s.n_cmp > 0;
    if (!k || (need_sel && !kbar)) return NSA_ERR_INVALID_ARG;
    if (need_cmp && (!v || !kcmp || !vcmp)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(kbar) || !aligned16(kcmp) || !aligned16(vcmp))
        return NSA_ERR_INVALID_ARG;
    return cuda_status(nsa::launch_pool_kv(
        s, static_cast<const __nv_bfloat16*>(k), static_cast<const __nv_bfloat16*>(v),
        need_sel ? kbar : nullptr, need_cmp ? static_cast<__nv_bfloat16*>(kcmp) : nullptr,
        need_cmp ? static_cast<__nv_bfloat16*>(vcmp) : nullptr, static_cast<cudaStream_t>(stream)));
}

// floor(a / b) for b > 0 and any a
static int floor_div(int a, int b) { return a >= 0 ? a / b : -((-a + b - 1) / b); }

nsa_status nsa_append_kv(const nsa_config* cfg, void* k, void* v, const void* k_new, const void* v_new,
                         float* kbar, void* kcmp, void* vcmp, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    if (s.Tq < 1) return NSA_ERR_INVALID_ARG;
    if (!k || !v || !k_new || !v_new) return NSA_ERR_INVALID_ARG;
    const int t0 = s.q0, t1 = s.q0 + s.Tq;      // new rows [t0, t1)
    // selection blocks ending inside [t0, t1): j * bs + bs - 1 in [t0, t1)
    const bool sel = (cfg->flags & NSA_BR_SEL) != 0;
    const int jb0 = t0 / s.bs, jb1 = sel ? std::min(t1 / s.bs, s.nb_full) : jb0;
    // compressed tokens whose window ends inside [t0, t1): j * sc + lc - 1 in [t0, t1)
    const bool cmp = (cfg->flags & NSA_BR_CMP) != 0;
    int jc0 = 0, jc1 = 0;
    if (cmp && s.n_cmp > 0) {
        jc0 = std::max(0, floor_div(t0 - s.lc + s.sc, s.sc));
        jc1 = std::min(s.n_cmp, std::max(0, floor_div(t1 - s.lc, s.sc) + 1));
        jc1 = std::max(jc1, jc0);
    }
    if ((jb1 > jb0 && !kbar) || (jc1 > jc0 && (!kcmp || !vcmp))) return NSA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(kbar) ||
        !aligned16(kcmp) || !aligned16(vcmp))
        return NSA_ERR_INVALID_ARG;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    __nv_bfloat16* kb = static_cast<__nv_bfloat16*>(k);
    __nv_bfloat16* vb = static_cast<__nv_bfloat16*>(v);
    st = cuda_status(nsa::launch_append_rows(s, static_cast<const __nv_bfloat16*>(k_new),
                                             static_cast<const __nv_bfloat16*>(v_new), kb, vb, t0, s.Tq, cs));
    if (st != NSA_OK) return st;
    return cuda_status(nsa::launch_pool_range(s, kb, vb, kbar, static_cast<__nv_bfloat16*>(kcmp),
                                              static_cast<__nv_bfloat16*>(vcmp), jb0, jb1, jc0, jc1, cs));
}

// The pooled inputs the configured scores read: kbar (scaled dot product,
// probability sums) or the compressed keys (scores from the compressed branch).
static bool score_inputs_ok(const Shape& s, const void* q, const float* kbar, const void* kcmp) {
    if (!q) return false;
    if (s.score_mode == 2) return s.n_cmp == 0 || kcmp != nullptr;
    return s.nb_full == 0 || kbar != nullptr;
}

// Scores (scores_out) and/or selected ids (idx) computed from q and the pooled keys.
static cudaError_t launch_selection(const Shape& s, const void* q, const float* kbar, const void* kcmp,
                             float* scores_out, int32_t* idx, cudaStream_t cs) {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    if (s.score_mode != 0)
        return nsa::launch_score_variant(s, qb, kbar, static_cast<const __nv_bfloat16*>(kcmp), scores_out,
                                         idx, cs);
    return nsa::launch_score_topk(s, qb, kbar, nullptr, scores_out, idx, cs);
}

nsa_status nsa_score_blocks_ex(const nsa_config* cfg, const void* q, const float* kbar, const void* kcmp,
                               float* scores, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    if (!(cfg->flags & NSA_BR_SEL)) return NSA_ERR_INVALID_ARG;
    if (!scores || !score_inputs_ok(s, q, kbar, kcmp)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kbar) || !aligned16(kcmp) || !aligned16(scores)) return NSA_ERR_INVALID_ARG;
    if (s.Tq == 0) return NSA_OK;
    return cuda_status(launch_selection(s, q, kbar, kcmp, scores, nullptr, static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_score_blocks(const nsa_config* cfg, const void* q, const float* kbar, float* scores,
                            void* stream) {
    return nsa_score_blocks_ex(cfg, q, kbar, nullptr, scores, stream);
}

nsa_status nsa_topk_select_ex(const nsa_config* cfg, const void* q, const float* kbar, const void* kcmp,
                              const float* scores, int32_t* idx, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    if (!(cfg->flags & NSA_BR_SEL)) return NSA_ERR_INVALID_ARG;
    if (!idx) return NSA_ERR_INVALID_ARG;
    if (!scores && !score_inputs_ok(s, q, kbar, kcmp)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(kbar) || !aligned16(kcmp) || !aligned16(scores) || !aligned16(idx))
        return NSA_ERR_INVALID_ARG;
    if (s.Tq == 0) return NSA_OK;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (scores)
        return cuda_status(nsa::launch_score_topk(s, nullptr, nullptr, scores, nullptr, idx, cs));
    return cuda_status(launch_selection(s, q, kbar, kcmp, nullptr, idx, cs));
}

nsa_status nsa_topk_select(const nsa_config* cfg, const void* q, const float* kbar,
                           const float* scores, int32_t* idx, void* stream) {
    return nsa_topk_select_ex(cfg, q, kbar, nullptr, scores, idx, stream);
}

nsa_status nsa_sparse_attn_fwd(const nsa_config* cfg, const void* q, const void* k, const void* v,
                               const float* kbar, const void* kcmp, const void* vcmp,
                               const float* gates, const int32_t* idx, void* out, void* workspace,
                               size_t ws_bytes, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    const bool sel = (cfg->flags & NSA_BR_SEL) != 0;
    const bool cmp = (cfg->flags & NSA_BR_CMP) != 0;
    if (!q || !k || !v || !out) return NSA_ERR_INVALID_ARG;
    if (cmp && s.n_cmp > 0 && (!kcmp || !vcmp)) return NSA_ERR_INVALID_ARG;
    if (sel && !idx && !score_inputs_ok(s, q, kbar, kcmp)) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kbar) || !aligned16(kcmp) ||
        !aligned16(vcmp) || !aligned16(gates) || !aligned16(idx) || !aligned16(out) ||
        !aligned16(workspace))
        return NSA_ERR_INVALID_ARG;
    const WsLayout wl = ws_layout(s);
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    int32_t* sel_idx = const_cast<int32_t*>(idx);
    if (sel && !idx) {
        if (!workspace || ws_bytes < wl.minimal) return NSA_ERR_WORKSPACE;
        sel_idx = reinterpret_cast<int32_t*>(ws + wl.idx);
    }
    if (s.Tq == 0) return NSA_OK;
    cudaStream_t cs = static_cast<cudaStream_t>(stream);
    if (sel && idx && (cfg->flags & NSA_DEBUG_CHECKS)) {
        // validate the caller's ids before any attention kernel reads them
        int bad = 0;
        st = cuda_status(nsa::check_idx_rows(s, idx, &bad, cs));
        if (st != NSA_OK) return st;
        if (bad > 0) return NSA_ERR_INVALID_ARG;
    }
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v);
    const __nv_bfloat16* kcb = static_cast<const __nv_bfloat16*>(kcmp);
    const __nv_bfloat16* vcb = static_cast<const __nv_bfloat16*>(vcmp);
    __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(out);
    TimingScope timing(cs);
    if (sel && !idx) {
        g_timing.mark("select", cs);
        if (wl.sc && ws_bytes >= wl.total)
            st = cuda_status(nsa::launch_score_tc(s, qb, kbar, reinterpret_cast<float*>(ws + wl.sc_qh),
                                                  reinterpret_cast<float*>(ws + wl.sc_ql),
                                                  reinterpret_cast<float*>(ws + wl.sc_kh),
                                                  reinterpret_cast<float*>(ws + wl.sc_kl), sel_idx, cs));
        else
            st = cuda_status(launch_selection(s, q, kbar, kcmp, nullptr, sel_idx, cs));
        if (st != NSA_OK) return st;
    }
    const Plan plan = make_plan(s, false, ws ? ws_bytes : 0, wl);
    if (plan.path == NSA_PATH_ROWWISE) {
        g_timing.mark("rowwise", cs);
        return cuda_status(nsa::launch_attn(s, qb, kb, vb, kcb, vcb, gates, sel_idx, ob, cs));
    }
    // block-major selected branch when the workspace holds its index and partials
    if (plan.path == NSA_PATH_BLOCK_MAJOR && wl.sub) {
        const Shape t = sub_block_shape(s);
        int32_t* idx_sub = reinterpret_cast<int32_t*>(ws + wl.idx_sub);
        nsa::SelIndex x;
        x.cnt = reinterpret_cast<int32_t*>(ws + wl.cnt);
        x.off = reinterpret_cast<int32_t*>(ws + wl.off);
        x.item_off = reinterpret_cast<int32_t*>(ws + wl.item_off);
        x.cursor = reinterpret_cast<int32_t*>(ws + wl.cursor);
        x.list = reinterpret_cast<int32_t*>(ws + wl.list);
        x.items = reinterpret_cast<int4*>(ws + wl.items);
        __nv_bfloat16* part_o = reinterpret_cast<__nv_bfloat16*>(ws + wl.part_o);
        float* part_lse = reinterpret_cast<float*>(ws + wl.part_lse);
        g_timing.mark("expand", cs);
        st = cuda_status(nsa::launch_sel_expand(s, sel_idx, idx_sub, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("index", cs);
        st = cuda_status(nsa::launch_sel_index(t, idx_sub, x, 128, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("sel_bm", cs);
        st = cuda_status(nsa::launch_sel_bm(t, qb, kb, vb, x, part_o, part_lse, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("sel_merge", cs);
        return cuda_status(nsa::launch_sel_merge_out(t, idx_sub, part_o, part_lse, gates, ob, cs));
    }
    if (plan.path == NSA_PATH_BLOCK_MAJOR) {
        nsa::SelIndex x;
        x.cnt = reinterpret_cast<int32_t*>(ws + wl.cnt);
        x.off = reinterpret_cast<int32_t*>(ws + wl.off);
        x.item_off = reinterpret_cast<int32_t*>(ws + wl.item_off);
        x.cursor = reinterpret_cast<int32_t*>(ws + wl.cursor);
        x.list = reinterpret_cast<int32_t*>(ws + wl.list);
        x.items = reinterpret_cast<int4*>(ws + wl.items);
        __nv_bfloat16* part_o = reinterpret_cast<__nv_bfloat16*>(ws + wl.part_o);
        float* part_lse = reinterpret_cast<float*>(ws + wl.part_lse);
        const int tok = 128 / s.heads_per_unit;
        g_timing.mark("index", cs);
        st = cuda_status(nsa::launch_sel_index(s, sel_idx, x, tok, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("sel_bm", cs);
        st = cuda_status(nsa::launch_sel_bm(s, qb, kb, vb, x, part_o, part_lse, cs));
        if (st != NSA_OK) return st;
        __nv_bfloat16* o_sel = reinterpret_cast<__nv_bfloat16*>(ws + wl.o_sel);
        g_timing.mark("sel_merge", cs);
        st = cuda_status(nsa::launch_sel_merge(s, sel_idx, part_o, part_lse, o_sel, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("attn_tc", cs);
        return cuda_status(nsa::launch_attn_tc(s, qb, kb, vb, kcb, vcb, gates, sel_idx, o_sel, 1,
                                               nullptr, nullptr, ob, cs));
    }
    if (plan.path == NSA_PATH_DECODE) {
        float* dec_o = reinterpret_cast<float*>(ws + wl.dec_o);
        float* dec_lse = reinterpret_cast<float*>(ws + wl.dec_lse);
        g_timing.mark("attn_dec", cs);
        st = cuda_status(nsa::launch_attn_dec(s, qb, kb, vb, kcb, vcb, sel_idx, dec_o, dec_lse, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("dec_merge", cs);
        return cuda_status(nsa::launch_dec_merge(s, dec_o, dec_lse, gates, ob, cs));
    }
    if (plan.path == NSA_PATH_SPLIT_K) {
        float* split_o = reinterpret_cast<float*>(ws + wl.split_o);
        float* split_lse = reinterpret_cast<float*>(ws + wl.split_lse);
        g_timing.mark("attn_tc", cs);
        st = cuda_status(nsa::launch_attn_tc(s, qb, kb, vb, kcb, vcb, gates, sel_idx, nullptr,
                                             wl.n_split, split_o, split_lse, ob, cs));
        if (st != NSA_OK) return st;
        g_timing.mark("split_merge", cs);
        return cuda_status(nsa::launch_split_merge(s, wl.n_split, split_o, split_lse, gates, ob, cs));
    }
    g_timing.mark("attn_tc", cs);
    return cuda_status(nsa::launch_attn_tc(s, qb, kb, vb, kcb, vcb, gates, sel_idx, nullptr, 1,
                                           nullptr, nullptr, ob, cs));
}

static size_t bwd_ws_bytes(const Shape& s) {
    if (!(s.flags & NSA_BR_CMP) || s.n_cmp == 0) return 0;
    return round_up((size_t)s.B * s.Hkv * s.n_cmp * s.dqk * 4, 256) +
           round_up((size_t)s.B * s.Hkv * s.n_cmp * s.dv * 4, 256);
}

nsa_status nsa_bwd_workspace_size(const nsa_config* cfg, size_t* bytes) {
    if (!bytes) return NSA_ERR_INVALID_ARG;
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    *bytes = bwd_ws_bytes(s);
    return NSA_OK;
}

nsa_status nsa_sparse_attn_bwd(const nsa_config* cfg, const void* q, const void* k, const void* v,
                               const void* kcmp, const void* vcmp, const float* gates, const int32_t* idx,
                               const void* d_out, float* dq, float* dk, float* dv, float* dgates,
                               void* workspace, size_t ws_bytes, void* stream) {
    Shape s;
    nsa_status st = make_shape(cfg, &s);
    if (st != NSA_OK) return st;
    const bool sel = (cfg->flags & NSA_BR_SEL) != 0;
    const bool cmp = (cfg->flags & NSA_BR_CMP) != 0 && s.n_cmp > 0;
    if (!q || !k || !v || !d_out || !dq || !dk || !dv) return NSA_ERR_INVALID_ARG;
    if ((sel && !idx) || (cmp && (!kcmp || !vcmp))) return NSA_ERR_INVALID_ARG;
    if (gates && !dgates) return NSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(kcmp) || !aligned16(vcmp) ||
        !aligned16(gates) || !aligned16(idx) || !aligned16(d_out) || !aligned16(dq) || !aligned16(dk) ||
        !aligned16(dv) || !aligned16(dgates) || !aligned16(workspace))
        return NSA_ERR_INVALID_ARG;
    if (!nsa::bwd_supported(s)) return NSA_ERR_UNSUPPORTED;
    const size_t need = bwd_ws_bytes(s);
    if (need && (!workspace || ws_bytes < need)) return NSA_ERR_WORKSPACE;
    if (s.Tq == 0) return NSA_OK;
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    float* dkc = need ? reinterpret_cast<float*>(ws) : nullptr;
    float* dvc = need ? reinterpret_cast<float*>(ws + round_up((size_t)s.B * s.Hkv * s.n_cmp * s.dqk * 4, 256))
                      : nullptr;
    return cuda_status(nsa::launch_attn_bwd(
        s, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
        static_cast<const __nv_bfloat16*>(v), static_cast<const __nv_bfloat16*>(kcmp),
        static_cast<const __nv_bfloat16*>(vcmp), gates, idx, static_cast<const __nv_bfloat16*>(d_out), dq, dk,
        dv, dgates, dkc, dvc, static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_check_bounded_wait(uint64_t limit_ns, void* stream) {
    if (limit_ns < 1 || limit_ns > 1000000000ull) return NSA_ERR_INVALID_ARG;
    return cuda_status(nsa::launch_wait_selftest(limit_ns, static_cast<cudaStream_t>(stream)));
}

nsa_status nsa_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns > 1000000000ull) return NSA_ERR_INVALID_ARG;
    return cuda_status(nsa::set_wait_limit(limit_ns));
}

nsa_status nsa_timing_enable(int32_t on) {
    StageTiming& t = g_timing;
    if (on && !t.created) {
        int d = -1;
        if (cudaGetDevice(&d) != cudaSuccess) return NSA_ERR_CUDA;
        int made = 0;
        for (; made <= NSA_TIMING_MAX_STAGES; ++made) {
            const cudaError_t e = cudaEventCreate(&t.ev[made]);
            if (e != cudaSuccess) {
                for (int i = 0; i < made; ++i) cudaEventDestroy(t.ev[i]);
                return cuda_status(e);
            }
        }
        t.created = true;
        t.dev = d;
    }
    t.on = on != 0;
    return NSA_OK;
}

nsa_status nsa_timing_read(int32_t max_stages, float* ms, const char** names, int32_t* n_stages) {
    if (!n_stages || max_stages < 0 || (max_stages > 0 && (!ms || !names))) return NSA_ERR_INVALID_ARG;
    StageTiming& t = g_timing;
    *n_stages = 0;
    if (!t.created || !t.closed || t.n == 0) return NSA_OK;
    nsa_status st = cuda_status(cudaEventSynchronize(t.ev[t.n]));
    if (st != NSA_OK) return st;
    for (int i = 0; i < t.n && i < max_stages; ++i) {
        float v = 0.f;
        st = cuda_status(cudaEventElapsedTime(&v, t.ev[i], t.ev[i + 1]));
        if (st != NSA_OK) return st;
        ms[i] = v;
        names[i] = t.names[i];
    }
    *n_stages = t.n;
    return NSA_OK;
}

const char* nsa_last_cuda_error(void) { return g_last_cuda_error; }

nsa_status nsa_get_device_status(int32_t* status) {
    if (!status) return NSA_ERR_INVALID_ARG;
    const int v1 = nsa::read_and_clear_tc_status();
    const int v2 = nsa::read_and_clear_bm_status();
    const int v3 = nsa::read_and_clear_dec_status();
    const int v4 = nsa::read_and_clear_select_status();
    const int v5 = nsa::read_and_clear_sctc_status();
    if (v1 < 0 || v2 < 0 || v3 < 0 || v4 < 0 || v5 < 0) return NSA_ERR_CUDA;
    *status = v1 ? v1 : (v2 ? v2 : (v3 ? v3 : (v4 ? v4 : v5)));
    return NSA_OK;
}

}  // extern "C"
