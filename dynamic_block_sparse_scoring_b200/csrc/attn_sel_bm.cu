// Selected-branch attention, block-major, on tcgen05: one KV block against
// every query that kept it.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §7 "Kimi Simplifies The Sparse
// Route": MoBA gathers, for each KV block, the queries that chose it into a
// contiguous batch and runs dense attention on it; §4 "Inside Native Sparse
// Attention": the selected branch attends over every token of the kept
// blocks.  With random selections neighbouring tokens rarely share blocks, so
// a query-major tile would either re-read each block per query or compute
// over the union of its tokens' blocks; block-major loads each 64-key block
// once per work item of up to 128/HPT queries.
//
// A work item is (sequence, selection unit, block j, up to TOK queries from
// the block's list).  Its 128 rows are the TOK queries x HPT heads, gathered
// by TMA (one 4D box per query).  S = Q K_j^T (M=128, N=64) and O = P V_j
// (M=128, N=d_v) run on tcgen05; the block is fully visible except for the
// query's own block, where key u is visible iff u <= t.  Each row writes a
// partial result for its (query, slot): o = (P V)/l in bf16 and
// lse = m + log2(l) in the scaled-log2 domain.  The partials of a query's
// slots are merged by sel_merge.cu.  Items come chunk by chunk (SEL_CHUNK
// queries); every CTA takes a contiguous share of each chunk, so consecutive
// items of a CTA share their K/V block.
//
// Roles (480 threads): warp 0 TMA producer (item descriptors, K/V once per run
// of items on the same block; with one head per unit also the Q rows), warp 1
// MMA lane + TMEM owner, warps 2-5 and 6-9 two softmax warpgroups taking
// alternate items (S/P double-buffered in TMEM), warps 10-13 the epilogue
// warpgroup (O double-buffered in TMEM, drained to the partial buffers while the
// next items' softmax runs), warp 14 the Q-row loader (groups of heads).  All
// waits are bounded; a timeout records NSA_ERR_TIMEOUT in g_bm_status and unwinds.
#include <cudaTypedefs.h>
#include <math.h>

#include <type_traits>

#include "common.cuh"
#include "sel_index.cuh"
#include "tc.cuh"

namespace nsa {

__device__ int g_bm_status = 0;

namespace {

constexpr int BM = 128;
constexpr int BLK = 64;             // keys per block (the path requires sel_block == 64)
constexpr int NTHREADS = 480;      // producer, MMA, 2 softmax warpgroups, epilogue warpgroup, Q loader
constexpr int NM = 8;               // item descriptors in flight
constexpr int CHUNK_Q = 16384;      // 128 rows x 64 columns bf16
constexpr int CHUNK_KV = 8192;      // 64 rows x 64 columns bf16
constexpr uint64_t WAIT_NS = 1000000000ull;
constexpr int NQ = 2;               // query-gather stages

// MT = most queries in one item: 16 when a unit stacks 8 or 16 heads under each
// query, 128 when a unit is one head (per-head selection).
template <int MT>
struct ItemMeta {
    int valid;          // 0 = end of the stream
    int lidx;           // list id = (chunk * B * Hsel + b * Hsel + u) * nb_all + j
    int n;              // queries in the item
    int kvs;            // K/V stage holding block j
    int new_block;      // first item on this K/V stage load
    int last_of_block;  // last item using this K/V stage load
    int pad[2];
    int tok[MT];        // query * SEL_SLOTS + slot
};

struct BmArgs {
    Shape s;
    const int4* items;
    const int32_t* item_off;  // [lists + 1] first item of each list (chunk boundaries)
    const int32_t* list;
    __nv_bfloat16* part_o;    // [B, Hsel, Tq, topk, hpt, d_v]
    float* part_lse;          // [B, Hsel, Tq, topk, hpt]
    int hpt, tok;
    int n_chunks;
    int lists_per_chunk;
    float scale_log2;
};

template <int DQK, int DV, int MT>
struct BmSmem {
    static constexpr int QC = DQK / 64, VC = DV / 64;
    static constexpr int Q_OFF = 0;                                  // NQ stages
    static constexpr int K_OFF = Q_OFF + NQ * QC * CHUNK_Q;           // 2 stages
    static constexpr int V_OFF = K_OFF + 2 * QC * CHUNK_KV;           // 2 stages
    static constexpr int STG_OFF = V_OFF + 2 * VC * CHUNK_KV;        // 2 x [BM rows x 128 B]
    static constexpr int META_OFF = STG_OFF + 2 * BM * 128;
    static constexpr int ROW_OFF = META_OFF + NM * (int)sizeof(ItemMeta<MT>);   // row m, l [2][2][BM]
    static constexpr int BAR_OFF = ROW_OFF + 4 * BM * 4;
    // q_full[NQ] q_empty[NQ] kv_full[2] kv_empty[2] meta_full[NM] meta_empty[NM]
    // s_full[2] p_full[2] o_full[2] o_free[2] drain
    static constexpr int NBAR = 2 * NQ + 4 + 2 * NM + 8 + 1;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int ALLOC = MISC_OFF + 64 + 1024;
};

struct BmBars {
    uint64_t* b;
    static constexpr int KV0 = 2 * NQ, MT0 = KV0 + 4, SB0 = MT0 + 2 * NM;
    __device__ __forceinline__ uint64_t* q_full(int i) const { return b + i; }
    __device__ __forceinline__ uint64_t* q_empty(int i) const { return b + NQ + i; }
    __device__ __forceinline__ uint64_t* kv_full(int i) const { return b + KV0 + i; }
    __device__ __forceinline__ uint64_t* kv_empty(int i) const { return b + KV0 + 2 + i; }
    __device__ __forceinline__ uint64_t* meta_full(int i) const { return b + MT0 + i; }
    __device__ __forceinline__ uint64_t* meta_empty(int i) const { return b + MT0 + NM + i; }
    __device__ __forceinline__ uint64_t* s_full(int i) const { return b + SB0 + i; }
    __device__ __forceinline__ uint64_t* p_full(int i) const { return b + SB0 + 2 + i; }
    __device__ __forceinline__ uint64_t* o_full(int i) const { return b + SB0 + 4 + i; }
    __device__ __forceinline__ uint64_t* o_free(int i) const { return b + SB0 + 6 + i; }
    __device__ __forceinline__ uint64_t* drain() const { return b + SB0 + 8; }
};

__device__ __forceinline__ bool bm_warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, tc::mbar_wait(b, parity, abort_flag, WAIT_NS));
}

__device__ __forceinline__ void bm_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_bm_status, (int)NSA_ERR_TIMEOUT);
}

template <int DQK, int DV, int MT>
__global__ void __launch_bounds__(NTHREADS, 1)
    sel_bm_kernel(const __grid_constant__ CUtensorMap map_qg, const __grid_constant__ CUtensorMap map_k,
                  const __grid_constant__ CUtensorMap map_v,
                  const __grid_constant__ CUtensorMap map_po, const BmArgs a) {
    using L = BmSmem<DQK, DV, MT>;
    using ItemMeta = nsa::ItemMeta<MT>;
    constexpr int NG = (MT + 31) / 32;      // lane groups covering an item's queries
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    BmBars bar{reinterpret_cast<uint64_t*>(sm + L::BAR_OFF)};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC_OFF + 8);
    ItemMeta* metas = reinterpret_cast<ItemMeta*>(sm + L::META_OFF);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < NQ; ++i) {
            tc::mbar_init(bar.q_full(i), 1);
            tc::mbar_init(bar.q_empty(i), 1);
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar.kv_full(i), 1);
            tc::mbar_init(bar.kv_empty(i), 1);
            tc::mbar_init(bar.s_full(i), 1);
            tc::mbar_init(bar.p_full(i), 4);
            tc::mbar_init(bar.o_full(i), 1);
            tc::mbar_init(bar.o_free(i), 4);
        }
        for (int i = 0; i < NM; ++i) {
            tc::mbar_init(bar.meta_full(i), 1);
            // MMA lane + owning softmax WG + epilogue WG (+ the Q-loader warp, groups of heads)
            tc::mbar_init(bar.meta_empty(i), MT <= 32 ? 10 : 9);
        }
        tc::mbar_init(bar.drain(), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        tc::prefetch_map(&map_qg);
        tc::prefetch_map(&map_k);
        tc::prefetch_map(&map_v);
        tc::prefetch_map(&map_po);
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    // S0 [0,64) S1 [64,128) O0 [128,128+DV) O1 [256,256+DV)
    auto tS = [&](int i) { return tmem + 64 * i; };
    auto tO = [&](int i) { return tmem + 128 + 128 * i; };

    const int nb_all = a.s.nb_all;
    const int bhsel = a.s.B * a.s.Hsel;
    // This CTA's share of chunk c's items: a contiguous range, so that
    // consecutive items mostly stay on one block (K/V loaded once for them),
    // while all CTAs advance through the chunks together.
    auto chunk_range = [&](int c, int& lo, int& hi) {
        const int c0 = a.item_off[(size_t)c * a.lists_per_chunk];
        const int c1 = a.item_off[(size_t)(c + 1) * a.lists_per_chunk];
        const int per = (c1 - c0 + gridDim.x - 1) / gridDim.x;
        lo = min(c1, c0 + (int)blockIdx.x * per);
        hi = min(c1, lo + per);
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        uint32_t kv_loads = 0, q_loads = 0;
        int prev_lidx = -1, kvs = 0;
        const uint64_t q_policy = tc::l2_policy_evict_last();
        int chunk = 0, i = 0, i_end = 0, li = 0, ends = 0;
        // register windows over the item and list arrays (both are consumed in
        // order, so one coalesced warp load serves many items)
        int4 iwin = make_int4(0, 0, 0, 0);
        int ibase = -1;
        int lwin0 = 0, lwin1 = 0, lbase = -1;
        auto item_at = [&](int k) -> int4 {
            if (ibase < 0 || k < ibase || k >= ibase + 32) {
                ibase = k;
                iwin = a.items[k + lane];          // the items array has 32 slack entries
            }
            int4 r;
            r.x = __shfl_sync(0xffffffffu, iwin.x, k - ibase);
            r.y = __shfl_sync(0xffffffffu, iwin.y, k - ibase);
            r.z = __shfl_sync(0xffffffffu, iwin.z, k - ibase);
            return r;
        };
        auto list_at = [&](int pos, int n) -> int {     // lane l < n gets list[pos + l]
            if (lbase < 0 || pos < lbase || pos + n > lbase + 64) {
                lbase = pos;
                lwin0 = a.list[pos + lane];
                lwin1 = a.list[pos + 32 + lane];       // the list array has 64 slack entries
            }
            const int o = pos - lbase + lane;
            const int v0 = __shfl_sync(0xffffffffu, lwin0, o & 31);
            const int v1 = __shfl_sync(0xffffffffu, lwin1, o & 31);
            return o < 32 ? v0 : v1;
        };
        chunk_range(0, i, i_end);
        while (ok && ends < 2) {
            while (i >= i_end && chunk + 1 < a.n_chunks) chunk_range(++chunk, i, i_end);
            ItemMeta m;
            bool meta_ready = false;     // this item's metadata slot already waited for
            m.valid = i < i_end;
            m.lidx = m.n = m.kvs = m.new_block = m.last_of_block = 0;
            if (m.valid) {
                const int4 it = item_at(i);
                m.lidx = it.x;
                m.n = it.z;
                m.new_block = it.x != prev_lidx;
                // the next item this CTA will take (possibly in a later chunk)
                if (i + 1 < i_end) {
                    m.last_of_block = item_at(i + 1).x != it.x;
                } else {
                    int nxt = i + 1, nxt_end = i_end, nchunk = chunk;
                    while (nxt >= nxt_end && nchunk + 1 < a.n_chunks) chunk_range(++nchunk, nxt, nxt_end);
                    m.last_of_block = nxt >= nxt_end || a.items[nxt].x != it.x;
                }
                const int bu = (it.x / nb_all) % bhsel, j = it.x % nb_all;
                const int b = bu / a.s.Hsel, u = bu % a.s.Hsel;
                const int kvh = a.s.per_head ? u / a.s.G : u;
                const int h0 = a.s.per_head ? u : u * a.s.G;
                if (m.new_block) {
                    kvs = kv_loads & 1;
                    if (!bm_warp_wait(bar.kv_empty(kvs), ((kv_loads >> 1) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) tc::mbar_arrive_expect_tx(bar.kv_full(kvs), (L::QC + L::VC) * CHUNK_KV);
                    __syncwarp();
                    const int plane = b * a.s.Hkv + kvh;
                    if (lane < L::QC)
                        tc::tma_load_3d(sm + L::K_OFF + (kvs * L::QC + lane) * CHUNK_KV, &map_k,
                                        bar.kv_full(kvs), 64 * lane, j * BLK, plane);
                    else if (lane < L::QC + L::VC)
                        tc::tma_load_3d(sm + L::V_OFF + (kvs * L::VC + lane - L::QC) * CHUNK_KV, &map_v,
                                        bar.kv_full(kvs), 64 * (lane - L::QC), j * BLK, plane);
                    ++kv_loads;
                    prev_lidx = it.x;
                }
                m.kvs = kvs;
                if constexpr (MT <= 32) {
                    // the Q-loader warp gathers the item's query rows from the metadata
                    const int tokv = list_at(it.y, m.n);
                    for (int tt = 0; tt < MT; ++tt) m.tok[tt] = __shfl_sync(0xffffffffu, tokv, tt);
                } else {
                    // more queries than lanes: they go straight into the item's
                    // metadata slot, which the Q loads then read back
                    const int slot = li % NM;
                    if (!bm_warp_wait(bar.meta_empty(slot), ((li / NM) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    meta_ready = true;
                    for (int g = 0; g < NG; ++g) {
                        const int n_g = min(32, m.n - 32 * g);
                        if (n_g <= 0) break;
                        const int tokv = list_at(it.y + 32 * g, n_g);
                        if (lane < n_g) metas[slot].tok[32 * g + lane] = tokv;
                    }
                    __syncwarp();
                    const int qs = li % NQ;
                    if (!bm_warp_wait(bar.q_empty(qs), ((li / NQ) & 1) ^ 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    // one head per query (hpt == 1): the query rows are gathered four
                    // at a time from q viewed as [B * Tq * Hq rows, DQK]; the last
                    // group repeats its final row (rows >= n are never used)
                    const int n4 = (m.n + 3) / 4;
                    if (lane == 0) tc::mbar_arrive_expect_tx(bar.q_full(qs), n4 * 4 * L::QC * 128);
                    __syncwarp();
                    const int* toks = metas[slot].tok;
                    const int qrow0 = (b * a.s.Tq) * a.s.Hq + h0;
                    for (int e = lane; e < n4 * L::QC; e += 32) {
                        const int g4 = e / L::QC, c = e % L::QC;
                        int r[4];
#pragma unroll
                        for (int k = 0; k < 4; ++k)
                            r[k] = qrow0 + pair_query(toks[min(4 * g4 + k, m.n - 1)]) * a.s.Hq;
                        tc::tma_gather4_hint(sm + L::Q_OFF + (qs * L::QC + c) * CHUNK_Q + 4 * g4 * 128, &map_qg,
                                             bar.q_full(qs), 64 * c, r[0], r[1], r[2], r[3], q_policy);
                    }
                }
                if constexpr (MT > 32) ++q_loads;
                ++i;
            } else {
                ++ends;    // two end markers: each softmax warpgroup sees one
            }
            const int slot = li % NM;
            if (!meta_ready && !bm_warp_wait(bar.meta_empty(slot), ((li / NM) & 1) ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                if constexpr (MT <= 32) {
                    metas[slot] = m;
                } else {
                    ItemMeta& d = metas[slot];
                    d.valid = m.valid;
                    d.lidx = m.lidx;
                    d.n = m.n;
                    d.kvs = m.kvs;
                    d.new_block = m.new_block;
                    d.last_of_block = m.last_of_block;
                }
                tc::mbar_arrive(bar.meta_full(slot));
            }
            ++li;
        }
        if (!ok) bm_abort(abort_flag);
        // wait for every copy still in flight before the CTA may exit
        for (uint32_t s = 0; s < 2; ++s) {
            if (kv_loads > s) {
                const uint32_t last = s + ((kv_loads - 1 - s) / 2) * 2;
                tc::mbar_wait_bounded(bar.kv_full(s), (last >> 1) & 1, WAIT_NS);
            }
        }
        for (uint32_t s = 0; s < NQ; ++s) {
            if (q_loads > s) {
                const uint32_t last = s + ((q_loads - 1 - s) / NQ) * NQ;
                tc::mbar_wait_bounded(bar.q_full(s), (last / NQ) & 1, WAIT_NS);
            }
        }
    } else if (warp == 14) {
        // ------------------------------------------------------------ Q loader (groups of
        // heads): one TMA per (query, 64-column chunk) of every item, spread over the
        // lanes, into the item's Q stage.  Issuing these 3 x TOK boxes per item from
        // the producer warp made it the slowest role, so they have their own warp.
        if constexpr (MT <= 32) {
            bool ok = true;
            uint32_t q_loads = 0;
            const uint64_t q_policy = tc::l2_policy_evict_last();
            for (int li = 0; ok; ++li) {
                const int slot = li % NM;
                if (!bm_warp_wait(bar.meta_full(slot), (li / NM) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                const ItemMeta& mref = metas[slot];
                const int valid = mref.valid, lidx = mref.lidx, n = mref.n;
                const int tokl = lane < MT ? mref.tok[lane] : 0;
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar.meta_empty(slot));
                if (!valid) break;
                const int bu = (lidx / nb_all) % bhsel;
                const int b = bu / a.s.Hsel, u = bu % a.s.Hsel;
                const int h0 = a.s.per_head ? u : u * a.s.G;
                const int qs = li % NQ;
                if (!bm_warp_wait(bar.q_empty(qs), ((li / NQ) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0) tc::mbar_arrive_expect_tx(bar.q_full(qs), n * L::QC * a.hpt * 128);
                __syncwarp();
                for (int e0 = 0; e0 < n * L::QC; e0 += 32) {
                    const int e = e0 + lane;
                    const int tt = e / L::QC, c = e % L::QC;
                    const int qtok = __shfl_sync(0xffffffffu, tokl, tt & 31);
                    if (e < n * L::QC)
                        tc::tma_load_4d_hint(sm + L::Q_OFF + (qs * L::QC + c) * CHUNK_Q + tt * a.hpt * 128,
                                             &map_qg, bar.q_full(qs), 64 * c, h0, pair_query(qtok), b, q_policy);
                }
                ++q_loads;
            }
            if (!ok) bm_abort(abort_flag);
            // wait for every copy still in flight before the CTA may exit
            for (uint32_t s = 0; s < NQ; ++s) {
                if (q_loads > s) {
                    const uint32_t last = s + ((q_loads - 1 - s) / NQ) * NQ;
                    tc::mbar_wait_bounded(bar.q_full(s), (last / NQ) & 1, WAIT_NS);
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc_qk = tc::idesc_bf16_f32(BM, BLK, false, false);
            const uint32_t idesc_pv = tc::idesc_bf16_f32(BM, DV, false, true);
            const uint32_t q_base = tc::smem_u32(sm + L::Q_OFF);
            const uint32_t k_base = tc::smem_u32(sm + L::K_OFF);
            const uint32_t v_base = tc::smem_u32(sm + L::V_OFF);
            bool ok = true, have_prev = false;
            int prev_li = 0, prev_kvs = 0, prev_last = 0;
            uint32_t kv_seen = 0;
            auto issue_pv = [&](int li, int kvs, int last) -> bool {
                const int sb = li & 1;
                if (!tc::mbar_wait(bar.p_full(sb), (li >> 1) & 1, abort_flag, WAIT_NS) ||
                    !tc::mbar_wait(bar.o_free(sb), ((li >> 1) & 1) ^ 1, abort_flag, WAIT_NS))
                    return false;
                tc::fence_after_sync();
                const uint32_t vst = v_base + kvs * L::VC * CHUNK_KV;
#pragma unroll
                for (int kk = 0; kk < BLK / 16; ++kk)
                    tc::mma_ts(tO(sb), tS(sb) + kk * 8, tc::sdesc_sw128(vst + kk * 2048, CHUNK_KV, 1024),
                               idesc_pv, kk > 0);
                tc::mma_commit(bar.o_full(sb));
                if (last) tc::mma_commit(bar.kv_empty(kvs));
                return true;
            };
            for (int li = 0; ok; ++li) {
                const int slot = li % NM;
                if (!tc::mbar_wait(bar.meta_full(slot), (li / NM) & 1, abort_flag, WAIT_NS)) {
                    ok = false;
                    break;
                }
                const ItemMeta& m = metas[slot];
                const int valid = m.valid, kvs = m.kvs, new_block = m.new_block, last = m.last_of_block;
                tc::mbar_arrive(bar.meta_empty(slot));
                if (!valid) {
                    if (have_prev && !issue_pv(prev_li, prev_kvs, prev_last)) ok = false;
                    break;
                }
                const int qs = li % NQ;
                if (!tc::mbar_wait(bar.q_full(qs), (li / NQ) & 1, abort_flag, WAIT_NS)) {
                    ok = false;
                    break;
                }
                if (new_block) {
                    if (!tc::mbar_wait(bar.kv_full(kvs), (kv_seen >> 1) & 1, abort_flag, WAIT_NS)) {
                        ok = false;
                        break;
                    }
                    ++kv_seen;
                }
                tc::fence_after_sync();
                const uint32_t qst = q_base + qs * L::QC * CHUNK_Q;
                const uint32_t kst = k_base + kvs * L::QC * CHUNK_KV;
#pragma unroll
                for (int kk = 0; kk < DQK / 16; ++kk) {
                    tc::mma_ss(tS(li & 1),
                               tc::sdesc_sw128(qst + (kk >> 2) * CHUNK_Q + (kk & 3) * 32, 16, 1024),
                               tc::sdesc_sw128(kst + (kk >> 2) * CHUNK_KV + (kk & 3) * 32, 16, 1024),
                               idesc_qk, kk > 0);
                }
                tc::mma_commit(bar.s_full(li & 1));
                tc::mma_commit(bar.q_empty(qs));
                if (have_prev && !issue_pv(prev_li, prev_kvs, prev_last)) {
                    ok = false;
                    break;
                }
                have_prev = true;
                prev_li = li;
                prev_kvs = kvs;
                prev_last = last;
            }
            if (!ok) bm_abort(abort_flag);
            tc::mma_commit(bar.drain());
            tc::mbar_wait_bounded(bar.drain(), 0, WAIT_NS);
        }
        __syncwarp();
    } else if (warp >= 2 && warp < 10) {
        // ------------------------------------------------------------ softmax (warps 2-5 and
        // 6-9, alternate items; S/P double-buffered in TMEM)
        const int wg = (warp - 2) >> 2;          // softmax warpgroup 0 / 1 takes items li % 2 == wg
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int tt = r / a.hpt;
        float* row_m = reinterpret_cast<float*>(sm + L::ROW_OFF);    // [2][BM] per O buffer
        float* row_l = row_m + 2 * BM;
        bool ok = true;
        for (int li = wg; ok; li += 2) {
            const int slot = li % NM;
            if (!bm_warp_wait(bar.meta_full(slot), (li / NM) & 1, abort_flag)) {
                ok = false;
                break;
            }
            const ItemMeta& mref = metas[slot];
            const int valid = mref.valid, lidx = mref.lidx, n = mref.n;
            const int tokr = tt < MT ? mref.tok[tt] : 0;
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar.meta_empty(slot));
            if (!valid) break;
            const bool row_valid = tt < n;
            const int j = lidx % nb_all;
            const int t = a.s.q0 + pair_query(tokr);
            const int sb = li & 1;
            if (!bm_warp_wait(bar.s_full(sb), (li >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            uint32_t sv[BLK];
            tc::tmem_ld32(tS(sb) + lane_off, sv);
            tc::tmem_ld32(tS(sb) + lane_off + 32, sv + 32);
            tc::tmem_wait_ld();
            // visible offsets: the whole block, or u <= t inside the query's own block
            const int hi = row_valid ? min(BLK - 1, t - j * BLK) : -1;
            float m = 0.f, l = 0.f;
            // P = 2^(s*scale*log2e - m) / l, normalised before the P V product so
            // the partial o comes out of the MMA already divided by l.  Specialised
            // on whether any row of the warp needs the causal mask (only items on
            // a query's own block do).
            auto softmax_row = [&](auto masked_tag) {
                constexpr bool MASKED = decltype(masked_tag)::value;
                float mx[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
#pragma unroll
                for (int k = 0; k < BLK; ++k) {
                    float x = __uint_as_float(sv[k]);
                    if (MASKED) {
                        x = k <= hi ? x : -INFINITY;
                        sv[k] = __float_as_uint(x);
                    }
                    mx[k & 7] = fmaxf(mx[k & 7], x);
                }
                const float m_raw = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                          fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                m = m_raw == -INFINITY ? 0.f : m_raw * a.scale_log2;
                float ps[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) ps[q] = 0.f;
#pragma unroll
                for (int k = 0; k < BLK; ++k) {
                    const float pk = tc::ex2(fmaf(__uint_as_float(sv[k]), a.scale_log2, -m));
                    ps[k & 7] += pk;
                    sv[k] = __float_as_uint(pk);
                }
                l = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
                for (int k = 0; k < BLK; k += 2)
                    sv[k >> 1] = tc::pack_bf16x2(__uint_as_float(sv[k]) * inv,
                                                 __uint_as_float(sv[k + 1]) * inv);
            };
            if (__all_sync(0xffffffffu, hi == BLK - 1))
                softmax_row(std::false_type{});
            else
                softmax_row(std::true_type{});
            // (m, l) of this item's rows go to the epilogue through shared memory;
            // buffer sb is free once the epilogue of item li - 2 has released it
            // (o_free); the p_full arrival below orders these writes before PV(li)
            // and hence before the epilogue reads them
            if (li >= 2 && !bm_warp_wait(bar.o_free(sb), ((li >> 1) & 1) ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            row_m[sb * BM + r] = m;
            row_l[sb * BM + r] = l;
            tc::tmem_st32(tS(sb) + lane_off, sv);
            tc::tmem_wait_st();
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar.p_full(sb));
        }
        if (!ok) bm_abort(abort_flag);
    } else if (warp >= 10 && warp < 14) {
        // ------------------------------------------------------------ epilogue (warps 10-13,
        // every item): o = P V (already divided by l) -> bf16 partial rows, staged in
        // shared memory in the 128-byte-swizzled layout and written by TMA stores
        // (one {64 columns x hpt rows} box per query and column half, whole lines
        // instead of a 256-byte row per lane); lse = m + log2(l) per row.  A warp's 32
        // rows are whole queries, so each warp stores its own queries' rows as soon as
        // it has staged them (warp-level ordering only; the stores of an item are
        // spread over the four warps).  The four warps decide every wait together
        // (barrier reduction), so none of them can be left alone at a named barrier.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int tt = r / a.hpt, hl = r % a.hpt;
        const float* row_m = reinterpret_cast<const float*>(sm + L::ROW_OFF);
        const float* row_l = row_m + 2 * BM;
        // queries whose rows this warp holds: qpw of them, one store per lane l < qpw
        // (one head per query: lanes 0..7 store four rows each with one scatter)
        const int qpw = MT > 32 ? 32 : 32 / a.hpt;
        const uint64_t st_policy = tc::l2_policy_evict_first();
        uint32_t halves = 0;
        bool ok = true;
        for (int li = 0;; ++li) {
            const int slot = li % NM;
            bool okw = bm_warp_wait(bar.meta_full(slot), (li / NM) & 1, abort_flag);
            int valid = 0, lidx = 0, n = 0, tokr = 0;
            int tok_lane[4];              // the queries whose stores this lane issues
#pragma unroll
            for (int g = 0; g < 4; ++g) tok_lane[g] = 0;
            if (okw) {
                const ItemMeta& mref = metas[slot];
                valid = mref.valid;
                lidx = mref.lidx;
                n = mref.n;
                tokr = tt < MT ? mref.tok[tt] : 0;
                // lane l of warp quarter w: query w * qpw + l (groups of heads), or
                // rows 32 w + 4 l .. 32 w + 4 l + 3 (one head per query, lanes 0..7)
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const int qi = MT > 32 ? 32 * quarter + 4 * lane + g : quarter * qpw + lane;
                    const bool mine = MT > 32 ? lane < 8 : (g == 0 && lane < qpw);
                    tok_lane[g] = mine && qi < MT ? mref.tok[qi] : 0;
                }
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar.meta_empty(slot));
            }
            if (!tc::named_bar_and(1, 128, okw)) {
                ok = false;
                break;
            }
            if (!valid) break;
            const int sb = li & 1;
            okw = bm_warp_wait(bar.o_full(sb), (li >> 1) & 1, abort_flag) &&
                  // acquire the softmax warpgroup's (m, l) writes directly from its
                  // p_full arrival (already complete, since o_full implies it)
                  bm_warp_wait(bar.p_full(sb), (li >> 1) & 1, abort_flag);
            if (!tc::named_bar_and(1, 128, okw)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
            const bool row_valid = tt < n;
            const int bu = (lidx / nb_all) % bhsel;
            const float m = row_m[sb * BM + r], l = row_l[sb * BM + r];
            const size_t prow = (((size_t)bu * a.s.Tq + pair_query(tokr)) * a.s.topk + pair_slot(tokr)) * a.hpt + hl;
            // first partial row of each query this lane stores
            int prow_q[4];
#pragma unroll
            for (int g = 0; g < 4; ++g)
                prow_q[g] = (int)((((size_t)bu * a.s.Tq + pair_query(tok_lane[g])) * a.s.topk + pair_slot(tok_lane[g])) *
                                  a.hpt);
#pragma unroll 1
            for (int c = 0; c < DV; c += 64, ++halves) {
                uint32_t o[64];
                tc::tmem_ld32(tO(sb) + lane_off + c, o);
                tc::tmem_ld32(tO(sb) + lane_off + c + 32, o + 32);
                tc::tmem_wait_ld();
                if (c + 64 == DV) {
                    // every column of O(sb) is in registers: MMA may reuse the buffer
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar.o_free(sb));
                }
                // staging buffer (halves & 1) was last read by the stores this warp
                // issued two halves ago; at most the latest group may still be reading
                tc::bulk_wait_read<1>();
                __syncwarp();
                uint8_t* rowp = sm + L::STG_OFF + (halves & 1) * (BM * 128) + r * 128;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 u4;
                    u4.x = tc::pack_bf16x2(__uint_as_float(o[8 * q + 0]), __uint_as_float(o[8 * q + 1]));
                    u4.y = tc::pack_bf16x2(__uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3]));
                    u4.z = tc::pack_bf16x2(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5]));
                    u4.w = tc::pack_bf16x2(__uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7]));
                    *reinterpret_cast<uint4*>(rowp + ((q ^ (r & 7)) << 4)) = u4;
                }
                tc::fence_proxy_async_smem();
                __syncwarp();
                uint8_t* stg = sm + L::STG_OFF + (halves & 1) * (BM * 128);
                if constexpr (MT > 32) {
                    const int r0 = 32 * quarter + 4 * lane;          // this lane's four rows
                    if (lane < 8) {
                        if (r0 + 3 < n) {
                            tc::tma_scatter4(&map_po, stg + r0 * 128, c, prow_q[0], prow_q[1], prow_q[2],
                                             prow_q[3]);
                        } else {
#pragma unroll
                            for (int g = 0; g < 4; ++g)
                                if (r0 + g < n) tc::tma_store_2d_hint(&map_po, stg + (r0 + g) * 128, c, prow_q[g],
                                                                      st_policy);
                        }
                    }
                } else {
                    const int qi = quarter * qpw + lane;
                    if (lane < qpw && qi < n)
                        tc::tma_store_2d_hint(&map_po, stg + qi * a.hpt * 128, c, prow_q[0], st_policy);
                }
                tc::bulk_commit();
            }
            if (row_valid) __stcs(a.part_lse + prow, m + __log2f(l));
        }
        tc::bulk_wait<0>();
        if (!ok) bm_abort(abort_flag);
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 bm_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
            const cuuint64_t* strides, const cuuint32_t* box) {
    auto enc = bm_encode_fn();
    if (!enc) return false;
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int DQK, int DV, int MT>
cudaError_t launch_bm_impl(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const SelIndex& x, __nv_bfloat16* part_o,
                           float* part_lse, cudaStream_t st) {
    BmArgs a;
    a.s = s;
    a.items = x.items;
    a.item_off = x.item_off;
    a.n_chunks = sel_chunks(s);
    a.lists_per_chunk = (int)sel_lists_per_chunk(s);
    a.list = x.list;
    a.part_o = part_o;
    a.part_lse = part_lse;
    a.hpt = s.heads_per_unit;
    a.tok = BM / a.hpt;
    a.scale_log2 = s.scale * 1.4426950408889634f;
    CUtensorMap mq, mk, mv;
    const cuuint64_t qd[4] = {(cuuint64_t)DQK, (cuuint64_t)s.Hq, (cuuint64_t)s.Tq, (cuuint64_t)s.B};
    const cuuint64_t qs[3] = {(cuuint64_t)DQK * 2, (cuuint64_t)DQK * 2 * s.Hq,
                              (cuuint64_t)DQK * 2 * s.Hq * s.Tq};
    const cuuint32_t qb[4] = {64, (cuuint32_t)a.hpt, 1, 1};
    const cuuint64_t kd[3] = {(cuuint64_t)DQK, (cuuint64_t)s.Tk, (cuuint64_t)s.B * s.Hkv};
    const cuuint64_t ks[2] = {(cuuint64_t)DQK * 2, (cuuint64_t)DQK * 2 * s.Tk};
    const cuuint64_t vd[3] = {(cuuint64_t)DV, (cuuint64_t)s.Tk, (cuuint64_t)s.B * s.Hkv};
    const cuuint64_t vs[2] = {(cuuint64_t)DV * 2, (cuuint64_t)DV * 2 * s.Tk};
    const cuuint32_t kb[3] = {64, (cuuint32_t)BLK, 1};
    // partial rows [B * Hsel * Tq * topk * hpt, DV] written in {64, hpt} boxes
    CUtensorMap mpo;
    const cuuint64_t pd[2] = {(cuuint64_t)DV, (cuuint64_t)sel_partial_rows(s)};
    const cuuint64_t ps[1] = {(cuuint64_t)DV * 2};
    const cuuint32_t pb[2] = {64, (cuuint32_t)a.hpt};
    // one head per query: q as [B * Tq * Hq rows, DQK], one-row boxes for the 4-row gathers
    const cuuint64_t qd2[2] = {(cuuint64_t)DQK, (cuuint64_t)s.B * s.Tq * s.Hq};
    const cuuint64_t qs2[1] = {(cuuint64_t)DQK * 2};
    const cuuint32_t qb2[2] = {64, 1};
    const bool q_ok = MT > 32 ? encode(&mq, q, 2, qd2, qs2, qb2) : encode(&mq, q, 4, qd, qs, qb);
    if (!q_ok || !encode(&mk, k, 3, kd, ks, kb) ||
        !encode(&mv, v, 3, vd, vs, kb) || !encode(&mpo, part_o, 2, pd, ps, pb))
        return cudaErrorInvalidValue;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int smem = BmSmem<DQK, DV, MT>::ALLOC;
    static_assert(BmSmem<DQK, DV, MT>::ALLOC <= 232448, "shared memory");
    cudaError_t e = cudaFuncSetAttribute(sel_bm_kernel<DQK, DV, MT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    sel_bm_kernel<DQK, DV, MT><<<nsm, NTHREADS, smem, st>>>(mq, mk, mv, mpo, a);
    return cudaGetLastError();
}

}  // namespace

bool sel_bm_supported(const Shape& s) {
    if (!(s.flags & NSA_BR_SEL)) return false;
    if (s.dqk != 64 && s.dqk != 128 && s.dqk != 192) return false;
    if (s.dv != 64 && s.dv != 128) return false;
    if (s.bs != BLK) return false;
    const int hpt = s.heads_per_unit;
    // a slot is SEL_SLOT_BITS of a list entry; the merge of groups takes up to 16 slots
    // (one head per query: q rows are gathered by a 32-bit row index)
    const bool shape_ok = ((hpt == 8 || hpt == 16) && s.topk <= 16) ||
                          (hpt == 1 && s.topk <= SEL_SLOTS && (size_t)s.B * s.Tq * s.Hq < (size_t(1) << 31));
    if (s.Tq >= (1 << (31 - SEL_SLOT_BITS))) return false;       // list entries are int32
    // partial rows are addressed by 32-bit TMA coordinates
    return shape_ok && sel_partial_rows(s) < (size_t(1) << 31);
}

cudaError_t launch_sel_bm(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const SelIndex& x, __nv_bfloat16* part_o,
                          float* part_lse, cudaStream_t st) {
#define NSA_BM_CASE(A, B)                                                              \
    if (s.dqk == A && s.dv == B)                                                       \
        return s.heads_per_unit == 1 ? launch_bm_impl<A, B, 128>(s, q, k, v, x, part_o, part_lse, st) \
                                     : launch_bm_impl<A, B, 16>(s, q, k, v, x, part_o, part_lse, st);
    NSA_BM_CASE(64, 64)
    NSA_BM_CASE(128, 128)
    NSA_BM_CASE(192, 128)
    NSA_BM_CASE(64, 128)
    NSA_BM_CASE(128, 64)
    NSA_BM_CASE(192, 64)
#undef NSA_BM_CASE
    return cudaErrorInvalidValue;
}

int read_and_clear_bm_status() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_bm_status, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_bm_status, &zero, sizeof(int));
    return v;
}

}  // namespace nsa
