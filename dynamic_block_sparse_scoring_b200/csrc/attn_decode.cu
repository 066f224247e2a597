// Few-query attention (decode) on tcgen05 with the keys as the MMA M dimension.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention": a query attends over the compressed tokens, the tokens of its
// kept blocks and its sliding window, one softmax per branch, and the three
// outputs are summed with per-head gates; §5 "Hardware Makes Sparsity Work":
// the heads of a GQA group share those keys.  At decode a (sequence, group)
// has one query token, i.e. G query rows.  A query-major tile would stack them
// as 16 of 128 MMA rows and pay the softmax of all 128; here the roles are
// transposed instead:
//
//   S^T = K Q^T     M = 128 keys of a tile, N = 16 (the group's heads), K = d_qk
//   O^T += V^T P^T  M = d_v = 128,          N = 16,                    K = 128 keys
//
// so a softmax thread owns one key and sees its 16 head scores, and a tile
// costs 16 exponentials per thread.  The per-head maxima are reduced across
// the 128 key threads; the running sums stay per thread (scaled on the rare
// rescale) and are reduced once per work item.
//
// Work item = (sequence, unit, query, branch, range of 128-key tiles).
// Compressed and window tiles are contiguous key ranges; a selected tile is
// two 64-key segments of the kept blocks.  Each item writes a partial result
// per head (o = O/l in fp32, lse = m + log2 l); dec_merge_kernel combines the
// items of a branch with the log-sum-exp rule and sums the branches with the
// gates.  CTAs are persistent and take items round-robin.
//
// Roles (192 threads): warp 0 TMA producer, warp 1 MMA lane + TMEM owner,
// warps 2-5 softmax and epilogue (TMEM lane quarter = warp % 4).  Every wait
// is bounded; a timeout records NSA_ERR_TIMEOUT in g_dec_status and unwinds.
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace nsa {

__device__ int g_dec_status = 0;

namespace {

constexpr int DT = 128;             // keys per tile
constexpr int NH = 16;              // MMA N: query rows (heads of one token), padded to 16
constexpr int DV = 128;             // value width = MMA M of O^T
constexpr int NTHREADS = 192;
constexpr int CH = DT * 128;        // one 64-column chunk of a 128-key tile (16 KB)
constexpr int QCH = NH * 128;       // one 64-column chunk of the 16 query rows (2 KB)
constexpr int PCH = NH * 128;       // one 64-key chunk of P^T (2 KB)
constexpr uint64_t WAIT_NS = 1000000000ull;

enum { B_CMP = 0, B_SEL = 1, B_WIN = 2 };

struct DecArgs {
    Shape s;
    const int32_t* idx;
    float* part_o;      // [items][NH][DV]
    float* part_lse;    // [items][NH]
    int hpt;
    int tpi;            // tiles per item
    int ni[3];          // items per unit and branch (0 = branch off)
    int ni_all;
    int n_items;
    int spb;            // 64-key segments per selection block
    float scale_log2;
};

constexpr int NKS = 3;              // K stages (released when QK completes)
constexpr int NVS = 2;              // V stages (released when PV completes)

template <int DQK>
struct DecSmem {
    static constexpr int QC = DQK / 64;
    static constexpr int K_OFF = 0;                             // NKS stages x QC chunks
    static constexpr int V_OFF = K_OFF + NKS * QC * CH;         // NVS stages x 2 chunks
    static constexpr int Q_OFF = V_OFF + NVS * 2 * CH;          // 2 buffers x QC chunks
    static constexpr int P_OFF = Q_OFF + 2 * QC * QCH;          // 1 buffer x 2 chunks
    static constexpr int RED_OFF = P_OFF + 2 * PCH;             // [3][4 warps][NH] fp32
    static constexpr int BAR_OFF = RED_OFF + 3 * 4 * NH * 4;
    // q_full[2] q_empty[2] k_full[3] k_empty[3] v_full[2] v_empty[2] s_full[2] s_free[2]
    // p_full pv_done o_full o_free
    static constexpr int NBAR = 22;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int ALLOC = MISC_OFF + 64 + 1024;
    static_assert(ALLOC <= 232448, "shared memory");
};

struct DecBars {
    uint64_t* b;
    __device__ __forceinline__ uint64_t* q_full(int i) const { return b + i; }
    __device__ __forceinline__ uint64_t* q_empty(int i) const { return b + 2 + i; }
    __device__ __forceinline__ uint64_t* k_full(int i) const { return b + 4 + i; }
    __device__ __forceinline__ uint64_t* k_empty(int i) const { return b + 7 + i; }
    __device__ __forceinline__ uint64_t* v_full(int i) const { return b + 10 + i; }
    __device__ __forceinline__ uint64_t* v_empty(int i) const { return b + 12 + i; }
    __device__ __forceinline__ uint64_t* s_full(int i) const { return b + 14 + i; }
    __device__ __forceinline__ uint64_t* s_free(int i) const { return b + 16 + i; }
    __device__ __forceinline__ uint64_t* p_full() const { return b + 18; }
    __device__ __forceinline__ uint64_t* pv_done() const { return b + 19; }
    __device__ __forceinline__ uint64_t* o_full() const { return b + 20; }
    __device__ __forceinline__ uint64_t* o_free() const { return b + 21; }
};

// What one work item covers; every role derives it the same way.
struct Item {
    int b, u, i, t;     // sequence, selection unit, query row, query position
    int br;             // B_CMP / B_SEL / B_WIN
    int t0, t1;         // tile range [t0, t1) (empty when t0 >= t1)
    int n_vis;          // compressed: visible tokens
    int win_lo;         // window: first key
    int nseg;           // selected: 64-key segments of the kept blocks
    const int32_t* irow;
    int blk_lane;       // warp form: lane e holds kept block e (selected items)
};

// `warp_form`: called by a whole warp, which reads the query's kept blocks
// once (one coalesced load, lane e = block e) instead of one load per use.
__device__ __forceinline__ Item item_info(const DecArgs& a, int item, bool warp_form = false) {
    const Shape& s = a.s;
    Item it;
    const int unit = item / a.ni_all;
    int k = item % a.ni_all;
    it.i = unit % s.Tq;
    const int bu = unit / s.Tq;
    it.u = bu % s.Hsel;
    it.b = bu / s.Hsel;
    it.t = s.q0 + it.i;
    it.br = k < a.ni[0] ? B_CMP : (k < a.ni[0] + a.ni[1] ? B_SEL : B_WIN);
    const int sub = it.br == B_CMP ? k : (it.br == B_SEL ? k - a.ni[0] : k - a.ni[0] - a.ni[1]);
    it.n_vis = 0;
    it.win_lo = 0;
    it.nseg = 0;
    it.irow = nullptr;
    it.blk_lane = -1;
    int ntiles = 0;
    if (it.br == B_CMP) {
        it.n_vis = it.t >= s.lc - 1 ? min((it.t - s.lc + 1) / s.sc + 1, s.n_cmp) : 0;
        ntiles = (it.n_vis + DT - 1) / DT;
    } else if (it.br == B_SEL) {
        it.irow = a.idx + (((size_t)it.b * s.Hsel + it.u) * s.Tq + it.i) * s.topk;
        int nv = 0;
        if (warp_form) {
            const int lane = threadIdx.x & 31;
            it.blk_lane = lane < s.topk ? it.irow[lane] : -1;
            nv = __popc(__ballot_sync(0xffffffffu, it.blk_lane >= 0));
        } else {
            for (int e = 0; e < s.topk; ++e) nv += it.irow[e] >= 0 ? 1 : 0;
        }
        it.nseg = nv * a.spb;
        ntiles = (it.nseg + 1) / 2;
    } else {
        it.win_lo = max(0, it.t - s.win + 1);
        ntiles = (it.t - it.win_lo + 1 + DT - 1) / DT;
    }
    it.t0 = sub * a.tpi;
    it.t1 = min(ntiles, it.t0 + a.tpi);
    return it;
}

// Item id of this CTA's k-th work item, or -1 past the last.  The items are
// taken branch by branch (every compressed item, then the selected, then the
// window ones, each in unit order) and dealt to the CTAs back and forth
// (0 .. G-1, G-1 .. 0, ...), so that every CTA gets a near-equal number of
// tiles: the compressed and selected items are the long ones.  The id itself
// stays unit-major (unit * ni_all + branch offset + sub-range), which is how
// the partials are laid out for the merge.
__device__ __forceinline__ int item_at(const DecArgs& a, int k) {
    const int G = gridDim.x, c = blockIdx.x;
    const int p = (k >> 1) * 2 * G + ((k & 1) ? 2 * G - 1 - c : c);
    if (p >= a.n_items) return -1;
    const int units = a.n_items / a.ni_all;
    int q = p, off = 0;
    for (int br = 0; br < 3; ++br) {
        const int nb = units * a.ni[br];
        if (q < nb) return (q / a.ni[br]) * a.ni_all + off + q % a.ni[br];
        q -= nb;
        off += a.ni[br];
    }
    return -1;
}

// First key of 64-key segment e of a selected item (kept blocks ascending, -1
// padded last), from the warp-form block list; every lane of the warp calls it.
__device__ __forceinline__ int seg_start(const DecArgs& a, const Item& it, int e) {
    const int blk = __shfl_sync(0xffffffffu, it.blk_lane, (e / a.spb) & 31);
    return blk * a.s.bs + (e % a.spb) * 64;
}

__device__ __forceinline__ bool dec_warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, tc::mbar_wait(b, parity, abort_flag, WAIT_NS));
}

__device__ __forceinline__ void dec_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_dec_status, (int)NSA_ERR_TIMEOUT);
}

// order-preserving int image of a float (for redux.sync.max)
__device__ __forceinline__ int f2ord(float x) {
    const int i = __float_as_int(x);
    return i >= 0 ? i : i ^ 0x7fffffff;
}
__device__ __forceinline__ float ord2f(int i) { return __int_as_float(i >= 0 ? i : i ^ 0x7fffffff); }

__device__ __forceinline__ int warp_max_i(int v) {
    int r;
    asm volatile("redux.sync.max.s32 %0, %1, 0xffffffff;" : "=r"(r) : "r"(v));
    return r;
}

template <int DQK>
__global__ void __launch_bounds__(NTHREADS, 1)
    dec_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k128,
               const __grid_constant__ CUtensorMap map_v128, const __grid_constant__ CUtensorMap map_k64,
               const __grid_constant__ CUtensorMap map_v64, const __grid_constant__ CUtensorMap map_kc,
               const __grid_constant__ CUtensorMap map_vc, const DecArgs a) {
    using L = DecSmem<DQK>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    DecBars bar{reinterpret_cast<uint64_t*>(sm + L::BAR_OFF)};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC_OFF + 8);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar.q_full(i), 1);
            tc::mbar_init(bar.q_empty(i), 1);
            tc::mbar_init(bar.v_full(i), 1);
            tc::mbar_init(bar.v_empty(i), 1);
            tc::mbar_init(bar.s_full(i), 1);
            tc::mbar_init(bar.s_free(i), 4);
        }
        for (int i = 0; i < NKS; ++i) {
            tc::mbar_init(bar.k_full(i), 1);
            tc::mbar_init(bar.k_empty(i), 1);
        }
        tc::mbar_init(bar.p_full(), 4);
        tc::mbar_init(bar.pv_done(), 1);
        tc::mbar_init(bar.o_full(), 1);
        tc::mbar_init(bar.o_free(), 4);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 64);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    auto tS = [&](int i) { return tmem + 16 * i; };   // S^T buffers: columns [0,16) [16,32)
    const uint32_t tO = tmem + 32;                      // O^T: columns [32,48)

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // K of tile n is loaded as soon as QK(n - NKS) has completed; V of tile n
        // is issued after K of tile n + 1, so the value loads never hold back
        // the key loads that the MMA needs first.
        bool ok = true;
        uint32_t kcount = 0, vcount = 0, qcount = 0;
        struct VJob {
            int cmp, sel, row0, row1, plane;
        } pend{0, 0, 0, 0, -1};
        auto issue_v = [&](const VJob& v) -> bool {
            const int vs = vcount & 1;
            if (!dec_warp_wait(bar.v_empty(vs), ((vcount >> 1) & 1) ^ 1, abort_flag)) return false;
            uint8_t* vst = sm + L::V_OFF + vs * 2 * CH;
            if (v.sel) {
                if (lane == 0) tc::mbar_arrive_expect_tx(bar.v_full(vs), 2 * CH);
                __syncwarp();
                if (lane < 4) {
                    const int h = lane >> 1, c = lane & 1;
                    tc::tma_load_3d(vst + c * CH + h * (CH / 2), &map_v64, bar.v_full(vs), 64 * c,
                                    h ? v.row1 : v.row0, v.plane);
                }
            } else {
                if (lane == 0) tc::mbar_arrive_expect_tx(bar.v_full(vs), 2 * CH);
                __syncwarp();
                if (lane < 2)
                    tc::tma_load_3d(vst + lane * CH, v.cmp ? &map_vc : &map_v128, bar.v_full(vs), 64 * lane,
                                    v.row0, v.plane);
            }
            ++vcount;
            return true;
        };
        for (int k = 0, item; ok && (item = item_at(a, k)) >= 0; ++k) {
            const Item it = item_info(a, item, true);
            if (it.t0 >= it.t1) continue;
            const int plane = it.b * s.Hkv + it.u;   // group-shared selection: unit = KV head
            const int qb = qcount & 1;
            if (!dec_warp_wait(bar.q_empty(qb), ((qcount >> 1) & 1) ^ 1, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) tc::mbar_arrive_expect_tx(bar.q_full(qb), L::QC * a.hpt * 128);
            __syncwarp();
            if (lane < L::QC)
                tc::tma_load_4d(sm + L::Q_OFF + (qb * L::QC + lane) * QCH, &map_q, bar.q_full(qb),
                                64 * lane, it.u * a.hpt, it.i, it.b);
            ++qcount;
            for (int j = it.t0; j < it.t1; ++j) {
                VJob cur{it.br == B_CMP, it.br == B_SEL, 0, 0, plane};
                if (it.br == B_SEL) {
                    // an odd last segment is paired with itself (masked by the softmax),
                    // so that a stage never holds stale or uninitialised rows
                    const int e1 = 2 * j + 1;
                    cur.row0 = seg_start(a, it, 2 * j);
                    const int s1 = seg_start(a, it, e1);
                    cur.row1 = e1 < it.nseg ? s1 : cur.row0;
                } else {
                    cur.row0 = cur.cmp ? j * DT : it.win_lo + j * DT;
                }
                const int ks = kcount % NKS;
                if (!dec_warp_wait(bar.k_empty(ks), ((kcount / NKS) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* kst = sm + L::K_OFF + ks * L::QC * CH;
                if (lane == 0) tc::mbar_arrive_expect_tx(bar.k_full(ks), L::QC * CH);
                __syncwarp();
                if (cur.sel) {
                    if (lane < 2 * L::QC) {
                        const int h = lane / L::QC, c = lane % L::QC;
                        tc::tma_load_3d(kst + c * CH + h * (CH / 2), &map_k64, bar.k_full(ks), 64 * c,
                                        h ? cur.row1 : cur.row0, plane);
                    }
                } else if (lane < L::QC) {
                    tc::tma_load_3d(kst + lane * CH, cur.cmp ? &map_kc : &map_k128, bar.k_full(ks), 64 * lane,
                                    cur.row0, plane);
                }
                ++kcount;
                if (pend.plane >= 0 && !issue_v(pend)) {
                    ok = false;
                    break;
                }
                pend = cur;
            }
        }
        if (ok && pend.plane >= 0 && !issue_v(pend)) ok = false;
        if (!ok) dec_abort(abort_flag);
        // wait for every copy still in flight before the CTA may exit
        for (uint32_t st = 0; st < NKS; ++st)
            if (kcount > st) {
                const uint32_t last = st + ((kcount - 1 - st) / NKS) * NKS;
                tc::mbar_wait_bounded(bar.k_full(st), (last / NKS) & 1, WAIT_NS);
            }
        for (uint32_t st = 0; st < 2; ++st) {
            if (vcount > st) {
                const uint32_t last = st + ((vcount - 1 - st) / 2) * 2;
                tc::mbar_wait_bounded(bar.v_full(st), (last >> 1) & 1, WAIT_NS);
            }
            if (qcount > st) {
                const uint32_t last = st + ((qcount - 1 - st) / 2) * 2;
                tc::mbar_wait_bounded(bar.q_full(st), (last >> 1) & 1, WAIT_NS);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc_qk = tc::idesc_bf16_f32(DT, NH, false, false);
            const uint32_t idesc_pv = tc::idesc_bf16_f32(DV, NH, true, false);
            const uint32_t k_base = tc::smem_u32(sm + L::K_OFF);
            const uint32_t v_base = tc::smem_u32(sm + L::V_OFF);
            const uint32_t q_base = tc::smem_u32(sm + L::Q_OFF);
            const uint32_t p_base = tc::smem_u32(sm + L::P_OFF);
            bool ok = true;
            uint32_t tcount = 0, qcount = 0, ocount = 0;
            // O^T += V^T P^T for tile n (V stage n & 1, the single P buffer)
            auto issue_pv = [&](uint32_t n, bool first) -> bool {
                const int vs = n & 1;
                if (!tc::mbar_wait(bar.p_full(), n & 1, abort_flag, WAIT_NS) ||
                    !tc::mbar_wait(bar.v_full(vs), (n >> 1) & 1, abort_flag, WAIT_NS))
                    return false;
                // the first PV of an item overwrites O: the previous item's epilogue must have read it
                if (first && ocount > 0 && !tc::mbar_wait(bar.o_free(), (ocount - 1) & 1, abort_flag, WAIT_NS))
                    return false;
                tc::fence_after_sync();
                const uint32_t vst = v_base + vs * 2 * CH;
#pragma unroll
                for (int kk = 0; kk < DT / 16; ++kk)
                    tc::mma_ss(tO, tc::sdesc_sw128(vst + kk * 2048, CH, 1024),
                               tc::sdesc_sw128(p_base + (kk >> 2) * PCH + (kk & 3) * 32, 16, 1024), idesc_pv,
                               (first && kk == 0) ? 0u : 1u);
                tc::mma_commit(bar.v_empty(vs));
                tc::mma_commit(bar.pv_done());
                return true;
            };
            for (int k = 0, item; ok && (item = item_at(a, k)) >= 0; ++k) {
                const Item it = item_info(a, item);
                if (it.t0 >= it.t1) continue;
                const int qb = qcount & 1;
                if (!tc::mbar_wait(bar.q_full(qb), (qcount >> 1) & 1, abort_flag, WAIT_NS)) {
                    ok = false;
                    break;
                }
                const uint32_t qst = q_base + qb * L::QC * QCH;
                for (int j = it.t0; j < it.t1; ++j, ++tcount) {
                    const int ks = tcount % NKS, sb = tcount & 1;
                    if (!tc::mbar_wait(bar.k_full(ks), (tcount / NKS) & 1, abort_flag, WAIT_NS) ||
                        (tcount >= 2 && !tc::mbar_wait(bar.s_free(sb), ((tcount >> 1) & 1) ^ 1, abort_flag, WAIT_NS))) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t kst = k_base + ks * L::QC * CH;
#pragma unroll
                    for (int kk = 0; kk < DQK / 16; ++kk)
                        tc::mma_ss(tS(sb), tc::sdesc_sw128(kst + (kk >> 2) * CH + (kk & 3) * 32, 16, 1024),
                                   tc::sdesc_sw128(qst + (kk >> 2) * QCH + (kk & 3) * 32, 16, 1024), idesc_qk,
                                   kk > 0 ? 1u : 0u);
                    tc::mma_commit(bar.s_full(sb));
                    tc::mma_commit(bar.k_empty(ks));
                    if (j == it.t1 - 1) tc::mma_commit(bar.q_empty(qb));
                    if (j > it.t0 && !issue_pv(tcount - 1, j - 1 == it.t0)) {
                        ok = false;
                        break;
                    }
                }
                if (!ok) break;
                if (!issue_pv(tcount - 1, it.t1 - 1 == it.t0)) {
                    ok = false;
                    break;
                }
                tc::mma_commit(bar.o_full());
                ++qcount;
                ++ocount;
            }
            if (!ok) dec_abort(abort_flag);
            // the last epilogue has read O (and every MMA before its commit completed)
            if (ocount > 0) tc::mbar_wait_bounded(bar.o_free(), (ocount - 1) & 1, WAIT_NS);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        // One vote barrier per tile: it publishes the warps' per-head maxima
        // (red[tile & 1]) and makes every wait's outcome uniform, so that all
        // four warps leave together if one of them timed out.
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;            // key of the tile; d_v lane of O^T
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* red = reinterpret_cast<float*>(sm + L::RED_OFF);     // [3][4][NH]
        uint8_t* pbuf = sm + L::P_OFF;
        const int wq = warp - 2;                      // 0..3, slot in red
        bool ok = true, ok_prev = true;
        uint32_t tcount = 0, ocount = 0;
        for (int k = 0, item; ok && (item = item_at(a, k)) >= 0; ++k) {
            const Item it = item_info(a, item, true);
            float* po = a.part_o + (size_t)item * NH * DV;
            float* pl = a.part_lse + (size_t)item * NH;
            if (it.t0 >= it.t1) {
                for (int h = 0; h < a.hpt; ++h) po[h * DV + r] = 0.f;
                if (r < NH) pl[r] = -INFINITY;
                continue;
            }
            float mrun[NH], lsum[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                mrun[h] = -INFINITY;
                lsum[h] = 0.f;
            }
            for (int j = it.t0; j < it.t1; ++j, ++tcount) {
                const int sb = tcount & 1;
                float* rt = red + sb * 4 * NH;
                // key of this thread and whether the query sees it
                bool valid;
                if (it.br == B_CMP) {
                    valid = j * DT + r < it.n_vis;
                } else if (it.br == B_SEL) {
                    const int e = 2 * j + (r >> 6);
                    const int st0 = seg_start(a, it, e);
                    valid = e < it.nseg && st0 + (r & 63) <= it.t;
                } else {
                    valid = it.win_lo + j * DT + r <= it.t;
                }
                bool okw = dec_warp_wait(bar.s_full(sb), (tcount >> 1) & 1, abort_flag);
                float x[NH];
                if (okw) {
                    tc::fence_after_sync();
                    uint32_t sv[NH];
                    tc::tmem_ld16(tS(sb) + lane_off, sv);
                    tc::tmem_wait_ld();
                    tc::fence_before_sync();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar.s_free(sb));
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        x[h] = (valid && h < a.hpt) ? __uint_as_float(sv[h]) * a.scale_log2 : -INFINITY;
                        const int m = warp_max_i(f2ord(x[h]));
                        if (lane == h) rt[wq * NH + h] = ord2f(m);
                    }
                }
                if (!tc::named_bar_and(1, 128, okw && ok_prev)) {
                    ok = false;
                    break;
                }
                // tile maxima; lazy rescale (only when a head's maximum grows by > 2^8)
                bool rescale = false;
                float alpha[NH];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float tm = fmaxf(fmaxf(rt[h], rt[NH + h]), fmaxf(rt[2 * NH + h], rt[3 * NH + h]));
                    alpha[h] = 1.f;
                    if (tm > mrun[h] + 8.f) {
                        alpha[h] = tc::ex2(mrun[h] - tm);      // 0 when mrun = -inf
                        mrun[h] = tm;
                        lsum[h] *= alpha[h];
                        rescale = true;
                    }
                }
                // the P buffer (and O, for a rescale) is free once PV of the previous tile completed
                ok_prev = tcount == 0 || dec_warp_wait(bar.pv_done(), (tcount - 1) & 1, abort_flag);
                if (ok_prev) {
                    if (rescale && j > it.t0) {
                        tc::fence_after_sync();
                        uint32_t ov[NH];
                        tc::tmem_ld16(tO + lane_off, ov);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int h = 0; h < NH; ++h) ov[h] = __float_as_uint(__uint_as_float(ov[h]) * alpha[h]);
                        tc::tmem_st16(tO + lane_off, ov);
                        tc::tmem_wait_st();
                    }
                    uint8_t* pb = pbuf + (r >> 6) * PCH;
                    const int unit16 = (r & 63) >> 3;
#pragma unroll
                    for (int h = 0; h < NH; ++h) {
                        const float p = x[h] == -INFINITY ? 0.f : tc::ex2(x[h] - mrun[h]);
                        lsum[h] += p;
                        *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((unit16 ^ (h & 7)) << 4) + (r & 7) * 2) =
                            __float2bfloat16_rn(p);
                    }
                    tc::fence_before_sync();
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) tc::mbar_arrive(bar.p_full());
                }
            }
            if (!ok) break;
            // epilogue: o = O^T / l per head, lse = m + log2 l
            bool okw = dec_warp_wait(bar.o_full(), ocount & 1, abort_flag);
            float* rs = red + 2 * 4 * NH;
            uint32_t ov[NH];
            if (okw) {
                tc::fence_after_sync();
                tc::tmem_ld16(tO + lane_off, ov);
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar.o_free());
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    const float v = warp_sum(lsum[h]);
                    if (lane == h) rs[wq * NH + h] = v;
                }
            }
            if (!tc::named_bar_and(1, 128, okw && ok_prev)) {
                ok = false;
                break;
            }
            ++ocount;
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                const float l = (rs[h] + rs[NH + h]) + (rs[2 * NH + h] + rs[3 * NH + h]);
                if (h < a.hpt) po[h * DV + r] = l > 0.f ? __uint_as_float(ov[h]) / l : 0.f;
                if (r == h) pl[h] = l > 0.f ? mrun[h] + __log2f(l) : -INFINITY;
            }
        }
        if (!ok) dec_abort(abort_flag);
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 64);
}

constexpr int MG_BATCH = 8;         // items of a branch whose loads the merge issues together

// out[b, i, h] = sum over branches of gate * (log-sum-exp merge of the branch's items)
__global__ void __launch_bounds__(256) dec_merge_kernel(Shape s, DecArgs a, const float* __restrict__ gates,
                                                        __nv_bfloat16* __restrict__ out) {
    const int c8n = DV / 8;
    const size_t total = (size_t)s.B * s.Tq * s.Hq * c8n;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int c8 = (int)(e % c8n);
        const size_t row = e / c8n;                  // (b, i, hq)
        const int hq = (int)(row % s.Hq);
        const int i = (int)((row / s.Hq) % s.Tq);
        const int b = (int)(row / ((size_t)s.Hq * s.Tq));
        const int u = hq / a.hpt, hl = hq % a.hpt;
        const size_t unit = ((size_t)b * s.Hsel + u) * s.Tq + i;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        int k0 = 0;
        for (int br = 0; br < 3; ++br) {
            const int n = a.ni[br];
            if (n == 0) continue;
            const size_t it0 = unit * a.ni_all + k0;
            k0 += n;
            float o[8] = {0, 0, 0, 0, 0, 0, 0, 0}, wsum = 0.f, m = -INFINITY;
            // up to MG_BATCH items of the branch: every load issued before any is used
            for (int kb = 0; kb < n; kb += MG_BATCH) {
                float lse[MG_BATCH];
                float4 x0[MG_BATCH], x1[MG_BATCH];
#pragma unroll
                for (int k = 0; k < MG_BATCH; ++k) {
                    lse[k] = -INFINITY;
                    if (kb + k < n) {
                        lse[k] = a.part_lse[(it0 + kb + k) * NH + hl];
                        const float4* src =
                            reinterpret_cast<const float4*>(a.part_o + ((it0 + kb + k) * NH + hl) * DV + c8 * 8);
                        x0[k] = src[0];
                        x1[k] = src[1];
                    }
                }
                float mb = m;
#pragma unroll
                for (int k = 0; k < MG_BATCH; ++k) mb = fmaxf(mb, lse[k]);
                if (mb == -INFINITY) continue;          // nothing visible so far
                // rescale what earlier batches accumulated to the new maximum
                const float sc = m == -INFINITY ? 0.f : exp2f(m - mb);
                wsum *= sc;
#pragma unroll
                for (int q = 0; q < 8; ++q) o[q] *= sc;
                m = mb;
#pragma unroll
                for (int k = 0; k < MG_BATCH; ++k) {
                    if (kb + k >= n) break;
                    const float w = exp2f(lse[k] - m);    // 0 for an empty item (lse = -inf)
                    wsum += w;
                    o[0] = fmaf(w, x0[k].x, o[0]); o[1] = fmaf(w, x0[k].y, o[1]);
                    o[2] = fmaf(w, x0[k].z, o[2]); o[3] = fmaf(w, x0[k].w, o[3]);
                    o[4] = fmaf(w, x1[k].x, o[4]); o[5] = fmaf(w, x1[k].y, o[5]);
                    o[6] = fmaf(w, x1[k].z, o[6]); o[7] = fmaf(w, x1[k].w, o[7]);
                }
            }
            if (m == -INFINITY) continue;                // empty branch: o = 0
            const float g = gates ? gates[row * 3 + br] : 1.f;
            const float f = g / wsum;
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(f, o[q], acc[q]);
        }
        *reinterpret_cast<uint4*>(out + row * DV + c8 * 8) = pack8(acc);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 dec_encode_fn() {
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

bool dec_encode(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                const cuuint64_t* strides, const cuuint32_t* box) {
    auto enc = dec_encode_fn();
    if (!enc) return false;
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

DecArgs make_args(const Shape& s, const int32_t* idx, float* part_o, float* part_lse) {
    DecArgs a;
    a.s = s;
    a.idx = idx;
    a.part_o = part_o;
    a.part_lse = part_lse;
    a.hpt = s.heads_per_unit;
    a.spb = s.bs / 64;
    a.scale_log2 = s.scale * 1.4426950408889634f;
    // most tiles any query of the problem has, per branch
    const int t_last = s.q0 + s.Tq - 1;
    const int cmp_tiles = (s.flags & NSA_BR_CMP) ? (s.n_cmp + DT - 1) / DT : 0;
    const int sel_tiles = (s.flags & NSA_BR_SEL) ? (s.topk * a.spb + 1) / 2 : 0;
    const int win_tiles = (s.flags & NSA_BR_WIN) ? (min(s.win, t_last + 1) + DT - 1) / DT : 0;
    const long units = (long)s.B * s.Hsel * s.Tq;
    const long tiles = units * (cmp_tiles + sel_tiles + win_tiles);
    // about ten items per SM
    a.tpi = (int)std::max<long>(1, std::min<long>(64, (tiles + 10 * 148 - 1) / (10 * 148)));
    a.ni[0] = (cmp_tiles + a.tpi - 1) / a.tpi;
    a.ni[1] = (sel_tiles + a.tpi - 1) / a.tpi;
    a.ni[2] = (win_tiles + a.tpi - 1) / a.tpi;
    a.ni_all = a.ni[0] + a.ni[1] + a.ni[2];
    a.n_items = (int)(units * a.ni_all);
    return a;
}

template <int DQK>
cudaError_t launch_dec_impl(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* kcmp, const __nv_bfloat16* vcmp,
                            const DecArgs& a, cudaStream_t st) {
    CUtensorMap mq, mk128, mv128, mk64, mv64, mkc, mvc;
    const cuuint64_t qd[4] = {(cuuint64_t)DQK, (cuuint64_t)s.Hq, (cuuint64_t)s.Tq, (cuuint64_t)s.B};
    const cuuint64_t qs[3] = {(cuuint64_t)DQK * 2, (cuuint64_t)DQK * 2 * s.Hq,
                              (cuuint64_t)DQK * 2 * s.Hq * s.Tq};
    const cuuint32_t qb[4] = {64, (cuuint32_t)a.hpt, 1, 1};
    const cuuint64_t kd[3] = {(cuuint64_t)DQK, (cuuint64_t)s.Tk, (cuuint64_t)s.B * s.Hkv};
    const cuuint64_t ks[2] = {(cuuint64_t)DQK * 2, (cuuint64_t)DQK * 2 * s.Tk};
    const cuuint64_t vd[3] = {(cuuint64_t)DV, (cuuint64_t)s.Tk, (cuuint64_t)s.B * s.Hkv};
    const cuuint64_t vs[2] = {(cuuint64_t)DV * 2, (cuuint64_t)DV * 2 * s.Tk};
    const cuuint32_t b128[3] = {64, (cuuint32_t)DT, 1};
    const cuuint32_t b64[3] = {64, 64, 1};
    if (!dec_encode(&mq, q, 4, qd, qs, qb) || !dec_encode(&mk128, k, 3, kd, ks, b128) ||
        !dec_encode(&mv128, v, 3, vd, vs, b128) || !dec_encode(&mk64, k, 3, kd, ks, b64) ||
        !dec_encode(&mv64, v, 3, vd, vs, b64))
        return cudaErrorInvalidValue;
    if ((s.flags & NSA_BR_CMP) && s.n_cmp > 0) {
        const cuuint64_t cd[3] = {(cuuint64_t)DQK, (cuuint64_t)s.n_cmp, (cuuint64_t)s.B * s.Hkv};
        const cuuint64_t cs[2] = {(cuuint64_t)DQK * 2, (cuuint64_t)DQK * 2 * s.n_cmp};
        const cuuint64_t cvd[3] = {(cuuint64_t)DV, (cuuint64_t)s.n_cmp, (cuuint64_t)s.B * s.Hkv};
        const cuuint64_t cvs[2] = {(cuuint64_t)DV * 2, (cuuint64_t)DV * 2 * s.n_cmp};
        if (!dec_encode(&mkc, kcmp, 3, cd, cs, b128) || !dec_encode(&mvc, vcmp, 3, cvd, cvs, b128))
            return cudaErrorInvalidValue;
    } else {
        mkc = mk128;      // never used: no compressed tile is enumerated
        mvc = mv128;
    }
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int smem = DecSmem<DQK>::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(dec_kernel<DQK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = std::min(nsm, a.n_items);
    dec_kernel<DQK><<<grid, NTHREADS, smem, st>>>(mq, mk128, mv128, mk64, mv64, mkc, mvc, a);
    return cudaGetLastError();
}

}  // namespace

bool attn_dec_supported(const Shape& s) {
    if (s.per_head) return false;
    if (s.dqk != 64 && s.dqk != 128 && s.dqk != 192) return false;
    if (s.dv != DV) return false;
    const int hpt = s.heads_per_unit;
    if (hpt != 8 && hpt != 16) return false;
    if ((s.flags & NSA_BR_SEL) && s.bs % 64 != 0) return false;
    return s.Tq >= 1 && s.Tq <= 4;
}

size_t attn_dec_items(const Shape& s) { return (size_t)make_args(s, nullptr, nullptr, nullptr).n_items; }
size_t attn_dec_part_floats() { return (size_t)NH * DV; }

cudaError_t launch_attn_dec(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* kcmp, const __nv_bfloat16* vcmp,
                            const int32_t* idx, float* part_o, float* part_lse, cudaStream_t st) {
    const DecArgs a = make_args(s, idx, part_o, part_lse);
    if (a.n_items == 0) return cudaSuccess;
    if (s.dqk == 64) return launch_dec_impl<64>(s, q, k, v, kcmp, vcmp, a, st);
    if (s.dqk == 128) return launch_dec_impl<128>(s, q, k, v, kcmp, vcmp, a, st);
    if (s.dqk == 192) return launch_dec_impl<192>(s, q, k, v, kcmp, vcmp, a, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_dec_merge(const Shape& s, const float* part_o, const float* part_lse,
                             const float* gates, __nv_bfloat16* out, cudaStream_t st) {
    DecArgs a = make_args(s, nullptr, const_cast<float*>(part_o), const_cast<float*>(part_lse));
    const size_t total = (size_t)s.B * s.Tq * s.Hq * (DV / 8);
    if (total == 0) return cudaSuccess;
    const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 8);
    dec_merge_kernel<<<grid, 256, 0, st>>>(s, a, gates, out);
    return cudaGetLastError();
}

int read_and_clear_dec_status() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_dec_status, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_dec_status, &zero, sizeof(int));
    return v;
}

}  // namespace nsa
