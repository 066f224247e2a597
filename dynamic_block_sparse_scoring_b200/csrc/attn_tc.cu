// Gated three-branch sparse attention on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), query-major.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention", Figure 2: compressed branch (pooled block tokens), selected
// branch (every token of the kept blocks), sliding-window branch; each
// branch output times its per-token gate, summed.  §5 "Hardware Makes
// Sparsity Work": the heads of a GQA group share their blocks, so they are
// stacked into the rows of one matrix product with the shared keys.
//
// A work tile is 128 query rows = TOK consecutive tokens x HPT heads that
// share their key/value head (HPT = the group for group-shared selection).
// Its key tiles are 128 keys made of two 64-key segments, each fetched by
// TMA straight from K/V (or the compressed K/V) into 128-byte-swizzled
// shared memory:
//   compressed branch - compressed tokens visible to the tile's last token;
//   selected branch   - the union of the tile tokens' selected blocks, every
//                       row masked to its own token's blocks;
//   window branch     - raw keys [t_first - window + 1, t_last].
// Per key tile: S = Q K^T (tcgen05.mma, both operands in smem, fp32 in
// TMEM); the softmax warpgroups (two threads per row) mask, track the
// running max (the reference max only moves when the row max grows by more
// than 2^8, so O rarely needs rescaling), writes P as bf16 over S in TMEM;
// O += P V (A operand from TMEM).  At a branch boundary the thread folds
// gate * O / l into an fp32 accumulator row in TMEM; the row is rounded to
// bf16 once at the end.
//
// Warp roles (384 threads): warp 0 TMA producer, warp 1 MMA issuer (one
// lane) and TMEM owner, warps 2-3 idle, warps 4-11 softmax/epilogue (two
// warpgroups, each thread half a row).  Warpgroup 0 hands registers to the
// softmax warpgroups (setmaxnreg), whose code would otherwise spill under the
// per-thread limit of a 384-thread CTA.  Persistent CTAs, one per SM.  Every wait is bounded; a timeout raises a CTA-wide abort, records
// NSA_ERR_TIMEOUT in g_tc_status, drains in-flight copies and MMAs, frees
// TMEM and returns.
#include <cudaTypedefs.h>
#include <math.h>

#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "tc.cuh"

namespace nsa {

__device__ int g_tc_status = 0;

namespace {

constexpr int BM = 128;          // query rows per work tile
constexpr int BN = 128;          // keys per key tile (two 64-key segments)
constexpr int SEG = 64;
constexpr int NS = 2;            // K/V pipeline stages
constexpr int NM = 8;            // key-tile descriptors in flight
constexpr int CHUNK = 16384;     // one 128-row x 64-column bf16 operand chunk
constexpr int HALF = 8192;       // one 64-row segment of a chunk
constexpr uint64_t WAIT_NS = 1000000000ull;   // 1 s per wait
constexpr int MAX_UNION = 1024;  // (tokens per tile) x top_k entries of the selected branch
constexpr int NTHREADS = 384;    // warpgroup 0: producer warp, MMA warp (+2 idle); two softmax warpgroups

enum { BR_CMP = 0, BR_SEL = 1, BR_WIN = 2, BR_END = 3 };

struct KeyTile {
    int br;
    int first;          // first key tile of its branch in this work tile
    int seg[2];         // key position of each 64-key segment, -1 = empty
    uint32_t member[2]; // selected branch: bit tt = token tt of the tile kept this segment
    int pad[2];
};

struct TcArgs {
    Shape s;
    const int32_t* idx;
    const float* gates;
    __nv_bfloat16* out;
    int tok;              // tokens per work tile
    int hpt;              // heads per work tile
    int n_tt;             // token tiles per (sequence, unit)
    int n_work;           // total work tiles
    float scale_log2;     // scale * log2(e)
    // selected branch computed block-major and merged: o_sel [B, Tq, Hq, d_v]
    // bf16 (ungated); null = the selected branch runs here over the union of
    // the tile's block sets
    const __nv_bfloat16* o_sel;
    // split-K (few work tiles, e.g. decode): each tile's key tiles are cut into
    // n_split contiguous shares processed by different CTAs; each writes, per row
    // and branch, o = O/l (fp32) and lse = m + log2(l) (scaled log2 units) to
    // split_o [B, Tq, Hq, 3, n_split, d_v] / split_lse [B, Tq, Hq, 3, n_split]
    // (lse = -inf: no key of that branch in this share), merged by
    // split_merge_kernel.  n_split = 1: no split, the gated output is written here.
    int n_split;
    float* split_o;
    float* split_lse;
};

template <int DQK, int DV>
struct Smem {
    static constexpr int QC = DQK / 64;
    static constexpr int VC = DV / 64;
    static constexpr int Q_OFF = 0;
    static constexpr int K_OFF = Q_OFF + QC * CHUNK;
    static constexpr int V_OFF = K_OFF + NS * QC * CHUNK;
    static constexpr int META_OFF = V_OFF + NS * VC * CHUNK;
    static constexpr int UNION_OFF = META_OFF + NM * (int)sizeof(KeyTile);
    static constexpr int XCH_OFF = UNION_OFF + MAX_UNION * 4;      // row max / sum exchange
    static constexpr int BAR_OFF = XCH_OFF + 6 * BM * 4 + 64;       // + pair status words
    // barriers: q_full, q_empty, k_full[NS], k_empty[NS], v_full[NS], v_empty[NS],
    // meta_full[NM], meta_empty[NM], s_full[2], p_full[2], pv_done[2], drain
    static constexpr int NBAR = 2 + 4 * NS + 2 * NM + 4 + 3;
    static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;
    static constexpr int BYTES = MISC_OFF + 64;
    static constexpr int ALLOC = BYTES + 1024;   // slack to align the base to 1024 B
};

// All barriers live at one shared-memory base; each accessor is a constant
// offset from it, so a role keeps one pointer live instead of twelve.
struct Bars {
    uint64_t* b;
    __device__ __forceinline__ uint64_t* q_full() const { return b; }
    __device__ __forceinline__ uint64_t* q_empty() const { return b + 1; }
    __device__ __forceinline__ uint64_t* k_full(int i) const { return b + 2 + i; }
    __device__ __forceinline__ uint64_t* k_empty(int i) const { return b + 2 + NS + i; }
    __device__ __forceinline__ uint64_t* v_full(int i) const { return b + 2 + 2 * NS + i; }
    __device__ __forceinline__ uint64_t* v_empty(int i) const { return b + 2 + 3 * NS + i; }
    __device__ __forceinline__ uint64_t* meta_full(int i) const { return b + 2 + 4 * NS + i; }
    __device__ __forceinline__ uint64_t* meta_empty(int i) const { return b + 2 + 4 * NS + NM + i; }
    __device__ __forceinline__ uint64_t* s_full(int i) const { return b + 2 + 4 * NS + 2 * NM + i; }
    __device__ __forceinline__ uint64_t* p_full(int i) const { return b + 4 + 4 * NS + 2 * NM + i; }
    // P V of key tile k completes pv_done(k & 1)
    __device__ __forceinline__ uint64_t* pv_done(int i) const { return b + 6 + 4 * NS + 2 * NM + i; }
    __device__ __forceinline__ uint64_t* drain() const { return b + 8 + 4 * NS + 2 * NM; }
};

__device__ __forceinline__ Bars make_bars(uint64_t* b) {
    Bars r;
    r.b = b;
    return r;
}

struct WorkTile {
    int b, unit, tt, kvh, h0, t0, ntok;
};

__device__ __forceinline__ WorkTile decode_work(const TcArgs& a, int w) {
    // heaviest (latest) token tiles first
    const int per_tt = a.s.B * a.s.Hsel;
    WorkTile t;
    t.tt = a.n_tt - 1 - w / per_tt;
    const int r = w % per_tt;
    t.b = r / a.s.Hsel;
    t.unit = r % a.s.Hsel;
    t.kvh = a.s.per_head ? t.unit / a.s.G : t.unit;
    t.h0 = a.s.per_head ? t.unit : t.unit * a.s.G;
    t.t0 = a.s.q0 + t.tt * a.tok;
    t.ntok = min(a.tok, a.s.Tq - t.tt * a.tok);
    return t;
}

// Limit of every wait on a copy, an MMA or another role (WAIT_NS unless a test
// shortened it through nsa_set_wait_limit_ns); the drains before TMEM is freed
// keep WAIT_NS.
__constant__ uint64_t c_wait_ns = WAIT_NS;

// Every lane waits (each acquires the barrier); the result is made warp-uniform
// so that a timeout seen by one lane unwinds the whole warp together.
__device__ __forceinline__ bool warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, tc::mbar_wait(b, parity, abort_flag, c_wait_ns));
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_tc_status, (int)NSA_ERR_TIMEOUT);
}

// ------------------------------------------------------------------ producer

template <int DQK, int DV>
struct Producer {
    using L = Smem<DQK, DV>;
    const TcArgs& a;
    uint8_t* sm;
    Bars bar;
    volatile int* abort_flag;
    const CUtensorMap* mq;
    const CUtensorMap* mk;
    const CUtensorMap* mv;
    const CUtensorMap* mkc;
    const CUtensorMap* mvc;
    uint32_t gm = 0, gk = 0;   // descriptors / key tiles issued so far
    int lane;

    bool prefetch_only = false;     // set for the L2 prefetch pass of a split share

    __device__ bool emit(const KeyTile& kt, const WorkTile& w) {
        if (prefetch_only) {
            if (kt.br == BR_END) return true;
            const bool cmp = kt.br == BR_CMP;
            const int plane = w.b * a.s.Hkv + w.kvh;
            const int e = lane;                   // one box per lane: 2 segments x (QC + VC) chunks
            const int per_seg = L::QC + L::VC;
            if (e < 2 * per_seg) {
                const int sg = e / per_seg, c = e % per_seg;
                const int row = sg ? kt.seg[1] : kt.seg[0];   // (a select keeps kt in registers)
                if (row >= 0) {
                    if (c < L::QC) tc::tma_prefetch_l2_3d(cmp ? mkc : mk, 64 * c, row, plane);
                    else tc::tma_prefetch_l2_3d(cmp ? mvc : mv, 64 * (c - L::QC), row, plane);
                }
            }
            return true;
        }
        const int slot = gm % NM;
        if (!warp_wait(bar.meta_empty(slot), ((gm / NM) & 1) ^ 1, abort_flag)) return false;
        if (lane == 0) {
            reinterpret_cast<KeyTile*>(sm + L::META_OFF)[slot] = kt;
            tc::mbar_arrive(bar.meta_full(slot));
        }
        ++gm;
        if (kt.br == BR_END) return true;
        const int st = gk % NS;
        const uint32_t ph = ((gk / NS) & 1) ^ 1;
        const bool cmp = kt.br == BR_CMP;
        const CUtensorMap* K = cmp ? mkc : mk;
        const CUtensorMap* V = cmp ? mvc : mv;
        const int rows = cmp ? a.s.n_cmp : a.s.Tk;     // a segment at `rows` is fully out of
        const int plane = w.b * a.s.Hkv + w.kvh;       // bounds: TMA fills it with zeros
        if (!warp_wait(bar.k_empty(st), ph, abort_flag)) return false;
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar.k_full(st), 2 * L::QC * HALF);
            uint8_t* dst = sm + L::K_OFF + st * L::QC * CHUNK;
            for (int sg = 0; sg < 2; ++sg) {
                const int row = kt.seg[sg] >= 0 ? kt.seg[sg] : rows;
                for (int c = 0; c < L::QC; ++c)
                    tc::tma_load_3d(dst + c * CHUNK + sg * HALF, K, bar.k_full(st), 64 * c, row,
                                    plane);
            }
        }
        if (!warp_wait(bar.v_empty(st), ph, abort_flag)) return false;
        if (lane == 0) {
            tc::mbar_arrive_expect_tx(bar.v_full(st), 2 * L::VC * HALF);
            uint8_t* dst = sm + L::V_OFF + st * L::VC * CHUNK;
            for (int sg = 0; sg < 2; ++sg) {
                const int row = kt.seg[sg] >= 0 ? kt.seg[sg] : rows;
                for (int c = 0; c < L::VC; ++c)
                    tc::tma_load_3d(dst + c * CHUNK + sg * HALF, V, bar.v_full(st), 64 * c, row,
                                    plane);
            }
        }
        ++gk;
        return true;
    }

    // Union of the tile tokens' selected blocks, ascending, with per-token
    // membership bits; the whole warp cooperates.  Returns the number of
    // distinct blocks; entries are (block << 5 | token) sorted then merged.
    __device__ int build_union(const WorkTile& w, uint32_t* keys, uint32_t* members) {
        const int k = a.s.topk;
        const int n = w.ntok * k;
        int np = 1;
        while (np < n) np <<= 1;
        const int32_t* base = a.idx + (((size_t)w.b * a.s.Hsel + w.unit) * a.s.Tq +
                                       (size_t)w.tt * a.tok) * k;
        for (int e = lane; e < np; e += 32) {
            uint32_t key = 0xFFFFFFFFu;
            if (e < n) {
                const int blk = base[e];
                const int tt = e / k;
                const int t = w.t0 + tt;
                if (blk >= 0 && blk <= t / a.s.bs) key = ((uint32_t)blk << 5) | (uint32_t)tt;
            }
            keys[e] = key;
        }
        __syncwarp();
        // bitonic sort of np keys
        for (int size = 2; size <= np; size <<= 1) {
            for (int stride = size >> 1; stride > 0; stride >>= 1) {
                for (int e = lane; e < np / 2; e += 32) {
                    const int lo = 2 * e - (e & (stride - 1));
                    const int hi = lo + stride;
                    const bool up = (lo & size) == 0;
                    const uint32_t x = keys[lo], y = keys[hi];
                    if ((x > y) == up) {
                        keys[lo] = y;
                        keys[hi] = x;
                    }
                }
                __syncwarp();
            }
        }
        // merge equal blocks: lane 0 walks the sorted list
        int nu = 0;
        if (lane == 0) {
            uint32_t prev = 0xFFFFFFFFu;
            for (int e = 0; e < n; ++e) {
                const uint32_t key = keys[e];
                if (key == 0xFFFFFFFFu) break;
                const uint32_t blk = key >> 5;
                if (blk != prev) {
                    keys[nu] = blk;
                    members[nu] = 0;
                    ++nu;
                    prev = blk;
                }
                members[nu - 1] |= 1u << (key & 31);
            }
        }
        nu = __shfl_sync(0xffffffffu, nu, 0);
        __syncwarp();
        return nu;
    }

    uint32_t q_loads = 0;

    __device__ bool run(int cta, int ncta) {
        uint32_t wt = 0;
        uint32_t* keys = reinterpret_cast<uint32_t*>(sm + L::UNION_OFF);
        uint32_t* members = keys + MAX_UNION / 2;
        for (int work = cta; work < a.n_work * a.n_split; work += ncta, ++wt) {
            const WorkTile w = decode_work(a, work % a.n_work);
            const int split = work / a.n_work;
            const int t_last = w.t0 + w.ntok - 1;
            // the selected blocks' union first: the sort overlaps the pipeline drain
            const bool sel_here = (a.s.flags & NSA_BR_SEL) && a.o_sel == nullptr;
            const int nu = sel_here ? build_union(w, keys, members) : 0;
            if (!warp_wait(bar.q_empty(), (wt & 1) ^ 1, abort_flag)) return false;
            if (lane == 0) {
                tc::mbar_arrive_expect_tx(bar.q_full(), L::QC * CHUNK);
                for (int c = 0; c < L::QC; ++c)
                    tc::tma_load_4d(sm + L::Q_OFF + c * CHUNK, mq, bar.q_full(), 64 * c, w.h0,
                                    w.tt * a.tok, w.b);
            }
            ++q_loads;
            KeyTile kt;
            kt.pad[0] = kt.pad[1] = 0;
            // key tiles of the three branches, numbered 0..n_total-1 in emission
            // order; this work item emits the tiles of its split share only
            int nvis = 0;
            if (a.s.flags & NSA_BR_CMP) {
                nvis = t_last - a.s.lc + 1 < 0 ? 0 : (t_last - a.s.lc + 1) / a.s.sc + 1;
                nvis = min(nvis, a.s.n_cmp);
            }
            const int nseg_sel = sel_here ? nu * (a.s.bs / SEG) : 0;
            const int win_lo = max(0, w.t0 - a.s.win + 1);
            const int n_tiles = (nvis + BN - 1) / BN + (nseg_sel + 1) / 2 +
                                ((a.s.flags & NSA_BR_WIN) ? (t_last - win_lo + BN) / BN : 0);
            const int g_lo = (int)((long long)split * n_tiles / a.n_split);
            const int g_hi = (int)((long long)(split + 1) * n_tiles / a.n_split);
            // split shares stream from HBM: first prefetch the share's K/V into L2,
            // then emit the tiles (two passes over the same enumeration)
            for (int pass = a.n_split > 1 ? 0 : 1; pass < 2; ++pass) {
            prefetch_only = pass == 0;
            int g = 0;
            if (a.s.flags & NSA_BR_CMP) {
                const int g_br = max(g, g_lo);      // first tile of this branch in the share
                for (int j0 = 0; j0 < nvis; j0 += BN, ++g) {
                    if (g < g_lo || g >= g_hi) continue;
                    kt.br = BR_CMP;
                    kt.first = g == g_br;
                    kt.seg[0] = j0;
                    kt.seg[1] = j0 + SEG < nvis ? j0 + SEG : -1;
                    kt.member[0] = kt.member[1] = 0xFFFFFFFFu;
                    if (!emit(kt, w)) return false;
                }
            }
            if (sel_here) {
                const int segs_per_blk = a.s.bs / SEG;
                const int nseg = nseg_sel;
                const int g_br = max(g, g_lo);
                for (int sgi = 0; sgi < nseg; sgi += 2, ++g) {
                    if (g < g_lo || g >= g_hi) continue;
                    kt.br = BR_SEL;
                    kt.first = g == g_br;
                    for (int h = 0; h < 2; ++h) {
                        const int q = sgi + h;
                        if (q < nseg) {
                            const int u = q / segs_per_blk;
                            kt.seg[h] = (int)keys[u] * a.s.bs + (q % segs_per_blk) * SEG;
                            kt.member[h] = members[u];
                        } else {
                            kt.seg[h] = -1;
                            kt.member[h] = 0;
                        }
                    }
                    if (!emit(kt, w)) return false;
                }
            }
            if (a.s.flags & NSA_BR_WIN) {
                const int lo = win_lo;
                const int g_br = max(g, g_lo);
                for (int u0 = lo; u0 <= t_last; u0 += BN, ++g) {
                    if (g < g_lo || g >= g_hi) continue;
                    kt.br = BR_WIN;
                    kt.first = g == g_br;
                    kt.seg[0] = u0;
                    kt.seg[1] = u0 + SEG <= t_last ? u0 + SEG : -1;
                    kt.member[0] = kt.member[1] = 0xFFFFFFFFu;
                    if (!emit(kt, w)) return false;
                }
            }
            }                                   // pass
            prefetch_only = false;
            kt.br = BR_END;
            kt.first = 0;
            kt.seg[0] = kt.seg[1] = -1;
            if (!emit(kt, w)) return false;
        }
        return true;
    }

    // Waits for every copy this warp issued (bounded, regardless of abort).
    __device__ void drain(uint32_t q_loads) {
        for (uint32_t s = 0; s < NS && s < gk; ++s) {
            const uint32_t last = s + ((gk - 1 - s) / NS) * NS;   // last key tile on stage s
            const uint32_t ph = (last / NS) & 1;
            tc::mbar_wait_bounded(bar.k_full(s), ph, WAIT_NS);
            tc::mbar_wait_bounded(bar.v_full(s), ph, WAIT_NS);
        }
        if (q_loads > 0) tc::mbar_wait_bounded(bar.q_full(), (q_loads - 1) & 1, WAIT_NS);
    }
};

// ------------------------------------------------------------------ kernel

template <int DQK, int DV>
__global__ void __launch_bounds__(NTHREADS, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ CUtensorMap map_kc,
                   const __grid_constant__ CUtensorMap map_vc, const TcArgs a) {
    using L = Smem<DQK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
    Bars bar = make_bars(reinterpret_cast<uint64_t*>(sm + L::BAR_OFF));
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L::MISC_OFF);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L::MISC_OFF + 8);
    KeyTile* metas = reinterpret_cast<KeyTile*>(sm + L::META_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        tc::mbar_init(bar.q_full(), 1);
        tc::mbar_init(bar.q_empty(), 1);
        for (int i = 0; i < NS; ++i) {
            tc::mbar_init(bar.k_full(i), 1);
            tc::mbar_init(bar.k_empty(i), 1);
            tc::mbar_init(bar.v_full(i), 1);
            tc::mbar_init(bar.v_empty(i), 1);
        }
        for (int i = 0; i < NM; ++i) {
            tc::mbar_init(bar.meta_full(i), 1);
            tc::mbar_init(bar.meta_empty(i), 9);   // MMA lane + 8 softmax warps
        }
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar.s_full(i), 1);
            tc::mbar_init(bar.p_full(i), 8);       // 8 softmax warps
        }
        tc::mbar_init(bar.pv_done(0), 1);
        tc::mbar_init(bar.pv_done(1), 1);
        tc::mbar_init(bar.drain(), 1);
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tc::prefetch_map(&map_q);
        tc::prefetch_map(&map_k);
        tc::prefetch_map(&map_v);
        tc::prefetch_map(&map_kc);
        tc::prefetch_map(&map_vc);
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS0 = tmem, tO = tmem + 256, tAcc = tmem + 384;

    if (warp < 4) {
        // warpgroup 0 gives registers to the softmax warpgroups: 4 x 32 x 56 + 8 x 32 x 216
        // = 62464 of the 384 x 168 = 64512 the block was launched with
        asm volatile("setmaxnreg.dec.sync.aligned.u32 56;" ::: "memory");
    if (warp == 0) {
        // ---------------------------------------------------------- producer
        Producer<DQK, DV> p{a, sm, bar, abort_flag, &map_q, &map_k, &map_v, &map_kc, &map_vc};
        p.lane = lane;
        if (!p.run(blockIdx.x, gridDim.x)) raise_abort(abort_flag);
        p.drain(p.q_loads);
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc_qk = tc::idesc_bf16_f32(BM, BN, false, false);
            const uint32_t idesc_pv = tc::idesc_bf16_f32(BM, DV, false, true);
            const uint32_t q_base = tc::smem_u32(sm + L::Q_OFF);
            const uint32_t k_base = tc::smem_u32(sm + L::K_OFF);
            const uint32_t v_base = tc::smem_u32(sm + L::V_OFF);
            uint32_t gm = 0, gi = 0, wt = 0;
            bool ok = true;
            for (int work = blockIdx.x; ok && work < a.n_work * a.n_split; work += gridDim.x, ++wt) {
                if (!tc::mbar_wait(bar.q_full(), wt & 1, abort_flag, c_wait_ns)) { ok = false; break; }
                bool have_prev = false;
                uint32_t prev_gi = 0;
                int prev_first = 0;
                while (true) {
                    const int slot = gm % NM;
                    if (!tc::mbar_wait(bar.meta_full(slot), (gm / NM) & 1, abort_flag, c_wait_ns)) {
                        ok = false;
                        break;
                    }
                    const int br = metas[slot].br;
                    const int first = metas[slot].first;
                    tc::mbar_arrive(bar.meta_empty(slot));
                    ++gm;
                    if (br != BR_END) {
                        const int st = gi % NS;
                        if (!tc::mbar_wait(bar.k_full(st), (gi / NS) & 1, abort_flag, c_wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                        const uint32_t dS = tS0 + (gi & 1) * 128;
                        const uint32_t kst = k_base + st * L::QC * CHUNK;
#pragma unroll
                        for (int kk = 0; kk < DQK / 16; ++kk) {
                            const uint32_t off = (kk >> 2) * CHUNK + (kk & 3) * 32;
                            tc::mma_ss(dS, tc::sdesc_sw128(q_base + off, 16, 1024),
                                       tc::sdesc_sw128(kst + off, 16, 1024), idesc_qk, kk > 0);
                        }
                        tc::mma_commit(bar.s_full(gi & 1));
                        tc::mma_commit(bar.k_empty(st));
                    } else {
                        tc::mma_commit(bar.q_empty());
                    }
                    if (have_prev) {
                        // O (+)= P V for the previous key tile
                        const int pst = prev_gi % NS;
                        if (!tc::mbar_wait(bar.p_full(prev_gi & 1), (prev_gi >> 1) & 1, abort_flag,
                                           c_wait_ns) ||
                            !tc::mbar_wait(bar.v_full(pst), (prev_gi / NS) & 1, abort_flag,
                                           c_wait_ns)) {
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                        const uint32_t aP = tS0 + (prev_gi & 1) * 128;
                        const uint32_t vst = v_base + pst * L::VC * CHUNK;
#pragma unroll
                        for (int kk = 0; kk < BN / 16; ++kk) {
                            tc::mma_ts(tO, aP + kk * 8, tc::sdesc_sw128(vst + kk * 2048, CHUNK, 1024),
                                       idesc_pv, (prev_first && kk == 0) ? 0u : 1u);
                        }
                        tc::mma_commit(bar.v_empty(pst));
                        tc::mma_commit(bar.pv_done(prev_gi & 1));
                    }
                    if (br == BR_END) break;
                    have_prev = true;
                    prev_gi = gi;
                    prev_first = first;
                    ++gi;
                }
            }
            if (!ok) raise_abort(abort_flag);
            // all issued MMAs must finish before TMEM is released
            tc::mma_commit(bar.drain());
            tc::mbar_wait_bounded(bar.drain(), 0, WAIT_NS);
        }
        __syncwarp();
    }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 216;" ::: "memory");
        // ---------------------------------------------------------- softmax / epilogue
        // Two warpgroups; thread (half, r) owns row r and key columns
        // [64*half, 64*half + 64) of every S tile (= segment `half`), and
        // columns [half*DV/2, (half+1)*DV/2) of O and Acc.  The two halves of a
        // row exchange their partial max (every tile) and partial sum (at
        // branch ends) through shared memory.
        const int half = (warp - 4) >> 2;
        const int quarter = warp & 3;               // TMEM lane quarter of this warp
        const int r = quarter * 32 + lane;          // tile row of this thread
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        float* xmax = reinterpret_cast<float*>(sm + L::XCH_OFF);   // [2 parity][2 half][BM]
        float* xsum = xmax + 4 * BM;                                 // [2 half][BM]
        int* xstat = reinterpret_cast<int*>(xsum + 2 * BM);          // [2 parity][8 warps]
        const int sw = warp - 4;                                     // partner warp: sw ^ 4
        uint32_t pseq = 0;                                           // pair barriers passed
        // Barrier between the two warps that hold the two halves of the same rows
        // (named barrier 2 + quarter, 64 threads).  It returns the AND of `pred` over
        // both warps and sets `fail` when either arrives failed: a warp whose wait
        // ran out raises the abort flag, arrives here once with failed = true and
        // leaves, and its partner, at whichever pair barrier it reaches next, learns
        // of it here and leaves too, so neither is left alone at a barrier.  A warp
        // can be at most one pair barrier ahead of its partner, so the status words
        // alternate between two slots.
        auto pair_sync = [&](bool pred, bool failed, bool& fail) {
            if (lane == 0) xstat[(pseq & 1) * 8 + sw] = failed ? 1 : 0;
            const bool all = tc::named_bar_and(2 + quarter, 64, pred && !failed);
            fail = failed || xstat[(pseq & 1) * 8 + (sw ^ 4)] != 0;
            ++pseq;
            return all;
        };
        auto fail_out = [&]() {
            raise_abort(abort_flag);
            bool f;
            pair_sync(false, true, f);
        };
        constexpr int DVH = DV / 2;
        uint32_t gm = 0, gi = 0;
        // P V of key tile k is the (k >> 1)-th completion of pv_done(k & 1).  When
        // this warp has S of tile k, P V of tile k - 2 has completed (the tensor
        // pipe runs in order) and that of tile k + 1 cannot have started, so the
        // parity wait for tile k - 1 is unambiguous however many earlier waits were
        // skipped.
        auto wait_pv = [&](uint32_t k) {
            return warp_wait(bar.pv_done(k & 1), (k >> 1) & 1, abort_flag);
        };
        bool ok = true;
        for (int work = blockIdx.x; ok && work < a.n_work * a.n_split; work += gridDim.x) {
            const WorkTile w = decode_work(a, work % a.n_work);
            const int split = work / a.n_work;
            const bool split_mode = a.n_split > 1;
            uint32_t visited = 0;                  // branches with at least one tile here
            const int tt = r / a.hpt;
            const int h = w.h0 + r % a.hpt;
            const bool row_valid = tt < w.ntok;
            const int t = w.t0 + tt;
            const int qi = w.tt * a.tok + tt;       // query index of the row
            const size_t grow = ((size_t)w.b * a.s.Tq + qi) * a.s.Hq + h;
            const int cmp_cap = t - a.s.lc + 1 < 0 ? -1 : min((t - a.s.lc + 1) / a.s.sc, a.s.n_cmp - 1);

            int cur_br = -1;
            bool acc_has = false, have_prev = false;
            float m_ref = -INFINITY, l = 0.f;      // l: this half's share of the row sum
            // the row's gates are read now and o_sel's half-row is brought into L2, so
            // that neither load's latency lands in a branch end or the epilogue
            float gate[3] = {1.f, 1.f, 1.f};
            if (a.gates && row_valid && !split_mode) {
                const float* grow_gates = a.gates + grow * 3;
                gate[0] = grow_gates[0];
                gate[1] = grow_gates[1];
                gate[2] = grow_gates[2];
            }
            if (a.o_sel != nullptr && row_valid && !split_mode)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.o_sel + grow * DV + half * (DV / 2)));

            // folds gate * O / l of the finished branch into Acc (warp-uniform); in
            // split mode writes this share's O / l and lse for the row instead
            auto correction = [&](int br) {
                bool fail;
                xsum[half * BM + r] = l;
                pair_sync(true, false, fail);
                if (fail) return false;
                const float lrow = l + xsum[(half ^ 1) * BM + r];
                pair_sync(true, false, fail);
                if (fail) return false;
                if (split_mode) {
                    const size_t pr = (grow * 3 + br) * a.n_split + split;
                    const float inv = lrow > 0.f ? 1.f / lrow : 0.f;
#pragma unroll 1
                    for (int c = half * DVH; c < (half + 1) * DVH; c += 32) {
                        uint32_t o[32];
                        tc::tmem_ld32(tO + lane_off + c, o);
                        tc::tmem_wait_ld();
                        if (row_valid) {
                            float4* dst = reinterpret_cast<float4*>(a.split_o + pr * DV + c);
#pragma unroll
                            for (int q4 = 0; q4 < 8; ++q4)
                                dst[q4] = make_float4(__uint_as_float(o[4 * q4]) * inv, __uint_as_float(o[4 * q4 + 1]) * inv,
                                                      __uint_as_float(o[4 * q4 + 2]) * inv, __uint_as_float(o[4 * q4 + 3]) * inv);
                        }
                    }
                    if (row_valid && half == 0)
                        a.split_lse[pr] = lrow > 0.f ? m_ref + __log2f(lrow) : -INFINITY;
                    visited |= 1u << br;
                    return true;
                }
                float wgt = 0.f;
                if (row_valid && lrow > 0.f) {
                    const float g = br == 0 ? gate[0] : br == 1 ? gate[1] : gate[2];
                    wgt = g / lrow;
                }
#pragma unroll 1
                for (int c = half * DVH; c < (half + 1) * DVH; c += 32) {
                    uint32_t o[32], acc[32];
                    tc::tmem_ld32(tO + lane_off + c, o);
                    if (acc_has) tc::tmem_ld32(tAcc + lane_off + c, acc);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float prev = acc_has ? __uint_as_float(acc[j]) : 0.f;
                        acc[j] = __float_as_uint(fmaf(wgt, __uint_as_float(o[j]), prev));
                    }
                    tc::tmem_st32(tAcc + lane_off + c, acc);
                }
                tc::tmem_wait_st();
                acc_has = true;
                return true;
            };

            while (true) {
                const int slot = gm % NM;
                if (!warp_wait(bar.meta_full(slot), (gm / NM) & 1, abort_flag)) {
                    fail_out();
                    ok = false;
                    break;
                }
                const KeyTile kt = metas[slot];
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar.meta_empty(slot));
                ++gm;
                if (kt.br == BR_END) break;

                const int sb = gi & 1;
                if (!warp_wait(bar.s_full(sb), (gi >> 1) & 1, abort_flag)) {
                    fail_out();
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                // valid key offsets [lo, hi] of this thread's segment for its row
                int lo = 0, hi = -1;
                const int s0 = half ? kt.seg[1] : kt.seg[0];
                if (s0 >= 0 && row_valid) {
                    if (kt.br == BR_CMP) {
                        hi = min(SEG - 1, cmp_cap - s0);
                    } else if (kt.br == BR_SEL) {
                        if (((half ? kt.member[1] : kt.member[0]) >> tt) & 1u) hi = min(SEG - 1, t - s0);
                    } else {
                        lo = max(0, t - a.s.win + 1 - s0);
                        hi = min(SEG - 1, t - s0);
                    }
                }
                if (hi < lo) lo = hi = SEG;    // empty: no offset 0..63 matches
                const bool new_branch = kt.first != 0;
                float m_use = 0.f, alpha = 1.f, psum = 0.f;
                bool rescale = false;
                uint32_t sv[SEG];
                // One tile of this half-row, specialised on whether any row of the
                // warp needs a mask (interior tiles of the compressed and window
                // branches are fully visible).
                auto half_row = [&](auto masked_tag) {
                    constexpr bool MASKED = decltype(masked_tag)::value;
                    tc::tmem_ld32(tS0 + sb * 128 + lane_off + half * SEG, sv);
                    tc::tmem_ld32(tS0 + sb * 128 + lane_off + half * SEG + 32, sv + 32);
                    tc::tmem_wait_ld();
                    float mx[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) mx[q] = -INFINITY;
                    const uint32_t span = (uint32_t)(hi - lo);
#pragma unroll
                    for (int k = 0; k < SEG; ++k) {
                        float x = __uint_as_float(sv[k]);
                        if (MASKED) {
                            x = (uint32_t)(k - lo) <= span ? x : -INFINITY;
                            sv[k] = __float_as_uint(x);
                        }
                        mx[k & 7] = fmaxf(mx[k & 7], x);
                    }
                    const float m_half = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                               fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                    // exchange with the other half of the row; after this barrier both
                    // halves have finished reading S, so P may overwrite it
                    xmax[((gi & 1) * 2 + half) * BM + r] = m_half;
                    bool fail;
                    pair_sync(true, false, fail);
                    if (fail) return false;
                    const float m_raw = fmaxf(m_half, xmax[((gi & 1) * 2 + (half ^ 1)) * BM + r]);
                    // scale > 0, so the scaled max is the max of the scaled scores
                    const float m_tile = m_raw * a.scale_log2;
                    m_use = new_branch ? -INFINITY : m_ref;
                    if (m_tile != -INFINITY) {
                        if (m_use == -INFINITY) {
                            m_use = m_tile;
                        } else if (m_tile > m_use + 8.f) {
                            alpha = tc::ex2(m_use - m_tile);
                            rescale = true;
                            m_use = m_tile;
                        }
                    }
                    // p = 2^(s*scale*log2e - m); masked scores are -inf and give 0
                    const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
                    float ps[8];
#pragma unroll
                    for (int q = 0; q < 8; ++q) ps[q] = 0.f;
#pragma unroll
                    for (int k = 0; k < SEG; k += 2) {
                        const float p0 = tc::ex2(fmaf(__uint_as_float(sv[k]), a.scale_log2, neg_m));
                        const float p1 = tc::ex2(fmaf(__uint_as_float(sv[k + 1]), a.scale_log2, neg_m));
                        ps[(k >> 1) & 7] += p0 + p1;
                        sv[k >> 1] = tc::pack_bf16x2(p0, p1);     // packed in place: k/2 < k
                    }
                    psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                    return true;
                };
                // Later tiles of a branch try one pass first: the exponentials use the
                // row's running reference max while the tile's max is taken alongside.
                // The two passes above would keep that reference unless a score
                // exceeds it by more than 8 (log2 units), so when no row of this warp
                // pair does (one barrier vote), the result is theirs; otherwise both
                // warps redo the tile with them (S is still in TMEM: no P is stored
                // before the vote).
                auto one_pass = [&](auto masked_tag) {
                    constexpr bool MASKED = decltype(masked_tag)::value;
                    tc::tmem_ld32(tS0 + sb * 128 + lane_off + half * SEG, sv);
                    tc::tmem_ld32(tS0 + sb * 128 + lane_off + half * SEG + 32, sv + 32);
                    tc::tmem_wait_ld();
                    const uint32_t span = (uint32_t)(hi - lo);
                    const float neg_m = m_ref == -INFINITY ? 0.f : -m_ref;
                    float ym[4], ps[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) ym[q] = -INFINITY;
#pragma unroll
                    for (int q = 0; q < 8; ++q) ps[q] = 0.f;
#pragma unroll
                    for (int k = 0; k < SEG; k += 2) {
                        float x0 = __uint_as_float(sv[k]), x1 = __uint_as_float(sv[k + 1]);
                        if (MASKED) {
                            x0 = (uint32_t)(k - lo) <= span ? x0 : -INFINITY;
                            x1 = (uint32_t)(k + 1 - lo) <= span ? x1 : -INFINITY;
                        }
                        const float y0 = fmaf(x0, a.scale_log2, neg_m);
                        const float y1 = fmaf(x1, a.scale_log2, neg_m);
                        ym[(k >> 1) & 3] = fmaxf(ym[(k >> 1) & 3], fmaxf(y0, y1));
                        const float p0 = tc::ex2(y0), p1 = tc::ex2(y1);
                        ps[(k >> 1) & 7] += p0 + p1;
                        sv[k >> 1] = tc::pack_bf16x2(p0, p1);     // packed in place: k/2 < k
                    }
                    psum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                    const float ymax = fmaxf(fmaxf(ym[0], ym[1]), fmaxf(ym[2], ym[3]));
                    // a row without a reference yet takes one from its first valid score
                    return m_ref == -INFINITY ? ymax != -INFINITY : ymax > 8.f;
                };
                const bool full_warp = __all_sync(0xffffffffu, lo == 0 && hi == SEG - 1);
                bool done = false;
                if (!new_branch) {
                    const bool over = full_warp ? one_pass(std::false_type{}) : one_pass(std::true_type{});
                    bool fail;
                    done = pair_sync(!over, false, fail);
                    if (fail) {
                        ok = false;
                        break;
                    }
                    if (done) m_use = m_ref;
                }
                if (!done && !(full_warp ? half_row(std::false_type{}) : half_row(std::true_type{}))) {
                    ok = false;
                    break;
                }
                tc::tmem_st32(tS0 + sb * 128 + lane_off + half * 32, sv);
                tc::tmem_wait_st();

                // O may be touched only after the previous P V has landed; the wait is
                // skipped when this tile neither rescales O nor closes a branch
                if (have_prev) {
                    const bool touch_o = (new_branch && cur_br >= 0) || __any_sync(0xffffffffu, rescale);
                    if (touch_o) {
                        if (!wait_pv(gi - 1)) {
                            fail_out();
                            ok = false;
                            break;
                        }
                        tc::fence_after_sync();
                    }
                }
                if (new_branch && cur_br >= 0 && !correction(cur_br)) {
                    ok = false;
                    break;
                }
                if (new_branch) l = 0.f;
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll 1
                    for (int c = half * DVH; c < (half + 1) * DVH; c += 32) {
                        uint32_t o[32];
                        tc::tmem_ld32(tO + lane_off + c, o);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            o[j] = __float_as_uint(__uint_as_float(o[j]) * alpha);
                        tc::tmem_st32(tO + lane_off + c, o);
                    }
                    tc::tmem_wait_st();
                    l *= alpha;
                }
                l += psum;
                m_ref = m_use;
                cur_br = kt.br;
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive(bar.p_full(sb));
                have_prev = true;
                ++gi;
            }
            if (!ok) break;
            if (have_prev) {
                if (!wait_pv(gi - 1)) {
                    fail_out();
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
                if (!correction(cur_br)) {
                    ok = false;
                    break;
                }
            }
            if (split_mode) {
                if (row_valid && half == 0)
                    for (int br = 0; br < 3; ++br)
                        if (!(visited & (1u << br)))
                            a.split_lse[(grow * 3 + br) * a.n_split + split] = -INFINITY;
                tc::fence_before_sync();
                continue;
            }
            // selected branch computed outside: out += g_sel * o_sel
            const bool add_sel = a.o_sel != nullptr && (a.s.flags & NSA_BR_SEL) && row_valid;
            const float g_sel = add_sel ? gate[1] : 0.f;
            // epilogue: this half of the Acc row (+ the selected branch) -> bf16 -> out
#pragma unroll 1
            for (int c = half * DVH; c < (half + 1) * DVH; c += 32) {
                uint32_t acc[32];
                if (acc_has) {
                    tc::tmem_ld32(tAcc + lane_off + c, acc);
                    tc::tmem_wait_ld();
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j) acc[j] = 0u;
                }
                if (add_sel) {
                    const uint4* src = reinterpret_cast<const uint4*>(a.o_sel + grow * DV + c);
                    uint4 raw[4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) raw[q4] = src[q4];
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        float f[8];
                        unpack8(raw[q4], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            acc[8 * q4 + e] = __float_as_uint(fmaf(g_sel, f[e], __uint_as_float(acc[8 * q4 + e])));
                    }
                }
                if (row_valid) {
                    uint4* dst = reinterpret_cast<uint4*>(a.out + grow * DV + c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        uint4 u;
                        u.x = tc::pack_bf16x2(__uint_as_float(acc[8 * q + 0]), __uint_as_float(acc[8 * q + 1]));
                        u.y = tc::pack_bf16x2(__uint_as_float(acc[8 * q + 2]), __uint_as_float(acc[8 * q + 3]));
                        u.z = tc::pack_bf16x2(__uint_as_float(acc[8 * q + 4]), __uint_as_float(acc[8 * q + 5]));
                        u.w = tc::pack_bf16x2(__uint_as_float(acc[8 * q + 6]), __uint_as_float(acc[8 * q + 7]));
                        dst[q] = u;
                    }
                }
            }
            tc::fence_before_sync();
        }
        if (!ok) raise_abort(abort_flag);
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// bf16 tensor [planes, rows, d] viewed as a 3D map {d, rows, planes}, box {64, 64, 1}
bool make_kv_map(CUtensorMap* m, const void* base, int d, int rows, int planes) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)(rows > 0 ? rows : 1), (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)d * 2 * (cuuint64_t)(rows > 0 ? rows : 1)};
    cuuint32_t box[3] = {64, 64, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// q [B, Tq, Hq, d] as a 4D map {d, Hq, Tq, B}, box {64, hpt, tok, 1}
bool make_q_map(CUtensorMap* m, const void* base, const Shape& s, int hpt, int tok) {
    auto enc = encode_fn();
    if (!enc) return false;
    cuuint64_t dims[4] = {(cuuint64_t)s.dqk, (cuuint64_t)s.Hq, (cuuint64_t)s.Tq, (cuuint64_t)s.B};
    cuuint64_t strides[3] = {(cuuint64_t)s.dqk * 2, (cuuint64_t)s.dqk * 2 * s.Hq,
                             (cuuint64_t)s.dqk * 2 * s.Hq * s.Tq};
    cuuint32_t box[4] = {64, (cuuint32_t)hpt, (cuuint32_t)tok, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

template <int DQK, int DV>
cudaError_t launch_tc_impl(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* kcmp,
                           const __nv_bfloat16* vcmp, const float* gates, const int32_t* idx,
                           const __nv_bfloat16* o_sel, int n_split, float* split_o,
                           float* split_lse, __nv_bfloat16* out, cudaStream_t st) {
    TcArgs a;
    a.s = s;
    a.o_sel = o_sel;
    a.n_split = n_split;
    a.split_o = split_o;
    a.split_lse = split_lse;
    a.idx = idx;
    a.gates = gates;
    a.out = out;
    a.hpt = s.heads_per_unit;
    a.tok = BM / a.hpt;
    a.n_tt = (s.Tq + a.tok - 1) / a.tok;
    a.n_work = a.n_tt * s.B * s.Hsel;
    a.scale_log2 = s.scale * 1.4426950408889634f;
    CUtensorMap mq, mk, mv, mkc, mvc;
    const int planes = s.B * s.Hkv;
    if (!make_q_map(&mq, q, s, a.hpt, a.tok) || !make_kv_map(&mk, k, DQK, s.Tk, planes) ||
        !make_kv_map(&mv, v, DV, s.Tk, planes))
        return cudaErrorInvalidValue;
    // without a compressed branch the compressed maps point at K/V (never read)
    const bool cmp = (s.flags & NSA_BR_CMP) && s.n_cmp > 0;
    if (!make_kv_map(&mkc, cmp ? (const void*)kcmp : (const void*)k, DQK, cmp ? s.n_cmp : s.Tk, planes) ||
        !make_kv_map(&mvc, cmp ? (const void*)vcmp : (const void*)v, DV, cmp ? s.n_cmp : s.Tk, planes))
        return cudaErrorInvalidValue;
    int dev = 0, nsm = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev);
    const int smem = Smem<DQK, DV>::ALLOC;
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<DQK, DV>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int grid = min(a.n_work * a.n_split, nsm);
    if (grid <= 0) return cudaSuccess;
    attn_tc_kernel<DQK, DV><<<grid, NTHREADS, smem, st>>>(mq, mk, mv, mkc, mvc, a);
    return cudaGetLastError();
}

}  // namespace

bool attn_tc_supported(const Shape& s) {
    if (s.dqk != 64 && s.dqk != 128 && s.dqk != 192) return false;
    if (s.dv != 64 && s.dv != 128) return false;
    const int hpt = s.heads_per_unit;
    if (hpt > 16 || (BM % hpt) != 0) return false;
    // the selected branch's per-segment membership masks hold 32 tokens per tile;
    // the window and compressed branches alone take one or two heads per unit too
    // (up to 128 tokens per tile: MHA, or full causal attention as a window >= Tkv)
    if ((s.flags & NSA_BR_SEL) && hpt < 4) return false;
    if ((s.flags & NSA_BR_SEL) && (s.bs % SEG != 0)) return false;
    if ((s.flags & NSA_BR_SEL) && (BM / hpt) * s.topk > MAX_UNION / 2) return false;
    return true;
}

cudaError_t launch_attn_tc(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* kcmp,
                           const __nv_bfloat16* vcmp, const float* gates, const int32_t* idx,
                           const __nv_bfloat16* o_sel, int n_split, float* split_o,
                           float* split_lse, __nv_bfloat16* out, cudaStream_t st) {
#define NSA_TC_CASE(A, B)                                                                  \
    if (s.dqk == A && s.dv == B)                                                           \
        return launch_tc_impl<A, B>(s, q, k, v, kcmp, vcmp, gates, idx, o_sel, n_split,   \
                                    split_o, split_lse, out, st);
    NSA_TC_CASE(64, 64)
    NSA_TC_CASE(128, 128)
    NSA_TC_CASE(192, 128)
    NSA_TC_CASE(64, 128)
    NSA_TC_CASE(128, 64)
    NSA_TC_CASE(192, 64)
#undef NSA_TC_CASE
    return cudaErrorInvalidValue;
}

namespace {

// out[row] = sum_br g_br * (sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M)) over the
// split shares of each branch (empty branches contribute 0).  One thread per
// 4 output columns of a (query, head) row.
__global__ void __launch_bounds__(256) split_merge_kernel(Shape s, int n_split,
                                                          const float* __restrict__ split_o,
                                                          const float* __restrict__ split_lse,
                                                          const float* __restrict__ gates,
                                                          __nv_bfloat16* __restrict__ out) {
    const int c4n = s.dv / 4;
    const size_t nrows = (size_t)s.B * s.Tq * s.Hq;
    const size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= nrows * c4n) return;
    const size_t row = e / c4n;
    const int c4 = (int)(e % c4n);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int br = 0; br < 3; ++br) {
        const uint32_t bit = br == 0 ? NSA_BR_CMP : br == 1 ? NSA_BR_SEL : NSA_BR_WIN;
        if (!(s.flags & bit)) continue;
        const float* lse = split_lse + (row * 3 + br) * n_split;
        float m = -INFINITY;
        for (int sp = 0; sp < n_split; ++sp) m = fmaxf(m, lse[sp]);
        if (m == -INFINITY) continue;
        float wsum = 0.f;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp = 0; sp < n_split; ++sp) {
            if (lse[sp] == -INFINITY) continue;
            const float w = exp2f(lse[sp] - m);
            wsum += w;
            const float4 v = reinterpret_cast<const float4*>(split_o + ((row * 3 + br) * n_split + sp) * s.dv)[c4];
            o.x = fmaf(w, v.x, o.x);
            o.y = fmaf(w, v.y, o.y);
            o.z = fmaf(w, v.z, o.z);
            o.w = fmaf(w, v.w, o.w);
        }
        const float g = (gates ? gates[row * 3 + br] : 1.f) / wsum;
        acc.x = fmaf(g, o.x, acc.x);
        acc.y = fmaf(g, o.y, acc.y);
        acc.z = fmaf(g, o.z, acc.z);
        acc.w = fmaf(g, o.w, acc.w);
    }
    __nv_bfloat162* dst = reinterpret_cast<__nv_bfloat162*>(out + row * s.dv + 4 * c4);
    dst[0] = __floats2bfloat162_rn(acc.x, acc.y);
    dst[1] = __floats2bfloat162_rn(acc.z, acc.w);
}

}  // namespace

int attn_tc_split_count(const Shape& s) {
    const int hpt = s.heads_per_unit;
    const int tok = BM / hpt;
    const int n_work = (s.Tq + tok - 1) / tok * s.B * s.Hsel;
    // enough work items to cover the SMs about eight times over
    if (n_work >= 2 * 148) return 1;
    return std::min(16, (8 * 148 + n_work - 1) / n_work);
}

cudaError_t launch_split_merge(const Shape& s, int n_split, const float* split_o,
                               const float* split_lse, const float* gates, __nv_bfloat16* out,
                               cudaStream_t st) {
    const size_t n = (size_t)s.B * s.Tq * s.Hq * (s.dv / 4);
    split_merge_kernel<<<(unsigned)((n + 255) / 256), 256, 0, st>>>(s, n_split, split_o, split_lse,
                                                                     gates, out);
    return cudaGetLastError();
}

// Self-test of the failure path shared by the tensor-core kernels: one warp
// waits, with the same bounded wait, on an mbarrier whose phase nothing ever
// completes, gives up after `limit_ns` and records NSA_ERR_TIMEOUT in the
// same status word, exactly as a kernel whose copy or MMA never arrived.
__global__ void wait_selftest_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(&bar, 1);
        abort_flag = 0;
        tc::fence_mbar_init();
    }
    __syncwarp();
    const bool ok = __all_sync(0xffffffffu, tc::mbar_wait(&bar, 0, &abort_flag, limit_ns));
    if (!ok && threadIdx.x == 0) raise_abort(&abort_flag);
}

cudaError_t set_wait_limit(uint64_t limit_ns) {
    const uint64_t v = limit_ns ? limit_ns : WAIT_NS;
    return cudaMemcpyToSymbol(c_wait_ns, &v, sizeof(v));
}

cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st) {
    wait_selftest_kernel<<<1, 32, 0, st>>>(limit_ns);
    return cudaGetLastError();
}

int read_and_clear_tc_status() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_tc_status, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_tc_status, &zero, sizeof(int));
    return v;
}

}  // namespace nsa
