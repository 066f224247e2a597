// Block scoring and top-k block selection.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention": every query has one score per KV block; under GQA the heads of
// a group add their scores into one selection score and take one top-k, so
// the whole group reads the same blocks.  LateTalk #103 (zjai.club) §13: the
// block holding the query is always selected.
//
// The group score is linear in the queries, so it is computed as
// scale * (sum_h q_h) . kbar_b in fp32: one dot product per (query, group,
// block) instead of one per head.  A CTA takes RT query rows of one
// selection unit, stages the rows' summed queries and chunks of KC pooled
// keys in shared memory, forms the RT x KC score tile with FFMA (a 4 x 4
// register tile per thread), and keeps a running top-(k-1) per row in the registers of one warp (one key per lane,
// sorted descending).  A key packs the order-preserving bits of the score
// with the inverted block id, so a single 64-bit comparison orders by score
// and then by lower block id.
#include <math.h>

#include "common.cuh"
#include "tc.cuh"


namespace nsa {

__device__ int g_select_status = 0;

constexpr int ST_RT = 64;   // query rows per CTA
constexpr int ST_KC = 64;   // pooled keys per chunk
constexpr int ST_NT = 256;  // threads per CTA (8 warps x 8 rows of top-k state)
constexpr int ST_RPW = ST_RT / 8;   // rows per warp

enum { MODE_SELECT = 0, MODE_SCORES = 1, MODE_SELECT_FROM_SCORES = 2 };

// Merges the 32 candidate keys of a warp (one per lane, 0 = none) into the
// warp's running list: the K1 largest keys so far, descending, one per lane
// (lanes >= K1 hold 0); `thr` is the list's smallest key (lane K1 - 1).
// A few survivors of the threshold are inserted one at a time; four or more
// are bitonic-sorted across the lanes and bitonic-merged with the list.
__device__ __forceinline__ void warp_list_merge(unsigned long long& key, unsigned long long& thr,
                                                unsigned long long ck, int K1, int lane) {
    unsigned mask = __ballot_sync(0xffffffffu, ck > thr);
    if (__popc(mask) >= 4) {
        unsigned long long v = ck > thr ? ck : 0ull;
#pragma unroll
        for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
            for (int j = k >> 1; j > 0; j >>= 1) {
                const unsigned long long o = __shfl_xor_sync(0xffffffffu, v, j);
                const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
                v = keep_max ? (v > o ? v : o) : (v < o ? v : o);
            }
        // v descending; the larger of key[l] and v[31 - l] is the top 32 of both, bitonic
        const unsigned long long vr = __shfl_sync(0xffffffffu, v, 31 - lane);
        unsigned long long w = key > vr ? key : vr;
#pragma unroll
        for (int j = 16; j > 0; j >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, w, j);
            w = (lane & j) == 0 ? (w > o ? w : o) : (w < o ? w : o);
        }
        key = lane < K1 ? w : 0ull;
        thr = __shfl_sync(0xffffffffu, key, K1 - 1);
        return;
    }
    while (mask) {
        const int src = __ffs(mask) - 1;
        const unsigned long long x = __shfl_sync(0xffffffffu, ck, src);
        const int p = __popc(__ballot_sync(0xffffffffu, lane < K1 && key > x));
        const unsigned long long up = __shfl_up_sync(0xffffffffu, key, 1);
        if (lane < K1) {
            if (lane == p) key = x;
            else if (lane > p) key = up;
        }
        thr = __shfl_sync(0xffffffffu, key, K1 - 1);
        mask &= ~(1u << src);
        mask &= __ballot_sync(0xffffffffu, ck > thr);
    }
}

template <int MODE>
__global__ void __launch_bounds__(ST_NT, 2) score_topk_kernel(Shape s, const __nv_bfloat16* __restrict__ q,
                                                           const float* __restrict__ kbar,
                                                           const float* __restrict__ scores_in,
                                                           float* __restrict__ scores_out,
                                                           int32_t* __restrict__ idx) {
    extern __shared__ float smem[];
    const int d = s.dqk;
    const int ld = d + 4;
    float* qs = smem;                       // [RT][ld]   summed queries
    float* ks = qs + ST_RT * ld;            // [KC][ld]   pooled keys
    float* ss = ks;                         // [RT][KC+1] score tile, reuses the key buffer
                                            // once the FFMA tile is in registers

    const int i0 = blockIdx.x * ST_RT;
    const int u = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = s.per_head ? u / s.G : u;
    const int h0 = s.per_head ? u : u * s.G;
    const int nh = s.heads_per_unit;
    const int nrows = min(ST_RT, s.Tq - i0);

    // current block of the last row bounds the candidates of the whole tile
    const int c_last = (s.q0 + i0 + nrows - 1) / s.bs;
    const int cmax = min(c_last, s.nb_full);

    if (MODE != MODE_SELECT_FROM_SCORES) {
        const int nvec = d / 8;
        for (int p = tid; p < ST_RT * nvec; p += ST_NT) {
            const int r = p / nvec, vec = p % nvec;
            float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (r < nrows) {
                const __nv_bfloat16* src = q + (((size_t)b * s.Tq + i0 + r) * s.Hq + h0) * d + vec * 8;
                // the unit's heads in groups of 8, every load of a group issued before
                // any is summed (the rows are far apart: one HBM round trip per group)
                for (int h8 = 0; h8 < nh; h8 += 8) {
                    uint4 raw[8];
#pragma unroll
                    for (int hh = 0; hh < 8; ++hh)
                        if (h8 + hh < nh) raw[hh] = *reinterpret_cast<const uint4*>(src + (size_t)(h8 + hh) * d);
#pragma unroll
                    for (int hh = 0; hh < 8; ++hh) {
                        if (h8 + hh >= nh) break;
                        float f[8];
                        unpack8(raw[hh], f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc[e] += f[e];
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) qs[r * ld + vec * 8 + e] = acc[e];
        }
    }

    // pooled-key chunks go through registers: the loads of chunk j + 1 are issued
    // before chunk j is scored, so their latency overlaps the FFMA and top-k work
    constexpr int KREG = ST_KC * 192 / 4 / ST_NT;    // float4 per thread; d = 256 loads the rest late
    float4 kreg[KREG];
    const float* kb_base = kbar + (size_t)(b * s.Hkv + kvh) * s.nb_full * d;
    auto load_chunk = [&](int c0) {
        const int nk = min(ST_KC, cmax - c0);
        const int nf4 = d / 4;
#pragma unroll
        for (int e = 0; e < KREG; ++e) {
            const int p = tid + e * ST_NT;
            if (p < nk * nf4)
                kreg[e] = *reinterpret_cast<const float4*>(kb_base + (size_t)(c0 + p / nf4) * d + (p % nf4) * 4);
        }
    };
    if (MODE != MODE_SELECT_FROM_SCORES && cmax > 0) load_chunk(0);

    const int K1 = s.topk - 1;               // past blocks kept per row
    unsigned long long key[ST_RPW];      // lane's slot of rows ST_RPW*warp + j
#pragma unroll
    for (int j = 0; j < ST_RPW; ++j) key[j] = 0ull;

    for (int b0 = 0; b0 < cmax; b0 += ST_KC) {
        const int nk = min(ST_KC, cmax - b0);
        if (MODE != MODE_SELECT_FROM_SCORES) {
            const int nf4 = d / 4;
#pragma unroll
            for (int e = 0; e < KREG; ++e) {
                const int p = tid + e * ST_NT;
                if (p < nk * nf4) *reinterpret_cast<float4*>(ks + (p / nf4) * ld + (p % nf4) * 4) = kreg[e];
            }
            for (int p = KREG * ST_NT + tid; p < nk * nf4; p += ST_NT)
                *reinterpret_cast<float4*>(ks + (p / nf4) * ld + (p % nf4) * 4) =
                    *reinterpret_cast<const float4*>(kb_base + (size_t)(b0 + p / nf4) * d + (p % nf4) * 4);
            __syncthreads();
            if (b0 + ST_KC < cmax) load_chunk(b0 + ST_KC);
            // register tile: thread -> rows 4*rg .. 4*rg+3, blocks bg, bg+16, bg+32, bg+48
            const int rg = tid >> 4, bg = tid & 15;
            float acc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int m = 0; m < 4; ++m) acc[i][m] = 0.f;
            for (int c = 0; c < d; c += 4) {
                float4 qv[4], kv[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) qv[i] = *reinterpret_cast<const float4*>(qs + (4 * rg + i) * ld + c);
#pragma unroll
                for (int m = 0; m < 4; ++m) kv[m] = *reinterpret_cast<const float4*>(ks + (bg + 16 * m) * ld + c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        acc[i][m] = fmaf(qv[i].x, kv[m].x, acc[i][m]);
                        acc[i][m] = fmaf(qv[i].y, kv[m].y, acc[i][m]);
                        acc[i][m] = fmaf(qv[i].z, kv[m].z, acc[i][m]);
                        acc[i][m] = fmaf(qv[i].w, kv[m].w, acc[i][m]);
                    }
            }
            __syncthreads();                 // every thread is done reading ks
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = 4 * rg + i;
                const int t = s.q0 + i0 + r;
                const int cr = t / s.bs;
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const int jj = bg + 16 * m;
                    const int blk = b0 + jj;
                    const bool valid = (r < nrows) && (jj < nk) && (blk < cr);
                    // forced leading (sink) blocks score +inf: always kept, like the own block
                    const float val = blk < s.n_sink ? INFINITY : s.scale * acc[i][m];
                    if (MODE == MODE_SCORES) {
                        if (r < nrows && jj < nk) {
                            float w = blk < cr ? val : (blk == cr ? INFINITY : -INFINITY);
                            scores_out[(((size_t)b * s.Hsel + u) * s.Tq + i0 + r) * s.nb_all + blk] = w;
                        }
                    } else {
                        ss[r * (ST_KC + 1) + jj] = valid ? val : -INFINITY;
                    }
                }
            }
        } else {
            for (int p = tid; p < ST_RT * ST_KC; p += ST_NT) {
                const int r = p / ST_KC, jj = p % ST_KC;
                const int blk = b0 + jj;
                float val = -INFINITY;
                if (r < nrows && jj < nk) {
                    const int cr = (s.q0 + i0 + r) / s.bs;
                    if (blk < cr)
                        val = blk < s.n_sink ? INFINITY   // forced leading blocks
                                             : scores_in[(((size_t)b * s.Hsel + u) * s.Tq + i0 + r) * s.nb_all + blk];
                }
                ss[r * (ST_KC + 1) + jj] = val;
            }
        }
        __syncthreads();

        if (MODE != MODE_SCORES && K1 > 0) {
#pragma unroll
            for (int j = 0; j < ST_RPW; ++j) {
                const int r = warp * ST_RPW + j;
                unsigned long long thr = __shfl_sync(0xffffffffu, key[j], K1 - 1);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int jj = lane + 32 * half;
                    const float sv = ss[r * (ST_KC + 1) + jj];
                    const unsigned long long ck = (sv != -INFINITY) ? score_key(sv, b0 + jj) : 0ull;
                    warp_list_merge(key[j], thr, ck, K1, lane);
                }
            }
        }
        __syncthreads();
    }

    if (MODE == MODE_SCORES) {
        // columns at and after the last chunk: +inf at the current block, -inf after it
        for (int p = tid; p < nrows * s.nb_all; p += ST_NT) {
            const int r = p / s.nb_all, j = p % s.nb_all;
            if (j < cmax) continue;
            const int cr = (s.q0 + i0 + r) / s.bs;
            scores_out[(((size_t)b * s.Hsel + u) * s.Tq + i0 + r) * s.nb_all + j] =
                j == cr ? INFINITY : -INFINITY;
        }
        return;
    }

#pragma unroll
    for (int j = 0; j < ST_RPW; ++j) {
        const int r = warp * ST_RPW + j;
        if (r >= nrows) continue;
        const int cr = (s.q0 + i0 + r) / s.bs;
        const bool have = lane < K1 && key[j] != 0ull;
        const int blk = have ? key_block(key[j]) : 0x7fffffff;
        const int npast = __popc(__ballot_sync(0xffffffffu, have));
        int rank = 0;
        for (int o = 0; o < 32; ++o) {
            const int other = __shfl_sync(0xffffffffu, blk, o);
            rank += (other < blk) ? 1 : 0;
        }
        int32_t* dst = idx + (((size_t)b * s.Hsel + u) * s.Tq + i0 + r) * s.topk;
        if (have) dst[rank] = blk;
        if (lane == 0) dst[npast] = cr;
        if (lane > npast && lane < s.topk) dst[lane] = -1;
    }
}

// Few query rows (decode): one 256-thread CTA per (query, unit, sequence),
// two per SM.  The row's pooled keys are contiguous in memory.  Every warp
// streams its own contiguous share of them through a private ring of
// shared-memory slots with bulk copies (TMA engine) on its own mbarriers, so
// no warp waits for another while keys arrive; the lanes split the d_qk dot
// product of a pooled row.  The scores collect in shared memory, every warp
// folds its share into a running top-(k-1), and the warp lists are merged as
// a tree.
// Eight warps with four 3 KB slots each measured faster at decode (64 x 65536
// tokens, d_qk 192) than 16 warps x 2 slots, 4 warps x 8 slots or 4 warps x
// 4 slots of 6 KB, all with the same 96 KB ring (53.5 us against 57-60 us).
constexpr int SR_NT = 256;
constexpr int SR_NW = SR_NT / 32;
constexpr int SR_MAXC = 2048;           // past blocks per row held in shared memory
constexpr int SR_NSLOT = 4;             // slots per warp (copies in flight)
constexpr int SR_SLOT = 3072;           // bytes per slot (4 pooled rows at d_qk = 192)
constexpr int SR_RING = SR_NW * SR_NSLOT * SR_SLOT;
constexpr int SR_SMEM = SR_RING + SR_MAXC * 4 + 256 * 4 + SR_NW * SR_NSLOT * 8;
static_assert(SR_NW * 32 * 8 <= SR_RING, "the warp lists reuse the ring");
static_assert(SR_SLOT % 1024 == 0, "a slot holds at least one pooled row at every d_qk");

template <int D>
__global__ void __launch_bounds__(SR_NT, 2)
    select_rows_kernel(Shape s, const __nv_bfloat16* __restrict__ q, const float* __restrict__ kbar,
                       int32_t* __restrict__ idx) {
    constexpr int RPS = SR_SLOT / (D * 4);       // pooled rows per slot
    constexpr int NSEG = D / 64;                 // float2 columns per lane
    extern __shared__ __align__(128) uint8_t sr_smem[];
    float* sc = reinterpret_cast<float*>(sr_smem + SR_RING);                 // [SR_MAXC]
    float* qs = sc + SR_MAXC;                                                  // [D]
    uint64_t* bars = reinterpret_cast<uint64_t*>(qs + 256);                   // [NW][NSLOT]
    // the warp lists reuse the ring once every warp has scored its share
    unsigned long long* lists = reinterpret_cast<unsigned long long*>(sr_smem);
    const int i = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = s.per_head ? u / s.G : u;
    const int h0 = s.per_head ? u : u * s.G;
    const int t = s.q0 + i;
    const int cr = t / s.bs;
    const int ncand = min(cr, s.nb_full);
    const int K1 = s.topk - 1;
    const float* kb = kbar + (size_t)(b * s.Hkv + kvh) * s.nb_full * D;
    // this warp's contiguous share of the candidates
    const int per = (ncand + SR_NW - 1) / SR_NW;
    const int w0 = min(ncand, warp * per), nw = min(ncand, w0 + per) - w0;
    const int nchunk = (nw + RPS - 1) / RPS;
    uint8_t* ring = sr_smem + (size_t)warp * SR_NSLOT * SR_SLOT;
    uint64_t* wb = bars + warp * SR_NSLOT;
    auto issue = [&](int c) {               // lane 0: chunk c into slot c % NSLOT
        const int nr = min(RPS, nw - c * RPS);
        const uint32_t bytes = (uint32_t)nr * D * 4;
        uint64_t* bar = wb + c % SR_NSLOT;
        tc::mbar_arrive_expect_tx(bar, bytes);
        tc::bulk_load(ring + (c % SR_NSLOT) * SR_SLOT, kb + (size_t)(w0 + c * RPS) * D, bytes, bar);
    };
    if (lane == 0) {
        for (int k = 0; k < SR_NSLOT; ++k) tc::mbar_init(wb + k, 1);
        tc::fence_mbar_init();
        for (int c = 0; c < SR_NSLOT && c < nchunk; ++c) issue(c);
    }
    // summed query, heads added in order (while the first copies are in flight)
    const __nv_bfloat16* qrow = q + (((size_t)b * s.Tq + i) * s.Hq + h0) * D;
    for (int c = tid; c < D; c += SR_NT) {
        float acc = 0.f;
        for (int hh = 0; hh < s.heads_per_unit; ++hh) acc += bf2f(qrow[hh * D + c]);
        qs[c] = acc;
    }
    __syncthreads();
    float2 qv[NSEG];
#pragma unroll
    for (int j = 0; j < NSEG; ++j) qv[j] = *reinterpret_cast<const float2*>(qs + 64 * j + 2 * lane);
    bool ok = true;
    for (int c = 0; c < nchunk; ++c) {
        ok = tc::mbar_wait_bounded(wb + c % SR_NSLOT, (c / SR_NSLOT) & 1, 1000000000ull) && ok;
        const float* buf = reinterpret_cast<const float*>(ring + (c % SR_NSLOT) * SR_SLOT);
        const int nr = min(RPS, nw - c * RPS);
        float part[RPS];
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr) {
            part[rr] = 0.f;
            if (rr < nr) {
#pragma unroll
                for (int j = 0; j < NSEG; ++j) {
                    const float2 kv = *reinterpret_cast<const float2*>(buf + rr * D + 64 * j + 2 * lane);
                    part[rr] = fmaf(qv[j].x, kv.x, part[rr]);
                    part[rr] = fmaf(qv[j].y, kv.y, part[rr]);
                }
            }
        }
        __syncwarp();                        // every lane has read the slot
        if (lane == 0 && c + SR_NSLOT < nchunk) issue(c + SR_NSLOT);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
            for (int rr = 0; rr < RPS; ++rr) part[rr] += __shfl_xor_sync(0xffffffffu, part[rr], off);
        float mine = 0.f;
#pragma unroll
        for (int rr = 0; rr < RPS; ++rr)
            if (lane == rr) mine = part[rr];
        if (lane < nr) {
            const int blk = w0 + c * RPS + lane;
            sc[blk] = blk < s.n_sink ? INFINITY : s.scale * mine;      // forced leading blocks
        }
    }
    // a copy that never landed only records an error (the row's ids are then invalid)
    if (!ok) atomicExch(&g_select_status, (int)NSA_ERR_TIMEOUT);
    __syncwarp();
    // the warp's top-(k-1) of its own share
    unsigned long long key = 0ull, thr = 0ull;
    if (K1 > 0) {
        for (int e0 = 0; e0 < nw; e0 += 32) {
            const int e = e0 + lane;
            const unsigned long long ck = e < nw ? score_key(sc[w0 + e], w0 + e) : 0ull;
            warp_list_merge(key, thr, ck, K1, lane);
        }
    }
    __syncthreads();                          // every warp is done with its ring
    lists[warp * 32 + lane] = key;
    __syncthreads();
    // tree merge of the warp lists
    for (int step = 1; step < SR_NW; step <<= 1) {
        if ((warp & (2 * step - 1)) == 0 && K1 > 0) {
            warp_list_merge(key, thr, lists[(warp + step) * 32 + lane], K1, lane);
            lists[warp * 32 + lane] = key;
        }
        __syncthreads();
    }
    if (warp == 0) {
        const bool have = lane < K1 && key != 0ull;
        const int blk = have ? key_block(key) : 0x7fffffff;
        const int npast = __popc(__ballot_sync(0xffffffffu, have));
        int rank = 0;
        for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xffffffffu, blk, o) < blk) ? 1 : 0;
        int32_t* dst = idx + (((size_t)b * s.Hsel + u) * s.Tq + i) * s.topk;
        if (have) dst[rank] = blk;
        if (lane == 0) dst[npast] = cr;
        if (lane > npast && lane < s.topk) dst[lane] = -1;
    }
}

// Selection-score variants (the probability sums of the unit's heads, or
// block scores gathered from the compressed branch's probabilities), one CTA
// per (query row, unit, sequence).  Both need every candidate's score before
// any is known (a softmax over the candidates), so the row is scored twice:
// pass 1 finds each head's softmax normaliser (online max and sum per thread,
// then combined across the CTA), pass 2 writes the normalised scores to
// shared memory.  The row is then written to `scores` and/or its top-(k-1)
// selected from shared memory (per-warp lists merged as a tree, as above).
//   VMODE 1: per head h, p_h(b) = softmax_b(scale q_h . kbar_b) over the
//            candidates b < c(t); score(b) = sum_h p_h(b).
//   VMODE 2: per head h, p_h(j) = softmax_j(scale q_h . kcmp_j) over the
//            visible compressed tokens (j * sc + lc - 1 <= t);
//            score(b) = sum_j (sum_h p_h(j)) |window_j ∩ block_b| / lc.
// One thread per candidate (block or compressed token) with the unit's query
// heads broadcast from shared memory; fp32 throughout.
constexpr int SV_NT = 256;
constexpr int SV_NW = SV_NT / 32;
constexpr int SV_MAXH = 16;
constexpr int SV_MAXC = 16384;          // candidate blocks / visible compressed tokens per row

// shared-memory entries kept for n candidates (a multiple of 4 floats, so the
// arrays after them stay 16-byte aligned)
__host__ __device__ __forceinline__ int sv_cap(int n) { return (n + 3) & ~3; }

template <int VMODE, int D>
__global__ void __launch_bounds__(SV_NT) score_variant_kernel(Shape s, const __nv_bfloat16* __restrict__ q,
                                                              const float* __restrict__ kbar,
                                                              const __nv_bfloat16* __restrict__ kcmp,
                                                              float* __restrict__ scores_out,
                                                              int32_t* __restrict__ idx) {
    extern __shared__ __align__(16) float sv_smem[];
    float* qs = sv_smem;                          // [nh][D]
    float* red_m = qs + SV_MAXH * D;              // [NW][MAXH]
    float* red_l = red_m + SV_NW * SV_MAXH;       // [NW][MAXH]
    float* hm = red_l + SV_NW * SV_MAXH;          // [MAXH] per-head max
    float* hl = hm + SV_MAXH;                     // [MAXH] per-head 1 / sum
    // (sized to this shape's candidates, so that several CTAs share an SM)
    float* sc = hl + SV_MAXH;                     // [nb_full] block scores
    float* pj = sc + sv_cap(s.nb_full);           // [n_cmp] compressed-token weights (VMODE 2)
    unsigned long long* lists = reinterpret_cast<unsigned long long*>(pj + (VMODE == 2 ? sv_cap(s.n_cmp) : 0));
    const int i = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int kvh = s.per_head ? u / s.G : u;
    const int h0 = s.per_head ? u : u * s.G;
    const int nh = s.heads_per_unit;
    const int t = s.q0 + i;
    const int cr = t / s.bs;
    const int ncand = min(cr, s.nb_full);
    // the candidates the softmax runs over: blocks, or visible compressed tokens
    const int nvis = t >= s.lc - 1 ? min(s.n_cmp, (t - s.lc + 1) / s.sc + 1) : 0;
    const int nsm = VMODE == 1 ? ncand : nvis;
    const __nv_bfloat16* qrow = q + (((size_t)b * s.Tq + i) * s.Hq + h0) * D;
    for (int e = tid; e < nh * D; e += SV_NT) qs[e] = bf2f(qrow[e]);
    __syncthreads();
    const float* kb = kbar + (size_t)(b * s.Hkv + kvh) * s.nb_full * D;
    const __nv_bfloat16* kc = kcmp + (size_t)(b * s.Hkv + kvh) * s.n_cmp * D;
    // scale * q_h . x for every head of the unit, x = candidate e's key row
    auto logits = [&](int e, float* lg) {
#pragma unroll
        for (int h = 0; h < SV_MAXH; ++h) lg[h] = 0.f;
        for (int c = 0; c < D; c += 8) {
            float x[8];
            if (VMODE == 1) {
                const float4 a = *reinterpret_cast<const float4*>(kb + (size_t)e * D + c);
                const float4 bq = *reinterpret_cast<const float4*>(kb + (size_t)e * D + c + 4);
                x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
                x[4] = bq.x; x[5] = bq.y; x[6] = bq.z; x[7] = bq.w;
            } else {
                unpack8(*reinterpret_cast<const uint4*>(kc + (size_t)e * D + c), x);
            }
#pragma unroll
            for (int h = 0; h < SV_MAXH; ++h) {
                if (h < nh) {
                    const float4 qa = *reinterpret_cast<const float4*>(qs + h * D + c);
                    const float4 qb = *reinterpret_cast<const float4*>(qs + h * D + c + 4);
                    float acc = lg[h];
                    acc = fmaf(qa.x, x[0], acc); acc = fmaf(qa.y, x[1], acc);
                    acc = fmaf(qa.z, x[2], acc); acc = fmaf(qa.w, x[3], acc);
                    acc = fmaf(qb.x, x[4], acc); acc = fmaf(qb.y, x[5], acc);
                    acc = fmaf(qb.z, x[6], acc); acc = fmaf(qb.w, x[7], acc);
                    lg[h] = acc;
                }
            }
        }
#pragma unroll
        for (int h = 0; h < SV_MAXH; ++h) lg[h] *= s.scale;
    };
    // pass 1: per-head online max / sum over this thread's candidates, then the CTA's
    float m[SV_MAXH], l[SV_MAXH];
#pragma unroll
    for (int h = 0; h < SV_MAXH; ++h) {
        m[h] = -INFINITY;
        l[h] = 0.f;
    }
    for (int e = tid; e < nsm; e += SV_NT) {
        float lg[SV_MAXH];
        logits(e, lg);
#pragma unroll
        for (int h = 0; h < SV_MAXH; ++h) {
            const float mn = fmaxf(m[h], lg[h]);
            l[h] = l[h] * expf(m[h] - mn) + expf(lg[h] - mn);
            m[h] = mn;
        }
    }
#pragma unroll
    for (int h = 0; h < SV_MAXH; ++h) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
            const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
            const float mn = fmaxf(m[h], mo);
            l[h] = (m[h] == -INFINITY ? 0.f : l[h] * expf(m[h] - mn)) +
                   (mo == -INFINITY ? 0.f : lo * expf(mo - mn));
            m[h] = mn;
        }
        if (lane == 0) {
            red_m[warp * SV_MAXH + h] = m[h];
            red_l[warp * SV_MAXH + h] = l[h];
        }
    }
    __syncthreads();
    if (tid < SV_MAXH) {
        float mm = -INFINITY, ll = 0.f;
        for (int w = 0; w < SV_NW; ++w) {
            const float mo = red_m[w * SV_MAXH + tid], lo = red_l[w * SV_MAXH + tid];
            const float mn = fmaxf(mm, mo);
            ll = (mm == -INFINITY ? 0.f : ll * expf(mm - mn)) + (mo == -INFINITY ? 0.f : lo * expf(mo - mn));
            mm = mn;
        }
        hm[tid] = mm;
        hl[tid] = ll > 0.f ? 1.f / ll : 0.f;
    }
    __syncthreads();
    // pass 2: the unit's summed probabilities per candidate
    float* dst2 = VMODE == 1 ? sc : pj;
    for (int e = tid; e < nsm; e += SV_NT) {
        float lg[SV_MAXH];
        logits(e, lg);
        float p = 0.f;
#pragma unroll
        for (int h = 0; h < SV_MAXH; ++h)
            if (h < nh) p += expf(lg[h] - hm[h]) * hl[h];
        dst2[e] = p;
    }
    __syncthreads();
    if (VMODE == 2) {
        // block b: the compressed tokens whose window [j sc, j sc + lc) overlaps it
        const float inv_lc = 1.f / (float)s.lc;
        for (int bb = tid; bb < ncand; bb += SV_NT) {
            const int lo_t = bb * s.bs, hi_t = (bb + 1) * s.bs;
            int j0 = lo_t - s.lc + 1;
            j0 = j0 <= 0 ? 0 : (j0 + s.sc - 1) / s.sc;
            const int j1 = min(nvis - 1, (hi_t - 1) / s.sc);
            float acc = 0.f;
            for (int j = j0; j <= j1; ++j) {
                const int ov = min(j * s.sc + s.lc, hi_t) - max(j * s.sc, lo_t);
                if (ov > 0) acc = fmaf(pj[j], (float)ov * inv_lc, acc);
            }
            sc[bb] = acc;
        }
        __syncthreads();
    }
    // forced leading blocks
    for (int bb = tid; bb < min(s.n_sink, ncand); bb += SV_NT) sc[bb] = INFINITY;
    __syncthreads();
    if (scores_out) {
        float* row = scores_out + (((size_t)b * s.Hsel + u) * s.Tq + i) * s.nb_all;
        for (int bb = tid; bb < s.nb_all; bb += SV_NT)
            row[bb] = bb < ncand ? sc[bb] : (bb == cr ? INFINITY : -INFINITY);
    }
    if (!idx) return;
    const int K1 = s.topk - 1;
    unsigned long long key = 0ull, thr = 0ull;
    const int per = (ncand + SV_NW - 1) / SV_NW;
    const int w0 = min(ncand, warp * per), nw = min(ncand, w0 + per) - w0;
    if (K1 > 0) {
        for (int e0 = 0; e0 < nw; e0 += 32) {
            const int e = e0 + lane;
            const unsigned long long ck = e < nw ? score_key(sc[w0 + e], w0 + e) : 0ull;
            warp_list_merge(key, thr, ck, K1, lane);
        }
    }
    lists[warp * 32 + lane] = key;
    __syncthreads();
    for (int step = 1; step < SV_NW; step <<= 1) {
        if ((warp & (2 * step - 1)) == 0 && K1 > 0) {
            warp_list_merge(key, thr, lists[(warp + step) * 32 + lane], K1, lane);
            lists[warp * 32 + lane] = key;
        }
        __syncthreads();
    }
    if (warp == 0) {
        const bool have = lane < K1 && key != 0ull;
        const int blk = have ? key_block(key) : 0x7fffffff;
        const int npast = __popc(__ballot_sync(0xffffffffu, have));
        int rank = 0;
        for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xffffffffu, blk, o) < blk) ? 1 : 0;
        int32_t* dst = idx + (((size_t)b * s.Hsel + u) * s.Tq + i) * s.topk;
        if (have) dst[rank] = blk;
        if (lane == 0) dst[npast] = cr;
        if (lane > npast && lane < s.topk) dst[lane] = -1;
    }
}

template <int VMODE, int D>
void launch_variant(const Shape& s, const __nv_bfloat16* q, const float* kbar, const __nv_bfloat16* kcmp,
                    float* scores_out, int32_t* idx, cudaStream_t st) {
    const int smem = (SV_MAXH * D + 2 * SV_NW * SV_MAXH + 2 * SV_MAXH + sv_cap(s.nb_full) +
                      (VMODE == 2 ? sv_cap(s.n_cmp) : 0)) * 4 + SV_NW * 32 * 8;
    cudaFuncSetAttribute(score_variant_kernel<VMODE, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    score_variant_kernel<VMODE, D><<<dim3(s.Tq, s.Hsel, s.B), SV_NT, smem, st>>>(s, q, kbar, kcmp, scores_out,
                                                                               idx);
}

bool score_variant_supported(const Shape& s) {
    return s.heads_per_unit <= SV_MAXH && s.nb_full <= SV_MAXC && s.n_cmp <= SV_MAXC &&
           (s.dqk == 64 || s.dqk == 128 || s.dqk == 192 || s.dqk == 256);
}

cudaError_t launch_score_variant(const Shape& s, const __nv_bfloat16* q, const float* kbar,
                                 const __nv_bfloat16* kcmp, float* scores_out, int32_t* idx,
                                 cudaStream_t st) {
#define NSA_SV_CASE(DD)                                                                          \
    if (s.dqk == DD) {                                                                           \
        if (s.score_mode == 1) launch_variant<1, DD>(s, q, kbar, kcmp, scores_out, idx, st);    \
        else launch_variant<2, DD>(s, q, kbar, kcmp, scores_out, idx, st);                      \
        return cudaGetLastError();                                                               \
    }
    NSA_SV_CASE(64)
    NSA_SV_CASE(128)
    NSA_SV_CASE(192)
    NSA_SV_CASE(256)
#undef NSA_SV_CASE
    return cudaErrorInvalidValue;
}

template <int D>
void launch_select_rows(const Shape& s, const __nv_bfloat16* q, const float* kbar, int32_t* idx,
                        cudaStream_t st) {
    cudaFuncSetAttribute(select_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, SR_SMEM);
    select_rows_kernel<D><<<dim3(s.Tq, s.Hsel, s.B), SR_NT, SR_SMEM, st>>>(s, q, kbar, idx);
}

cudaError_t launch_score_topk(const Shape& s, const __nv_bfloat16* q, const float* kbar,
                              const float* scores_in, float* scores_out, int32_t* idx,
                              cudaStream_t st) {
    const int ld = s.dqk + 4;
    const size_t key_buf = (size_t)ST_KC * ld > (size_t)ST_RT * (ST_KC + 1)
                               ? (size_t)ST_KC * ld : (size_t)ST_RT * (ST_KC + 1);
    const size_t smem = ((size_t)ST_RT * ld + key_buf) * sizeof(float);
    dim3 grid((s.Tq + ST_RT - 1) / ST_RT, s.Hsel, s.B);
    if (scores_out) {
        cudaFuncSetAttribute(score_topk_kernel<MODE_SCORES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        score_topk_kernel<MODE_SCORES><<<grid, ST_NT, smem, st>>>(s, q, kbar, nullptr, scores_out,
                                                                  nullptr);
    } else if (scores_in) {
        cudaFuncSetAttribute(score_topk_kernel<MODE_SELECT_FROM_SCORES>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        score_topk_kernel<MODE_SELECT_FROM_SCORES><<<grid, ST_NT, smem, st>>>(
            s, nullptr, nullptr, scores_in, nullptr, idx);
    } else if (s.Tq <= 16 && s.heads_per_unit <= 16 && s.nb_full <= SR_MAXC && s.dqk <= 256) {
        // few query rows: a 64-row score tile would be mostly empty
        if (s.dqk == 64) launch_select_rows<64>(s, q, kbar, idx, st);
        else if (s.dqk == 128) launch_select_rows<128>(s, q, kbar, idx, st);
        else if (s.dqk == 192) launch_select_rows<192>(s, q, kbar, idx, st);
        else launch_select_rows<256>(s, q, kbar, idx, st);
    } else {
        cudaFuncSetAttribute(score_topk_kernel<MODE_SELECT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        score_topk_kernel<MODE_SELECT><<<grid, ST_NT, smem, st>>>(s, q, kbar, nullptr, nullptr,
                                                                  idx);
    }
    return cudaGetLastError();
}

int read_and_clear_select_status() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_select_status, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_select_status, &zero, sizeof(int));
    return v;
}

}  // namespace nsa
