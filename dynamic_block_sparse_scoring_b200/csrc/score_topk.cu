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

namespace nsa {

constexpr int ST_RT = 64;   // query rows per CTA
constexpr int ST_KC = 64;   // pooled keys per chunk
constexpr int ST_NT = 256;  // threads per CTA (8 warps x 8 rows of top-k state)
constexpr int ST_RPW = ST_RT / 8;   // rows per warp

enum { MODE_SELECT = 0, MODE_SCORES = 1, MODE_SELECT_FROM_SCORES = 2 };

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
                    const float val = s.scale * acc[i][m];
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
                        val = scores_in[(((size_t)b * s.Hsel + u) * s.Tq + i0 + r) * s.nb_all + blk];
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
                    unsigned mask = __ballot_sync(0xffffffffu, ck > thr);
                    while (mask) {
                        const int src = __ffs(mask) - 1;
                        const unsigned long long x = __shfl_sync(0xffffffffu, ck, src);
                        const unsigned long long mine = key[j];
                        const int p = __popc(__ballot_sync(0xffffffffu, lane < K1 && mine > x));
                        const unsigned long long up = __shfl_up_sync(0xffffffffu, mine, 1);
                        if (lane < K1) {
                            if (lane == p) key[j] = x;
                            else if (lane > p) key[j] = up;
                        }
                        thr = __shfl_sync(0xffffffffu, key[j], K1 - 1);
                        mask &= ~(1u << src);
                        mask &= __ballot_sync(0xffffffffu, ck > thr);
                    }
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

// Few query rows (decode): one CTA per (query, unit, sequence).  Each of its
// 32 warps scores a contiguous range of past blocks (the lanes split the d_qk
// dot product, so a pooled key row is one coalesced read) and keeps its own
// running top-(k-1); the warp lists are then merged by warp 0.
constexpr int SR_NT = 1024;             // 32 warps: more pooled rows in flight per CTA
constexpr int SR_NW = SR_NT / 32;

__global__ void __launch_bounds__(SR_NT, 1) select_rows_kernel(Shape s, const __nv_bfloat16* __restrict__ q,
                                                            const float* __restrict__ kbar,
                                                            int32_t* __restrict__ idx) {
    __shared__ float qs[256];
    __shared__ unsigned long long lists[SR_NW][32];
    const int i = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d = s.dqk;
    const int kvh = s.per_head ? u / s.G : u;
    const int h0 = s.per_head ? u : u * s.G;
    const int t = s.q0 + i;
    const int cr = t / s.bs;
    const int ncand = min(cr, s.nb_full);
    const int K1 = s.topk - 1;
    for (int c = tid; c < d; c += SR_NT) {
        float acc = 0.f;
        const __nv_bfloat16* src = q + (((size_t)b * s.Tq + i) * s.Hq + h0) * d + c;
        for (int hh = 0; hh < s.heads_per_unit; ++hh) acc += bf2f(src[(size_t)hh * d]);
        qs[c] = acc;
    }
    __syncthreads();
    unsigned long long key = 0ull;               // this lane's slot of the warp's list
    unsigned long long thr = 0ull;
    const int per = (ncand + SR_NW - 1) / SR_NW;
    const int j0 = warp * per, j1 = min(ncand, j0 + per);
    const float* kb = kbar + (size_t)(b * s.Hkv + kvh) * s.nb_full * d;
    for (int jb = j0; jb < j1; jb += 32) {
        // 32 blocks per round: every lane ends up holding the score of block jb + lane
        float mine = -INFINITY;
        for (int jj = 0; jj < 32 && jb + jj < j1; jj += 8) {
            // eight pooled rows in flight at once
            float part[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                part[e] = 0.f;
                if (jb + jj + e < j1) {
                    const float* row = kb + (size_t)(jb + jj + e) * d;
#pragma unroll
                    for (int cc = 0; cc < 8; ++cc) {      // d <= 256: all loads issued together
                        const int c = lane + 32 * cc;
                        if (c < d) part[e] = fmaf(qs[c], row[c], part[e]);
                    }
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float tot = warp_sum(part[e]);
                if (lane == jj + e) mine = s.scale * tot;
            }
        }
        if (K1 > 0) {
            const unsigned long long ck = (jb + lane < j1) ? score_key(mine, jb + lane) : 0ull;
            unsigned mask = __ballot_sync(0xffffffffu, ck > thr);
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
    }
    lists[warp][lane] = key;
    __syncthreads();
    if (warp != 0) return;
    // merge the other warps' lists into warp 0's
    for (int w = 1; w < SR_NW && K1 > 0; ++w) {
        const unsigned long long ck = lists[w][lane];
        unsigned mask = __ballot_sync(0xffffffffu, ck > thr);
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
    } else if (s.Tq <= 16) {
        // few query rows: a 64-row score tile would be mostly empty
        select_rows_kernel<<<dim3(s.Tq, s.Hsel, s.B), SR_NT, 0, st>>>(s, q, kbar, idx);
    } else {
        cudaFuncSetAttribute(score_topk_kernel<MODE_SELECT>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        score_topk_kernel<MODE_SELECT><<<grid, ST_NT, smem, st>>>(s, q, kbar, nullptr, nullptr,
                                                                  idx);
    }
    return cudaGetLastError();
}

}  // namespace nsa
