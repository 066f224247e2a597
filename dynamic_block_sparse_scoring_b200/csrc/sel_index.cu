// Inverted index of the selected blocks: for every (sequence, selection unit,
// block) the (query, slot) pairs whose top-k set holds that block.
//
// This is the gathering step of MoBA's execution (Zhang Xiaojun #94
// transcript (bidclub.ai), §7 "Kimi Simplifies The Sparse Route": for each KV
// block, collect the queries that chose it into one contiguous batch), used
// here for group-shared NSA selection too, so that a block's keys are loaded
// once for every query that kept it.
//
// Four launches: count pairs per list (atomics), one-CTA exclusive scans of
// the counts and of the work items per list, fill the lists (atomic cursors;
// the order inside a list does not matter because every row of an attention
// tile is computed independently), and cut each list into work items of at
// most `tok` queries.
#include "common.cuh"
#include "sel_index.cuh"

namespace nsa {

namespace {

// One thread per row of idx (a (sequence, unit, query)): the row's pairs all
// fall in lists of one chunk and unit, so the list base is one division per
// row.  A warp's 32 rows are consecutive queries, which mostly keep the same
// blocks in the same slots (the own block above all, and with per-head
// selection whole runs of sub-blocks), so at every slot the lanes that hit the
// same list are combined into one atomic (warp-aggregated, __match_any_sync).
// All 32 lanes run every slot (rows past the end take no part), so the warp
// stays converged at the collectives.
__device__ __forceinline__ size_t warp_row0() {
    return ((size_t)blockIdx.x * blockDim.x + threadIdx.x) & ~size_t(31);
}

__global__ void count_pairs_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ cnt,
                                   int BHsel, int Tq, int topk, int nb_all, size_t rows) {
    const int lane = threadIdx.x & 31;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t r0 = warp_row0(); r0 < rows; r0 += stride) {
        const size_t r = r0 + lane;
        const bool in = r < rows;
        const size_t bu = in ? r / Tq : 0;
        const int qi = in ? (int)(r - bu * Tq) : 0;
        const int lbase = (int)(((size_t)(qi / SEL_CHUNK) * BHsel + bu) * nb_all);
        const int32_t* row = idx + r * topk;
        for (int k = 0; k < topk; ++k) {
            const int blk = in ? row[k] : -1;
            const unsigned valid = __ballot_sync(0xffffffffu, blk >= 0);
            if (blk >= 0) {
                const int lid = lbase + blk;
                const unsigned peers = __match_any_sync(valid, lid);
                if (lane == __ffs(peers) - 1) atomicAdd(&cnt[lid], __popc(peers));
            }
        }
    }
}

// Single CTA of 1024 threads: off = exclusive scan of cnt, item_off =
// exclusive scan of ceil(cnt / tok); writes the totals at index L.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t* __restrict__ cnt,
                                                    int32_t* __restrict__ off,
                                                    int32_t* __restrict__ item_off,
                                                    int32_t* __restrict__ cursor, int L, int tok) {
    __shared__ int32_t wsum_a[32], wsum_b[32];
    __shared__ int32_t carry_a, carry_b;
    if (threadIdx.x == 0) carry_a = carry_b = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < L; base += 1024) {
        const int i = base + threadIdx.x;
        const int c = i < L ? cnt[i] : 0;
        const int n = (c + tok - 1) / tok;
        int a = c, b = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int ya = __shfl_up_sync(0xffffffffu, a, o);
            const int yb = __shfl_up_sync(0xffffffffu, b, o);
            if (lane >= o) {
                a += ya;
                b += yb;
            }
        }
        if (lane == 31) {
            wsum_a[warp] = a;
            wsum_b[warp] = b;
        }
        __syncthreads();
        if (warp == 0) {
            int sa = wsum_a[lane], sb = wsum_b[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int ya = __shfl_up_sync(0xffffffffu, sa, o);
                const int yb = __shfl_up_sync(0xffffffffu, sb, o);
                if (lane >= o) {
                    sa += ya;
                    sb += yb;
                }
            }
            wsum_a[lane] = sa;
            wsum_b[lane] = sb;
        }
        __syncthreads();
        const int pa = (warp ? wsum_a[warp - 1] : 0) + a - c + carry_a;   // exclusive
        const int pb = (warp ? wsum_b[warp - 1] : 0) + b - n + carry_b;
        if (i < L) {
            off[i] = pa;
            cursor[i] = pa;
            item_off[i] = pb;
        }
        __syncthreads();
        if (threadIdx.x == 1023) {
            carry_a = pa + c;
            carry_b = pb + n;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        off[L] = carry_a;
        item_off[L] = carry_b;
    }
}

__global__ void fill_pairs_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ cursor,
                                  int32_t* __restrict__ list, int BHsel, int Tq, int topk,
                                  int nb_all, size_t rows) {
    const int lane = threadIdx.x & 31;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (size_t r0 = warp_row0(); r0 < rows; r0 += stride) {
        const size_t r = r0 + lane;
        const bool in = r < rows;
        const size_t bu = in ? r / Tq : 0;
        const int qi = in ? (int)(r - bu * Tq) : 0;
        const int lbase = (int)(((size_t)(qi / SEL_CHUNK) * BHsel + bu) * nb_all);
        const int32_t* row = idx + r * topk;
        for (int k = 0; k < topk; ++k) {
            const int blk = in ? row[k] : -1;
            const unsigned valid = __ballot_sync(0xffffffffu, blk >= 0);
            if (blk >= 0) {
                const int lid = lbase + blk;
                const unsigned peers = __match_any_sync(valid, lid);
                const int leader = __ffs(peers) - 1;
                int pos = 0;
                if (lane == leader) pos = atomicAdd(&cursor[lid], __popc(peers));
                pos = __shfl_sync(peers, pos, leader) + __popc(peers & ((1u << lane) - 1u));
                list[pos] = qi * SEL_SLOTS + k;
            }
        }
    }
}

__global__ void make_items_kernel(const int32_t* __restrict__ off,
                                  const int32_t* __restrict__ item_off, int4* __restrict__ items,
                                  int L, int tok) {
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < L; i += gridDim.x * blockDim.x) {
        const int c = off[i + 1] - off[i];
        int it = item_off[i];
        for (int q = 0; q < c; q += tok, ++it) items[it] = make_int4(i, off[i] + q, min(tok, c - q), 0);
    }
}

// One head per unit with blocks longer than 64 keys: a kept block becomes its
// 64-key sub-blocks, so that the block-major kernel (64 keys per item) serves
// it unchanged.  The selected branch is one softmax over every key of the kept
// blocks up to the query, and the sub-blocks starting after the query hold
// none of those keys, so they are dropped.  Row r of idx_sub lists the
// sub-blocks of row r's kept blocks in order (ascending), -1 padded to
// top_k * (sel_block / 64) entries.
__global__ void expand_kernel(const int32_t* __restrict__ idx, int32_t* __restrict__ idx_sub, size_t rows,
                              int Tq, int q0, int topk, int bs, int spb) {
    for (size_t r = (size_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
         r += (size_t)gridDim.x * blockDim.x) {
        const int t = q0 + (int)(r % Tq);
        const int32_t* src = idx + r * topk;
        int32_t* dst = idx_sub + r * (size_t)topk * spb;
        int n = 0;
        for (int e = 0; e < topk; ++e) {
            const int blk = src[e];
            if (blk < 0 || blk > t / bs) continue;      // only causal blocks are attended
            for (int sb = 0; sb < spb && blk * bs + sb * 64 <= t; ++sb) dst[n++] = blk * spb + sb;
        }
        for (; n < topk * spb; ++n) dst[n] = -1;
    }
}

// Debug check of a caller-supplied idx: a row is valid when its ids lie in
// [0, c(t)] and below nb_all, are strictly ascending, are followed only by -1,
// and include the own block c(t).  Reads idx only; counts the invalid rows.
__device__ int g_idx_bad = 0;

__global__ void check_idx_kernel(const int32_t* __restrict__ idx, size_t rows, int Tq, int q0, int topk,
                                 int bs, int nb_all) {
    for (size_t r = (size_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows;
         r += (size_t)gridDim.x * blockDim.x) {
        const int c = (q0 + (int)(r % Tq)) / bs;
        const int32_t* row = idx + r * topk;
        bool bad = false, pad = false, own = false;
        int prev = -1;
        for (int e = 0; e < topk; ++e) {
            const int v = row[e];
            if (v == -1) {
                pad = true;
                continue;
            }
            if (pad || v < 0 || v > c || v >= nb_all || v <= prev) bad = true;
            own |= v == c;
            prev = v;
        }
        if (bad || !own) atomicAdd(&g_idx_bad, 1);
    }
}

}  // namespace

cudaError_t check_idx_rows(const Shape& s, const int32_t* idx, int* bad, cudaStream_t st) {
    const size_t rows = (size_t)s.B * s.Hsel * s.Tq;
    static const int zero = 0;
    *bad = 0;
    cudaError_t e = cudaMemcpyToSymbolAsync(g_idx_bad, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, st);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<size_t>((rows + 255) / 256, 148 * 8);
    check_idx_kernel<<<grid, 256, 0, st>>>(idx, rows, s.Tq, s.q0, s.topk, s.bs, s.nb_all);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbolAsync(bad, g_idx_bad, sizeof(int), 0, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return e;
    return cudaStreamSynchronize(st);
}

cudaError_t launch_sel_expand(const Shape& s, const int32_t* idx, int32_t* idx_sub, cudaStream_t st) {
    const size_t rows = (size_t)s.B * s.Hsel * s.Tq;
    if (rows == 0) return cudaSuccess;
    const int grid = (int)std::min<size_t>((rows + 255) / 256, 148 * 16);
    expand_kernel<<<grid, 256, 0, st>>>(idx, idx_sub, rows, s.Tq, s.q0, s.topk, s.bs, s.bs / 64);
    return cudaGetLastError();
}

cudaError_t launch_sel_index(const Shape& s, const int32_t* idx, const SelIndex& x, int tok,
                             cudaStream_t st) {
    const int L = (int)sel_lists(s);
    const int BHsel = s.B * s.Hsel;
    const size_t rows = (size_t)s.B * s.Hsel * s.Tq;
    cudaError_t e = cudaMemsetAsync(x.cnt, 0, sizeof(int32_t) * L, st);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<size_t>((rows + 255) / 256, 148 * 16);
    count_pairs_kernel<<<grid, 256, 0, st>>>(idx, x.cnt, BHsel, s.Tq, s.topk, s.nb_all, rows);
    scan_kernel<<<1, 1024, 0, st>>>(x.cnt, x.off, x.item_off, x.cursor, L, tok);
    fill_pairs_kernel<<<grid, 256, 0, st>>>(idx, x.cursor, x.list, BHsel, s.Tq, s.topk, s.nb_all,
                                            rows);
    make_items_kernel<<<(L + 255) / 256, 256, 0, st>>>(x.off, x.item_off, x.items, L, tok);
    return cudaGetLastError();
}

}  // namespace nsa
