// Merge of the block-major selected-branch partials into one output per
// (query, head): o_sel = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M).
//
// Each slot's partial is a softmax over one kept block (Zhang Xiaojun #94
// transcript (bidclub.ai), §4 "Inside Native Sparse Attention": the selected
// branch is one softmax over every token of the kept blocks); weighting the
// per-block results by their normalisers recovers that single softmax.
//
// HBM-bound: a thread owns 8 output columns of one (query, head) and issues
// its slots' 16-byte partial loads eight at a time (after one read of the
// query's block ids) before combining them.
#include "common.cuh"

namespace nsa {

namespace {

constexpr int MG_MAXK = 16;   // slots per query handled here (the block-major path needs top_k <= 16)
constexpr int MG_BATCH = 8;

__global__ void __launch_bounds__(256, 4) sel_merge_kernel(Shape s, const int32_t* __restrict__ idx,
                                                        const __nv_bfloat16* __restrict__ part_o,
                                                        const float* __restrict__ part_lse,
                                                        __nv_bfloat16* __restrict__ o_sel) {
    // one CTA per query: the query's slot count and its (slot, head) log-sum-exps
    // are staged once in shared memory (one coalesced read), so that every thread
    // issues only its 16-byte partial loads
    __shared__ float lse_s[MG_MAXK * 16];
    __shared__ int nvalid_s;
    const int hpt = s.heads_per_unit, c8n = s.dv / 8;
    const int qi = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int h = threadIdx.x / c8n, c8 = threadIdx.x % c8n;
    const size_t prow0 = ((size_t)(b * s.Hsel + u) * s.Tq + qi) * s.topk;
    if (threadIdx.x < 32) {
        // the kept blocks fill the first slots (ascending, -1 padded)
        const int blk = threadIdx.x < s.topk ? idx[prow0 + threadIdx.x] : -1;
        const int nv = __popc(__ballot_sync(0xffffffffu, blk >= 0));
        if (threadIdx.x == 0) nvalid_s = nv;
    }
    for (int e = threadIdx.x; e < s.topk * hpt; e += blockDim.x)
        lse_s[e] = __ldcs(part_lse + prow0 * hpt + e);
    __syncthreads();
    if (h >= hpt) return;
    const int nvalid = nvalid_s;
    float m = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < MG_MAXK; ++sl)
        if (sl < nvalid) m = fmaxf(m, lse_s[sl * hpt + h]);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float wsum = 0.f;
    // slots in batches of MG_BATCH whose loads are issued together: a batch fits the
    // 64 registers that four CTAs of 256 threads per SM leave each thread, and four
    // CTAs keep more bytes in flight than three with the whole row at once
#pragma unroll
    for (int b0 = 0; b0 < MG_MAXK; b0 += MG_BATCH) {
        if (b0 >= nvalid) break;
        uint4 raw[MG_BATCH];
#pragma unroll
        for (int k = 0; k < MG_BATCH; ++k)
            if (b0 + k < nvalid)
                raw[k] = __ldcs(reinterpret_cast<const uint4*>(part_o + ((prow0 + b0 + k) * hpt + h) * s.dv + c8 * 8));
#pragma unroll
        for (int k = 0; k < MG_BATCH; ++k) {
            if (b0 + k >= nvalid) break;
            const float w = exp2f(lse_s[(b0 + k) * hpt + h] - m);
            wsum += w;
            float f[8];
            unpack8(raw[k], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, f[e], acc[e]);
        }
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= inv;
    const int hq = s.per_head ? u : u * s.G + h;
    *reinterpret_cast<uint4*>(o_sel + (((size_t)b * s.Tq + qi) * s.Hq + hq) * s.dv + c8 * 8) =
        pack8(acc);
}

// Selected branch alone with one head per unit (MoBA's per-head selection;
// Zhang Xiaojun #94 transcript (bidclub.ai), §7: every head keeps its own
// blocks and the output is that branch alone).  A kept block reaches here as
// its 64-key sub-blocks, each one slot with its own partial; the merge is the
// same normaliser-weighted sum, written to out with the branch's gate.  One
// CTA per (query, group of MO_NT / (d_v / 8) heads): the heads' block ids and
// log-sum-exps are staged in shared memory with one coalesced pass, so every
// thread (8 output columns of one head) knows its slot count and maximum
// before it issues its 16-byte partial loads, eight slots at a time.
constexpr int MO_NT = 256;
constexpr int MO_MAXK = 64;    // slots per (query, head): kept 64-key sub-blocks
constexpr int MO_MAXH = 32;    // heads per CTA (d_v = 64)
constexpr int MO_BATCH = 8;

__global__ void __launch_bounds__(MO_NT, 3) sel_merge_out_kernel(Shape s, const int32_t* __restrict__ idx,
                                                               const __nv_bfloat16* __restrict__ part_o,
                                                               const float* __restrict__ part_lse,
                                                               const float* __restrict__ gates,
                                                               __nv_bfloat16* __restrict__ out) {
    __shared__ float lse_s[MO_MAXH * MO_MAXK];
    __shared__ int nvalid_s[MO_MAXH];
    const int c8n = s.dv / 8, hpc = MO_NT / c8n;
    const int qi = blockIdx.x, b = blockIdx.z;
    const int h0 = blockIdx.y * hpc;
    const int nh = min(hpc, s.Hq - h0);
    if (threadIdx.x < MO_MAXH) nvalid_s[threadIdx.x] = 0;
    __syncthreads();
    // unit = head: the partial rows of (b, head, query) are ((b * Hsel + head) * Tq + qi) * topk + slot
    for (int e = threadIdx.x; e < nh * s.topk; e += MO_NT) {
        const int hl = e / s.topk, sl = e % s.topk;
        const size_t pr = ((size_t)(b * s.Hsel + h0 + hl) * s.Tq + qi) * s.topk + sl;
        const int blk = idx[pr];
        const float lse = __ldcs(part_lse + pr);
        lse_s[hl * MO_MAXK + sl] = blk >= 0 ? lse : -INFINITY;
        if (blk >= 0) atomicAdd(&nvalid_s[hl], 1);       // the kept sub-blocks fill the first slots
    }
    __syncthreads();
    const int hl = threadIdx.x / c8n, c8 = threadIdx.x % c8n;
    if (hl >= nh) return;
    const int h = h0 + hl;
    const int nvalid = nvalid_s[hl];
    const float* lrow = lse_s + hl * MO_MAXK;
    float m = -INFINITY;
    for (int k = 0; k < nvalid; ++k) m = fmaxf(m, lrow[k]);
    const size_t prow0 = ((size_t)(b * s.Hsel + h) * s.Tq + qi) * s.topk;
    float o[8] = {0, 0, 0, 0, 0, 0, 0, 0}, wsum = 0.f;
    for (int kb = 0; kb < nvalid; kb += MO_BATCH) {
        uint4 raw[MO_BATCH];
#pragma unroll
        for (int k = 0; k < MO_BATCH; ++k)
            if (kb + k < nvalid)
                raw[k] = __ldcs(reinterpret_cast<const uint4*>(part_o + (prow0 + kb + k) * s.dv + c8 * 8));
#pragma unroll
        for (int k = 0; k < MO_BATCH; ++k) {
            if (kb + k >= nvalid) break;
            const float w = exp2f(lrow[kb + k] - m);
            wsum += w;
            float f[8];
            unpack8(raw[k], f);
#pragma unroll
            for (int q = 0; q < 8; ++q) o[q] = fmaf(w, f[q], o[q]);
        }
    }
    const size_t row = ((size_t)b * s.Tq + qi) * s.Hq + h;      // (b, query, head) of out
    const float g = gates ? gates[row * 3 + 1] : 1.f;
    const float scale = wsum > 0.f ? g / wsum : 0.f;
#pragma unroll
    for (int q = 0; q < 8; ++q) o[q] *= scale;
    *reinterpret_cast<uint4*>(out + row * s.dv + c8 * 8) = pack8(o);
}

}  // namespace

cudaError_t launch_sel_merge_out(const Shape& s, const int32_t* idx, const __nv_bfloat16* part_o,
                                 const float* part_lse, const float* gates, __nv_bfloat16* out,
                                 cudaStream_t st) {
    if ((size_t)s.B * s.Tq * s.Hq == 0) return cudaSuccess;
    if (s.topk > MO_MAXK || (s.dv != 64 && s.dv != 128)) return cudaErrorInvalidValue;
    const int hpc = MO_NT / (s.dv / 8);
    dim3 grid(s.Tq, (s.Hq + hpc - 1) / hpc, s.B);
    sel_merge_out_kernel<<<grid, MO_NT, 0, st>>>(s, idx, part_o, part_lse, gates, out);
    return cudaGetLastError();
}

cudaError_t launch_sel_merge(const Shape& s, const int32_t* idx, const __nv_bfloat16* part_o,
                             const float* part_lse, __nv_bfloat16* o_sel, cudaStream_t st) {
    // one CTA per query row: heads x 16-byte columns threads (<= 16 x 16)
    const int threads = ((s.heads_per_unit * (s.dv / 8) + 31) / 32) * 32;
    dim3 grid(s.Tq, s.Hsel, s.B);
    sel_merge_kernel<<<grid, std::max(threads, 32), 0, st>>>(s, idx, part_o, part_lse, o_sel);
    return cudaGetLastError();
}

}  // namespace nsa
