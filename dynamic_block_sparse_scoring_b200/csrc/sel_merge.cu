// Merge of the block-major selected-branch partials into one output per
// (query, head): o_sel = sum_s 2^(lse_s - M) o_s / sum_s 2^(lse_s - M).
//
// Each slot's partial is a softmax over one kept block (Zhang Xiaojun #94
// transcript (bidclub.ai), §4 "Inside Native Sparse Attention": the selected
// branch is one softmax over every token of the kept blocks); weighting the
// per-block results by their normalisers recovers that single softmax.
//
// HBM-bound: a thread owns 8 output columns of one (query, head) and issues
// all of its slots' 16-byte partial loads (after one read of the query's
// block ids) before combining them.
#include "common.cuh"

namespace nsa {

namespace {

constexpr int MG_MAXK = 16;   // slots per query handled here (the block-major path needs top_k <= 16)

__global__ void __launch_bounds__(256) sel_merge_kernel(Shape s, const int32_t* __restrict__ idx,
                                                        const __nv_bfloat16* __restrict__ part_o,
                                                        const float* __restrict__ part_lse,
                                                        __nv_bfloat16* __restrict__ o_sel) {
    const int hpt = s.heads_per_unit, c8n = s.dv / 8;
    const int per_tok = hpt * c8n;
    const int tok_per_cta = blockDim.x / per_tok;
    const int tl = threadIdx.x / per_tok, rem = threadIdx.x % per_tok;
    const int h = rem / c8n, c8 = rem % c8n;
    const int qi = blockIdx.x * tok_per_cta + tl;
    const int u = blockIdx.y, b = blockIdx.z;
    if (tl >= tok_per_cta || qi >= s.Tq) return;
    const size_t prow0 = ((size_t)(b * s.Hsel + u) * s.Tq + qi) * s.topk;
    // the kept blocks fill the first slots (ascending, -1 padded)
    const int32_t* irow = idx + prow0;
    int nvalid = 0;
#pragma unroll
    for (int sl = 0; sl < MG_MAXK; ++sl) nvalid += (sl < s.topk && irow[sl] >= 0) ? 1 : 0;
    float lse[MG_MAXK];
    uint4 raw[MG_MAXK];
    float m = -INFINITY;
#pragma unroll
    for (int sl = 0; sl < MG_MAXK; ++sl) {             // every load of the row issued at once
        lse[sl] = -INFINITY;
        if (sl < nvalid) {
            lse[sl] = __ldcs(part_lse + (prow0 + sl) * hpt + h);
            raw[sl] = __ldcs(reinterpret_cast<const uint4*>(part_o + ((prow0 + sl) * hpt + h) * s.dv + c8 * 8));
        }
    }
#pragma unroll
    for (int sl = 0; sl < MG_MAXK; ++sl) m = fmaxf(m, lse[sl]);
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    float wsum = 0.f;
#pragma unroll
    for (int sl = 0; sl < MG_MAXK; ++sl) {
        if (sl >= nvalid) break;
        const float w = exp2f(lse[sl] - m);
        wsum += w;
        float f[8];
        unpack8(raw[sl], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, f[e], acc[e]);
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] *= inv;
    const int hq = s.per_head ? u : u * s.G + h;
    *reinterpret_cast<uint4*>(o_sel + (((size_t)b * s.Tq + qi) * s.Hq + hq) * s.dv + c8 * 8) =
        pack8(acc);
}

}  // namespace

cudaError_t launch_sel_merge(const Shape& s, const int32_t* idx, const __nv_bfloat16* part_o,
                             const float* part_lse, __nv_bfloat16* o_sel, cudaStream_t st) {
    const int per_tok = s.heads_per_unit * (s.dv / 8);
    const int tok_per_cta = per_tok >= 256 ? 1 : 256 / per_tok;
    dim3 grid((s.Tq + tok_per_cta - 1) / tok_per_cta, s.Hsel, s.B);
    sel_merge_kernel<<<grid, tok_per_cta * per_tok, 0, st>>>(s, idx, part_o, part_lse, o_sel);
    return cudaGetLastError();
}

}  // namespace nsa
