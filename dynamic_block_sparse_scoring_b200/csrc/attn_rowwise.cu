// Gated three-branch sparse attention, one query row and one selection unit
// per CTA (FFMA, fp32 online softmax).
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention", Figure 2: a compressed branch over pooled block tokens, a
// selected branch over every token of the kept blocks, and a sliding-window
// branch; each branch output is multiplied by its gate and the three are
// summed.  §2 "Attention From First Principles": scaled dot products, causal
// mask, softmax, weighted sum of values.
//
// The CTA holds the unit's heads (the GQA group, or one head for per-head
// selection) and walks each branch's key list in chunks of 32 keys staged
// in shared memory: logits for all heads x 32 keys, an online-softmax update
// of (max, sum) per head, then the rescaled value accumulation.  Each branch
// is normalised by its own sum and added to the output with its gate.
#include <math.h>

#include "common.cuh"

namespace nsa {

constexpr int RW_NT = 256;
constexpr int RW_KC = 32;     // keys per chunk
constexpr int RW_MAXH = 16;   // heads per unit

struct RwSmem {
    float* qs;     // [nh][dqk]
    float* ks;     // [KC][dqk+1]
    float* vs;     // [KC][dv]
    float* ps;     // [nh][KC]
    float* os;     // [nh][dv]  branch accumulator
    float* oacc;   // [nh][dv]  gated sum over branches
    float* m;      // [nh]
    float* l;      // [nh]
    float* alpha;  // [nh]
};

__device__ void rw_chunk(const Shape& s, RwSmem& sm, int nh, const __nv_bfloat16* kbase,
                         const __nv_bfloat16* vbase, int n) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int dqk = s.dqk, dv = s.dv, ldk = dqk + 1;
    {
        const int nv = dqk / 8;
        for (int p = tid; p < n * nv; p += RW_NT) {
            const int r = p / nv, vec = p % nv;
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(kbase + (size_t)r * dqk + vec * 8), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) sm.ks[r * ldk + vec * 8 + e] = f[e];
        }
        const int nvv = dv / 8;
        for (int p = tid; p < n * nvv; p += RW_NT) {
            const int r = p / nvv, vec = p % nvv;
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(vbase + (size_t)r * dv + vec * 8), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) sm.vs[r * dv + vec * 8 + e] = f[e];
        }
    }
    __syncthreads();
    for (int p = tid; p < nh * RW_KC; p += RW_NT) {
        const int h = p / RW_KC, j = p % RW_KC;
        float acc = -INFINITY;
        if (j < n) {
            acc = 0.f;
            const float* qh = sm.qs + h * dqk;
            const float* kj = sm.ks + j * ldk;
            for (int c = 0; c < dqk; ++c) acc = fmaf(qh[c], kj[c], acc);
            acc *= s.scale;
        }
        sm.ps[h * RW_KC + j] = acc;
    }
    __syncthreads();
    for (int h = warp; h < nh; h += RW_NT / 32) {
        const float x = sm.ps[h * RW_KC + lane];
        const float mold = sm.m[h];
        const float mnew = fmaxf(mold, warp_max(x));
        const float p = (x == -INFINITY) ? 0.f : expf(x - mnew);
        const float sum = warp_sum(p);
        const float a = (mold == -INFINITY) ? 0.f : expf(mold - mnew);
        sm.ps[h * RW_KC + lane] = p;
        __syncwarp();
        if (lane == 0) {
            sm.l[h] = sm.l[h] * a + sum;
            sm.m[h] = mnew;
            sm.alpha[h] = a;
        }
    }
    __syncthreads();
    for (int p = tid; p < nh * dv; p += RW_NT) {
        const int h = p / dv, c = p % dv;
        float acc = sm.os[p] * sm.alpha[h];
        const float* ph = sm.ps + h * RW_KC;
        for (int j = 0; j < n; ++j) acc = fmaf(ph[j], sm.vs[j * dv + c], acc);
        sm.os[p] = acc;
    }
    __syncthreads();
}

__device__ void rw_begin_branch(RwSmem& sm, int nh, int dv) {
    for (int p = threadIdx.x; p < nh * dv; p += RW_NT) sm.os[p] = 0.f;
    for (int h = threadIdx.x; h < nh; h += RW_NT) {
        sm.m[h] = -INFINITY;
        sm.l[h] = 0.f;
    }
    __syncthreads();
}

__device__ void rw_end_branch(const Shape& s, RwSmem& sm, int nh, const float* gates, size_t grow,
                              int h0, int br) {
    for (int p = threadIdx.x; p < nh * s.dv; p += RW_NT) {
        const int h = p / s.dv;
        const float l = sm.l[h];
        const float w = gates ? gates[(grow + h0 + h) * 3 + br] : 1.0f;
        if (l > 0.f) sm.oacc[p] += w * sm.os[p] / l;
    }
    __syncthreads();
}

__global__ void __launch_bounds__(RW_NT) attn_rowwise_kernel(
    Shape s, const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
    const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ kcmp,
    const __nv_bfloat16* __restrict__ vcmp, const float* __restrict__ gates,
    const int32_t* __restrict__ idx, __nv_bfloat16* __restrict__ out) {
    extern __shared__ float smem[];
    const int i = blockIdx.x, u = blockIdx.y, b = blockIdx.z;
    const int nh = s.heads_per_unit;
    const int kvh = s.per_head ? u / s.G : u;
    const int h0 = s.per_head ? u : u * s.G;
    const int t = s.q0 + i;
    RwSmem sm;
    sm.qs = smem;
    sm.ks = sm.qs + nh * s.dqk;
    sm.vs = sm.ks + RW_KC * (s.dqk + 1);
    sm.ps = sm.vs + RW_KC * s.dv;
    sm.os = sm.ps + nh * RW_KC;
    sm.oacc = sm.os + nh * s.dv;
    sm.m = sm.oacc + nh * s.dv;
    sm.l = sm.m + RW_MAXH;
    sm.alpha = sm.l + RW_MAXH;

    const size_t qrow = (size_t)b * s.Tq + i;        // row of q / gates / out
    for (int p = threadIdx.x; p < nh * s.dqk; p += RW_NT)
        sm.qs[p] = bf2f(q[(qrow * s.Hq + h0) * s.dqk + p]);
    for (int p = threadIdx.x; p < nh * s.dv; p += RW_NT) sm.oacc[p] = 0.f;
    __syncthreads();

    const size_t kvoff = (size_t)(b * s.Hkv + kvh) * s.Tk;
    if (s.flags & NSA_BR_CMP) {
        rw_begin_branch(sm, nh, s.dv);
        // compressed token j is visible once its last source token j*sc + lc - 1 <= t
        int nvis = t - s.lc + 1 < 0 ? 0 : (t - s.lc + 1) / s.sc + 1;
        nvis = min(nvis, s.n_cmp);
        const size_t coff = (size_t)(b * s.Hkv + kvh) * s.n_cmp;
        for (int j0 = 0; j0 < nvis; j0 += RW_KC)
            rw_chunk(s, sm, nh, kcmp + (coff + j0) * s.dqk, vcmp + (coff + j0) * s.dv,
                     min(RW_KC, nvis - j0));
        rw_end_branch(s, sm, nh, gates, qrow * s.Hq, h0, 0);
    }
    if (s.flags & NSA_BR_SEL) {
        rw_begin_branch(sm, nh, s.dv);
        const int32_t* sel = idx + (((size_t)b * s.Hsel + u) * s.Tq + i) * s.topk;
        for (int slot = 0; slot < s.topk; ++slot) {
            const int blk = sel[slot];
            if (blk < 0 || blk > t / s.bs) continue;   // only causal blocks are attended
            const int lo = blk * s.bs;
            const int hi = min(min(lo + s.bs, t + 1), s.Tk);
            for (int j0 = lo; j0 < hi; j0 += RW_KC)
                rw_chunk(s, sm, nh, k + (kvoff + j0) * s.dqk, v + (kvoff + j0) * s.dv,
                         min(RW_KC, hi - j0));
        }
        rw_end_branch(s, sm, nh, gates, qrow * s.Hq, h0, 1);
    }
    if (s.flags & NSA_BR_WIN) {
        rw_begin_branch(sm, nh, s.dv);
        const int lo = max(0, t - s.win + 1);
        for (int j0 = lo; j0 <= t; j0 += RW_KC)
            rw_chunk(s, sm, nh, k + (kvoff + j0) * s.dqk, v + (kvoff + j0) * s.dv,
                     min(RW_KC, t + 1 - j0));
        rw_end_branch(s, sm, nh, gates, qrow * s.Hq, h0, 2);
    }
    for (int p = threadIdx.x; p < nh * s.dv; p += RW_NT)
        out[(qrow * s.Hq + h0) * s.dv + p] = __float2bfloat16_rn(sm.oacc[p]);
}

cudaError_t launch_attn(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                        const __nv_bfloat16* v, const __nv_bfloat16* kcmp,
                        const __nv_bfloat16* vcmp, const float* gates, const int32_t* idx,
                        __nv_bfloat16* out, cudaStream_t st) {
    const int nh = s.heads_per_unit;
    const size_t smem = ((size_t)nh * s.dqk + (size_t)RW_KC * (s.dqk + 1) + (size_t)RW_KC * s.dv +
                         (size_t)nh * RW_KC + 2 * (size_t)nh * s.dv + 3 * RW_MAXH) *
                        sizeof(float);
    cudaFuncSetAttribute(attn_rowwise_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)smem);
    dim3 grid(s.Tq, s.Hsel, s.B);
    attn_rowwise_kernel<<<grid, RW_NT, smem, st>>>(s, q, k, v, kcmp, vcmp, gates, idx, out);
    return cudaGetLastError();
}

}  // namespace nsa
