// Backward pass of the gated three-branch sparse attention for fixed block
// sets.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §2 "Attention From First
// Principles": each branch is a softmax-weighted sum of values; §4, Figure 2:
// the branch outputs are gated and summed; §6 "Why Sparse Attention Wins":
// the top-k choice is discrete and passes no gradient, while the compressed
// branch carries gradient back to the keys and values it pools.  For one
// query row and head, with d_out its output gradient and g_br the branch gate:
//   o_br = sum_e P_e v_e,  dgate_br = d_out . o_br,  d_o = g_br d_out,
//   D = d_o . o_br,  ds_e = P_e (d_o . v_e - D),
//   dq += scale sum_e ds_e k_e,  dk_e += scale ds_e q,  dv_e += P_e d_o.
// Keys of the compressed branch are the compressed tokens; their gradients
// are collected per token (fp32) and then spread over the token's window with
// weight 1 / cmp_block, the derivative of the window mean.
//
// One CTA (128 threads) per (query row, head, sequence): the branch's scores,
// then probabilities, then ds live in shared memory (one value per key), the
// dot products run over the threads, and dk / dv (shared by the heads of a
// KV group and by many queries) accumulate with fp32 atomic adds.  This is a
// plain FFMA formulation, written for clarity of the gradient rather than
// speed.
#include <math.h>

#include <algorithm>

#include "common.cuh"

namespace nsa {

namespace {

constexpr int BW_NT = 128;
constexpr int BW_MAXK = 16384;          // keys of one branch held in shared memory
constexpr int BW_MAXB = 32;             // kept blocks per row

struct BwdArgs {
    Shape s;
    const __nv_bfloat16 *q, *k, *v, *kcmp, *vcmp, *d_out;
    const float* gates;
    const int32_t* idx;
    float *dq, *dk, *dv, *dgates, *dkc, *dvc;
};

__device__ __forceinline__ float block_sum(float x, float* red) {
    x = warp_sum(x);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < BW_NT / 32; ++w) t += red[w];
    return t;
}

__device__ __forceinline__ float block_max(float x, float* red) {
    x = warp_max(x);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float t = -INFINITY;
    for (int w = 0; w < BW_NT / 32; ++w) t = fmaxf(t, red[w]);
    return t;
}

__global__ void __launch_bounds__(BW_NT) bwd_rows_kernel(BwdArgs a) {
    extern __shared__ float bw_smem[];
    const Shape& s = a.s;
    const int dqk = s.dqk, dv = s.dv;
    float* qs = bw_smem;                  // [dqk] the query row
    float* dos = qs + dqk;                // [dv] d_out of the row
    float* dob = dos + dv;                // [dv] gate * d_out
    float* os = dob + dv;                 // [dv] branch output
    float* red = os + dv;                 // [4] reductions
    int* blk_start = reinterpret_cast<int*>(red + 4);   // [BW_MAXB + 1] kept blocks' key offsets
    int* blk_id = blk_start + BW_MAXB + 1;               // [BW_MAXB]
    float* pe = reinterpret_cast<float*>(blk_id + BW_MAXB);   // [BW_MAXK] scores -> P -> ds
    const int i = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x;
    const int t = s.q0 + i;
    const int kvh = h / s.G;
    const size_t row = ((size_t)b * s.Tq + i) * s.Hq + h;
    for (int c = tid; c < dqk; c += BW_NT) qs[c] = bf2f(a.q[row * dqk + c]);
    for (int c = tid; c < dv; c += BW_NT) dos[c] = bf2f(a.d_out[row * dv + c]);
    __syncthreads();
    float dq_acc[2] = {0.f, 0.f};         // columns tid and tid + 128 of dq (dqk <= 256)
    const size_t plane = (size_t)b * s.Hkv + kvh;
    for (int br = 0; br < 3; ++br) {
        if (!(s.flags & (1u << br))) {
            // the output does not depend on a disabled branch's gate
            if (tid == 0 && a.dgates) a.dgates[row * 3 + br] = 0.f;
            continue;
        }
        // the branch's keys: e -> (key row, whether it is a compressed token)
        int nkeys = 0, win_lo = 0, nblk = 0;
        if (br == 0) {
            nkeys = t >= s.lc - 1 ? min(s.n_cmp, (t - s.lc + 1) / s.sc + 1) : 0;
        } else if (br == 2) {
            win_lo = max(0, t - s.win + 1);
            nkeys = t - win_lo + 1;
        } else {
            if (tid == 0) {
                const int u = s.per_head ? h : kvh;
                const int32_t* r = a.idx + (((size_t)b * s.Hsel + u) * s.Tq + i) * s.topk;
                int n = 0, tot = 0;
                for (int e = 0; e < s.topk && n < BW_MAXB; ++e) {
                    const int j = r[e];
                    if (j < 0 || j * s.bs > t) continue;
                    blk_id[n] = j;
                    blk_start[n] = tot;
                    tot += min(s.bs, t - j * s.bs + 1);
                    ++n;
                }
                blk_start[n] = tot;
                red[3] = __int_as_float(n);
            }
            __syncthreads();
            nblk = __float_as_int(red[3]);
            nkeys = blk_start[nblk];
        }
        nkeys = min(nkeys, BW_MAXK);
        const float g = a.gates ? a.gates[row * 3 + br] : 1.f;
        auto key_row = [&](int e) -> size_t {         // row of k / v (or of kcmp / vcmp)
            if (br == 0) return plane * s.n_cmp + e;
            if (br == 2) return plane * s.Tk + win_lo + e;
            int lo = 0;
            while (lo + 1 < nblk && blk_start[lo + 1] <= e) ++lo;
            return plane * s.Tk + (size_t)blk_id[lo] * s.bs + (e - blk_start[lo]);
        };
        const __nv_bfloat16* K = br == 0 ? a.kcmp : a.k;
        const __nv_bfloat16* V = br == 0 ? a.vcmp : a.v;
        // scores, max, probabilities
        float mloc = -INFINITY;
        for (int e = tid; e < nkeys; e += BW_NT) {
            const __nv_bfloat16* kr = K + key_row(e) * dqk;
            float acc = 0.f;
            for (int c = 0; c < dqk; c += 8) {
                float f[8];
                unpack8(*reinterpret_cast<const uint4*>(kr + c), f);
#pragma unroll
                for (int x = 0; x < 8; ++x) acc = fmaf(qs[c + x], f[x], acc);
            }
            pe[e] = s.scale * acc;
            mloc = fmaxf(mloc, pe[e]);
        }
        const float m = block_max(mloc, red);
        float lloc = 0.f;
        for (int e = tid; e < nkeys; e += BW_NT) {
            const float p = expf(pe[e] - m);
            pe[e] = p;
            lloc += p;
        }
        const float l = block_sum(lloc, red);
        const float inv = l > 0.f ? 1.f / l : 0.f;
        for (int e = tid; e < nkeys; e += BW_NT) pe[e] *= inv;
        __syncthreads();
        // branch output, gate gradient, D
        for (int c = tid; c < dv; c += BW_NT) {
            float acc = 0.f;
            for (int e = 0; e < nkeys; ++e) acc = fmaf(pe[e], bf2f(V[key_row(e) * dv + c]), acc);
            os[c] = acc;
            dob[c] = g * dos[c];
        }
        __syncthreads();
        float part = 0.f;
        for (int c = tid; c < dv; c += BW_NT) part += dos[c] * os[c];
        const float dgate = block_sum(part, red);
        if (tid == 0 && a.dgates) a.dgates[row * 3 + br] = dgate;
        const float D = g * dgate;
        // ds_e = P_e (d_o . v_e - D); dv_e += P_e d_o
        for (int e = tid; e < nkeys; e += BW_NT) {
            const size_t kr = key_row(e);
            const __nv_bfloat16* vr = V + kr * dv;
            float dp = 0.f;
            for (int c = 0; c < dv; c += 8) {
                float f[8];
                unpack8(*reinterpret_cast<const uint4*>(vr + c), f);
#pragma unroll
                for (int x = 0; x < 8; ++x) dp = fmaf(dob[c + x], f[x], dp);
            }
            const float p = pe[e];
            float* dvr = (br == 0 ? a.dvc : a.dv) + kr * dv;
            for (int c = 0; c < dv; ++c) atomicAdd(dvr + c, p * dob[c]);
            pe[e] = p * (dp - D);
        }
        __syncthreads();
        // dq += scale sum_e ds_e k_e;  dk_e += scale ds_e q
        for (int cc = 0; cc < 2; ++cc) {
            const int c = tid + cc * BW_NT;
            if (c >= dqk) break;
            float acc = 0.f;
            for (int e = 0; e < nkeys; ++e) acc = fmaf(pe[e], bf2f(K[key_row(e) * dqk + c]), acc);
            dq_acc[cc] += s.scale * acc;
        }
        for (int e = tid; e < nkeys; e += BW_NT) {
            float* dkr = (br == 0 ? a.dkc : a.dk) + key_row(e) * dqk;
            const float w = s.scale * pe[e];
            for (int c = 0; c < dqk; ++c) atomicAdd(dkr + c, w * qs[c]);
        }
        __syncthreads();
    }
    for (int cc = 0; cc < 2; ++cc) {
        const int c = tid + cc * BW_NT;
        if (c < dqk) a.dq[row * dqk + c] = dq_acc[cc];
    }
}

// dk[u] += sum over the compressed tokens j whose window holds u of dkc[j] /
// cmp_block (and the same for v): each output element gathers its tokens.
__global__ void bwd_spread_kernel(const float* __restrict__ dkc, const float* __restrict__ dvc,
                                  float* __restrict__ dk, float* __restrict__ dv, Shape s) {
    const size_t nk = (size_t)s.B * s.Hkv * s.Tk * s.dqk;
    const size_t nv = (size_t)s.B * s.Hkv * s.Tk * s.dv;
    const float inv = 1.f / (float)s.lc;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < nk + nv;
         e += (size_t)gridDim.x * blockDim.x) {
        const bool val = e >= nk;
        const size_t x = val ? e - nk : e;
        const int d = val ? s.dv : s.dqk;
        const int c = (int)(x % d);
        const size_t pu = x / d;                  // plane * Tk + u
        const int u = (int)(pu % s.Tk);
        const size_t plane = pu / s.Tk;
        int j0 = u - s.lc + 1;
        j0 = j0 <= 0 ? 0 : (j0 + s.sc - 1) / s.sc;
        const int j1 = min(s.n_cmp - 1, u / s.sc);
        float acc = 0.f;
        for (int j = j0; j <= j1; ++j) acc += (val ? dvc : dkc)[(plane * s.n_cmp + j) * d + c];
        (val ? dv : dk)[x] += acc * inv;
    }
}

}  // namespace

size_t bwd_smem_bytes(const Shape& s) {
    return (size_t)(s.dqk + 3 * s.dv + 4) * 4 + (2 * BW_MAXB + 1) * 4 + (size_t)BW_MAXK * 4;
}

bool bwd_supported(const Shape& s) {
    if (s.dqk % 8 || s.dv % 8 || s.dqk > 2 * BW_NT) return false;
    if ((s.flags & NSA_BR_SEL) && (s.topk > BW_MAXB || (size_t)s.topk * s.bs > BW_MAXK)) return false;
    if ((s.flags & NSA_BR_WIN) && s.win > BW_MAXK) return false;
    if ((s.flags & NSA_BR_CMP) && s.n_cmp > BW_MAXK) return false;
    return true;
}

cudaError_t launch_attn_bwd(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* kcmp, const __nv_bfloat16* vcmp,
                            const float* gates, const int32_t* idx, const __nv_bfloat16* d_out, float* dq,
                            float* dk, float* dv, float* dgates, float* dkc, float* dvc, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(dk, 0, (size_t)s.B * s.Hkv * s.Tk * s.dqk * 4, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dv, 0, (size_t)s.B * s.Hkv * s.Tk * s.dv * 4, st);
    const bool cmp = (s.flags & NSA_BR_CMP) && s.n_cmp > 0;
    if (e == cudaSuccess && cmp) e = cudaMemsetAsync(dkc, 0, (size_t)s.B * s.Hkv * s.n_cmp * s.dqk * 4, st);
    if (e == cudaSuccess && cmp) e = cudaMemsetAsync(dvc, 0, (size_t)s.B * s.Hkv * s.n_cmp * s.dv * 4, st);
    if (e != cudaSuccess) return e;
    BwdArgs a{s, q, k, v, kcmp, vcmp, d_out, gates, idx, dq, dk, dv, dgates, dkc, dvc};
    const size_t smem = bwd_smem_bytes(s);
    e = cudaFuncSetAttribute(bwd_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_rows_kernel<<<dim3(s.Tq, s.Hq, s.B), BW_NT, smem, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || !cmp) return e;
    const size_t n = (size_t)s.B * s.Hkv * s.Tk * (s.dqk + s.dv);
    const int grid = (int)std::min<size_t>((n + 255) / 256, 148 * 16);
    bwd_spread_kernel<<<grid, 256, 0, st>>>(dkc, dvc, dk, dv, s);
    return cudaGetLastError();
}

}  // namespace nsa
