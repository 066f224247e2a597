// Block representations: mean-pooled selection keys (fp32) and compressed
// keys/values (bf16).
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention", Figure 2: every block of keys/values is compressed into one
// representation; §7 "Kimi Simplifies The Sparse Route": MoBA's block
// representation is the parameter-free mean of the block's keys.
//
// Both kernels stream K/V once with 16-byte loads (8 bf16 per thread and
// row) and accumulate in fp32; the work is HBM-bound (it reads Tkv*(d_qk+d_v)
// bf16 per KV head and writes a few percent of that).
#include <algorithm>

#include "common.cuh"

namespace nsa {

// kbar[b,h,j,:] = mean of k[b,h,j*bs:(j+1)*bs,:] for blocks j = j0 + blockIdx.x.
// One CTA per (j, h, b); the block's rows are split over the threads that
// share a 16-byte column, then the row partial sums are reduced through shared
// memory in a fixed order, so a block's mean does not depend on which launch
// (whole cache or incremental update) computes it.
__global__ void __launch_bounds__(256) pool_block_keys_kernel(const __nv_bfloat16* __restrict__ k,
                                                              float* __restrict__ kbar, int Tk,
                                                              int d, int bs, int nb_full, int Hkv,
                                                              int j0) {
    extern __shared__ float red[];
    const int j = j0 + blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int nvec = d / 8;
    const int nsplit = blockDim.x / nvec;
    const int tid = threadIdx.x;
    const int vec = tid % nvec, split = tid / nvec;
    if (split < nsplit) {
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        const __nv_bfloat16* base = k + ((size_t)(b * Hkv + h) * Tk + (size_t)j * bs) * d + vec * 8;
        for (int r = split; r < bs; r += nsplit) {
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(base + (size_t)r * d), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += f[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) red[split * d + vec * 8 + e] = acc[e];
    }
    __syncthreads();
    const float inv = 1.0f / (float)bs;
    float* dst = kbar + ((size_t)(b * Hkv + h) * nb_full + j) * d;
    for (int c = tid; c < d; c += blockDim.x) {
        float s = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) s += red[sp * d + c];
        dst[c] = s * inv;
    }
}

// Compressed tokens x_cmp[j] = mean of x over [j*sc, j*sc + lc), lc a multiple
// of sc, for j in [j_first, j_end).  A CTA produces JT consecutive compressed
// tokens: it first sums the (JT + lc/sc - 1) stride-long segments they cover
// into shared memory, then adds lc/sc neighbouring segments per output, so
// every input row is read once per CTA.  Each segment is summed row by row and
// each output adds its segments in order, so a token's value does not depend
// on where its CTA's range starts.  blockIdx.z = 2*b + (0: keys, 1: values).
constexpr int CMP_JT = 16;

__global__ void __launch_bounds__(256) compress_kernel(const __nv_bfloat16* __restrict__ k,
                                                       const __nv_bfloat16* __restrict__ v,
                                                       __nv_bfloat16* __restrict__ kcmp,
                                                       __nv_bfloat16* __restrict__ vcmp, int Tk,
                                                       int dqk, int dv, int lc, int sc, int n_cmp,
                                                       int Hkv, int j_first, int j_end) {
    extern __shared__ float seg[];
    const int which = blockIdx.z & 1, b = blockIdx.z >> 1, h = blockIdx.y;
    const int d = which ? dv : dqk;
    const __nv_bfloat16* x = which ? v : k;
    __nv_bfloat16* out = which ? vcmp : kcmp;
    const int j0 = j_first + blockIdx.x * CMP_JT;
    const int jn = min(CMP_JT, j_end - j0);
    const int m = lc / sc;
    const int nseg = jn + m - 1;
    const int nvec = d / 8;
    const __nv_bfloat16* base = x + ((size_t)(b * Hkv + h) * Tk + (size_t)j0 * sc) * d;
    for (int p = threadIdx.x; p < nseg * nvec; p += blockDim.x) {
        const int sg = p / nvec, vec = p % nvec;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        const __nv_bfloat16* row = base + (size_t)sg * sc * d + vec * 8;
        for (int r = 0; r < sc; ++r) {
            float f[8];
            unpack8(*reinterpret_cast<const uint4*>(row + (size_t)r * d), f);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += f[e];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) seg[sg * d + vec * 8 + e] = acc[e];
    }
    __syncthreads();
    const float inv = 1.0f / (float)lc;
    for (int p = threadIdx.x; p < jn * nvec; p += blockDim.x) {
        const int jj = p / nvec, vec = p % nvec;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int t = 0; t < m; ++t)
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] += seg[(jj + t) * d + vec * 8 + e];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] *= inv;
        *reinterpret_cast<uint4*>(out + ((size_t)(b * Hkv + h) * n_cmp + j0 + jj) * d + vec * 8) =
            pack8(acc);
    }
}

// Pooled tokens of the selection blocks [jb0, jb1) and the compressed tokens
// [jc0, jc1) (either range may be empty).
cudaError_t launch_pool_range(const Shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v,
                              float* kbar, __nv_bfloat16* kcmp, __nv_bfloat16* vcmp, int jb0, int jb1,
                              int jc0, int jc1, cudaStream_t st) {
    if (kbar && jb1 > jb0) {
        const int nvec = s.dqk / 8;
        const int nsplit = 256 / nvec;
        const size_t smem = (size_t)nsplit * s.dqk * sizeof(float);
        cudaFuncSetAttribute(pool_block_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        dim3 grid(jb1 - jb0, s.Hkv, s.B);
        pool_block_keys_kernel<<<grid, 256, smem, st>>>(k, kbar, s.Tk, s.dqk, s.bs, s.nb_full,
                                                        s.Hkv, jb0);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    if (kcmp && vcmp && jc1 > jc0) {
        const int m = s.lc / s.sc;
        const int dmax = s.dqk > s.dv ? s.dqk : s.dv;
        const size_t smem = (size_t)(CMP_JT + m - 1) * dmax * sizeof(float);
        cudaFuncSetAttribute(compress_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
        dim3 grid((jc1 - jc0 + CMP_JT - 1) / CMP_JT, s.Hkv, 2 * s.B);
        compress_kernel<<<grid, 256, smem, st>>>(k, v, kcmp, vcmp, s.Tk, s.dqk, s.dv, s.lc, s.sc,
                                                 s.n_cmp, s.Hkv, jc0, jc1);
        return cudaGetLastError();
    }
    return cudaSuccess;
}

cudaError_t launch_pool_kv(const Shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v,
                           float* kbar, __nv_bfloat16* kcmp, __nv_bfloat16* vcmp,
                           cudaStream_t st) {
    return launch_pool_range(s, k, v, kbar, kcmp, vcmp, 0, kbar ? s.nb_full : 0, 0,
                             (kcmp && vcmp) ? s.n_cmp : 0, st);
}

// New tokens x_new [B, Hkv, n_new, d] written into x [B, Hkv, Tk, d] at rows
// [t0, t0 + n_new), 16 bytes per thread; blockIdx.y: 0 keys, 1 values.
__global__ void append_rows_kernel(const __nv_bfloat16* __restrict__ k_new, const __nv_bfloat16* __restrict__ v_new,
                                   __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v, int BH, int Tk,
                                   int t0, int n_new, int dqk, int dv) {
    const bool val = blockIdx.y == 1;
    const int d = val ? dv : dqk;
    const __nv_bfloat16* src = val ? v_new : k_new;
    __nv_bfloat16* dst = val ? v : k;
    const int nvec = d / 8;
    const size_t total = (size_t)BH * n_new * nvec;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (size_t)gridDim.x * blockDim.x) {
        const int vec = (int)(e % nvec);
        const size_t row = e / nvec;                 // (plane, new row)
        const size_t plane = row / n_new;
        const int r = (int)(row % n_new);
        *reinterpret_cast<uint4*>(dst + (plane * Tk + t0 + r) * d + vec * 8) =
            *reinterpret_cast<const uint4*>(src + row * d + vec * 8);
    }
}

cudaError_t launch_append_rows(const Shape& s, const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                               __nv_bfloat16* k, __nv_bfloat16* v, int t0, int n_new, cudaStream_t st) {
    const size_t rows = (size_t)s.B * s.Hkv * n_new;
    const int grid = (int)std::min<size_t>((rows * (s.dqk / 8) + 255) / 256, 148 * 8);
    append_rows_kernel<<<dim3(grid, v ? 2 : 1), 256, 0, st>>>(k_new, v_new, k, v, s.B * s.Hkv, s.Tk, t0, n_new,
                                                              s.dqk, s.dv);
    return cudaGetLastError();
}

}  // namespace nsa
