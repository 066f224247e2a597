// Block scoring and top-k block selection for prefill on the tensor cores.
//
// Zhang Xiaojun #94 transcript (bidclub.ai), §4 "Inside Native Sparse
// Attention": every query scores every past KV block against the block's
// pooled key; under GQA the heads of a group add their scores, so the group
// shares one top-k.  LateTalk #103 (zjai.club) §13: the query's own block is
// always kept.
//
// The group score is linear in the queries: s = scale * (sum_h q_h) . kbar,
// one fp32 dot product per (query, unit, block).  Over a prefill these form a
// (queries x blocks) GEMM with K = d_qk.  The selection must separate scores
// 1e-5 apart, more than one tf32 or bf16 product resolves, so each operand is
// split into a tf32 high part and a tf32 low part (x = hi + lo, |lo| <=
// 2^-11 |x|) and a product is accumulated as hi.hi + hi.lo + lo.hi (the
// dropped lo.lo is below 2^-22 of it): three kind::tf32 MMAs per K step, fp32
// accumulation in TMEM.
//
//   qsplit_kernel   summed query rows (heads added in order), split
//   ksplit_kernel   pooled keys, split
//   score_tc_kernel a CTA takes 128 query rows of one (sequence, unit) and
//                   the blocks in N tiles of 256 (a 128 x 256 fp32 score tile
//                   in TMEM, double-buffered); the operands come by TMA in
//                   32-column chunks (128-byte swizzle).  An epilogue thread
//                   owns one query row and keeps its running top-(k-1) in
//                   registers; blocks arrive in ascending order, so a strict
//                   score comparison keeps the lower index among equal scores.
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "tc.cuh"

namespace nsa {

__device__ int g_sctc_status = 0;

namespace {

constexpr int SQ = 128;             // query rows per CTA
constexpr int SN = 256;             // candidate blocks per N tile
constexpr int SKC = 32;             // fp32 columns per chunk (128 bytes)
constexpr int SNT = 192;            // producer warp, MMA warp, 4 epilogue warps
constexpr int A_CH = SQ * 128;      // 16 KB
constexpr int B_CH = SN * 128;      // 32 KB
constexpr int STAGE = 2 * A_CH + 2 * B_CH;   // hi/lo of both operands: 96 KB
constexpr uint64_t WAIT_NS = 1000000000ull;

__device__ __forceinline__ float to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

// qh/ql [B, Hsel, Tq, d]: split of the unit's summed query row
__global__ void __launch_bounds__(256) qsplit_kernel(Shape s, const __nv_bfloat16* __restrict__ q,
                                                     float* __restrict__ qh, float* __restrict__ ql) {
    const int d = s.dqk, nvec = d / 8;
    const size_t total = (size_t)s.B * s.Hsel * s.Tq * nvec;
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (size_t)gridDim.x * blockDim.x) {
        const int v = (int)(e % nvec);
        const size_t row = e / nvec;                 // (b * Hsel + u) * Tq + t
        const int t = (int)(row % s.Tq);
        const int bu = (int)(row / s.Tq);
        const int u = bu % s.Hsel, b = bu / s.Hsel;
        const int h0 = s.per_head ? u : u * s.G;
        const __nv_bfloat16* src = q + (((size_t)b * s.Tq + t) * s.Hq + h0) * d + v * 8;
        float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        for (int h8 = 0; h8 < s.heads_per_unit; h8 += 8) {
            uint4 raw[8];
#pragma unroll
            for (int hh = 0; hh < 8; ++hh)
                if (h8 + hh < s.heads_per_unit) raw[hh] = *reinterpret_cast<const uint4*>(src + (size_t)(h8 + hh) * d);
#pragma unroll
            for (int hh = 0; hh < 8; ++hh) {
                if (h8 + hh >= s.heads_per_unit) break;
                float f[8];
                unpack8(raw[hh], f);
#pragma unroll
                for (int k = 0; k < 8; ++k) acc[k] += f[k];
            }
        }
        float hi[8], lo[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            hi[k] = to_tf32(acc[k]);
            lo[k] = to_tf32(acc[k] - hi[k]);
        }
        float4* dh = reinterpret_cast<float4*>(qh + row * d + v * 8);
        float4* dl = reinterpret_cast<float4*>(ql + row * d + v * 8);
        dh[0] = make_float4(hi[0], hi[1], hi[2], hi[3]);
        dh[1] = make_float4(hi[4], hi[5], hi[6], hi[7]);
        dl[0] = make_float4(lo[0], lo[1], lo[2], lo[3]);
        dl[1] = make_float4(lo[4], lo[5], lo[6], lo[7]);
    }
}

// kh/kl [B, Hkv, nb_full, d]: split of the pooled keys
__global__ void __launch_bounds__(256) ksplit_kernel(size_t n4, const float4* __restrict__ kbar,
                                                     float4* __restrict__ kh, float4* __restrict__ kl) {
    for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n4;
         e += (size_t)gridDim.x * blockDim.x) {
        const float4 x = kbar[e];
        float4 h, l;
        h.x = to_tf32(x.x); l.x = to_tf32(x.x - h.x);
        h.y = to_tf32(x.y); l.y = to_tf32(x.y - h.y);
        h.z = to_tf32(x.z); l.z = to_tf32(x.z - h.z);
        h.w = to_tf32(x.w); l.w = to_tf32(x.w - h.w);
        kh[e] = h;
        kl[e] = l;
    }
}

struct ScArgs {
    Shape s;
    int32_t* idx;
    int n_tt;           // query tiles per (sequence, unit)
};

struct ScBars {
    uint64_t* b;
    __device__ __forceinline__ uint64_t* full(int i) const { return b + i; }
    __device__ __forceinline__ uint64_t* empty(int i) const { return b + 2 + i; }
    __device__ __forceinline__ uint64_t* s_full(int i) const { return b + 4 + i; }
    __device__ __forceinline__ uint64_t* s_free(int i) const { return b + 6 + i; }
};

__device__ __forceinline__ bool sc_warp_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag) {
    return __all_sync(0xffffffffu, tc::mbar_wait(b, parity, abort_flag, WAIT_NS));
}

__device__ __forceinline__ void sc_abort(volatile int* abort_flag) {
    *abort_flag = 1;
    atomicExch(&g_sctc_status, (int)NSA_ERR_TIMEOUT);
}

template <int D, int K1>
__global__ void __launch_bounds__(SNT, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap map_qh, const __grid_constant__ CUtensorMap map_ql,
                    const __grid_constant__ CUtensorMap map_kh, const __grid_constant__ CUtensorMap map_kl,
                    const ScArgs a) {
    constexpr int NCH = D / SKC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    ScBars bar{reinterpret_cast<uint64_t*>(sm + 2 * STAGE)};
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + 2 * STAGE + 64);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + 2 * STAGE + 72);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const Shape& s = a.s;
    const int tt = a.n_tt - 1 - (int)blockIdx.x;     // latest (heaviest) query tiles first
    const int u = blockIdx.y, b = blockIdx.z;
    const int kvh = s.per_head ? u / s.G : u;
    const int t0 = tt * SQ;
    const int nrows = min(SQ, s.Tq - t0);
    // candidates of the tile's last row bound the N tiles
    const int c_last = (s.q0 + t0 + nrows - 1) / s.bs;
    const int cmax = min(c_last, s.nb_full);
    const int n_nt = (cmax + SN - 1) / SN;

    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            tc::mbar_init(bar.full(i), 1);
            tc::mbar_init(bar.empty(i), 1);
            tc::mbar_init(bar.s_full(i), 1);
            tc::mbar_init(bar.s_free(i), 4);
        }
        *abort_flag = 0;
        tc::fence_mbar_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, 512);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        bool ok = true;
        uint32_t cnt = 0;
        const int qplane = b * s.Hsel + u, kplane = b * s.Hkv + kvh;
        for (int nt = 0; ok && nt < n_nt; ++nt)
            for (int c = 0; c < NCH; ++c, ++cnt) {
                const int st = cnt & 1;
                if (!sc_warp_wait(bar.empty(st), ((cnt >> 1) & 1) ^ 1, abort_flag)) {
                    ok = false;
                    break;
                }
                uint8_t* base = sm + st * STAGE;
                if (lane == 0) {
                    tc::mbar_arrive_expect_tx(bar.full(st), STAGE);
                    tc::tma_load_3d(base, &map_qh, bar.full(st), SKC * c, t0, qplane);
                    tc::tma_load_3d(base + A_CH, &map_ql, bar.full(st), SKC * c, t0, qplane);
                    tc::tma_load_3d(base + 2 * A_CH, &map_kh, bar.full(st), SKC * c, nt * SN, kplane);
                    tc::tma_load_3d(base + 2 * A_CH + B_CH, &map_kl, bar.full(st), SKC * c, nt * SN, kplane);
                }
                __syncwarp();
            }
        if (!ok) sc_abort(abort_flag);
        for (uint32_t st = 0; st < 2; ++st)
            if (cnt > st) {
                const uint32_t last = st + ((cnt - 1 - st) / 2) * 2;
                tc::mbar_wait_bounded(bar.full(st), (last >> 1) & 1, WAIT_NS);
            }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA
        if (lane == 0) {
            const uint32_t idesc = tc::idesc_tf32_f32(SQ, SN);
            const uint32_t base0 = tc::smem_u32(sm);
            bool ok = true;
            uint32_t cnt = 0;
            for (int nt = 0; ok && nt < n_nt; ++nt) {
                const int sb = nt & 1;
                // the epilogue has read S buffer sb (N tile nt - 2)
                if (nt >= 2 && !tc::mbar_wait(bar.s_free(sb), ((nt >> 1) & 1) ^ 1, abort_flag, WAIT_NS)) {
                    ok = false;
                    break;
                }
                const uint32_t dS = tmem + sb * SN;
                for (int c = 0; c < NCH; ++c, ++cnt) {
                    const int st = cnt & 1;
                    if (!tc::mbar_wait(bar.full(st), (cnt >> 1) & 1, abort_flag, WAIT_NS)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    const uint32_t ah = base0 + st * STAGE, al = ah + A_CH, bh = ah + 2 * A_CH, bl = bh + B_CH;
#pragma unroll
                    for (int kk = 0; kk < SKC / 8; ++kk) {
                        const uint32_t o = kk * 32;
                        tc::mma_ss_tf32(dS, tc::sdesc_sw128(ah + o, 16, 1024), tc::sdesc_sw128(bh + o, 16, 1024),
                                        idesc, (c > 0 || kk > 0) ? 1u : 0u);
                        tc::mma_ss_tf32(dS, tc::sdesc_sw128(ah + o, 16, 1024), tc::sdesc_sw128(bl + o, 16, 1024),
                                        idesc, 1u);
                        tc::mma_ss_tf32(dS, tc::sdesc_sw128(al + o, 16, 1024), tc::sdesc_sw128(bh + o, 16, 1024),
                                        idesc, 1u);
                    }
                    tc::mma_commit(bar.empty(st));
                }
                if (!ok) break;
                tc::mma_commit(bar.s_full(sb));
            }
            if (!ok) sc_abort(abort_flag);
            // every MMA completes before TMEM is released
            if (n_nt > 0) tc::mbar_wait_bounded(bar.s_full((n_nt - 1) & 1), ((n_nt - 1) >> 1) & 1, WAIT_NS);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue: one query row per thread
        const int quarter = warp & 3;
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int t = s.q0 + t0 + r;
        const int cr = t / s.bs;
        const int ncand = min(cr, s.nb_full);
        float ls[K1];
        int lb[K1];
#pragma unroll
        for (int i = 0; i < K1; ++i) {
            ls[i] = -INFINITY;
            lb[i] = 0;
        }
        float thr = -INFINITY;
        float* cand = reinterpret_cast<float*>(sm + 2 * STAGE + 1024);   // [SQ][33]
        bool ok = true;
        for (int nt = 0; nt < n_nt; ++nt) {
            const int sb = nt & 1;
            if (!sc_warp_wait(bar.s_full(sb), (nt >> 1) & 1, abort_flag)) {
                ok = false;
                break;
            }
            tc::fence_after_sync();
#pragma unroll 1
            for (int cc = 0; cc < SN / 32; ++cc) {
                uint32_t v[32];
                tc::tmem_ld32(tmem + sb * SN + lane_off + cc * 32, v);
                tc::tmem_wait_ld();
                const int blk0 = nt * SN + cc * 32;
                // candidates above the threshold go to this thread's shared-memory slots
                // and a bit mask; the list update then runs once per such candidate
                // (one copy of the insertion code keeps the loop small)
                uint32_t pass = 0;
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    // forced leading (sink) blocks score +inf: always kept
                    const float sc = blk0 + j < s.n_sink ? INFINITY : s.scale * __uint_as_float(v[j]);
                    if (blk0 + j < ncand && sc > thr) {
                        pass |= 1u << j;
                        cand[r * 33 + j] = sc;
                    }
                }
                while (pass) {
                    const int j = __ffs(pass) - 1;
                    pass &= pass - 1;
                    const float xs = cand[r * 33 + j];
                    if (!(xs > thr)) continue;
                    const int xb = blk0 + j;
#pragma unroll
                    for (int i = K1 - 1; i > 0; --i) {
                        const bool gp = xs > ls[i - 1], gc = xs > ls[i];
                        ls[i] = gp ? ls[i - 1] : (gc ? xs : ls[i]);
                        lb[i] = gp ? lb[i - 1] : (gc ? xb : lb[i]);
                    }
                    if (xs > ls[0]) {
                        ls[0] = xs;
                        lb[0] = xb;
                    }
                    thr = ls[K1 - 1];
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(bar.s_free(sb));
        }
        if (!ok) sc_abort(abort_flag);
        if (r < nrows) {
            // kept past blocks ascending, then the query's own block, then -1
            int npast = 0;
#pragma unroll
            for (int i = 0; i < K1; ++i) {
                if (ls[i] == -INFINITY) lb[i] = 0x7fffffff;
                else ++npast;
            }
#pragma unroll
            for (int i = 0; i < K1; ++i)
#pragma unroll
                for (int k = 0; k < K1 - 1 - i; ++k) {
                    const int lo = min(lb[k], lb[k + 1]), hi = max(lb[k], lb[k + 1]);
                    lb[k] = lo;
                    lb[k + 1] = hi;
                }
            int32_t* dst = a.idx + (((size_t)b * s.Hsel + u) * s.Tq + t0 + r) * s.topk;
#pragma unroll
            for (int i = 0; i < K1; ++i)
                if (i < npast) dst[i] = lb[i];
            dst[npast] = cr;
            for (int i = npast + 1; i < s.topk; ++i) dst[i] = -1;
        }
    }

    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc(tmem, 512);
}

PFN_cuTensorMapEncodeTiled_v12000 sc_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) == cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

bool sc_encode(CUtensorMap* m, const float* base, int d, size_t rows, size_t planes, uint32_t box_rows) {
    auto enc = sc_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)d * 4 * rows};
    const cuuint32_t box[3] = {SKC, box_rows, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float*>(base), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int K1>
cudaError_t launch_sc_impl(const Shape& s, const float* qh, const float* ql, const float* kh, const float* kl,
                           int32_t* idx, cudaStream_t st) {
    CUtensorMap mqh, mql, mkh, mkl;
    if (!sc_encode(&mqh, qh, D, s.Tq, (size_t)s.B * s.Hsel, SQ) ||
        !sc_encode(&mql, ql, D, s.Tq, (size_t)s.B * s.Hsel, SQ) ||
        !sc_encode(&mkh, kh, D, s.nb_full, (size_t)s.B * s.Hkv, SN) ||
        !sc_encode(&mkl, kl, D, s.nb_full, (size_t)s.B * s.Hkv, SN))
        return cudaErrorInvalidValue;
    ScArgs a;
    a.s = s;
    a.idx = idx;
    a.n_tt = (s.Tq + SQ - 1) / SQ;
    const int smem = 2 * STAGE + 1024 + SQ * 33 * 4 + 1024;
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D, K1>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    score_tc_kernel<D, K1><<<dim3(a.n_tt, s.Hsel, s.B), SNT, smem, st>>>(mqh, mql, mkh, mkl, a);
    return cudaGetLastError();
}

}  // namespace

bool score_tc_supported(const Shape& s) {
    if (!(s.flags & NSA_BR_SEL) || s.nb_full < 1) return false;
    if (s.dqk != 64 && s.dqk != 128 && s.dqk != 192) return false;
    return s.topk == 4 || s.topk == 8 || s.topk == 16;
}

size_t score_tc_q_floats(const Shape& s) { return (size_t)s.B * s.Hsel * s.Tq * s.dqk; }
size_t score_tc_k_floats(const Shape& s) { return (size_t)s.B * s.Hkv * s.nb_full * s.dqk; }

cudaError_t launch_score_tc(const Shape& s, const __nv_bfloat16* q, const float* kbar, float* qh, float* ql,
                            float* kh, float* kl, int32_t* idx, cudaStream_t st) {
    {
        const size_t total = (size_t)s.B * s.Hsel * s.Tq * (s.dqk / 8);
        const int grid = (int)std::min<size_t>((total + 255) / 256, 148 * 16);
        qsplit_kernel<<<grid, 256, 0, st>>>(s, q, qh, ql);
        const size_t n4 = score_tc_k_floats(s) / 4;
        const int grid_k = (int)std::min<size_t>((n4 + 255) / 256, 148 * 8);
        ksplit_kernel<<<grid_k, 256, 0, st>>>(n4, reinterpret_cast<const float4*>(kbar),
                                              reinterpret_cast<float4*>(kh), reinterpret_cast<float4*>(kl));
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
#define NSA_SC_CASE(DD, KK) \
    if (s.dqk == DD && s.topk - 1 == KK) return launch_sc_impl<DD, KK>(s, qh, ql, kh, kl, idx, st);
    NSA_SC_CASE(64, 3) NSA_SC_CASE(64, 7) NSA_SC_CASE(64, 15)
    NSA_SC_CASE(128, 3) NSA_SC_CASE(128, 7) NSA_SC_CASE(128, 15)
    NSA_SC_CASE(192, 3) NSA_SC_CASE(192, 7) NSA_SC_CASE(192, 15)
#undef NSA_SC_CASE
    return cudaErrorInvalidValue;
}

int read_and_clear_sctc_status() {
    int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, g_sctc_status, sizeof(int)) != cudaSuccess) return -1;
    cudaMemcpyToSymbol(g_sctc_status, &zero, sizeof(int));
    return v;
}

}  // namespace nsa
