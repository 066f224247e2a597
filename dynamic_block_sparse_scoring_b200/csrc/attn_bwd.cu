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
// One CTA (256 threads) per (query row, selection unit, sequence) covering
// the unit's heads (the group's G heads, or one head with per-head selection),
// which share every key of every branch.  A branch's keys are taken 64 at a
// time into shared memory (rows padded to an odd number of 32-bit words, so
// that threads reading the same column of different keys hit different
// banks) and passed over three times: the softmax statistics of every head,
// then the branch output (for the gate gradient and D), then ds with the
// gradients.  dk and dv of a key receive one fp32 atomic add per column and
// row, summed over the CTA's heads first and issued by consecutive threads on
// consecutive columns; dq stays in registers over all branches.  A plain
// FFMA formulation of the gradient.
#include <math.h>

#include <algorithm>

#include "common.cuh"

namespace nsa {

namespace {

constexpr int BG_NT = 256;
constexpr int BG_KC = 64;               // keys per chunk
constexpr int BG_MAXH = 16;             // heads per CTA
constexpr int BG_MAXD = 256;            // d_qk, d_v
constexpr int BG_RO4 = BG_MAXH * BG_MAXD / 4 / BG_NT;   // per-thread column quads of o / dq
constexpr int BW_MAXB = 32;             // kept blocks per row

struct BwdArgs {
    Shape s;
    const __nv_bfloat16 *q, *k, *v, *kcmp, *vcmp, *d_out;
    const float* gates;
    const int32_t* idx;
    float *dq, *dk, *dv, *dgates, *dkc, *dvc;
};

// shared-memory layout (in 4-byte words) for a shape
struct BgLayout {
    int hb, dqk, dv, ks, vs;   // heads, dims, padded key / value row strides (bf16)
    int q, dos, dob, ps, ds, stat, red, krow, blk, kc, vc, total;
    __host__ __device__ BgLayout(const Shape& s) {
        hb = s.per_head ? 1 : s.G;
        dqk = s.dqk;
        dv = s.dv;
        ks = dqk + 2;                 // (dqk / 2 + 1) words: odd
        vs = dv + 2;
        q = 0;                        // [hb][dqk] fp32
        dos = q + hb * dqk;           // [hb][dv] d_out
        dob = dos + hb * dv;          // [hb][dv] gate * d_out
        ps = dob + hb * dv;           // [hb][KC] P
        ds = ps + hb * BG_KC;         // [hb][KC] ds
        stat = ds + hb * BG_KC;       // m, l, D, g, dgate: [5][BG_MAXH]
        red = stat + 5 * BG_MAXH;     // [2 warps][4][BG_MAXH / 4] reduction scratch, x2
        krow = red + 4 * BG_MAXH;     // [KC] key rows (int64: 2 words each)
        blk = krow + 2 * BG_KC;       // [BW_MAXB + 1] starts, [BW_MAXB] ids, [1] count
        kc = blk + 2 * BW_MAXB + 2;   // [KC][ks] bf16
        vc = kc + BG_KC * ks / 2;     // [KC][vs] bf16
        total = vc + BG_KC * vs / 2;
    }
};

// acc += w * sum_e p[e] * rows[e][0..3] for e < n (rows of `stride` bf16, four
// columns at a time; p four keys at a time)
__device__ __forceinline__ float4 fma_rows(const float* p, const __nv_bfloat16* rows, int stride, int n,
                                           float4 acc, float w = 1.f) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    int e = 0;
    for (; e + 4 <= n; e += 4) {
        const float4 p4 = *reinterpret_cast<const float4*>(p + e);
        const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const __nv_bfloat162* r = reinterpret_cast<const __nv_bfloat162*>(rows + (e + u) * stride);
            const float2 a0 = __bfloat1622float2(r[0]), a1 = __bfloat1622float2(r[1]);
            t.x = fmaf(pv[u], a0.x, t.x); t.y = fmaf(pv[u], a0.y, t.y);
            t.z = fmaf(pv[u], a1.x, t.z); t.w = fmaf(pv[u], a1.y, t.w);
        }
    }
    for (; e < n; ++e) {
        const __nv_bfloat162* r = reinterpret_cast<const __nv_bfloat162*>(rows + e * stride);
        const float2 a0 = __bfloat1622float2(r[0]), a1 = __bfloat1622float2(r[1]);
        t.x = fmaf(p[e], a0.x, t.x); t.y = fmaf(p[e], a0.y, t.y);
        t.z = fmaf(p[e], a1.x, t.z); t.w = fmaf(p[e], a1.y, t.w);
    }
    return make_float4(fmaf(w, t.x, acc.x), fmaf(w, t.y, acc.y), fmaf(w, t.z, acc.z), fmaf(w, t.w, acc.w));
}

__global__ void __launch_bounds__(BG_NT) bwd_group_kernel(BwdArgs a) {
    extern __shared__ float sm[];
    const Shape& s = a.s;
    const BgLayout L(s);
    const int hb = L.hb, dqk = s.dqk, dv = s.dv;
    float* qs = sm + L.q;
    float* dos = sm + L.dos;
    float* dob = sm + L.dob;
    float* ps = sm + L.ps;
    float* dss = sm + L.ds;
    float* st_m = sm + L.stat;
    float* st_l = st_m + BG_MAXH;
    float* st_D = st_l + BG_MAXH;
    float* st_g = st_D + BG_MAXH;
    float* st_dg = st_g + BG_MAXH;
    float* red = sm + L.red;                                   // [2][4][4]
    long long* krow = reinterpret_cast<long long*>(sm + L.krow);
    int* blk_start = reinterpret_cast<int*>(sm + L.blk);
    int* blk_id = blk_start + BW_MAXB + 1;
    int* blk_n = blk_id + BW_MAXB;
    __nv_bfloat16* kcs = reinterpret_cast<__nv_bfloat16*>(sm + L.kc);
    __nv_bfloat16* vcs = reinterpret_cast<__nv_bfloat16*>(sm + L.vc);

    const int i = blockIdx.x, unit = blockIdx.y, b = blockIdx.z;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t = s.q0 + i;
    const int h0 = s.per_head ? unit : unit * s.G;
    const int kvh = s.per_head ? unit / s.G : unit;
    const size_t row0 = ((size_t)b * s.Tq + i) * s.Hq + h0;        // row of head h0; heads follow
    const size_t plane = (size_t)b * s.Hkv + kvh;
    for (int x = tid; x < hb * dqk; x += BG_NT) qs[x] = bf2f(a.q[row0 * dqk + x]);
    for (int x = tid; x < hb * dv; x += BG_NT) dos[x] = bf2f(a.d_out[row0 * dv + x]);
    // score thread: key e_s of the chunk, heads 4 hq .. 4 hq + 3
    const int e_s = tid % BG_KC, hq = tid / BG_KC;
    const bool score_thread = 4 * hq < hb;
    float4 dq_acc[BG_RO4];
#pragma unroll
    for (int r = 0; r < BG_RO4; ++r) dq_acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncthreads();

    for (int br = 0; br < 3; ++br) {
        if (!(s.flags & (1u << br))) {
            // the output does not depend on a disabled branch's gate
            if (tid < hb && a.dgates) a.dgates[(row0 + tid) * 3 + br] = 0.f;
            continue;
        }
        int nkeys = 0, win_lo = 0;
        if (br == 0) {
            nkeys = t >= s.lc - 1 ? min(s.n_cmp, (t - s.lc + 1) / s.sc + 1) : 0;
        } else if (br == 2) {
            win_lo = max(0, t - s.win + 1);
            nkeys = t - win_lo + 1;
        } else {
            if (tid == 0) {
                const int32_t* r = a.idx + (((size_t)b * s.Hsel + unit) * s.Tq + i) * s.topk;
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
                *blk_n = n;
            }
            __syncthreads();
            nkeys = blk_start[*blk_n];
        }
        if (tid < hb) {
            st_g[tid] = a.gates ? a.gates[(row0 + tid) * 3 + br] : 1.f;
            st_m[tid] = -INFINITY;
            st_l[tid] = 0.f;
            st_dg[tid] = 0.f;
        }
        __syncthreads();
        for (int x = tid; x < hb * dv; x += BG_NT) dob[x] = st_g[x / dv] * dos[x];
        const __nv_bfloat16* K = br == 0 ? a.kcmp : a.k;
        const __nv_bfloat16* V = br == 0 ? a.vcmp : a.v;
        float* dK = br == 0 ? a.dkc : a.dk;
        float* dV = br == 0 ? a.dvc : a.dv;
        const int nchunk = (nkeys + BG_KC - 1) / BG_KC;
        float4 o_acc[BG_RO4];
#pragma unroll
        for (int r = 0; r < BG_RO4; ++r) o_acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);

        // one chunk: key rows, K (and V) rows into shared memory, then the four heads'
        // scores of this thread's key (scaled; -inf past the last key)
        auto load_chunk = [&](int c0, bool with_v, float* sc4) {
            const int nk = min(BG_KC, nkeys - c0);
            __syncthreads();                                   // the previous chunk is consumed
            if (tid < nk) {
                const int e = c0 + tid;
                long long r;
                if (br == 0) {
                    r = (long long)(plane * s.n_cmp + e);
                } else if (br == 2) {
                    r = (long long)(plane * s.Tk + win_lo + e);
                } else {
                    int lo = 0;
                    while (lo + 1 < *blk_n && blk_start[lo + 1] <= e) ++lo;
                    r = (long long)(plane * s.Tk + (size_t)blk_id[lo] * s.bs + (e - blk_start[lo]));
                }
                krow[tid] = r;
            }
            __syncthreads();
            const int kv8 = dqk / 8, vv8 = dv / 8;
            for (int x = tid; x < nk * kv8; x += BG_NT) {
                const int e = x / kv8, c = (x % kv8) * 8;
                const uint4 u = *reinterpret_cast<const uint4*>(K + krow[e] * dqk + c);
                uint32_t* d = reinterpret_cast<uint32_t*>(kcs + e * L.ks + c);
                d[0] = u.x; d[1] = u.y; d[2] = u.z; d[3] = u.w;
            }
            if (with_v)
                for (int x = tid; x < nk * vv8; x += BG_NT) {
                    const int e = x / vv8, c = (x % vv8) * 8;
                    const uint4 u = *reinterpret_cast<const uint4*>(V + krow[e] * dv + c);
                    uint32_t* d = reinterpret_cast<uint32_t*>(vcs + e * L.vs + c);
                    d[0] = u.x; d[1] = u.y; d[2] = u.z; d[3] = u.w;
                }
            __syncthreads();
#pragma unroll
            for (int j = 0; j < 4; ++j) sc4[j] = -INFINITY;
            if (score_thread && e_s < nk) {
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                const __nv_bfloat162* kr = reinterpret_cast<const __nv_bfloat162*>(kcs + e_s * L.ks);
                for (int c = 0; c < dqk; c += 4) {
                    const float2 k0 = __bfloat1622float2(kr[c / 2]), k1 = __bfloat1622float2(kr[c / 2 + 1]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int h = min(4 * hq + j, hb - 1);
                        const float4 qv = *reinterpret_cast<const float4*>(qs + h * dqk + c);
                        acc[j] = fmaf(qv.w, k1.y, fmaf(qv.z, k1.x, fmaf(qv.y, k0.y, fmaf(qv.x, k0.x, acc[j]))));
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (4 * hq + j < hb) sc4[j] = s.scale * acc[j];
            }
            return nk;
        };

        // pass 1: per-head max and sum of exponentials (online over chunks)
        for (int ch = 0; ch < nchunk; ++ch) {
            float sc4[4];
            load_chunk(ch * BG_KC, false, sc4);
            // the two warps of each head quad reduce their 32 keys, then combine
            float cm[4], cl[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                cm[j] = warp_max(sc4[j]);
                cl[j] = warp_sum(sc4[j] == -INFINITY ? 0.f : expf(sc4[j] - cm[j]));
            }
            if (lane == 0)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    red[(warp * 4 + j) * 2 + 0] = cm[j];
                    red[(warp * 4 + j) * 2 + 1] = cl[j];
                }
            __syncthreads();
            if (tid < hb) {
                const int qd = tid / 4, j = tid % 4;
                const int w0 = 2 * qd, w1 = 2 * qd + 1;              // the quad's two warps
                const float m0 = red[(w0 * 4 + j) * 2], l0 = red[(w0 * 4 + j) * 2 + 1];
                const float m1 = red[(w1 * 4 + j) * 2], l1 = red[(w1 * 4 + j) * 2 + 1];
                const float mc = fmaxf(m0, m1);
                if (mc != -INFINITY) {
                    const float lc = (m0 == -INFINITY ? 0.f : l0 * expf(m0 - mc)) +
                                     (m1 == -INFINITY ? 0.f : l1 * expf(m1 - mc));
                    const float mo = st_m[tid], mn = fmaxf(mo, mc);
                    st_l[tid] = (mo == -INFINITY ? 0.f : st_l[tid] * expf(mo - mn)) + lc * expf(mc - mn);
                    st_m[tid] = mn;
                }
            }
        }
        __syncthreads();
        if (tid < hb) st_l[tid] = st_l[tid] > 0.f ? 1.f / st_l[tid] : 0.f;    // now 1 / l

        // pass 2: branch output o = sum_e P_e v_e (this thread's outputs)
        for (int ch = 0; ch < nchunk; ++ch) {
            float sc4[4];
            const int nk = load_chunk(ch * BG_KC, true, sc4);
            if (score_thread)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int h = 4 * hq + j;
                    if (h < hb) ps[h * BG_KC + e_s] = sc4[j] == -INFINITY ? 0.f : expf(sc4[j] - st_m[h]) * st_l[h];
                }
            __syncthreads();
#pragma unroll
            for (int r = 0; r < BG_RO4; ++r) {
                const int x = tid + r * BG_NT;                 // column quad of o
                if (x < hb * dv / 4) {
                    const int h = 4 * x / dv, c = 4 * x % dv;
                    o_acc[r] = fma_rows(ps + h * BG_KC, vcs + c, L.vs, nk, o_acc[r]);
                }
            }
        }
        // gate gradient d_out . o and D = g d_out . o per head
#pragma unroll
        for (int r = 0; r < BG_RO4; ++r) {
            const int x = tid + r * BG_NT;
            if (x < hb * dv / 4) {
                const float4 d = *reinterpret_cast<const float4*>(dos + 4 * x);
                atomicAdd(&st_dg[4 * x / dv], d.x * o_acc[r].x + d.y * o_acc[r].y + d.z * o_acc[r].z + d.w * o_acc[r].w);
            }
        }
        __syncthreads();
        if (tid < hb) {
            if (a.dgates) a.dgates[(row0 + tid) * 3 + br] = st_dg[tid];
            st_D[tid] = st_g[tid] * st_dg[tid];
        }

        // pass 3: ds_e = P_e (d_o . v_e - D); dv_e += sum_h P_e d_o; dk_e += scale sum_h ds_e q;
        // dq += scale sum_e ds_e k_e
        for (int ch = 0; ch < nchunk; ++ch) {
            float sc4[4];
            const int nk = load_chunk(ch * BG_KC, true, sc4);
            if (score_thread && e_s < nk) {
                float dp[4] = {0.f, 0.f, 0.f, 0.f};
                const __nv_bfloat162* vr = reinterpret_cast<const __nv_bfloat162*>(vcs + e_s * L.vs);
                for (int c = 0; c < dv; c += 4) {
                    const float2 v0 = __bfloat1622float2(vr[c / 2]), v1 = __bfloat1622float2(vr[c / 2 + 1]);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int h = min(4 * hq + j, hb - 1);
                        const float4 dv4 = *reinterpret_cast<const float4*>(dob + h * dv + c);
                        dp[j] = fmaf(dv4.w, v1.y, fmaf(dv4.z, v1.x, fmaf(dv4.y, v0.y, fmaf(dv4.x, v0.x, dp[j]))));
                    }
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int h = 4 * hq + j;
                    if (h < hb) {
                        const float p = sc4[j] == -INFINITY ? 0.f : expf(sc4[j] - st_m[h]) * st_l[h];
                        ps[h * BG_KC + e_s] = p;
                        dss[h * BG_KC + e_s] = p * (dp[j] - st_D[h]);
                    }
                }
            }
            __syncthreads();
            // dv and dk of the chunk's keys: four columns per thread and atomic add
            for (int x = tid; x < nk * dv / 4; x += BG_NT) {
                const int e = 4 * x / dv, c = 4 * x % dv;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int h = 0; h < hb; ++h) {
                    const float p = ps[h * BG_KC + e];
                    const float4 d = *reinterpret_cast<const float4*>(dob + h * dv + c);
                    acc.x = fmaf(p, d.x, acc.x); acc.y = fmaf(p, d.y, acc.y);
                    acc.z = fmaf(p, d.z, acc.z); acc.w = fmaf(p, d.w, acc.w);
                }
                atomicAdd(reinterpret_cast<float4*>(dV + krow[e] * dv + c), acc);
            }
            for (int x = tid; x < nk * dqk / 4; x += BG_NT) {
                const int e = 4 * x / dqk, c = 4 * x % dqk;
                float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                for (int h = 0; h < hb; ++h) {
                    const float d = s.scale * dss[h * BG_KC + e];
                    const float4 qv = *reinterpret_cast<const float4*>(qs + h * dqk + c);
                    acc.x = fmaf(d, qv.x, acc.x); acc.y = fmaf(d, qv.y, acc.y);
                    acc.z = fmaf(d, qv.z, acc.z); acc.w = fmaf(d, qv.w, acc.w);
                }
                atomicAdd(reinterpret_cast<float4*>(dK + krow[e] * dqk + c), acc);
            }
#pragma unroll
            for (int r = 0; r < BG_RO4; ++r) {
                const int x = tid + r * BG_NT;                 // column quad of dq
                if (x < hb * dqk / 4) {
                    const int h = 4 * x / dqk, c = 4 * x % dqk;
                    dq_acc[r] = fma_rows(dss + h * BG_KC, kcs + c, L.ks, nk, dq_acc[r], s.scale);
                }
            }
        }
        __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < BG_RO4; ++r) {
        const int x = tid + r * BG_NT;
        if (x < hb * dqk / 4) *reinterpret_cast<float4*>(a.dq + row0 * dqk + 4 * x) = dq_acc[r];
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

size_t bwd_smem_bytes(const Shape& s) { return (size_t)BgLayout(s).total * 4; }

bool bwd_supported(const Shape& s) {
    if (s.dqk % 8 || s.dv % 8 || s.dqk > BG_MAXD || s.dv > BG_MAXD) return false;
    if ((s.per_head ? 1 : s.G) > BG_MAXH) return false;
    if ((s.flags & NSA_BR_SEL) && s.topk > BW_MAXB) return false;
    return bwd_smem_bytes(s) <= 200 * 1024;
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
    e = cudaFuncSetAttribute(bwd_group_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_group_kernel<<<dim3(s.Tq, s.per_head ? s.Hq : s.Hkv, s.B), BG_NT, smem, st>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess || !cmp) return e;
    const size_t n = (size_t)s.B * s.Hkv * s.Tk * (s.dqk + s.dv);
    const int grid = (int)std::min<size_t>((n + 255) / 256, 148 * 16);
    bwd_spread_kernel<<<grid, 256, 0, st>>>(dkc, dvc, dk, dv, s);
    return cudaGetLastError();
}

}  // namespace nsa
