// Shared device helpers for the sm_100a kernels of libnsa_b200.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nsa.h"

namespace nsa {

// Derived sizes of one problem, computed once on the host.
struct Shape {
    int B, Tq, Tk, q0, Hq, Hkv, G, dqk, dv;
    int bs, topk, win, lc, sc;
    int nb_full;    // complete selection blocks
    int nb_all;     // selection blocks including a ragged tail
    int n_cmp;      // compressed tokens
    int Hsel;       // selection units (KV heads or query heads)
    int heads_per_unit;
    int score_mode; // 0 scaled dot product, 1 probability sums, 2 from the compressed branch
    int n_sink;     // leading blocks always kept
    bool per_head;
    float scale;
    uint32_t flags;
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ void unpack8(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float2 t = __bfloat1622float2(h[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}

__device__ __forceinline__ uint4 pack8(const float* f) {
    uint4 u;
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    return u;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Order-preserving map of a finite fp32 score to uint32 (-0 treated as +0),
// packed with the inverted block id so that a larger key means a higher
// score, and for equal scores a lower block id.
__device__ __forceinline__ unsigned long long score_key(float s, int blk) {
    uint32_t u = __float_as_uint(s == 0.0f ? 0.0f : s);
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);
    return ((unsigned long long)u << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)blk);
}

__device__ __forceinline__ int key_block(unsigned long long key) {
    return (int)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
}

}  // namespace nsa

// Host-side launchers (defined in the kernel files, called by nsa_abi.cu).
namespace nsa {
cudaError_t launch_pool_kv(const Shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v,
                           float* kbar, __nv_bfloat16* kcmp, __nv_bfloat16* vcmp,
                           cudaStream_t st);
// pooled tokens of selection blocks [jb0, jb1) and compressed tokens [jc0, jc1)
cudaError_t launch_pool_range(const Shape& s, const __nv_bfloat16* k, const __nv_bfloat16* v,
                              float* kbar, __nv_bfloat16* kcmp, __nv_bfloat16* vcmp, int jb0, int jb1,
                              int jc0, int jc1, cudaStream_t st);
// rows [t0, t0 + n_new) of every (sequence, KV head) plane of k / v (v may be null)
cudaError_t launch_append_rows(const Shape& s, const __nv_bfloat16* k_new, const __nv_bfloat16* v_new,
                               __nv_bfloat16* k, __nv_bfloat16* v, int t0, int n_new, cudaStream_t st);
cudaError_t launch_score_topk(const Shape& s, const __nv_bfloat16* q, const float* kbar,
                              const float* scores_in, float* scores_out, int32_t* idx,
                              cudaStream_t st);
// backward pass for fixed block sets (attn_bwd.cu)
bool bwd_supported(const Shape& s);
cudaError_t launch_attn_bwd(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* kcmp, const __nv_bfloat16* vcmp,
                            const float* gates, const int32_t* idx, const __nv_bfloat16* d_out, float* dq,
                            float* dk, float* dv, float* dgates, float* dkc, float* dvc, cudaStream_t st);
// selection-score variants (score_mode 1 or 2): scores and/or top-k per row
bool score_variant_supported(const Shape& s);
cudaError_t launch_score_variant(const Shape& s, const __nv_bfloat16* q, const float* kbar,
                                 const __nv_bfloat16* kcmp, float* scores_out, int32_t* idx,
                                 cudaStream_t st);
cudaError_t launch_attn(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                        const __nv_bfloat16* v, const __nv_bfloat16* kcmp,
                        const __nv_bfloat16* vcmp, const float* gates, const int32_t* idx,
                        __nv_bfloat16* out, cudaStream_t st);
// tensor-core path (attn_tc.cu)
bool attn_tc_supported(const Shape& s);
cudaError_t launch_attn_tc(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                           const __nv_bfloat16* v, const __nv_bfloat16* kcmp,
                           const __nv_bfloat16* vcmp, const float* gates, const int32_t* idx,
                           const __nv_bfloat16* o_sel, int n_split, float* split_o,
                           float* split_lse, __nv_bfloat16* out, cudaStream_t st);
int attn_tc_split_count(const Shape& s);
cudaError_t launch_split_merge(const Shape& s, int n_split, const float* split_o,
                               const float* split_lse, const float* gates, __nv_bfloat16* out,
                               cudaStream_t st);
int read_and_clear_tc_status();
// the bounded wait's failure path on a barrier nothing completes (attn_tc.cu)
cudaError_t launch_wait_selftest(uint64_t limit_ns, cudaStream_t st);
// limit of the tensor-core attention kernel's waits (0: the default of one second)
cudaError_t set_wait_limit(uint64_t limit_ns);
// number of invalid rows of a caller-supplied idx into *bad (synchronises st) (sel_index.cu)
cudaError_t check_idx_rows(const Shape& s, const int32_t* idx, int* bad, cudaStream_t st);
cudaError_t launch_sel_merge(const Shape& s, const int32_t* idx, const __nv_bfloat16* part_o,
                             const float* part_lse, __nv_bfloat16* o_sel, cudaStream_t st);
// selected branch alone, one head per unit: out = g_sel * (merge of the row's
// sub-block partials), written directly (sel_merge.cu); s is the sub-block shape
cudaError_t launch_sel_merge_out(const Shape& s, const int32_t* idx, const __nv_bfloat16* part_o,
                                 const float* part_lse, const float* gates, __nv_bfloat16* out,
                                 cudaStream_t st);
// kept blocks -> the 64-key sub-blocks at or before the query (sel_index.cu)
cudaError_t launch_sel_expand(const Shape& s, const int32_t* idx, int32_t* idx_sub, cudaStream_t st);
// block-major selected branch (attn_sel_bm.cu)
struct SelIndex;
bool sel_bm_supported(const Shape& s);
cudaError_t launch_sel_bm(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                          const __nv_bfloat16* v, const SelIndex& x, __nv_bfloat16* part_o,
                          float* part_lse, cudaStream_t st);
int read_and_clear_bm_status();
// few-query attention with the keys as the MMA M dimension (attn_decode.cu)
bool attn_dec_supported(const Shape& s);
size_t attn_dec_items(const Shape& s);
size_t attn_dec_part_floats();   // fp32 values of one item's partial output (16 rows x 128)
cudaError_t launch_attn_dec(const Shape& s, const __nv_bfloat16* q, const __nv_bfloat16* k,
                            const __nv_bfloat16* v, const __nv_bfloat16* kcmp, const __nv_bfloat16* vcmp,
                            const int32_t* idx, float* part_o, float* part_lse, cudaStream_t st);
cudaError_t launch_dec_merge(const Shape& s, const float* part_o, const float* part_lse,
                             const float* gates, __nv_bfloat16* out, cudaStream_t st);
int read_and_clear_dec_status();
int read_and_clear_select_status();
// selection on the tensor cores, 3xTF32 (score_tc.cu)
bool score_tc_supported(const Shape& s);
size_t score_tc_q_floats(const Shape& s);   // each of qh, ql
size_t score_tc_k_floats(const Shape& s);   // each of kh, kl
cudaError_t launch_score_tc(const Shape& s, const __nv_bfloat16* q, const float* kbar, float* qh, float* ql,
                            float* kh, float* kl, int32_t* idx, cudaStream_t st);
int read_and_clear_sctc_status();
}  // namespace nsa
