// Types and helpers shared by the side-path kernels (routing, GEMV, token-parallel
// and tensor-core paths).
//
// One call applies the side path of one or more output slices that share x: each
// slice is a projection with its own factors, ranks, output width and place in y
// ("Compress then Serve" (academ.us/article/2407.00066), section 13.4 "Punica":
// the LoRA buffer is computed per token from x and added to y per output slice).
// Routing depends only on the token ids, so its work items carry no factor
// information; each kernel looks up (k, offsets) of the adapter for its slice.
#pragma once
#include "common.cuh"

namespace lf {

constexpr int kMaxSlices = 4;
constexpr int kGemvTok = 8;   // tokens per GEMV work item

struct Seg {
    int32_t adapter, start, len;
};
// GEMV work item (64 bytes): up to kGemvTok tokens of one adapter.
struct GemvItem {
    int32_t adapter, ntok, tok0, pad0;   // tok0: position of the first token in the permutation
    int64_t pad1, pad2;
    int32_t tok[kGemvTok];               // token indices
};
// Tensor-core work item: up to 128 consecutive permutation positions of one adapter.
struct TcItem {
    int32_t adapter, ntok, tok0, pad0;
};

// Factor tables of one output slice.
struct SliceTab {
    int32_t d_out;      // output columns of the slice
    int32_t t_col;      // first column of the slice's t in the t buffers
    int32_t chunk0;     // first grid column chunk of the slice (set per expand launch)
    int32_t k_shared;   // ranks == nullptr: every adapter uses the slice's shared factors (rank k_shared, offset 0)
    int32_t max_rank;   // 0, or the caller's bound on the slice's ranks (a rank above it is an error)
    int32_t pad;
    int64_t y_off;      // first column of the slice in y
    const int32_t* ranks;
    const int64_t* off_A;
    const int64_t* off_Bt;
    const __nv_bfloat16* A_pool;
    const __nv_bfloat16* Bt_pool;
    int64_t pool_A, pool_Bt;   // pool capacities (elements)
};

struct ApplyArgs {
    int32_t T, d_in, n_adapters, n_slices;
    int64_t y_ld;              // row stride of y (elements)
    int32_t ldt;               // row stride of t_buf / t_part (64 per slice)
    int32_t n_chunks;          // expand grid column chunks over all slices (set per launch)
    const __nv_bfloat16* x;    // T x d_in
    __nv_bfloat16* y;          // T rows of y_ld
    const int32_t* ids;        // T
    float scale;
    const float* scales;       // per adapter (nullable): replaces `scale`
    // Sigma-sandwich serving: t <- Sigma_a t before the expand (0 = none, 1 = diagonal
    // Sigma, n_adapters x k fp32, 2 = full Sigma, n_adapters x k x k fp32 row-major)
    int32_t sigma_mode;
    const float* sigma;
    SliceTab sl[kMaxSlices];
    // routing (sorted path)
    const int32_t* counts;     // [0] segments, [1] routed tokens, [2] GEMV items, [3] tensor-core items,
                               // [4] tokens in tok_list
    const Seg* segs;
    const int32_t* perm;
    const GemvItem* items;
    const TcItem* tc_items;
    const int32_t* tok_list;   // nullable: tokens for the token-parallel kernel (counts[4] of them)
    float* t_buf;              // T x ldt fp32, row = permutation position
    float* t_part;             // kTcMaxSplit x T x ldt fp32 split-K partials
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 v = __bfloat1622float2(h[i]);
        f[2 * i] = v.x;
        f[2 * i + 1] = v.y;
    }
}

// Slice that owns expand grid column chunk c.
__device__ __forceinline__ int slice_of_chunk(const ApplyArgs& a, int c) {
    int s = 0;
#pragma unroll
    for (int i = 1; i < kMaxSlices; ++i)
        if (i < a.n_slices && c >= a.sl[i].chunk0) s = i;
    return s;
}

// Rank and pool offsets of adapter `ad` in slice `s`, validated against the slice's
// pools: k > 64 -> LF_ERR_SHAPE, offsets not 16-byte aligned -> LF_ERR_ALIGNMENT,
// rows past a pool -> LF_ERR_WORKSPACE (latched when `report`); an invalid adapter
// contributes nothing.  Returns true when there is work (k > 0).
__device__ __forceinline__ bool factor_lookup(const int32_t* ranks, const int64_t* off_A, const int64_t* off_Bt,
                                              int k_shared, int max_rank, int d_in, int d_out, int64_t pool_A,
                                              int64_t pool_Bt, int ad, bool report, int& k, int64_t& oa, int64_t& ob) {
    if (ranks) {
        k = ranks[ad];
        oa = off_A[ad];
        ob = off_Bt[ad];
    } else {   // shared factors
        k = k_shared;
        oa = 0;
        ob = 0;
    }
    int err = 0;
    if (k > kMaxRank || (max_rank > 0 && k > max_rank)) err = LF_ERR_SHAPE;
    else if (k > 0 && ((oa & 7) || (ob & 7))) err = LF_ERR_ALIGNMENT;
    else if (k > 0 && (oa < 0 || ob < 0 || oa + (int64_t)k * d_in > pool_A || ob + (int64_t)k * d_out > pool_Bt))
        err = LF_ERR_WORKSPACE;
    if (err) {
        if (report) latch_error(err);
        k = 0;
        return false;
    }
    if (k < 0) k = 0;
    return k > 0;
}

__device__ __forceinline__ bool slice_factors(const ApplyArgs& a, int s, int ad, bool report, int& k, int64_t& oa,
                                              int64_t& ob) {
    const SliceTab& t = a.sl[s];
    return factor_lookup(t.ranks, t.off_A, t.off_Bt, t.k_shared, t.max_rank, a.d_in, t.d_out, t.pool_A, t.pool_Bt, ad,
                         report, k, oa, ob);
}

// Several projections of one batch (same tokens and ids), each with its own x, y and
// factor tables, applied by one launch in the decode regime.
constexpr int kMaxProj = 8;
struct ProjTab {
    const __nv_bfloat16* x;     // T x d_in
    __nv_bfloat16* y;           // T rows of y_ld
    int64_t y_ld, y_off;
    int32_t d_in, d_out;
    int32_t chunk0;             // first grid column chunk of the projection
    int32_t max_rank;           // 0, or the caller's bound on the projection's ranks
    const int32_t* ranks;
    const int64_t* off_A;
    const int64_t* off_Bt;
    const __nv_bfloat16* A_pool;
    const __nv_bfloat16* Bt_pool;
    int64_t pool_A, pool_Bt;
};
struct ProjArgs {
    int32_t T, n_adapters, n_proj, n_chunks;
    const int32_t* ids;
    float scale;
    const float* scales;        // per adapter (nullable): replaces `scale`
    ProjTab p[kMaxProj];
};

__device__ __forceinline__ float adapter_scale(const ApplyArgs& a, int ad) {
    return a.scales ? a.scales[ad] : a.scale;
}

// Sigma-sandwich step on one token's t (k values, fp32, in `t`): w = Sigma_ad t, written to
// `w` (may not alias `t`).  Called by `nthreads` threads with thread index `ti`; each
// output i is formed by one thread in a fixed order.
__device__ __forceinline__ void sigma_apply(const ApplyArgs& a, int ad, int k, const float* t, float* w, int ti,
                                            int nthreads) {
    if (a.sigma_mode == 1) {
        const float* d = a.sigma + (size_t)ad * k;
        for (int i = ti; i < k; i += nthreads) w[i] = d[i] * t[i];
    } else {
        const float* S = a.sigma + (size_t)ad * k * k;
        for (int i = ti; i < k; i += nthreads) {
            float acc = 0.f;
            for (int j = 0; j < k; ++j) acc = fmaf(S[i * k + j], t[j], acc);
            w[i] = acc;
        }
    }
}

}  // namespace lf
