// Multi-LoRA side path: routing, then shrink (t = A' x, fp32) and expand
// (y += s B' t, one bf16 rounding), never padding the retained rank.
//
// "Compress then Serve" (academ.us/article/2407.00066), section 3: (W0 + B A) x
// with the LoRA term computed apart from W0 x; section 11: a batch mixes
// requests for different adapters; section 13.4 "Punica": buffer = A x in fp32
// per token through an adapter index, then y += scale * B buffer.
// LoRAForge (kongchang.com), "The Bottleneck of Multi-LoRA Serving" and the
// rank-specialised kernels paragraph: adapters of different ranks run together,
// at their retained ranks, without padding.
#pragma once
#include "common.cuh"

namespace lf {

constexpr int kRouteThreads = 1024;
constexpr int kGemvTok = 8;        // tokens per GEMV work item
constexpr int kGemvThreads = 256;
constexpr int kGemvCols = kGemvThreads * 8;   // d_out columns per CTA

struct Seg {
    int32_t adapter, start, len;
};
struct GemvItem {
    int32_t seg, tok0, ntok, pad;
};

struct RouteOut {
    int32_t* counts;     // [0] n_seg, [1] n_valid, [2] n_items
    Seg* segs;           // min(T, n_adapters)
    int32_t* perm;       // T
    GemvItem* items;     // T / kGemvTok + min(T, n_adapters)
    int32_t* seg_out;    // optional caller copy
};

// One CTA: counting sort of token ids (stable), segments and GEMV work items.
// Shared memory: n_adapters ints (counts, then running positions).
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const int32_t* __restrict__ ids, int T,
                                                              int n_adapters, RouteOut o) {
    extern __shared__ int32_t rsm[];
    int32_t* pos = rsm;                         // n_adapters
    __shared__ int32_t wbase[32][32];
    __shared__ int32_t s_tot[3];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int a = tid; a < n_adapters; a += kRouteThreads) pos[a] = 0;
    __syncthreads();
    for (int t = tid; t < T; t += kRouteThreads) {
        const int a = ids[t];
        if (a < -1 || a >= n_adapters) {
            latch_error(LF_ERR_BAD_INDEX);
        } else if (a >= 0) {
            atomicAdd(&pos[a], 1);
        }
    }
    __syncthreads();
    // serial scan over adapters by thread 0 (n_adapters is small); emits segments/items
    if (tid == 0) {
        int run = 0, nseg = 0, nitem = 0;
        for (int a = 0; a < n_adapters; ++a) {
            const int c = pos[a];
            pos[a] = run;
            if (c > 0) {
                o.segs[nseg] = Seg{a, run, c};
                for (int q = 0; q < c; q += kGemvTok) o.items[nitem++] = GemvItem{nseg, q, min(kGemvTok, c - q), 0};
                ++nseg;
            }
            run += c;
        }
        s_tot[0] = nseg;
        s_tot[1] = run;
        s_tot[2] = nitem;
        o.counts[0] = nseg;
        o.counts[1] = run;
        o.counts[2] = nitem;
    }
    __syncthreads();
    // stable scatter, chunk by chunk; warps take their turn in token order
    for (int base = 0; base < T; base += kRouteThreads) {
        const int t = base + tid;
        int a = t < T ? ids[t] : -1;
        if (a < -1 || a >= n_adapters) a = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, a);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < kRouteThreads / 32; ++w) {
            if (warp == w && a >= 0 && lane == leader) {
                wbase[warp][lane] = pos[a];
                pos[a] += __popc(peers);
            }
            __syncthreads();
        }
        if (a >= 0) o.perm[wbase[warp][leader] + rank] = t;
        __syncthreads();
    }
    if (o.seg_out) {
        __syncthreads();
        const int nseg = s_tot[0], nval = s_tot[1];
        if (tid == 0) {
            o.seg_out[0] = nseg;
            o.seg_out[1] = nval;
        }
        for (int s = tid; s < nseg; s += kRouteThreads) {
            o.seg_out[2 + 3 * s] = o.segs[s].adapter;
            o.seg_out[3 + 3 * s] = o.segs[s].start;
            o.seg_out[4 + 3 * s] = o.segs[s].len;
        }
        for (int q = tid; q < nval; q += kRouteThreads) o.seg_out[2 + 3 * nseg + q] = o.perm[q];
    }
}

struct GemvArgs {
    int32_t d_in, d_out;
    const __nv_bfloat16* x;
    __nv_bfloat16* y;
    const int32_t* ranks;
    const int64_t* off_A;
    const int64_t* off_Bt;
    const __nv_bfloat16* A_pool;
    const __nv_bfloat16* Bt_pool;
    int64_t pool_A, pool_Bt;
    float scale;
    const int32_t* counts;
    const Seg* segs;
    const int32_t* perm;
    const GemvItem* items;
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

// grid: (max items, ceil(d_out / kGemvCols)).  Each CTA recomputes t for its
// <= kGemvTok tokens (A' rows and x rows come from L2 after the first CTA), then
// updates its d_out slice of y for those tokens.
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(GemvArgs a) {
    __shared__ float tsm[kGemvTok][kMaxRank];
    __shared__ int32_t toks[kGemvTok];
    const int it = blockIdx.x;
    if (it >= a.counts[2]) return;
    const GemvItem item = a.items[it];
    const Seg sg = a.segs[item.seg];
    const int ad = sg.adapter;
    const int k = a.ranks[ad];
    if (k <= 0) return;
    if (k > kMaxRank) {
        latch_error(LF_ERR_SHAPE);
        return;
    }
    const int64_t oa = a.off_A[ad], ob = a.off_Bt[ad];
    if ((oa & 7) || (ob & 7)) {
        latch_error(LF_ERR_ALIGNMENT);
        return;
    }
    if (oa < 0 || ob < 0 || oa + (int64_t)k * a.d_in > a.pool_A || ob + (int64_t)k * a.d_out > a.pool_Bt) {
        latch_error(LF_ERR_WORKSPACE);
        return;
    }
    const int nt = item.ntok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < nt) toks[tid] = a.perm[sg.start + item.tok0 + tid];
    __syncthreads();

    // shrink: warp w computes rows j = w, w+8, ... of t
    const __nv_bfloat16* Ap = a.A_pool + oa;
    for (int j = warp; j < k; j += kGemvThreads / 32) {
        float acc[kGemvTok];
#pragma unroll
        for (int q = 0; q < kGemvTok; ++q) acc[q] = 0.f;
        const __nv_bfloat16* arow = Ap + (int64_t)j * a.d_in;
        for (int d0 = lane * 8; d0 < a.d_in; d0 += 256) {
            float af[8], xf[8];
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(arow + d0)), af);
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q) {
                if (q < nt) {
                    bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)toks[q] * a.d_in + d0)), xf);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[q] = fmaf(af[e], xf[e], acc[q]);
                }
            }
        }
#pragma unroll
        for (int q = 0; q < kGemvTok; ++q) {
            const float v = warp_sum(acc[q]);
            if (lane == 0 && q < nt) tsm[q][j] = v;
        }
    }
    __syncthreads();

    // expand: 8 consecutive columns per thread
    const int e = blockIdx.y * kGemvCols + tid * 8;
    if (e >= a.d_out) return;
    float acc[kGemvTok][8];
#pragma unroll
    for (int q = 0; q < kGemvTok; ++q)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[q][c] = 0.f;
    const __nv_bfloat16* Bt = a.Bt_pool + ob + e;
    for (int j = 0; j < k; ++j) {
        float bf[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(Bt + (int64_t)j * a.d_out)), bf);
#pragma unroll
        for (int q = 0; q < kGemvTok; ++q) {
            if (q < nt) {
                const float tv = tsm[q][j];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[q][c] = fmaf(tv, bf[c], acc[q][c]);
            }
        }
    }
#pragma unroll
    for (int q = 0; q < kGemvTok; ++q) {
        if (q < nt) {
            __nv_bfloat16* yp = a.y + (int64_t)toks[q] * a.d_out + e;
            float yf[8];
            uint4 u = *reinterpret_cast<const uint4*>(yp);
            bf16x8_to_f32(u, yf);
            __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
            for (int c = 0; c < 4; ++c)
                h[c] = __floats2bfloat162_rn(fmaf(a.scale, acc[q][2 * c], yf[2 * c]),
                                             fmaf(a.scale, acc[q][2 * c + 1], yf[2 * c + 1]));
            *reinterpret_cast<uint4*>(yp) = u;
        }
    }
}

}  // namespace lf
