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
#include "prefill_tc.cuh"

namespace lf {

constexpr int kRouteThreads = 1024;
constexpr int kRouteChunk = 4096;  // tokens staged per pass of the run detection
constexpr int kGemvThreads = 256;
constexpr int kGemvCols = kGemvThreads * 8;   // d_out columns per CTA

struct RouteOut {
    int32_t* counts;     // [0] n_seg, [1] n_valid, [2] n_items, [3] n_tc_items, [4] n_tok (with tok_list)
    Seg* segs;           // min(T, n_adapters)
    int32_t* perm;       // T
    GemvItem* items;     // T / kGemvTok + min(T, n_adapters)
    int32_t* seg_out;    // optional caller copy
    TcItem* tc_items;    // T / kTcM + min(T, n_adapters) + 1
    int32_t tc_enable;   // segments with >= kTcMin tokens become tensor-core items
    // Run scratch (nullable, T ints each): with it the sort works on runs of equal
    // consecutive ids (the histogram and the stable scatter touch runs, not tokens).
    int32_t* run_start;  // first token of run i
    int32_t* run_pos;    // position of run i's first token in the permutation
    int32_t* tag;        // nullable: {kRouteTagMagic, T, n_adapters, tc_enable} once the tables are complete
    // nullable, T ints: the tokens of every segment that is not a tensor-core segment,
    // in routing order (adapter by adapter), for the token-parallel kernel
    int32_t* tok_list;
};

// Tag of a workspace whose routing tables were written for a batch of T tokens over
// n_adapters (checked by route_check_kernel before a routed call reuses them).
constexpr int32_t kRouteTagMagic = 0x52545447;

// Block-wide exclusive scan of one int per thread (blockDim.x a multiple of 32, <= 1024).
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) wsum[warp] = x;
    __syncthreads();
    if (warp == 0) {
        const int nw = (int)(blockDim.x >> 5);
        int w = lane < nw ? wsum[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        wsum[lane] = w;   // inclusive over warps
    }
    __syncthreads();
    const int base = warp > 0 ? wsum[warp - 1] : 0;
    const int tot = wsum[(blockDim.x >> 5) - 1];
    __syncthreads();
    if (total) *total = tot;
    return base + x - v;
}

// One CTA: stable counting sort of token ids into segments (adapter, start, len),
// the token permutation, GEMV work items of <= kGemvTok tokens and tensor-core items
// of <= 128 tokens.  Depends on the ids only (no factor tables), so one routing
// serves every slice and projection of a batch.
// Shared memory: 2 * n_adapters ints.
__global__ void __launch_bounds__(kRouteThreads) route_kernel(const int32_t* __restrict__ ids, int T,
                                                              int n_adapters, RouteOut o) {
    extern __shared__ int32_t rsm[];
    int32_t* cnt = rsm;                  // n_adapters: counts, then running positions
    int32_t* tokoff = rsm + n_adapters;  // n_adapters: first tok_list position of each adapter
    __shared__ int32_t wbase[32][32];
    __shared__ int wsum[32];
    __shared__ int s_carry[5];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nthr = (int)blockDim.x;
    for (int a = tid; a < n_adapters; a += nthr) cnt[a] = 0;
    if (tid == 0) s_carry[0] = 0;
    __syncthreads();
    const bool runs = o.run_start != nullptr;
    auto valid_id = [&](int t) {
        const int a = ids[t];
        return (a < -1 || a >= n_adapters) ? -1 : a;
    };
    int n_runs = 0;
    if (runs) {
        // runs of equal consecutive (valid) ids, in chunks of kRouteChunk tokens staged
        // through shared memory (coalesced loads); each thread owns a contiguous slice
        // of the chunk, counts its run starts, and one block scan numbers the runs
        __shared__ int32_t s_idc[kRouteChunk + 1];
        for (int base = 0; base < T; base += kRouteChunk) {
            const int len = min(kRouteChunk, T - base);
            for (int i = tid; i < len; i += nthr) {
                const int raw = ids[base + i];
                const bool bad = raw < -1 || raw >= n_adapters;
                if (bad) latch_error(LF_ERR_BAD_INDEX);
                s_idc[i + 1] = bad ? -1 : raw;
            }
            if (tid == 0) s_idc[0] = base > 0 ? valid_id(base - 1) : -2;
            __syncthreads();
            const int per = (len + nthr - 1) / nthr;
            const int t0 = min(len, tid * per), t1 = min(len, t0 + per);
            int nf = 0;
            for (int i = t0; i < t1; ++i) nf += (s_idc[i + 1] != s_idc[i]);
            int tot;
            int ri = block_excl_scan(nf, wsum, &tot) + s_carry[0] - 1;
            for (int i = t0; i < t1; ++i)
                if (s_idc[i + 1] != s_idc[i]) o.run_start[++ri] = base + i;
            __syncthreads();
            if (tid == 0) s_carry[0] += tot;
            __syncthreads();
        }
        n_runs = s_carry[0];
        for (int ri = tid; ri < n_runs; ri += nthr) {
            const int t0 = o.run_start[ri];
            const int a = valid_id(t0);
            if (a >= 0) atomicAdd(&cnt[a], (ri + 1 < n_runs ? o.run_start[ri + 1] : T) - t0);
        }
    } else {
        for (int t = tid; t < T; t += nthr) {
            const int a = ids[t];
            if (a < -1 || a >= n_adapters) latch_error(LF_ERR_BAD_INDEX);
            else if (a >= 0) atomicAdd(&cnt[a], 1);
        }
    }
    __syncthreads();
    if (tid == 0) s_carry[0] = s_carry[1] = s_carry[2] = s_carry[3] = s_carry[4] = 0;
    __syncthreads();
    // scans over adapters in chunks of kRouteThreads: token start, segment index, item
    // index, tensor-core item index, token-list position
    for (int a0 = 0; a0 < n_adapters; a0 += nthr) {
        const int a = a0 + tid;
        const int c = a < n_adapters ? cnt[a] : 0;
        const bool use_tc = o.tc_enable && c >= kTcMin;
        const int ni = use_tc ? 0 : (c + kGemvTok - 1) / kGemvTok;
        const int nti = use_tc ? (c + kTcM - 1) / kTcM : 0;
        int tt, ts, ti, tq, tb;
        const int start = block_excl_scan(c, wsum, &tt) + s_carry[0];
        const int sidx = block_excl_scan(c > 0 ? 1 : 0, wsum, &ts) + s_carry[1];
        const int iidx = block_excl_scan(ni, wsum, &ti) + s_carry[2];
        const int qidx = block_excl_scan(nti, wsum, &tq) + s_carry[3];
        const int bidx = block_excl_scan(use_tc ? 0 : c, wsum, &tb) + s_carry[4];
        if (a < n_adapters) {
            cnt[a] = start;
            tokoff[a] = use_tc ? -1 : bidx;
            if (c > 0) {
                o.segs[sidx] = Seg{a, start, c};
                for (int q = 0; q < nti; ++q) {
                    TcItem ti2;
                    ti2.adapter = a;
                    ti2.ntok = min(kTcM, c - q * kTcM);
                    ti2.tok0 = start + q * kTcM;
                    ti2.pad0 = 0;
                    o.tc_items[qidx + q] = ti2;
                }
                for (int q = 0; q < ni; ++q) {
                    GemvItem it{};
                    it.adapter = a;
                    it.ntok = min(kGemvTok, c - q * kGemvTok);
                    it.tok0 = start + q * kGemvTok;
                    o.items[iidx + q] = it;
                }
            }
        }
        __syncthreads();
        if (tid == 0) {
            s_carry[0] += tt;
            s_carry[1] += ts;
            s_carry[2] += ti;
            s_carry[3] += tq;
            s_carry[4] += tb;
        }
        __syncthreads();
    }
    const int nval = s_carry[0], nseg = s_carry[1];
    if (tid == 0) {
        o.counts[0] = nseg;
        o.counts[1] = nval;
        o.counts[2] = s_carry[2];
        o.counts[3] = s_carry[3];
        if (o.tok_list) o.counts[4] = s_carry[4];
        if (o.tag) {
            o.tag[0] = kRouteTagMagic;
            o.tag[1] = T;
            o.tag[2] = n_adapters;
            o.tag[3] = o.tc_enable;
        }
    }
    if (runs) {
        // stable scatter of runs (warp turns in run order), then every token in parallel
        const int nwr = min(nthr / 32, (n_runs + 31) / 32);
        for (int base = 0; base < n_runs; base += nthr) {
            const int ri = base + tid;
            int a = -1, len = 0;
            if (ri < n_runs) {
                const int t0 = o.run_start[ri];
                a = valid_id(t0);
                len = (ri + 1 < n_runs ? o.run_start[ri + 1] : T) - t0;
            }
            const unsigned peers = __match_any_sync(0xffffffffu, a);
            const int leader = __ffs(peers) - 1;
            int before = 0, total = 0;   // lengths of this warp's earlier / all runs of the same id
            for (int l = 0; l < 32; ++l) {
                const int v = __shfl_sync(0xffffffffu, len, l);
                if ((peers >> l) & 1u) {
                    total += v;
                    if (l < lane) before += v;
                }
            }
            for (int w = 0; w < nwr; ++w) {
                if (warp == w && a >= 0 && lane == leader) {
                    wbase[warp][lane] = cnt[a];
                    cnt[a] += total;
                }
                __syncthreads();
            }
            if (a >= 0) o.run_pos[ri] = wbase[warp][leader] + before;
            __syncthreads();
        }
        // permutation: one warp per run writes the run's consecutive token indices
        for (int ri = warp; ri < n_runs; ri += nthr / 32) {
            const int t0 = o.run_start[ri];
            if (valid_id(t0) < 0) continue;
            const int len = (ri + 1 < n_runs ? o.run_start[ri + 1] : T) - t0;
            const int p0 = o.run_pos[ri];
            for (int i = lane; i < len; i += 32) o.perm[p0 + i] = t0 + i;
        }
        __syncthreads();
    }
    if (!runs && T <= nthr) {
        // small batch: rank = number of earlier tokens with the same id (ids staged in smem)
        __shared__ int32_t s_ids[kRouteThreads];
        int a = -1;
        if (tid < T) {
            a = ids[tid];
            if (a < -1 || a >= n_adapters) a = -1;
            s_ids[tid] = a;
        }
        __syncthreads();
        if (a >= 0) {
            int rank = 0;
            for (int t2 = 0; t2 < tid; ++t2) rank += (s_ids[t2] == a);
            o.perm[cnt[a] + rank] = tid;
        }
        __syncthreads();
    }
    // stable scatter, chunk by chunk; warps take their turn in token order
    const int nwarps_live = min(nthr / 32, (T + 31) / 32);
    for (int base = 0; !runs && T > nthr && base < T; base += nthr) {
        const int t = base + tid;
        int a = t < T ? ids[t] : -1;
        if (a < -1 || a >= n_adapters) a = -1;
        const unsigned peers = __match_any_sync(0xffffffffu, a);
        const int leader = __ffs(peers) - 1;
        const int rank = __popc(peers & ((1u << lane) - 1u));
        for (int w = 0; w < nwarps_live; ++w) {
            if (warp == w && a >= 0 && lane == leader) {
                wbase[warp][lane] = cnt[a];
                cnt[a] += __popc(peers);
            }
            __syncthreads();
        }
        if (a >= 0) o.perm[wbase[warp][leader] + rank] = t;
        __syncthreads();
    }
    __syncthreads();
    for (int it = tid; it < s_carry[2]; it += nthr) {
        GemvItem& g = o.items[it];
        const int n = g.ntok, p0 = g.tok0;
#pragma unroll
        for (int q = 0; q < kGemvTok; ++q) g.tok[q] = q < n ? o.perm[p0 + q] : 0;
    }
    if (o.tok_list) {
        // tokens of the segments left to the token-parallel kernel, segment by segment
        // (one warp per segment; the permutation is complete after the barrier above)
        for (int sg = warp; sg < nseg; sg += nthr / 32) {
            const Seg sgm = o.segs[sg];
            const int off = tokoff[sgm.adapter];
            if (off < 0) continue;
            for (int q = lane; q < sgm.len; q += 32) o.tok_list[off + q] = o.perm[sgm.start + q];
        }
    }
    if (o.seg_out) {
        if (tid == 0) {
            o.seg_out[0] = nseg;
            o.seg_out[1] = nval;
        }
        for (int s = tid; s < nseg; s += nthr) {
            o.seg_out[2 + 3 * s] = o.segs[s].adapter;
            o.seg_out[3 + 3 * s] = o.segs[s].start;
            o.seg_out[4 + 3 * s] = o.segs[s].len;
        }
        for (int q = tid; q < nval; q += nthr) o.seg_out[2 + 3 * nseg + q] = o.perm[q];
    }
}

__device__ __forceinline__ bool item_ok(const ApplyArgs& a, int it, GemvItem& item) {
    if (it >= a.counts[2]) return false;
    item = a.items[it];
    return true;
}

// y[tok][e .. e+7] = bf16(y + scale * acc) for one 16-byte vector of y.
__device__ __forceinline__ void y_update8(__nv_bfloat16* yp, const float (&acc)[8], float scale) {
    uint4 u = *reinterpret_cast<const uint4*>(yp);
    float yf[8];
    bf16x8_to_f32(u, yf);
    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&u);
#pragma unroll
    for (int c = 0; c < 4; ++c)
        h[c] = __floats2bfloat162_rn(fmaf(scale, acc[2 * c], yf[2 * c]), fmaf(scale, acc[2 * c + 1], yf[2 * c + 1]));
    *reinterpret_cast<uint4*>(yp) = u;
}

constexpr int kShrinkJ = 4;   // rows of A' per pass

// Shrink: t[item][q][j] = A'_a[j] . x[tok_q] (fp32) for every (work item, slice); a
// bounded grid strides over the items the routing produced.  The d_in range is
// split across all warps so each warp keeps many 16-byte loads in flight; partial
// sums are reduced through shared memory in a fixed order.
__global__ void __launch_bounds__(kGemvThreads) shrink_kernel(ApplyArgs a) {
    __shared__ float part[kGemvThreads / 32][kShrinkJ][kGemvTok];
    __shared__ int32_t toks[kGemvTok];
    const int n_units = a.counts[2] * a.n_slices;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int itx = u / a.n_slices, sl = u - itx * a.n_slices;
        const GemvItem& item = a.items[itx];
        int k;
        int64_t oa, ob;
        if (!slice_factors(a, sl, item.adapter, true, k, oa, ob)) continue;   // uniform
        const int nt = item.ntok;
        if (tid < nt) toks[tid] = item.tok[tid];
        __syncthreads();
        const __nv_bfloat16* Ap = a.sl[sl].A_pool + oa;
        float* tout = a.t_buf + (size_t)item.tok0 * a.ldt + a.sl[sl].t_col;
        for (int j0 = 0; j0 < k; j0 += kShrinkJ) {
            float acc[kShrinkJ][kGemvTok];
#pragma unroll
            for (int jj = 0; jj < kShrinkJ; ++jj)
#pragma unroll
                for (int q = 0; q < kGemvTok; ++q) acc[jj][q] = 0.f;
            for (int d0 = tid * 8; d0 < a.d_in; d0 += kGemvThreads * 8) {
                float xf[kGemvTok][8];
#pragma unroll
                for (int q = 0; q < kGemvTok; ++q)
                    if (q < nt)
                        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)toks[q] * a.d_in + d0)), xf[q]);
#pragma unroll
                for (int jj = 0; jj < kShrinkJ; ++jj) {
                    if (j0 + jj < k) {
                        float af[8];
                        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(Ap + (int64_t)(j0 + jj) * a.d_in + d0)), af);
#pragma unroll
                        for (int q = 0; q < kGemvTok; ++q) {
                            if (q < nt) {
#pragma unroll
                                for (int e = 0; e < 8; ++e) acc[jj][q] = fmaf(af[e], xf[q][e], acc[jj][q]);
                            }
                        }
                    }
                }
            }
            const int nj = min(kShrinkJ, k - j0);   // block-uniform bounds: reduce live slots only
#pragma unroll
            for (int jj = 0; jj < kShrinkJ; ++jj)
#pragma unroll
                for (int q = 0; q < kGemvTok; ++q) {
                    if (jj < nj && q < nt) {
                        const float v = warp_sum(acc[jj][q]);
                        if (lane == 0) part[warp][jj][q] = v;
                    }
                }
            __syncthreads();
            if (tid < kShrinkJ * kGemvTok) {
                const int jj = tid / kGemvTok, q = tid % kGemvTok;
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kGemvThreads / 32; ++w) v += part[w][jj][q];
                if (j0 + jj < k && q < nt) tout[q * a.ldt + j0 + jj] = v;
            }
            __syncthreads();
        }
    }
}

// Expand: y[tok_q][e..e+7] = bf16(y + s * sum_j t[q][j] B'^T[j][e..e+7]) for every
// (work item, column chunk of kGemvCols over all slices); bounded grid, strided.
__global__ void __launch_bounds__(kGemvThreads) expand_kernel(ApplyArgs a) {
    __shared__ float tsm[kGemvTok][kMaxRank];
    __shared__ float tsw[kGemvTok][kMaxRank];
    __shared__ int32_t toks[kGemvTok];
    const int n_units = a.counts[2] * a.n_chunks;
    const int tid = threadIdx.x;
    for (int u = blockIdx.x; u < n_units; u += gridDim.x) {
        const int itx = u / a.n_chunks, chunk = u - itx * a.n_chunks;
        const GemvItem& item = a.items[itx];
        const int sl = slice_of_chunk(a, chunk);
        const SliceTab& S = a.sl[sl];
        int k;
        int64_t oa, ob;
        if (!slice_factors(a, sl, item.adapter, false, k, oa, ob)) continue;   // reported by the shrink; uniform
        const int nt = item.ntok;
        if (tid < nt) toks[tid] = item.tok[tid];
        const float* tin = a.t_buf + (size_t)item.tok0 * a.ldt + S.t_col;
        for (int e = tid; e < nt * kMaxRank; e += kGemvThreads) {
            const int q = e / kMaxRank, j = e % kMaxRank;
            tsm[q][j] = j < k ? tin[q * a.ldt + j] : 0.f;
        }
        __syncthreads();
        if (a.sigma_mode) {   // Sigma-sandwich: every token's t <- Sigma_a t (one adapter per item)
            const int q = tid / 32;   // 8 warps, one token each
            if (q < nt) sigma_apply(a, item.adapter, k, tsm[q], tsw[q], tid & 31, 32);
            __syncthreads();
            for (int e = tid; e < nt * kMaxRank; e += kGemvThreads) {
                const int q2 = e / kMaxRank, j = e % kMaxRank;
                tsm[q2][j] = j < k ? tsw[q2][j] : 0.f;
            }
            __syncthreads();
        }
        const int e = (chunk - S.chunk0) * kGemvCols + tid * 8;
        if (e < S.d_out) {
            float acc[kGemvTok][8];
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[q][c] = 0.f;
            const __nv_bfloat16* Bt = S.Bt_pool + ob + e;
#pragma unroll 4
            for (int j = 0; j < k; ++j) {
                float bf[8];
                bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(Bt + (int64_t)j * S.d_out)), bf);
#pragma unroll
                for (int q = 0; q < kGemvTok; ++q) {
                    if (q < nt) {
                        const float tv = tsm[q][j];
#pragma unroll
                        for (int c = 0; c < 8; ++c) acc[q][c] = fmaf(tv, bf[c], acc[q][c]);
                    }
                }
            }
            const float scale = adapter_scale(a, item.adapter);
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q)
                if (q < nt) y_update8(a.y + (int64_t)toks[q] * a.y_ld + S.y_off + e, acc[q], scale);
        }
        __syncthreads();   // tsm / toks are rewritten by the next unit
    }
}


// Routed calls reuse the routing tables already in the workspace.  If the tag does not
// name this batch shape (no routing pass on this workspace, or one for another T or
// adapter count), every work count is cleared, so no kernel of the call reads the tables,
// and LF_ERR_INVALID_ARG is latched.
__global__ void route_check_kernel(int32_t* tag, int32_t* counts, int T, int n_adapters, int tc_enable) {
    if (threadIdx.x != 0) return;
    if (!(tag[0] == kRouteTagMagic && tag[1] == T && tag[2] == n_adapters && tag[3] == tc_enable)) {
        counts[0] = counts[1] = counts[2] = counts[3] = counts[4] = 0;
        latch_error(LF_ERR_INVALID_ARG);
    }
}

// Decode regime, token-parallel (BGMV form: every token carries its adapter index,
// no sorting).  CTA (token, 16384-column chunk of one slice): t = A' x (k fp32 dot
// products over d_in, reduced across the CTA in a fixed order), then
// y[chunk] += s * B'^T t with 16-byte loads of the k rows of B'^T.  A chunk covers a
// whole projection up to 16384 columns, so t is formed once per (token, slice); wider
// slices recompute it per chunk (identical arithmetic; x and A' come from L2).  Tokens
// of one adapter read its factors from L2 after the first touch, so HBM sees every
// distinct factor row, x and y once.  512 threads: a 4096-wide x row is one 16-byte
// load per thread, so the shrink's loads are all in flight together (swept 256 / 512 / 1024
// threads and 8192 / 12288 / 16384 columns on the decode workload).
constexpr int kBgmvThreads = 512;
constexpr int kBgmvVec = 4;                                  // 8-column vectors per thread in the expand
constexpr int kBgmvCols = kBgmvThreads * 8 * kBgmvVec;       // d_out columns per CTA
constexpr int kBgmvJ = 8;                                    // retained directions per shrink pass

// t = A' x_t for one token (k values of fp32 into ts): every thread takes 8-element
// pieces of the row, kBgmvJ directions per pass, reduced over the warps in a fixed
// order.  CTA-uniform control flow (block barriers inside).
__device__ __forceinline__ void bgmv_shrink(const __nv_bfloat16* xr, int d_in, const __nv_bfloat16* Ap, int k,
                                            float (&red)[kBgmvThreads / 32][kBgmvJ], float* ts) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    for (int j0 = 0; j0 < k; j0 += kBgmvJ) {
        const int nj = min(kBgmvJ, k - j0);
        float acc[kBgmvJ];
#pragma unroll
        for (int jj = 0; jj < kBgmvJ; ++jj) acc[jj] = 0.f;
        for (int d0 = tid * 8; d0 < d_in; d0 += kBgmvThreads * 8) {
            uint4 ar[kBgmvJ];
            const uint4 xv = __ldg(reinterpret_cast<const uint4*>(xr + d0));
#pragma unroll
            for (int jj = 0; jj < kBgmvJ; ++jj)
                if (jj < nj) ar[jj] = __ldg(reinterpret_cast<const uint4*>(Ap + (int64_t)(j0 + jj) * d_in + d0));
            float xf[8];
            bf16x8_to_f32(xv, xf);
#pragma unroll
            for (int jj = 0; jj < kBgmvJ; ++jj) {
                if (jj < nj) {
                    float af[8];
                    bf16x8_to_f32(ar[jj], af);
#pragma unroll
                    for (int e = 0; e < 8; ++e) acc[jj] = fmaf(af[e], xf[e], acc[jj]);
                }
            }
        }
#pragma unroll
        for (int jj = 0; jj < kBgmvJ; ++jj) {
            if (jj < nj) {
                const float v = warp_sum(acc[jj]);
                if (lane == 0) red[warp][jj] = v;
            }
        }
        __syncthreads();
        if (tid < nj) {
            float v = 0.f;
#pragma unroll
            for (int w = 0; w < kBgmvThreads / 32; ++w) v += red[w][tid];
            ts[j0 + tid] = v;
        }
        __syncthreads();
    }
}

// The token row's chunk y[cbase ..) that the expand reads (always an HBM miss: each chunk
// is read once) and, for ranks up to 8, the k rows of B'^T, fetched into L2 by bulk
// prefetches (one thread per row) before the shrink, so that their latency overlaps the
// shrink instead of following it.  Larger ranks skip the B'^T rows: those mostly come from
// L2 already (every token of the adapter reads them), and a prefetch per CTA of up to 64
// rows adds L2 requests that cost more than the first touch saves.  Rows, offsets and
// chunk widths are multiples of 8 elements (16 bytes), as the bulk copy requires.
__device__ __forceinline__ void bgmv_prefetch(const __nv_bfloat16* yr, const __nv_bfloat16* Bt, int k, int d_out,
                                              int cbase) {
    const int tid = threadIdx.x;
    const int ncols = min(kBgmvCols, d_out - cbase);
    if (tid <= (k <= 8 ? k : 0) && ncols > 0) {
        const __nv_bfloat16* src = tid == 0 ? yr + cbase : Bt + (int64_t)(tid - 1) * d_out + cbase;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(ncols * 2) : "memory");
    }
}

// y[cbase .. cbase + kBgmvCols) of one token row (within d_out) += scale * B'^T tv,
// rounded once to bf16; 16-byte loads of the k rows of B'^T.
__device__ __forceinline__ void bgmv_expand(const float* tv, int k, const __nv_bfloat16* Bt, int d_out,
                                            __nv_bfloat16* yr, int cbase, float scale) {
    const int tid = threadIdx.x;
#pragma unroll
    for (int h = 0; h < kBgmvVec; ++h) {
        const int e = cbase + h * (kBgmvThreads * 8) + tid * 8;
        if (e >= d_out) break;
        uint4 yv = *reinterpret_cast<const uint4*>(yr + e);   // issued before the k-row loads are consumed
        float acc[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[c] = 0.f;
#pragma unroll 4
        for (int j = 0; j < k; ++j) {
            float bf[8];
            bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(Bt + (int64_t)j * d_out + e)), bf);
            const float tj = tv[j];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = fmaf(tj, bf[c], acc[c]);
        }
        __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(&yv);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float2 yf = __bfloat1622float2(y2[q]);
            y2[q] = __floats2bfloat162_rn(fmaf(scale, acc[2 * q], yf.x), fmaf(scale, acc[2 * q + 1], yf.y));
        }
        *reinterpret_cast<uint4*>(yr + e) = yv;
    }
}

// One (token, column chunk) of the token-parallel side path; CTA-uniform control flow.
__device__ __forceinline__ void bgmv_token(const ApplyArgs& a, int tok, float (&red)[kBgmvThreads / 32][kBgmvJ],
                                           float* ts, float* tw) {
    const int ad = a.ids[tok];
    if (ad == -1) return;
    const int sl = slice_of_chunk(a, blockIdx.y);
    const SliceTab& S = a.sl[sl];
    const bool lead = (int)blockIdx.y == S.chunk0 && threadIdx.x == 0;   // one CTA per (token, slice) reports
    if (ad < -1 || ad >= a.n_adapters) {
        if (lead && sl == 0) latch_error(LF_ERR_BAD_INDEX);
        return;
    }
    int k;
    int64_t oa, ob;
    if (!slice_factors(a, sl, ad, lead, k, oa, ob)) return;
    bgmv_shrink(a.x + (int64_t)tok * a.d_in, a.d_in, S.A_pool + oa, k, red, ts);
    const float* tv = ts;
    if (a.sigma_mode) {   // Sigma-sandwich: t <- Sigma_a t
        sigma_apply(a, ad, k, ts, tw, threadIdx.x, kBgmvThreads);
        __syncthreads();
        tv = tw;
    }
    bgmv_expand(tv, k, S.Bt_pool + ob, S.d_out, a.y + (int64_t)tok * a.y_ld + S.y_off,
                ((int)blockIdx.y - S.chunk0) * kBgmvCols, adapter_scale(a, ad));
}

// LIST = false: CTA blockIdx.x applies token blockIdx.x (decode regime, no routing pass).
// LIST = true: grid.x strides over the routing's list of tokens outside the tensor-core
// segments (tok_list, counts[4] of them, adapter by adapter, so consecutive CTAs read the
// same factors from L2).
template <bool LIST>
__global__ void __launch_bounds__(kBgmvThreads, 2) bgmv_kernel(ApplyArgs a) {
    __shared__ float red[kBgmvThreads / 32][kBgmvJ];
    __shared__ float ts[kMaxRank];
    __shared__ float tw[kMaxRank];
    if (!LIST) {
        bgmv_token(a, blockIdx.x, red, ts, tw);
        return;
    }
    const int n_tok = a.counts[4];
    for (int u = blockIdx.x; u < n_tok; u += gridDim.x) {
        bgmv_token(a, __ldg(a.tok_list + u), red, ts, tw);
        __syncthreads();   // red / ts / tw are rewritten by the next token
    }
}

// Several projections of one decode batch in one launch: CTA (token, column chunk),
// the chunks of all projections laid end to end along grid.y (each projection's first
// chunk at its chunk0).  Per projection the same arithmetic as bgmv_kernel<false>; each
// CTA first prefetches its y chunk (and small-rank B'^T rows) into L2.
__global__ void __launch_bounds__(kBgmvThreads, 2) bgmv_proj_kernel(ProjArgs a) {
    __shared__ float red[kBgmvThreads / 32][kBgmvJ];
    __shared__ float ts[kMaxRank];
    const int tok = blockIdx.x, c = blockIdx.y;
    int p = 0;
#pragma unroll
    for (int i = 1; i < kMaxProj; ++i)
        if (i < a.n_proj && c >= a.p[i].chunk0) p = i;
    const ProjTab& P = a.p[p];
    const int ad = a.ids[tok];
    if (ad == -1) return;
    const bool lead = c == P.chunk0 && threadIdx.x == 0;   // one CTA per (token, projection) reports
    if (ad < -1 || ad >= a.n_adapters) {
        if (lead && p == 0) latch_error(LF_ERR_BAD_INDEX);
        return;
    }
    int k;
    int64_t oa, ob;
    if (!factor_lookup(P.ranks, P.off_A, P.off_Bt, 0, P.max_rank, P.d_in, P.d_out, P.pool_A, P.pool_Bt, ad, lead, k,
                       oa, ob))
        return;
    __nv_bfloat16* yr = P.y + (int64_t)tok * P.y_ld + P.y_off;
    const int cbase = (c - P.chunk0) * kBgmvCols;
    bgmv_prefetch(yr, P.Bt_pool + ob, k, P.d_out, cbase);
    bgmv_shrink(P.x + (int64_t)tok * P.d_in, P.d_in, P.A_pool + oa, k, red, ts);
    bgmv_expand(ts, k, P.Bt_pool + ob, P.d_out, yr, cbase, a.scales ? a.scales[ad] : a.scale);
}

// Decode regime of the no-allocation entry point (one slice, sorted items): CTA
// (item, d_out chunk): all warps share the dot products of each A' row over d_in
// (16-byte loads issued together), t is reduced in a fixed order in shared memory,
// then the CTA updates its d_out chunk of y.  CTAs of one item in different chunks
// recompute the same t (identical arithmetic, A' and x served from L2).
__global__ void __launch_bounds__(kGemvThreads) fused_gemv_kernel(ApplyArgs a) {
    __shared__ float part[kGemvThreads / 32][kShrinkJ][kGemvTok];
    __shared__ float tsm[kGemvTok][kMaxRank];
    __shared__ int32_t toks[kGemvTok];
    GemvItem item;
    if (!item_ok(a, blockIdx.x, item)) return;
    const SliceTab& S = a.sl[0];
    int k;
    int64_t oa, ob;
    if (!slice_factors(a, 0, item.adapter, blockIdx.y == 0, k, oa, ob)) return;
    const int nt = item.ntok;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (tid < nt) toks[tid] = a.items[blockIdx.x].tok[tid];
    __syncthreads();
    const __nv_bfloat16* Ap = S.A_pool + oa;
    for (int j0 = 0; j0 < k; j0 += kShrinkJ) {
        const int nj = min(kShrinkJ, k - j0);
        float acc[kShrinkJ][kGemvTok];
#pragma unroll
        for (int jj = 0; jj < kShrinkJ; ++jj)
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q) acc[jj][q] = 0.f;
        for (int d0 = tid * 8; d0 < a.d_in; d0 += kGemvThreads * 8) {
            uint4 xr[kGemvTok], ar[kShrinkJ];
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q)
                if (q < nt) xr[q] = __ldg(reinterpret_cast<const uint4*>(a.x + (int64_t)toks[q] * a.d_in + d0));
#pragma unroll
            for (int jj = 0; jj < kShrinkJ; ++jj)
                if (jj < nj) ar[jj] = __ldg(reinterpret_cast<const uint4*>(Ap + (int64_t)(j0 + jj) * a.d_in + d0));
#pragma unroll
            for (int jj = 0; jj < kShrinkJ; ++jj) {
                if (jj < nj) {
                    float af[8];
                    bf16x8_to_f32(ar[jj], af);
#pragma unroll
                    for (int q = 0; q < kGemvTok; ++q) {
                        if (q < nt) {
                            float xf[8];
                            bf16x8_to_f32(xr[q], xf);
#pragma unroll
                            for (int e = 0; e < 8; ++e) acc[jj][q] = fmaf(af[e], xf[e], acc[jj][q]);
                        }
                    }
                }
            }
        }
#pragma unroll
        for (int jj = 0; jj < kShrinkJ; ++jj)
#pragma unroll
            for (int q = 0; q < kGemvTok; ++q) {
                if (jj < nj && q < nt) {
                    const float v = warp_sum(acc[jj][q]);
                    if (lane == 0) part[warp][jj][q] = v;
                }
            }
        __syncthreads();
        if (tid < kShrinkJ * kGemvTok) {
            const int jj = tid / kGemvTok, q = tid % kGemvTok;
            if (jj < nj && q < nt) {
                float v = 0.f;
#pragma unroll
                for (int w = 0; w < kGemvThreads / 32; ++w) v += part[w][jj][q];
                tsm[q][j0 + jj] = v;
            }
        }
        __syncthreads();
    }
    const int e = blockIdx.y * kGemvCols + tid * 8;
    if (e >= S.d_out) return;
    float acc[kGemvTok][8];
#pragma unroll
    for (int q = 0; q < kGemvTok; ++q)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[q][c] = 0.f;
    const __nv_bfloat16* Bt = S.Bt_pool + ob + e;
#pragma unroll 4
    for (int j = 0; j < k; ++j) {
        float bf[8];
        bf16x8_to_f32(__ldg(reinterpret_cast<const uint4*>(Bt + (int64_t)j * S.d_out)), bf);
#pragma unroll
        for (int q = 0; q < kGemvTok; ++q) {
            if (q < nt) {
                const float tv = tsm[q][j];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[q][c] = fmaf(tv, bf[c], acc[q][c]);
            }
        }
    }
    const float scale = adapter_scale(a, item.adapter);
#pragma unroll
    for (int q = 0; q < kGemvTok; ++q)
        if (q < nt) y_update8(a.y + (int64_t)toks[q] * a.y_ld + S.y_off + e, acc[q], scale);
}

}  // namespace lf
