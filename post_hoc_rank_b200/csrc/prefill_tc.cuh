// Multi-LoRA shrink / expand for segments with many tokens, on tcgen05 tensor
// cores (sm_100a).  Same arithmetic contract as the GEMV path: t = A' x kept in
// fp32, y = bf16(y + s * B'^T... ) rounded once ("Compress then Serve",
// academ.us/article/2407.00066, section 13.4 "Punica": fp32 intermediate buffer,
// then the scaled B step into y).  Only the prefill-shaped case is a real dense
// contraction (M = tokens of one adapter), so only it uses the tensor cores.
//
// Shrink: D[128 tokens x N] = X[128 x d_in] * [A'_1; A'_2; ...]^T, bf16 in, fp32 in
//   TMEM, N = the sum of the slices' ranks rounded up to 16 (padding lives in shared
//   memory only): x is read once for every slice that shares it.  X rows are
//   gathered through the token permutation with 16-byte cp.async into a 4-stage
//   ring of K-major core matrices, or, when the tile's tokens are consecutive rows
//   of x (a prefill request), loaded by one 2-D TMA copy per stage; one thread
//   issues the MMAs and commits each stage to an mbarrier that frees the stage for
//   the next copy.
// Expand (per slice): D[128 x 128] = t_hi * B + t_lo * B with t = t_hi + t_lo split
//   into two bf16 values (about 16 significant bits of the fp32 t); B = B'^T tile,
//   MN-major; the epilogue reads D from tensor memory and updates y once.
#pragma once
#include <cuda.h>   // CUtensorMap (type only)

#include "apply_common.cuh"
#include "tc.cuh"

namespace lf {

constexpr int kTcMin = 64;       // segments with at least this many tokens use the tensor cores
constexpr int kTcM = 128;        // tokens per tile (UMMA M)
constexpr int kTcKB = 64;        // d_in elements per pipeline stage (128 bytes per row)
constexpr int kTcStages = 4;
constexpr int kTcThreads = 128;  // shrink: 4 warps, warp w owns tensor-memory lanes 32w .. 32w+31
constexpr int kTcCols = 2048;    // d_out columns per expand CTA
constexpr int kTcMaxSplit = 8;   // d_in is split over at most this many CTAs per token tile

// d_in elements per split: d_in is cut into min(kTcMaxSplit, ceil(d_in / kTcSplitTarget))
// splits of equal length rounded up to the stage width (3584 -> 2 x 1792, 18944 -> 8 x
// 2368), so the CTAs of one token tile carry the same work.
constexpr int kTcSplitTarget = 2048;
__host__ __device__ inline int tc_split_len(int d_in) {
    int n = (d_in + kTcSplitTarget - 1) / kTcSplitTarget;
    n = n < 1 ? 1 : (n > kTcMaxSplit ? kTcMaxSplit : n);
    const int len = (d_in + n - 1) / n;
    return ((len + kTcKB - 1) / kTcKB) * kTcKB;
}

// ---- shrink ---------------------------------------------------------------
// CTA (token tile of one segment, split of d_in), 4 warps in roles:
//   warps 0, 2, 3, producers: gather the stage's 128 x rows (64 d_in elements,
//     through the token permutation) and the k rows of A' into a kTcStages ring
//     with 16-byte cp.async; kTcAhead stages stay in flight; once a stage's copies
//     have landed (cp.async.wait_group) each lane fences them to the async proxy and
//     arrives on the stage's `full` barrier; a stage is refilled after the
//     tcgen05.commit of the MMAs that read it arrives on its `empty` barrier.
//     When the tile's tokens are consecutive rows of x and the caller encoded a
//     tensor map of x (box 64 x 128, 128-byte swizzle), warp 0 lane 0 loads the x
//     stage with one TMA copy counted on the stage's `xfull` barrier instead, and
//     before leaving waits for every copy it issued;
//   warp 1 lane 0, MMA issuer: waits on `full` (and `xfull`), issues four K = 16
//     MMAs into TMEM, commits to `empty`, and at the end to `done`;
//   all warps: epilogue from TMEM (warp w reads lanes 32w ..) into t_part.
constexpr int kTcAhead = 2;      // stages in flight before the producers signal the oldest
constexpr int kTcProducers = 3;  // producer warps: 0, 2, 3 (warp 1 issues the MMAs)
// MAXN = most B rows (summed ranks) a CTA can take: 64 for one slice, 256 for up to 4.
template <int MAXN>
struct ShrinkTcSmem {
    __nv_bfloat16 a[kTcStages][kTcM * kTcKB];    // 16 KB per stage
    __nv_bfloat16 b[kTcStages][MAXN * kTcKB];    //  8 KB (MAXN 64) or 32 KB (MAXN 256) per stage
    uint64_t full[kTcStages];
    uint64_t empty[kTcStages];
    uint64_t xfull[kTcStages];   // TMA x stages (tx bytes)
    uint64_t done;
    uint32_t tmem;
    int32_t toks[kTcM];
    int32_t kcum[kMaxSlices + 1];   // B rows of slice s: kcum[s] .. kcum[s+1]-1
    int64_t oa[kMaxSlices];
};

// byte offset of element (row, kk) of a K-major operand tile with 64 K-elements per row
__device__ __forceinline__ uint32_t kmaj64(int row, int kk) {
    return (uint32_t)((row >> 3) * 1024 + (kk >> 3) * 128 + (row & 7) * 16 + (kk & 7) * 2);
}

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;   // src-size 0 fills the 16 bytes with zeros
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}


constexpr uint32_t kTcXStageBytes = kTcM * kTcKB * 2;   // one TMA box of x

// x_tma: the caller encoded `xmap` (x as d_in x T bf16, box 64 x 128, 128-byte swizzle).
template <int MAXN>
__global__ void __launch_bounds__(kTcThreads) shrink_tc_kernel(ApplyArgs a, const __grid_constant__ CUtensorMap xmap,
                                                               int x_tma) {
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    auto& s = *reinterpret_cast<ShrinkTcSmem<MAXN>*>(tc_raw);
    if ((int)blockIdx.x >= a.counts[3]) return;
    const TcItem it = a.tc_items[blockIdx.x];
    const int split = blockIdx.y, slen = tc_split_len(a.d_in);
    const int kbeg = split * slen;
    if (kbeg >= a.d_in) return;   // uniform: this split has no columns
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = it.ntok;
    if (tid < a.n_slices) {   // each slice's rank and A' offset, looked up in parallel
        int k;
        int64_t oa, ob;
        slice_factors(a, tid, it.adapter, split == 0, k, oa, ob);
        s.kcum[tid + 1] = k;
        s.oa[tid] = oa;
    }
    for (int m = tid; m < kTcM; m += kTcThreads) s.toks[m] = m < nt ? a.perm[it.tok0 + m] : 0;
    __syncthreads();
    if (tid == 0) {   // prefix sums: B rows of slice q are kcum[q] .. kcum[q+1]-1
        s.kcum[0] = 0;
        for (int q = 1; q <= a.n_slices; ++q) s.kcum[q] += s.kcum[q - 1];
    }
    bool consecutive = true;
    for (int m = tid; m < nt; m += kTcThreads) consecutive = consecutive && s.toks[m] == s.toks[0] + m;
    // uniform: x stages by TMA (rows toks[0] .. +127; rows past nt are never stored)
    const bool tma = __syncthreads_and(consecutive) && x_tma != 0 && (smem_u32(s.a[0]) & 1023u) == 0;
    const int ktot = s.kcum[a.n_slices];
    if (ktot <= 0) return;   // uniform
    const int npad = (ktot + 15) & ~15;
    // rows ktot..npad-1 of every B stage stay zero (never written by the copies)
    for (int e = tid; e < kTcStages * (npad - ktot) * kTcKB; e += kTcThreads) {
        const int st = e / ((npad - ktot) * kTcKB), r2 = e % ((npad - ktot) * kTcKB);
        const int n = ktot + r2 / kTcKB, kk = r2 % kTcKB;
        *reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(s.b[st]) + kmaj64(n, kk)) = __float2bfloat16(0.f);
    }
    if (warp == 0) tc::tmem_alloc(&s.tmem, MAXN);
    if (tid == 0) {
        for (int i = 0; i < kTcStages; ++i) {
            mbar_init(&s.full[i], 32 * kTcProducers);
            mbar_init(&s.empty[i], 1);
            mbar_init(&s.xfull[i], 1);
        }
        mbar_init(&s.done, 1);
        fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem;
    const int kend = min(a.d_in, kbeg + slen);
    const int nK = (kend - kbeg + kTcKB - 1) / kTcKB;
    bool ok = true;

    const int pidx = warp == 0 ? 0 : warp - 1;   // producer index (warps 0, 2, 3)
    if (warp != 1 && pidx < kTcProducers) {   // producers
        const __nv_bfloat16* A0 = a.sl[0].A_pool + s.oa[0];   // the only slice when MAXN == 64
        const bool x_issuer = tma && warp == 0 && lane == 0;
        int x_issued = 0;   // TMA x stages issued by this thread
        for (int kb = 0; kb < nK && ok; ++kb) {
            const int st = kb % kTcStages;
            if (kb >= kTcStages) ok = mbar_wait(&s.empty[st], (uint32_t)((kb / kTcStages - 1) & 1));
            if (!ok) break;
            char* abase = reinterpret_cast<char*>(s.a[st]);
            char* bbase = reinterpret_cast<char*>(s.b[st]);
            const int k0 = kbeg + kb * kTcKB;   // a multiple of 64 elements (128 bytes)
            if (x_issuer) {
                mbar_arrive_expect_tx(&s.xfull[st], kTcXStageBytes);
                tc::tma_load_2d(abase, &xmap, k0, s.toks[0], &s.xfull[st]);
                ++x_issued;
            }
            // chunk mapping: a half-warp covers 8 rows x 32 contiguous bytes (full sectors);
            // each quarter-warp writes 8 rows of one 16-byte column (distinct banks)
            for (int i = pidx; !tma && i < (kTcM * kTcKB / 8) / 32; i += kTcProducers) {
                const int u = 2 * i + (lane >> 4);
                const int m = 8 * (u & 15) + (lane & 7);
                const int kc = 2 * (u >> 4) + ((lane >> 3) & 1);
                const int kk = k0 + kc * 8;
                const bool v = m < nt && kk < kend;
                cp_async16_zfill(abase + kmaj64(m, kc * 8), v ? a.x + (int64_t)s.toks[m] * a.d_in + kk : a.x, v);
            }
            const int nrb = (ktot + 7) >> 3;
            for (int c = lane + 32 * pidx; c < nrb * 64; c += 32 * kTcProducers) {
                const int u = c >> 4;
                const int n = 8 * (u % nrb) + (c & 7);
                const int kc = 2 * (u / nrb) + ((c >> 3) & 1);
                const int kk = k0 + kc * 8;
                if (n < ktot) {
                    int q = 0;
                    if (MAXN > kMaxRank)
                        while (q + 1 < a.n_slices && n >= s.kcum[q + 1]) ++q;
                    const __nv_bfloat16* Ap = (MAXN > kMaxRank ? a.sl[q].A_pool + s.oa[q] : A0);
                    const bool v = kk < kend;
                    cp_async16_zfill(bbase + kmaj64(n, kc * 8),
                                     v ? Ap + (int64_t)(n - s.kcum[q]) * a.d_in + kk : Ap, v);
                }
            }
            tc::cp_async_commit();
            if (kb >= kTcAhead) {   // stage kb - kTcAhead has landed: hand it to the MMA issuer
                tc::cp_async_wait<kTcAhead>();
                tc::fence_proxy_async();
                mbar_arrive1(&s.full[(kb - kTcAhead) % kTcStages]);
            }
        }
        tc::cp_async_wait<0>();
        tc::fence_proxy_async();
        if (ok)
            for (int kb = max(0, nK - kTcAhead); kb < nK; ++kb) mbar_arrive1(&s.full[kb % kTcStages]);
        // no TMA copy of this thread is still in flight when the CTA leaves (on the
        // normal path these phases completed before the MMAs that read them)
        for (int kb = max(0, x_issued - kTcStages); kb < x_issued; ++kb)
            if (!mbar_wait(&s.xfull[kb % kTcStages], (uint32_t)((kb / kTcStages) & 1))) ok = false;
    } else if (warp == 1 && lane == 0) {   // MMA issuer
        const uint32_t idesc = tc::idesc_bf16(kTcM, npad, 0, 0);
        for (int kb = 0; kb < nK && ok; ++kb) {
            const int st = kb % kTcStages;
            ok = mbar_wait(&s.full[st], (uint32_t)((kb / kTcStages) & 1));
            if (ok && tma) ok = mbar_wait(&s.xfull[st], (uint32_t)((kb / kTcStages) & 1));
            if (!ok) break;
            tc::fence_after_sync();
#pragma unroll
            for (int ks = 0; ks < kTcKB / 16; ++ks) {
                const uint64_t ad = tma ? tc::smem_desc_sw128(reinterpret_cast<char*>(s.a[st]) + ks * 32)
                                        : tc::smem_desc(reinterpret_cast<char*>(s.a[st]) + ks * 256, 128, 1024);
                const uint64_t bd = tc::smem_desc(reinterpret_cast<char*>(s.b[st]) + ks * 256, 128, 1024);
                tc::mma_bf16(tmem, ad, bd, idesc, kb > 0 || ks > 0);
            }
            tc::commit(&s.empty[st]);
        }
        if (ok) tc::commit(&s.done);
    }
    __syncwarp();
    // epilogue: every thread waits for the final commit (a failed role above makes this
    // wait run out as well; the error is latched either way)
    ok = ok && mbar_wait(&s.done, 0);
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    if (ok) {
        const int m = warp * 32 + lane;
        float* trow = a.t_part + ((size_t)split * a.T + it.tok0 + m) * a.ldt;
        int q = 0;
        for (int c0 = 0; c0 < npad; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            if (m < nt) {
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int c = c0 + i;
                    if (c < ktot) {
                        if (MAXN > kMaxRank) {
                            while (q + 1 < a.n_slices && c >= s.kcum[q + 1]) ++q;
                            trow[a.sl[q].t_col + c - s.kcum[q]] = v[i];
                        } else {
                            trow[c] = v[i];   // one slice, t columns 0 .. k-1
                        }
                    }
                }
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, MAXN);
}

template <int MAXN>
constexpr size_t shrink_tc_smem() { return sizeof(ShrinkTcSmem<MAXN>) + 1024; }

// ---- expand ---------------------------------------------------------------
// CTA (token tile of one segment, kTcCols columns of d_out), 256 threads.  The
// column range is walked in kTcN2-wide steps through a software pipeline:
//   y tiles stream into a 3-buffer shared-memory ring, B'^T tiles into 2 buffers
//   (cp.async), so the loads of steps i+1 and i+2 are in flight while step i runs.
//   A y tile is gathered row by row through the permutation with cp.async or, when
//   the tile's tokens are consecutive rows of y and the caller encoded a tensor map
//   of y (box 64 x 128, 128-byte swizzle), loaded by thread 0 with two TMA copies;
//   either way it is held as two 64-column halves in the 128-byte swizzle layout;
//   one thread issues D = t_hi B + t_lo B (M = 128, N = kTcN2, fp32 in TMEM) and
//   commits to an mbarrier;
//   8 warps read D (warp w: lanes 32(w%4).., columns 64(w/4)..), add s*D to the
//   staged y in shared memory with one bf16 rounding, then the tile is written
//   back: by two TMA stores when it is a full TMA tile (128 tokens, 128 columns
//   inside the CTA's range), else with 16-byte stores of its rows < ntok and columns
//   in range (rows past the tile belong to other CTAs and are never written).
constexpr int kTcYBuf = 3;
constexpr int kTcExpThreads = 256;
constexpr uint32_t kTcYHalf = kTcM * 128;   // bytes of one 64-column half of a staged y tile
// KMAX: largest rank the variant takes (64: every rank, 97 KB of shared memory, two CTAs
// per SM; 16: ranks up to 16, 62 KB, three CTAs per SM); N2: expand step width (UMMA N).
template <int KMAX, int N2>
struct ExpandTcSmem {
    __nv_bfloat16 ahi[kTcM * KMAX];              // t_hi, K-major
    __nv_bfloat16 alo[kTcM * KMAX];              // t_lo
    __nv_bfloat16 b[2][KMAX * N2];               // B'^T tiles, MN-major
    union {
        __nv_bfloat16 yt[kTcYBuf][kTcM * N2];        // staged y tiles (1024-byte aligned when the block
                                                     // is: the members above are multiples of 1 KB;
                                                     // checked before TMA)
        float tw[kTcM][kMaxRank + 1];                // summed t rows (Sigma-sandwich only, prologue)
    };
    uint64_t bar;
    uint64_t ybar[kTcYBuf];   // TMA y tiles (tx bytes)
    uint32_t tmem;
    int32_t toks[kTcM];
};

// Byte offset of (row, col) in a staged y tile: 64-column halves of 128 rows x 128
// bytes, the 16-byte chunk c of row r stored at chunk c ^ (r % 8) (the layout a TMA
// copy with 128-byte swizzle writes; 16-byte row accesses of 8 consecutive rows hit
// distinct banks).
__device__ __forceinline__ uint32_t ytile_off(int row, int col) {
    return (uint32_t)(col >> 6) * kTcYHalf + (uint32_t)row * 128 +
           ((uint32_t)(((col >> 3) & 7) ^ (row & 7)) << 4) + (uint32_t)(col & 7) * 2;
}

// y_tma: the caller encoded `ymap` (y as y_ld x T bf16, box 64 x 128, 128-byte swizzle).
// The two variants split the (item, slice) pairs between them: KMAX = 16 takes ranks up
// to 16 (without Sigma-sandwich), KMAX = 64 the rest.
template <int KMAX, int N2>
__global__ void __launch_bounds__(kTcExpThreads, KMAX == 16 ? 3 : 2)
    expand_tc_kernel(ApplyArgs a, const __grid_constant__ CUtensorMap ymap, int y_tma) {
    static_assert(N2 % 64 == 0 && N2 <= 128, "steps of whole 64-column halves");
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    auto& s = *reinterpret_cast<ExpandTcSmem<KMAX, N2>*>(tc_raw);
    if ((int)blockIdx.x >= a.counts[3]) return;
    const TcItem it = a.tc_items[blockIdx.x];
    const int sl = slice_of_chunk(a, blockIdx.y);
    const SliceTab& S = a.sl[sl];
    int k;
    int64_t oa, ob;
    if (!slice_factors(a, sl, it.adapter, false, k, oa, ob)) return;   // reported by the shrink
    const bool small = k <= 16 && a.sigma_mode == 0;
    if (small != (KMAX == 16)) return;   // the other variant's pair
    const int e_begin = ((int)blockIdx.y - S.chunk0) * kTcCols;
    if (e_begin >= S.d_out) return;
    const int e_end = min(S.d_out, e_begin + kTcCols);
    const int nit = (e_end - e_begin + N2 - 1) / N2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nt = it.ntok;
    const float scale = adapter_scale(a, it.adapter);
    __nv_bfloat16* ybase = a.y + S.y_off;
    const int kpad = (k + 15) & ~15;
    const uint32_t sbo = (uint32_t)(kpad / 8) * 128;   // 8-row groups of t / 8-column groups of B
    for (int m = tid; m < kTcM; m += kTcExpThreads) s.toks[m] = m < nt ? a.perm[it.tok0 + m] : 0;
    // t tile -> (t_hi, t_lo) bf16, K-major: element (m, j) at (m/8)*sbo + (j/8)*128 + (m%8)*16 + (j%8)*2
    const int nsplit = (a.d_in + tc_split_len(a.d_in) - 1) / tc_split_len(a.d_in);
    auto t_of = [&](int m, int j) {   // t = sum of the split-K partials, fixed order: bitwise reproducible
        float acc = 0.f;
        if (m < nt && j < k)
            for (int sp = 0; sp < nsplit; ++sp) acc += a.t_part[((size_t)sp * a.T + it.tok0 + m) * a.ldt + S.t_col + j];
        return acc;
    };
    if (a.sigma_mode) {   // Sigma-sandwich: stage t rows, then t <- Sigma_a t per row
        for (int c = tid; c < kTcM * k; c += kTcExpThreads) {
            const int m = c / k, j = c % k;
            s.tw[m][j] = t_of(m, j);
        }
        __syncthreads();
    }
    for (int c = tid; c < kTcM * (kpad / 8); c += kTcExpThreads) {
        const int m = c % kTcM, jc = c / kTcM;
        float tv[8];
        if (a.sigma_mode) {
            const float* row = s.tw[m];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int j = jc * 8 + i;
                float acc = 0.f;
                if (m < nt && j < k) {
                    if (a.sigma_mode == 1) {
                        acc = a.sigma[(size_t)it.adapter * k + j] * row[j];
                    } else {
                        const float* Sr = a.sigma + ((size_t)it.adapter * k + j) * k;
                        for (int l = 0; l < k; ++l) acc = fmaf(Sr[l], row[l], acc);
                    }
                }
                tv[i] = acc;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) tv[i] = t_of(m, jc * 8 + i);
        }
        __align__(16) __nv_bfloat16 hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            hi[i] = __float2bfloat16_rn(tv[i]);
            lo[i] = __float2bfloat16_rn(tv[i] - __bfloat162float(hi[i]));
        }
        const uint32_t off = (uint32_t)(m >> 3) * sbo + (uint32_t)jc * 128 + (uint32_t)(m & 7) * 16;
        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(s.ahi) + off) = *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(s.alo) + off) = *reinterpret_cast<const uint4*>(lo);
    }
    if (warp == 0) tc::tmem_alloc(&s.tmem, N2);
    if (tid == 0) {
        mbar_init(&s.bar, 1);
        for (int b2 = 0; b2 < kTcYBuf; ++b2) mbar_init(&s.ybar[b2], 1);
        fence_barrier_init();
    }
    __syncthreads();   // toks visible to the copies below
    bool consecutive = true;
    for (int m = tid; m < nt; m += kTcExpThreads) consecutive = consecutive && s.toks[m] == s.toks[0] + m;
    // uniform: y tiles by TMA
    const bool ytma = __syncthreads_and(consecutive) && y_tma != 0 && (smem_u32(s.yt[0]) & 1023u) == 0;
    int y_issued = 0;   // TMA y tiles issued by thread 0

    const __nv_bfloat16* Bt = S.Bt_pool + ob;
    auto issue_y = [&](int i) {   // y rows of step i -> yt[i % 3]
        const int e0 = e_begin + i * N2;
        char* dst = reinterpret_cast<char*>(s.yt[i % kTcYBuf]);
        if (ytma) {   // rows toks[0] .. +127, columns y_off + e0 .. +127 (a multiple of 8 elements)
            if (tid == 0) {
                tc::bulk_wait_read0();   // the TMA store of the tile this buffer held has read it
                uint64_t* bar = &s.ybar[i % kTcYBuf];
                mbar_arrive_expect_tx(bar, (N2 / 64) * kTcYHalf);
#pragma unroll
                for (int hh = 0; hh < N2 / 64; ++hh)
                    tc::tma_load_2d(dst + hh * kTcYHalf, &ymap, (int)S.y_off + e0 + 64 * hh, s.toks[0], bar);
                ++y_issued;
            }
            return;
        }
        // rows past the tile / columns past the range zero-filled
        for (int c = tid; c < kTcM * (N2 / 8); c += kTcExpThreads) {
            const int row = c / (N2 / 8), ch = c % (N2 / 8);
            const int e = e0 + ch * 8;
            const bool ok = row < nt && e < e_end;
            cp_async16_zfill(dst + ytile_off(row, ch * 8), ok ? ybase + (int64_t)s.toks[row] * a.y_ld + e : ybase, ok);
        }
    };
    auto issue_b = [&](int i) {   // B'^T rows 0..kpad-1 of step i -> b[i % 2], MN-major
        const int e0 = e_begin + i * N2;
        char* dst = reinterpret_cast<char*>(s.b[i & 1]);
        for (int c = tid; c < kpad * (N2 / 8); c += kTcExpThreads) {
            const int j = c / (N2 / 8), nc = c % (N2 / 8);
            const int e = e0 + nc * 8;
            const bool ok = j < k && e < e_end;
            cp_async16_zfill(dst + (uint32_t)nc * sbo + (uint32_t)(j >> 3) * 128 + (uint32_t)(j & 7) * 16,
                             ok ? Bt + (int64_t)j * S.d_out + e : Bt, ok);
        }
    };
    issue_y(0);
    issue_b(0);
    tc::cp_async_commit();
    if (nit > 1) {
        issue_y(1);
        issue_b(1);
    }
    tc::cp_async_commit();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem;
    const uint32_t idesc = tc::idesc_bf16(kTcM, N2, 0, 1);
    const int q = warp & 3, h = warp >> 2;   // TMEM lane quadrant, column half
    const int m = 32 * q + lane;             // tile row of this thread in the epilogue
    bool ok = true;
    for (int i = 0; i < nit && ok; ++i) {
        tc::cp_async_wait<1>();              // step i's y and B tiles (this thread's copies)
        tc::fence_proxy_async();             // B tile -> visible to the tensor core
        if (ytma) ok = mbar_wait(&s.ybar[i % kTcYBuf], (uint32_t)((i / kTcYBuf) & 1));
        ok = __syncthreads_and(ok);
        if (!ok) break;
        if (tid == 0) {
            tc::fence_after_sync();
            const char* bb = reinterpret_cast<const char*>(s.b[i & 1]);
            for (int ks = 0; ks < kpad / 16; ++ks) {
                const uint64_t bd = tc::smem_desc(bb + ks * 256, 128, sbo);
                const uint64_t ah = tc::smem_desc(reinterpret_cast<char*>(s.ahi) + ks * 256, 128, sbo);
                const uint64_t al = tc::smem_desc(reinterpret_cast<char*>(s.alo) + ks * 256, 128, sbo);
                tc::mma_bf16(tmem, ah, bd, idesc, ks > 0);
                tc::mma_bf16(tmem, al, bd, idesc, true);
            }
            tc::commit(&s.bar);
        }
        if (i + 2 < nit) issue_y(i + 2);     // yt[(i+2) % 3] held step i-1, already written back
        ok = mbar_wait(&s.bar, (uint32_t)(i & 1));
        tc::fence_after_sync();
        if (i + 2 < nit) issue_b(i + 2);     // b[i % 2] is free once the MMAs of step i completed
        tc::cp_async_commit();
        __nv_bfloat16* yt = s.yt[i % kTcYBuf];
        if (ok) {
#pragma unroll
            for (int c16 = 0; c16 < N2 / 32; ++c16) {
                float v[16];
                tc::tmem_ld16(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((N2 / 2) * h + 16 * c16), v);
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    uint4* yp = reinterpret_cast<uint4*>(reinterpret_cast<char*>(yt) +
                                                         ytile_off(m, (N2 / 2) * h + 16 * c16 + 8 * half));
                    uint4 yv = *yp;
                    __nv_bfloat162* y2 = reinterpret_cast<__nv_bfloat162*>(&yv);
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const float2 yf = __bfloat1622float2(y2[p]);
                        y2[p] = __floats2bfloat162_rn(fmaf(scale, v[8 * half + 2 * p], yf.x),
                                                      fmaf(scale, v[8 * half + 2 * p + 1], yf.y));
                    }
                    *yp = yv;
                }
            }
        }
        tc::fence_proxy_async();             // staged tile -> visible to a TMA store / next TMA load
        tc::fence_before_sync();
        ok = __syncthreads_and(ok);          // staged tile complete; TMEM free for the next MMA
        if (ok) {
            const int e0 = e_begin + i * N2;
            if (ytma && nt == kTcM && e0 + N2 <= e_end) {   // the whole box is this CTA's
                if (tid == 0) {
                    const char* src = reinterpret_cast<const char*>(yt);
#pragma unroll
                    for (int hh = 0; hh < N2 / 64; ++hh)
                        tc::tma_store_2d(&ymap, (int)S.y_off + e0 + 64 * hh, s.toks[0], src + hh * kTcYHalf);
                    tc::bulk_commit();
                }
            } else {
                for (int c = tid; c < kTcM * (N2 / 8); c += kTcExpThreads) {
                    const int row = c / (N2 / 8), ch = c % (N2 / 8);
                    const int e = e0 + ch * 8;
                    if (row < nt && e < e_end)
                        *reinterpret_cast<uint4*>(ybase + (int64_t)s.toks[row] * a.y_ld + e) =
                            *reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(yt) + ytile_off(row, ch * 8));
                }
                tc::fence_proxy_async();     // reads of the buffer before a later TMA copy refills it
            }
        }
    }
    if (tid == 0 && ytma) {   // nothing of this CTA's TMA traffic is in flight when it leaves
        tc::bulk_wait0();
        for (int j = max(0, y_issued - kTcYBuf); j < y_issued; ++j)
            mbar_wait(&s.ybar[j % kTcYBuf], (uint32_t)((j / kTcYBuf) & 1));
    }
    tc::cp_async_wait<0>();
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    if (warp == 0) tc::tmem_dealloc(tmem, N2);
}

template <int KMAX, int N2>
constexpr size_t expand_tc_smem() { return sizeof(ExpandTcSmem<KMAX, N2>) + 1024; }

}  // namespace lf
