// Multi-LoRA shrink / expand for segments with many tokens, on tcgen05 tensor
// cores (sm_100a).  Same arithmetic contract as the GEMV path: t = A' x kept in
// fp32, y = bf16(y + s * B'^T... ) rounded once ("Compress then Serve",
// academ.us/article/2407.00066, section 13.4 "Punica": fp32 intermediate buffer,
// then the scaled B step into y).  Only the prefill-shaped case is a real dense
// contraction (M = tokens of one adapter), so only it uses the tensor cores.
//
// Shrink: D[128 tokens x N] = X[128 x d_in] * A'^T[d_in x N], bf16 in, fp32 in TMEM,
//   N = k rounded up to 16 (padding lives in shared memory only).  X rows are
//   gathered through the token permutation with 16-byte cp.async into a 4-stage
//   ring of K-major core matrices; one thread issues the MMAs and commits each
//   stage to an mbarrier that frees the stage for the next copy.
// Expand: D[128 x 256] = t_hi * B + t_lo * B with t = t_hi + t_lo split into two
//   bf16 values (about 16 significant bits of the fp32 t); B = B'^T tile,
//   MN-major; the epilogue reads D from tensor memory and updates y once.
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace lf {

constexpr int kTcMin = 64;       // segments with at least this many tokens use the tensor cores
constexpr int kTcM = 128;        // tokens per tile (UMMA M)
constexpr int kTcKB = 64;        // d_in elements per pipeline stage (128 bytes per row)
constexpr int kTcStages = 4;
constexpr int kTcThreads = 128;  // 4 warps: warp w owns tensor-memory lanes 32w .. 32w+31
constexpr int kTcN = 256;        // expand tile width (UMMA N)
constexpr int kTcCols = 2048;    // d_out columns per expand CTA
constexpr int kTcMaxSplit = 8;   // d_in is split over at most this many CTAs per token tile

// d_in elements per split: a multiple of the stage width, at least 1024, at most kTcMaxSplit splits
__host__ __device__ inline int tc_split_len(int d_in) {
    int len = (d_in + kTcMaxSplit - 1) / kTcMaxSplit;
    len = ((len + kTcKB - 1) / kTcKB) * kTcKB;
    return len < 1024 ? 1024 : len;
}

struct TcItem {
    int32_t adapter, k, ntok, tok0;   // tok0: position of the first token in the permutation
    int64_t oa, ob;
};

struct TcArgs {
    int32_t d_in, d_out;
    const __nv_bfloat16* x;
    __nv_bfloat16* y;
    const __nv_bfloat16* A_pool;
    const __nv_bfloat16* Bt_pool;
    float scale;
    const int32_t* counts;   // [3] = number of tensor-core items
    const TcItem* items;
    const int32_t* perm;
    float* t_part;           // kTcMaxSplit x T x kMaxRank fp32 partial sums, row = permutation position
    int32_t T;
};

// ---- shrink ---------------------------------------------------------------
struct ShrinkTcSmem {
    __nv_bfloat16 a[kTcStages][kTcM * kTcKB];       // 16 KB per stage
    __nv_bfloat16 b[kTcStages][kMaxRank * kTcKB];   //  8 KB per stage
    uint64_t bar[kTcStages];
    uint32_t tmem;
    int32_t toks[kTcM];
};

// byte offset of element (row, kk) of a K-major operand tile with 64 K-elements per row
__device__ __forceinline__ uint32_t kmaj64(int row, int kk) {
    return (uint32_t)((row >> 3) * 1024 + (kk >> 3) * 128 + (row & 7) * 16 + (kk & 7) * 2);
}

__device__ __forceinline__ void cp_async16_zfill(void* dst, const void* src, bool valid) {
    const int n = valid ? 16 : 0;   // src-size 0 fills the 16 bytes with zeros
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}

__global__ void __launch_bounds__(kTcThreads) shrink_tc_kernel(TcArgs a) {
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    auto& s = *reinterpret_cast<ShrinkTcSmem*>(tc_raw);
    if ((int)blockIdx.x >= a.counts[3]) return;
    const TcItem it = a.items[blockIdx.x];
    if (it.k <= 0) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = it.k, nt = it.ntok;
    const int npad = (k + 15) & ~15;
    for (int m = tid; m < kTcM; m += kTcThreads) s.toks[m] = m < nt ? a.perm[it.tok0 + m] : 0;
    // rows k..npad-1 of every B stage stay zero (never written by the copies)
    for (int e = tid; e < kTcStages * (npad - k) * kTcKB; e += kTcThreads) {
        const int st = e / ((npad - k) * kTcKB), r2 = e % ((npad - k) * kTcKB);
        const int n = k + r2 / kTcKB, kk = r2 % kTcKB;
        *reinterpret_cast<__nv_bfloat16*>(reinterpret_cast<char*>(s.b[st]) + kmaj64(n, kk)) = __float2bfloat16(0.f);
    }
    if (warp == 0) tc::tmem_alloc(&s.tmem, 64);
    if (tid == 0) {
        for (int i = 0; i < kTcStages; ++i) mbar_init(&s.bar[i], 1);
        fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem;
    const int split = blockIdx.y, slen = tc_split_len(a.d_in);
    const int kbeg = split * slen;
    if (kbeg >= a.d_in) {   // uniform: this split has no columns (before any async work)
        tc::fence_before_sync();
        __syncthreads();
        if (warp == 0) tc::tmem_dealloc(s.tmem, 64);
        return;
    }
    const int kend = min(a.d_in, kbeg + slen);
    const int nK = (kend - kbeg + kTcKB - 1) / kTcKB;
    const __nv_bfloat16* Ap = a.A_pool + it.oa;
    const uint32_t idesc = tc::idesc_bf16(kTcM, npad, 0, 0);

    auto load_stage = [&](int kb, int st) {
        char* abase = reinterpret_cast<char*>(s.a[st]);
        char* bbase = reinterpret_cast<char*>(s.b[st]);
        const int k0 = kbeg + kb * kTcKB;
#pragma unroll
        for (int i = 0; i < (kTcM * kTcKB / 8) / kTcThreads; ++i) {   // 8 chunks per thread
            const int c = tid + i * kTcThreads;
            const int m = c % kTcM, kc = c / kTcM;
            const int kk = k0 + kc * 8;
            const bool ok = m < nt && kk < kend;
            const __nv_bfloat16* src = ok ? a.x + (int64_t)s.toks[m] * a.d_in + kk : a.x;
            cp_async16_zfill(abase + kmaj64(m, kc * 8), src, ok);
        }
        for (int c = tid; c < k * (kTcKB / 8); c += kTcThreads) {
            const int n = c / (kTcKB / 8), kc = c % (kTcKB / 8);
            const int kk = k0 + kc * 8;
            const bool ok = kk < kend;
            const __nv_bfloat16* src = ok ? Ap + (int64_t)n * a.d_in + kk : Ap;
            cp_async16_zfill(bbase + kmaj64(n, kc * 8), src, ok);
        }
    };

    for (int p = 0; p < kTcStages - 1; ++p) {
        if (p < nK) load_stage(p, p);
        tc::cp_async_commit();
    }
    bool ok = true;
    for (int kb = 0; kb < nK && ok; ++kb) {
        const int nxt = kb + kTcStages - 1;
        if (nxt < nK) {
            const int st = nxt % kTcStages;
            if (nxt >= kTcStages) ok = mbar_wait(&s.bar[st], (uint32_t)((nxt / kTcStages - 1) & 1));
            if (ok) load_stage(nxt, st);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<kTcStages - 1>();
        tc::fence_proxy_async();
        ok = __syncthreads_and(ok);   // block-uniform: a timed-out wait stops every thread
        if (!ok) break;
        if (tid == 0) {
            tc::fence_after_sync();
            const int st = kb % kTcStages;
#pragma unroll
            for (int ks = 0; ks < kTcKB / 16; ++ks) {
                const uint64_t ad = tc::smem_desc(reinterpret_cast<char*>(s.a[st]) + ks * 256, 128, 1024);
                const uint64_t bd = tc::smem_desc(reinterpret_cast<char*>(s.b[st]) + ks * 256, 128, 1024);
                tc::mma_bf16(tmem, ad, bd, idesc, kb > 0 || ks > 0);
            }
            tc::commit(&s.bar[st]);
        }
    }
    tc::cp_async_wait<0>();
    if (ok) {
        const int last = nK - 1;
        ok = mbar_wait(&s.bar[last % kTcStages], (uint32_t)((last / kTcStages) & 1));
    }
    ok = __syncthreads_and(ok);
    tc::fence_after_sync();
    if (ok) {
        const int m = warp * 32 + lane;
        float* trow = a.t_part + ((size_t)split * a.T + it.tok0 + m) * kMaxRank;
        for (int c0 = 0; c0 < npad; c0 += 16) {
            float v[16];
            tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)c0, v);
            if (m < nt) {
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    if (c0 + i < k) trow[c0 + i] = v[i];
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 0) tc::tmem_dealloc(tmem, 64);
}

constexpr size_t kShrinkTcSmem = sizeof(ShrinkTcSmem) + 1024;

// ---- expand ---------------------------------------------------------------
constexpr int kTcStageLd = 68;   // 64 columns + 4: rows stay 16-byte aligned, 4-bank shift per row
struct ExpandTcSmem {
    __nv_bfloat16 ahi[kTcM * kMaxRank];   // t_hi, K-major, 16 KB
    __nv_bfloat16 alo[kTcM * kMaxRank];   // t_lo
    __nv_bfloat16 b[kMaxRank * kTcN];     // B'^T tile, MN-major, 32 KB
    float stage[kTcThreads / 32][32][kTcStageLd];   // per-warp accumulator transpose, 34 KB
    uint64_t bar;
    uint32_t tmem;
    int32_t toks[kTcM];
};

__global__ void __launch_bounds__(kTcThreads) expand_tc_kernel(TcArgs a) {
    extern __shared__ __align__(1024) unsigned char tc_raw[];
    auto& s = *reinterpret_cast<ExpandTcSmem*>(tc_raw);
    if ((int)blockIdx.x >= a.counts[3]) return;
    const TcItem it = a.items[blockIdx.x];
    if (it.k <= 0) return;
    const int e_begin = blockIdx.y * kTcCols;
    if (e_begin >= a.d_out) return;
    const int e_end = min(a.d_out, e_begin + kTcCols);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int k = it.k, nt = it.ntok;
    const int kpad = (k + 15) & ~15;
    const uint32_t sbo_a = (uint32_t)(kpad / 8) * 128;   // 8-row groups of the K-major t tiles
    const uint32_t sbo_b = (uint32_t)(kpad / 8) * 128;   // 8-column groups of the MN-major B tile
    for (int m = tid; m < kTcM; m += kTcThreads) s.toks[m] = m < nt ? a.perm[it.tok0 + m] : 0;
    // t tile -> (t_hi, t_lo) bf16, K-major: element (m, j) at (m/8)*sbo_a + (j/8)*128 + (m%8)*16 + (j%8)*2
    for (int c = tid; c < kTcM * (kpad / 8); c += kTcThreads) {
        const int m = c % kTcM, jc = c / kTcM;
        float tv[8];
        const int nsplit = (a.d_in + tc_split_len(a.d_in) - 1) / tc_split_len(a.d_in);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int j = jc * 8 + i;
            float acc = 0.f;
            if (m < nt && j < k)
                for (int sp = 0; sp < nsplit; ++sp)   // fixed order: bitwise reproducible
                    acc += a.t_part[((size_t)sp * a.T + it.tok0 + m) * kMaxRank + j];
            tv[i] = acc;
        }
        __align__(16) __nv_bfloat16 hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            hi[i] = __float2bfloat16_rn(tv[i]);
            lo[i] = __float2bfloat16_rn(tv[i] - __bfloat162float(hi[i]));
        }
        const uint32_t off = (uint32_t)(m >> 3) * sbo_a + (uint32_t)jc * 128 + (uint32_t)(m & 7) * 16;
        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(s.ahi) + off) = *reinterpret_cast<const uint4*>(hi);
        *reinterpret_cast<uint4*>(reinterpret_cast<char*>(s.alo) + off) = *reinterpret_cast<const uint4*>(lo);
    }
    if (warp == 0) tc::tmem_alloc(&s.tmem, kTcN);
    if (tid == 0) {
        mbar_init(&s.bar, 1);
        fence_barrier_init();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem;
    const uint32_t idesc = tc::idesc_bf16(kTcM, kTcN, 0, 1);
    const __nv_bfloat16* Bt = a.Bt_pool + it.ob;
    bool ok = true;
    int phase = 0;
    for (int e0 = e_begin; e0 < e_end && ok; e0 += kTcN, ++phase) {
        // B tile: element (j, n) = B'^T[j][e0 + n] at (n/8)*sbo_b + (j/8)*128 + (j%8)*16 + (n%8)*2
        for (int c = tid; c < kpad * (kTcN / 8); c += kTcThreads) {
            const int j = c / (kTcN / 8), nc = c % (kTcN / 8);
            const int e = e0 + nc * 8;
            const bool valid = j < k && e < e_end;
            const __nv_bfloat16* src = valid ? Bt + (int64_t)j * a.d_out + e : Bt;
            cp_async16_zfill(reinterpret_cast<char*>(s.b) + (uint32_t)nc * sbo_b + (uint32_t)(j >> 3) * 128 +
                                 (uint32_t)(j & 7) * 16,
                             src, valid);
        }
        tc::cp_async_commit();
        tc::cp_async_wait<0>();
        tc::fence_proxy_async();
        __syncthreads();
        if (tid == 0) {
            tc::fence_after_sync();
            for (int ks = 0; ks < kpad / 16; ++ks) {
                const uint64_t bd = tc::smem_desc(reinterpret_cast<char*>(s.b) + ks * 256, 128, sbo_b);
                const uint64_t ah = tc::smem_desc(reinterpret_cast<char*>(s.ahi) + ks * 256, 128, sbo_a);
                const uint64_t al = tc::smem_desc(reinterpret_cast<char*>(s.alo) + ks * 256, 128, sbo_a);
                tc::mma_bf16(tmem, ah, bd, idesc, ks > 0);
                tc::mma_bf16(tmem, al, bd, idesc, true);
            }
            tc::commit(&s.bar);
        }
        // y for this warp's 32 token rows, loaded while the MMAs run, in the coalesced
        // mapping of the epilogue: iteration i covers rows 4*(i%8) + lane/8 of column
        // block i/8, eight lanes per 128-byte row segment
        const int cl = (lane & 7) * 8;   // column offset of this lane inside a 64-column block
        uint4 yv[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            const int rr = warp * 32 + 4 * (i & 7) + (lane >> 3);
            const int e = e0 + 64 * (i >> 3) + cl;
            yv[i] = (rr < nt && e < e_end)
                        ? *reinterpret_cast<const uint4*>(a.y + (int64_t)s.toks[rr] * a.d_out + e)
                        : make_uint4(0, 0, 0, 0);
        }
        ok = mbar_wait(&s.bar, (uint32_t)(phase & 1));
        tc::fence_after_sync();
        if (ok) {
            float (*st)[kTcStageLd] = s.stage[warp];
#pragma unroll
            for (int blk = 0; blk < kTcN / 64; ++blk) {
                // accumulator rows (one per lane) of this 64-column block -> shared memory
#pragma unroll
                for (int c16 = 0; c16 < 4; ++c16) {
                    float v[16];
                    tc::tmem_ld16(tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)(blk * 64 + c16 * 16), v);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        *reinterpret_cast<float4*>(&st[lane][c16 * 16 + 4 * q]) =
                            make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
                }
                __syncwarp();
#pragma unroll
                for (int i8 = 0; i8 < 8; ++i8) {
                    const int i = blk * 8 + i8;
                    const int rl = 4 * i8 + (lane >> 3);   // row inside the warp's 32
                    const int rr = warp * 32 + rl;
                    const int e = e0 + 64 * blk + cl;
                    const float4 p0 = *reinterpret_cast<const float4*>(&st[rl][cl]);
                    const float4 p1 = *reinterpret_cast<const float4*>(&st[rl][cl + 4]);
                    const float acc[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
                    __nv_bfloat162* p2 = reinterpret_cast<__nv_bfloat162*>(&yv[i]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 yf = __bfloat1622float2(p2[q]);
                        p2[q] = __floats2bfloat162_rn(fmaf(a.scale, acc[2 * q], yf.x), fmaf(a.scale, acc[2 * q + 1], yf.y));
                    }
                    if (rr < nt && e < e_end)
                        *reinterpret_cast<uint4*>(a.y + (int64_t)s.toks[rr] * a.d_out + e) = yv[i];
                }
                __syncwarp();
            }
        }
        tc::fence_before_sync();
        ok = __syncthreads_and(ok);   // B tile and tensor memory free for the next tile; uniform ok
    }
    if (warp == 0) tc::tmem_dealloc(tmem, kTcN);
}

constexpr size_t kExpandTcSmem = sizeof(ExpandTcSmem) + 1024;

}  // namespace lf
