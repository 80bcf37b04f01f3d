// TSQR leaf by an exact integer Gram on the tcgen05 tensor cores (kind::i8).
//
// LoRAForge (kongchang.com), "FlashTSQR: An Accelerator for Batched Factor
// Construction": R of each tall-skinny factor comes from local work on row blocks
// followed by a merge, parallel across modules and row blocks.  As in the fp64 Gram
// leaf (gram.cuh), the local product of a row block X_c is its Gram matrix, the merge
// is the fixed-order sum of the Grams and the root is R = chol(G), the unique
// upper-triangular factor with positive diagonal (R^T R = X^T X).
//
// What this leaf computes.  Every column j of a work item (up to kI8MaxRows rows of
// one factor) gets a power-of-two scale 2^E_j above its largest magnitude (taken on
// the item's first 128 rows with kI8HeadBits bits of headroom); each value becomes the
// 32-bit fixed-point integer N = trunc(x 2^(31 - E_j)), so x~ = N 2^(E_j - 31) differs
// from x by less than 2^(E_j - 31) (about 2^-27 of the column's largest value, finer
// than the fp32 input itself for most entries).  The four bytes of U = N + 2^31 are
// unsigned 8-bit digits b3..b0 (b3 - 128 is the signed top digit), and
//     X~^T X~ = sum over digit pairs (s, t) of 2^(8(s+t)) Bhat_s^T Bhat_t,
// every Bhat_s^T Bhat_t an integer matrix that the int8 tensor cores form exactly in
// int32.  The Gram of X~ is therefore exact up to the final fp64 roundings, so R is
// the R of X~ to ~1e-16 kappa^2, i.e. the leaf is backward stable with a columnwise
// backward error below 2^-27 of the column maximum.  A value at or above 2^E_j (or a
// non-finite one) marks the matrix for the fp64 leaf instead, as does a matrix whose
// rows the bulk copies cannot address (row or offset not 16-byte aligned).
//
// Data flow per CTA (persistent, one per SM, static round-robin over the work items,
// longest first):
//   warp 0        producer: 1-D bulk copies (cp.async.bulk, no multicast) of 64-row
//                 fp32 stages into a kI8FStages ring (B: one contiguous block; A^T:
//                 one 256-byte run per column), completion counted in bytes;
//   warp 1        MMA issuer (one thread): per 128-row digit stage, D1 += [P3;P2] x
//                 [P3;P2;P1;P0]^T (M 128, N 256) and D2 += [P1;P0] x [P1;P0]^T (M 128,
//                 N 128) in four K = 32 steps each, into 384 TMEM columns;
//   warps 2..9    converters: column scales, fp32 -> digit planes (K-major, 128-byte
//                 swizzle, plane p = byte 3 - p) and the planes' column sums;
//   warps 10..13  epilogue: int32 accumulators -> signed-digit corrections ->
//                 fp64 Gram (packed upper triangle) -> fp64 Cholesky -> R.
// The 16 digit-pair products of a column pair live in two TMEM lanes (a column's
// planes 0 and 2 in lane i, planes 1 and 3 in lane 64 + i) and, for four of the pairs,
// in the transposed position; the epilogue combines them through shared memory in a
// fixed order, so the result does not depend on scheduling.  Converters hand the fp32
// stages back as soon as their values are in registers, so the ring keeps up to six
// 16 KB stages of the producer's copies in flight.
#pragma once
#include <float.h>

#include "common.cuh"
#include "gram.cuh"
#include "tc.cuh"

namespace lf {

constexpr int kI8Rows = 128;         // rows (the MMA's K) per digit stage
constexpr int kI8FRows = 64;         // rows per fp32 stage (two per digit stage)
constexpr int kI8FStages = 6;
constexpr int kI8DStages = 2;
constexpr int kI8ConvWarps = 8;
constexpr int kI8EpiWarps = 4;
constexpr int kI8ConvWarp0 = 2;
constexpr int kI8EpiWarp0 = kI8ConvWarp0 + kI8ConvWarps;       // 10
constexpr int kI8Threads = 32 * (kI8EpiWarp0 + kI8EpiWarps);   // 448
constexpr int kI8HeadBits = 2;       // 2^E is 4x to 8x the largest value of the first 128 rows
// Rows per work item: the largest accumulator, 255^2 * rows, stays below 2^31, and the
// corrected top-digit product times 2^24 stays below 2^53 (exact in fp64).
constexpr int kI8MaxRows = 24576;
constexpr int kI8LdS = 65;           // fp64 row stride of the epilogue's row buffers
constexpr int kI8LdA = 68;           // fp32 column stride of an A^T stage (64 rows + 4)
constexpr int kI8FStageFloats = kI8LdA * kI8FRows;
constexpr uint32_t kI8TmemCols = 512;

struct GramI8Meta {
    int32_t colsum[4][64];   // column sums of the digit planes over the item (plane 0 = top byte)
    int32_t E[64];           // column exponents: every |x| of the column is below 2^E
    int32_t ovf;             // a value reached 2^E, or was not finite
};

struct GramI8Smem {
    uint8_t dig[kI8DStages][256 * 128];     // digit stages: 4 planes x 64 columns x 128 rows (first: 1024-aligned)
    float f32[kI8FStages][kI8FStageFloats];
    double W[64 * kI8LdS];                  // fp64 rows: lanes i and 64 + i of the accumulators, summed
    double G[tri_size<64>()];               // packed Gram of a one-item matrix, then its Cholesky factor
    double diag[64];
    uint16_t kc[tri_size<64>()];            // packed index -> (row << 8) | column
    GramI8Meta meta[2];
    float cmax[4][64];
    uint64_t full_f[kI8FStages], empty_f[kI8FStages];
    uint64_t full_d[kI8DStages], empty_d[kI8DStages];
    uint64_t acc_full, acc_empty, drain;
    uint64_t meta_full[2], meta_empty[2];
    uint32_t tmem;
    int abort;
    int flag;
    int redo;
};

constexpr size_t gram_i8_smem() { return sizeof(GramI8Smem) + 1024; }

struct GramI8Args {
    const lf_module* mods;
    const float* B_base;
    const float* A_base;
    const TsqrWork* work;      // work items of <= kI8MaxRows rows, longest first
    int32_t n_work;
    const TsqrInfo* info;      // per mf: items of the matrix and its first partial slot
    int32_t* counters;         // per mf, zero on entry
    double* partial;           // slot s: packed Gram (tri_size<RT> doubles) of one item
    int32_t* fb;               // per mf: set to 1 when the matrix is left to the fp64 leaf
    int32_t* flags;            // per mf: set to 1 when the Cholesky rejects a pivot
    float* R_B;
    float* R_A;
    int32_t rs;
};

// Barrier among `nthreads` threads on hardware barrier `id` that also ANDs a predicate:
// every participant gets the same answer.
__device__ __forceinline__ bool named_and(int id, int nthreads, bool v) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\tbar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return out != 0;
}

// The four digit-plane words of four consecutive rows: word p holds byte 3 - p of
// u[0..3] (row order = byte order, lowest row in the lowest byte).
__device__ __forceinline__ void planes4(const uint32_t (&u)[4], uint32_t (&w)[4]) {
    const uint32_t hi01 = __byte_perm(u[0], u[1], 0x7362), lo01 = __byte_perm(u[0], u[1], 0x5140);
    const uint32_t hi23 = __byte_perm(u[2], u[3], 0x7362), lo23 = __byte_perm(u[2], u[3], 0x5140);
    w[0] = __byte_perm(hi01, hi23, 0x7632);
    w[1] = __byte_perm(hi01, hi23, 0x5410);
    w[2] = __byte_perm(lo01, lo23, 0x7632);
    w[3] = __byte_perm(lo01, lo23, 0x5410);
}

// 16 values of column c, rows 16 * qs .. 16 * qs + 15 of an fp32 stage (qs in 0..3);
// rows at or past `nvalid` and columns at or past r read as zero.
__device__ __forceinline__ void i8_load_unit(float (&x)[16], const float* st, int factor, int c, int qs, int r,
                                             int nvalid) {
    if (c >= r) {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = 0.f;
        return;
    }
    if (factor == 0) {   // B stage: row-major, row stride r
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = e < nvalid ? st[(16 * qs + e) * r + c] : 0.f;
    } else {             // A^T stage: column c at c * kI8LdA, rows contiguous
        const float4* p = reinterpret_cast<const float4*>(st + c * kI8LdA + 16 * qs);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const float4 f = p[v];
            x[4 * v + 0] = 4 * v + 0 < nvalid ? f.x : 0.f;
            x[4 * v + 1] = 4 * v + 1 < nvalid ? f.y : 0.f;
            x[4 * v + 2] = 4 * v + 2 < nvalid ? f.z : 0.f;
            x[4 * v + 3] = 4 * v + 3 < nvalid ? f.w : 0.f;
        }
    }
}

// Right-looking Cholesky of the packed Gram G (r x r used, packed for RT columns) by the
// 128 epilogue threads: per column j the pivot test (d_j <= kGramPivotTol G_jj rejects, as
// in the fp64 leaf), row j divided by r_jj, then the trailing triangle (packed entries
// from (j+1, j+1) on, each updated by one thread) less the outer product of row j.
// Returns false (for every thread alike) when a pivot is rejected.
template <int RT>
__device__ __forceinline__ bool i8_cholesky(double* G, double* diag, const uint16_t* kc, int r, int et) {
    constexpr int TRI = tri_size<RT>();
    constexpr int NT = 32 * kI8EpiWarps;
    for (int j = et; j < r; j += NT) diag[j] = G[tri_off<RT>(j, j)];
    tc::named_sync(2, NT);
    for (int j = 0; j < r; ++j) {
        const double d = G[tri_off<RT>(j, j)];
        if (!(d > kGramPivotTol * diag[j])) return false;
        const double rjj = sqrt(d);
        for (int c = j + 1 + et; c < r; c += NT) G[tri_off<RT>(j, c)] /= rjj;
        tc::named_sync(2, NT);
        if (et == 0) G[tri_off<RT>(j, j)] = rjj;
        const double* rowj = G + tri_off<RT>(j, j) - j;   // rowj[c] = G[j][c] for c >= j
        for (int e = (j + 1 < RT ? tri_off<RT>(j + 1, j + 1) : TRI) + et; e < TRI; e += NT) {
            const int k = kc[e] >> 8, c = kc[e] & 255;
            if (c < r) G[e] -= rowj[k] * rowj[c];
        }
        tc::named_sync(2, NT);
    }
    return true;
}

template <int RT>
__global__ void __launch_bounds__(kI8Threads, 1) gram_i8_kernel(GramI8Args a) {
    extern __shared__ __align__(1024) unsigned char i8_raw[];
    GramI8Smem& s = *reinterpret_cast<GramI8Smem*>(i8_raw + ((1024u - (smem_u32(i8_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int i = 0; i < kI8FStages; ++i) {
            mbar_init(&s.full_f[i], 1);
            mbar_init(&s.empty_f[i], kI8ConvWarps);
        }
        for (int i = 0; i < kI8DStages; ++i) {
            mbar_init(&s.full_d[i], kI8ConvWarps);
            mbar_init(&s.empty_d[i], 1);
        }
        mbar_init(&s.acc_full, 1);
        mbar_init(&s.acc_empty, kI8EpiWarps);
        mbar_init(&s.drain, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.meta_full[i], kI8ConvWarps);
            mbar_init(&s.meta_empty[i], kI8EpiWarps);
        }
        s.abort = 0;
        fence_barrier_init();
    }
    for (int rr = 0, e0 = 0; rr < RT; e0 += RT - rr, ++rr)
        for (int cc = rr + tid; cc < RT; cc += kI8Threads) s.kc[e0 + cc - rr] = (uint16_t)((rr << 8) | cc);
    if (warp == 1) tc::tmem_alloc(&s.tmem, kI8TmemCols);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = s.tmem;
    volatile int* abort_flag = &s.abort;
    // every wait is bounded; the first that runs out stops every role of the CTA
    auto wait = [&](uint64_t* bar, uint32_t parity) -> bool {
        if (*abort_flag) return false;
        if (mbar_wait(bar, parity)) return true;
        *abort_flag = 1;
        return false;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        int g = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < a.n_work && ok; it += gridDim.x) {
            const TsqrWork w = a.work[it];
            const int factor = w.mf & 1;
            const lf_module md = a.mods[w.mf >> 1];
            const int r = md.r;
            const float* X = factor == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
            const int nf = 2 * (int)cdiv(w.nrows, kI8Rows);
            for (int f = 0; f < nf; ++f, ++g) {
                const int slot = g % kI8FStages;
                if (g >= kI8FStages) ok = wait(&s.empty_f[slot], (uint32_t)((g / kI8FStages - 1) & 1));
                if (!ok) break;
                const int rows = max(0, min(kI8FRows, w.nrows - kI8FRows * f));
                const uint32_t bytes = (uint32_t)rows * (uint32_t)r * 4u;
                if (lane == 0) {
                    if (bytes) mbar_arrive_expect_tx(&s.full_f[slot], bytes);
                    else mbar_arrive1(&s.full_f[slot]);
                }
                __syncwarp();
                if (bytes) {
                    const int64_t row = (int64_t)w.row0 + (int64_t)kI8FRows * f;
                    if (factor == 0) {
                        if (lane == 0) bulk_g2s(s.f32[slot], X + row * r, bytes, &s.full_f[slot]);
                    } else {
                        for (int c = lane; c < r; c += 32)
                            bulk_g2s(s.f32[slot] + c * kI8LdA, X + (int64_t)c * md.d_in + row, (uint32_t)rows * 4u,
                                     &s.full_f[slot]);
                    }
                }
            }
        }
        // no bulk copy of this warp may still be writing shared memory when the CTA
        // leaves (on the normal path these phases completed before their conversion)
        for (int q = max(0, g - kI8FStages); q < g; ++q)
            mbar_wait(&s.full_f[q % kI8FStages], (uint32_t)((q / kI8FStages) & 1));
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t id1 = tc::idesc_u8(128, 256), id2 = tc::idesc_u8(128, 128);
            int gd = 0, k = 0;
            bool ok = true;
            for (int it = blockIdx.x; it < a.n_work && ok; it += gridDim.x, ++k) {
                const TsqrWork w = a.work[it];
                const int nd = (int)cdiv(w.nrows, kI8Rows);
                if (k >= 1) ok = wait(&s.acc_empty, (uint32_t)((k - 1) & 1));
                if (!ok) break;
                tc::fence_after_sync();
                for (int ds = 0; ds < nd; ++ds, ++gd) {
                    const int slot = gd % kI8DStages;
                    ok = wait(&s.full_d[slot], (uint32_t)((gd / kI8DStages) & 1));
                    if (!ok) break;
                    tc::fence_after_sync();
                    const char* base = reinterpret_cast<const char*>(s.dig[slot]);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // planes 0, 1 (rows 0..127) x planes 0..3
                        const uint64_t d = tc::smem_desc_sw128(base + 32 * q);
                        tc::mma_i8(tmem, d, d, id1, ds > 0 || q > 0);
                    }
#pragma unroll
                    for (int q = 0; q < 4; ++q) {   // planes 2, 3 x planes 2, 3
                        const uint64_t d = tc::smem_desc_sw128(base + 128 * 128 + 32 * q);
                        tc::mma_i8(tmem + 256, d, d, id2, ds > 0 || q > 0);
                    }
                    tc::commit(&s.empty_d[slot]);
                }
                if (!ok) break;
                tc::commit(&s.acc_full);
            }
            // every MMA issued above has completed before the tensor memory is freed
            tc::commit(&s.drain);
            mbar_wait(&s.drain, 0);
        }
        __syncwarp();
    } else if (warp < kI8EpiWarp0) {
        // ---------------------------------------------------------- converters
        const int cw = warp - kI8ConvWarp0;
        const int ct = tid - 32 * kI8ConvWarp0;
        int g = 0, gd = 0, k = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < a.n_work && ok; it += gridDim.x, ++k) {
            const TsqrWork w = a.work[it];
            const int factor = w.mf & 1;
            const int r = a.mods[w.mf >> 1].r;
            const int nd = (int)cdiv(w.nrows, kI8Rows);
            const int ms = k & 1;
            if (k >= 2) ok = wait(&s.meta_empty[ms], (uint32_t)(((k >> 1) - 1) & 1));
            ok = named_and(1, 32 * kI8ConvWarps, ok);
            if (!ok) break;
            GramI8Meta& M = s.meta[ms];
            // this thread's column and its two 16-row chunks (q0 and q0 + 4) of every
            // digit stage: B stages are read across columns (one row per load), A^T
            // stages across chunks of 8 columns (16-byte loads, conflict-free at stride 68)
            const int c = factor == 0 ? 32 * (cw & 1) + lane : 8 * cw + (lane & 7);
            const int q0 = factor == 0 ? (cw >> 1) : (lane >> 3);
            for (int e = ct; e < 4 * 64; e += 32 * kI8ConvWarps) (&M.colsum[0][0])[e] = 0;
            if (ct == 0) M.ovf = 0;
            uint32_t cs[4] = {0u, 0u, 0u, 0u};
            bool vok = true;
            float mult = 0.f, lim = 0.f;
            for (int ds = 0; ds < nd; ++ds, g += 2, ++gd) {
                const int f0 = g % kI8FStages, f1 = (g + 1) % kI8FStages;
                ok = wait(&s.full_f[f0], (uint32_t)((g / kI8FStages) & 1)) &&
                     wait(&s.full_f[f1], (uint32_t)(((g + 1) / kI8FStages) & 1));
                ok = named_and(1, 32 * kI8ConvWarps, ok);
                if (!ok) break;
                const int rbase = kI8Rows * ds;
                // this thread's two 16-row chunks into registers, then the fp32 stages go
                // back to the producer before any conversion work
                float xv[2][16];
                i8_load_unit(xv[0], s.f32[f0], factor, c, q0, r, w.nrows - rbase - 16 * q0);
                i8_load_unit(xv[1], s.f32[f1], factor, c, q0, r, w.nrows - rbase - 16 * (q0 + 4));
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive1(&s.empty_f[f0]);
                    mbar_arrive1(&s.empty_f[f1]);
                }
                if (ds == 0) {
                    // column exponents from the item's first 128 rows
                    float mx = 0.f;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(xv[h][e]));
                    s.cmax[q0][c] = mx;
                    tc::named_sync(1, 32 * kI8ConvWarps);
                    const float m = fmaxf(fmaxf(s.cmax[0][c], s.cmax[1][c]), fmaxf(s.cmax[2][c], s.cmax[3][c]));
                    int E = -90;   // an all-zero start: any nonzero value later overflows the scale
                    if (m > 0.f && m <= FLT_MAX) {
                        int e2;
                        frexpf(m, &e2);   // m < 2^e2
                        E = e2 + kI8HeadBits;
                    }
                    if (E > 127 || E < -96) {   // outside the fp32 powers of two used below: fp64 leaf
                        vok = false;
                        E = E > 127 ? 127 : -96;
                    }
                    mult = __int_as_float((158 - E) << 23);   // 2^(31 - E)
                    lim = __int_as_float((127 + E) << 23);    // 2^E
                    if (q0 == 0) M.E[c] = E;
                    tc::named_sync(1, 32 * kI8ConvWarps);     // cmax is rewritten by the next item
                }
                if (gd >= kI8DStages) ok = wait(&s.empty_d[gd % kI8DStages], (uint32_t)((gd / kI8DStages - 1) & 1));
                ok = named_and(1, 32 * kI8ConvWarps, ok);
                if (!ok) break;
                uint8_t* dig = s.dig[gd % kI8DStages];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int q = q0 + 4 * h;   // chunk: rows 16q .. 16q + 15 of the digit stage
                    uint32_t pw[4][4];
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {
                        uint32_t u[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float x = xv[h][4 * j4 + e];
                            vok = vok && fabsf(x) < lim;   // false for NaN as well
                            u[e] = (uint32_t)__float2int_rz(x * mult) ^ 0x80000000u;
                        }
                        uint32_t wd[4];
                        planes4(u, wd);
#pragma unroll
                        for (int p = 0; p < 4; ++p) {
                            pw[p][j4] = wd[p];
                            cs[p] = __dp4a(wd[p], 0x01010101u, cs[p]);
                        }
                    }
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        const int R = 64 * p + c;   // operand row (plane p, column c), 128 bytes
                        *reinterpret_cast<uint4*>(dig + R * 128 + ((q ^ (R & 7)) << 4)) =
                            make_uint4(pw[p][0], pw[p][1], pw[p][2], pw[p][3]);
                    }
                }
                tc::fence_proxy_async();   // the digit planes, to the tensor core's proxy
                __syncwarp();
                if (lane == 0) mbar_arrive1(&s.full_d[gd % kI8DStages]);
            }
            if (!ok) break;
#pragma unroll
            for (int p = 0; p < 4; ++p) atomicAdd(&M.colsum[p][c], (int)cs[p]);
            if (!vok) M.ovf = 1;
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.meta_full[ms]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = tid - 32 * kI8EpiWarp0;   // 0..127
        const int lq = warp & 3;                 // the TMEM lane quarter this warp may read
        const int m = 32 * lq + lane;            // accumulator row
        const bool hi = m >= 64;                 // planes 1 and 3 of column i (else planes 0 and 2)
        const int i = m & 63;
        constexpr int TRI = tri_size<RT>();
        int k = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < a.n_work && ok; it += gridDim.x, ++k) {
            const TsqrWork w = a.work[it];
            const int mf = w.mf, factor = mf & 1;
            const int r = a.mods[mf >> 1].r;
            const int nch = a.info[mf].nchunks;
            const int64_t Krows = (int64_t)cdiv(w.nrows, kI8Rows) * kI8Rows;   // zero rows included
            const int ms = k & 1;
            ok = wait(&s.acc_full, (uint32_t)(k & 1)) && wait(&s.meta_full[ms], (uint32_t)((k >> 1) & 1));
            ok = named_and(2, 32 * kI8EpiWarps, ok);
            if (!ok) break;
            tc::fence_after_sync();
            const GramI8Meta& M = s.meta[ms];
            // row i of this lane's products -> fp64 (exact integer combination, then at
            // most two roundings); D1 columns 0..255: column planes 0..3 (byte 3..0);
            // D2 columns 256..383: column planes 2, 3.  Lanes 0..63 (planes 0 and 2 of
            // column i) store W[i][j]; after a barrier lanes 64..127 (planes 1 and 3) add
            // theirs, so W = V1 + V2 in a fixed order.
            double* Wrow = s.W + i * kI8LdS;
            const int64_t Si0 = M.colsum[0][i], Si1 = M.colsum[1][i];
            const uint32_t tb = tmem + ((uint32_t)(32 * lq) << 16);
            for (int pass = 0; pass < 2; ++pass) {
                if (pass == 1) tc::named_sync(2, 32 * kI8EpiWarps);
                if ((int)hi != pass) continue;
                for (int jb = 0; jb < 8; ++jb) {
                    const uint32_t ta[6] = {tb + 8 * jb, tb + 64 + 8 * jb, tb + 128 + 8 * jb,
                                            tb + 192 + 8 * jb, tb + 256 + 8 * jb, tb + 320 + 8 * jb};
                    int32_t v[48];
                    tc::tmem_ld8x6(ta, v);
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const int j = 8 * jb + jj;
                        const int64_t p0 = v[jj], p1 = v[8 + jj], p2 = v[16 + jj], p3 = v[24 + jj];
                        const int64_t p4 = v[32 + jj], p5 = v[40 + jj];
                        double H, L;
                        if (!hi) {
                            // row plane 0 (top digit, signed as b3 - 128) and row plane 2
                            const int64_t q33 = p0 - 128 * (Si0 + M.colsum[0][j]) + 16384 * Krows;
                            const int64_t q32 = p1 - 128 * (int64_t)M.colsum[1][j];
                            const int64_t q31 = p2 - 128 * (int64_t)M.colsum[2][j];
                            const int64_t q30 = p3 - 128 * (int64_t)M.colsum[3][j];
                            H = (double)(q33 * (1ll << 24) + q32 * (1ll << 16) + q31 * (1ll << 8) + q30) * 0x1p24 +
                                (double)(p4 * (1ll << 8) + p5) * 0x1p8;
                            L = (double)(q31 * (1ll << 8) + q30) * 0x1p24;
                        } else {
                            // row plane 1 and row plane 3
                            const int64_t q23 = p0 - 128 * Si1;
                            H = (double)(q23 * (1ll << 24) + p1 * (1ll << 16) + p2 * (1ll << 8) + p3) * 0x1p16 +
                                (double)(p4 * (1ll << 8) + p5);
                            L = (double)(p2 * (1ll << 8) + p3) * 0x1p16;
                        }
                        const double V = j > i ? H : (j < i ? L : H + L);
                        Wrow[j] = hi ? Wrow[j] + V : V;
                    }
                }
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.acc_empty);   // the next item's MMAs may overwrite D
            tc::named_sync(2, 32 * kI8EpiWarps);
            // packed upper triangle: G_ab = 2^(E_a + E_b - 62) (W_ab + W_ba)
            double* dst = nch > 1 ? a.partial + (int64_t)w.slot * TRI : s.G;
            for (int ra = 0; ra < RT; ++ra) {
                const int cb = ra + et;
                if (cb < RT) {
                    double gv = 0.0;
                    if (ra < r && cb < r) {
                        gv = ra == cb ? s.W[ra * kI8LdS + ra] : s.W[ra * kI8LdS + cb] + s.W[cb * kI8LdS + ra];
                        // times 2^(E_a + E_b - 62), exact (E in [-96, 127])
                        gv *= __longlong_as_double((long long)(M.E[ra] + M.E[cb] - 62 + 1023) << 52);
                    }
                    dst[tri_off<RT>(ra, cb)] = gv;
                }
            }
            const int ovf = M.ovf;
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.meta_empty[ms]);
            bool redo;
            if (nch > 1) {
                __threadfence();
                tc::named_sync(2, 32 * kI8EpiWarps);
                if (et == 0) {
                    if (ovf) atomicExch(&a.fb[mf], 1);
                    __threadfence();
                    s.flag = atomicAdd(&a.counters[mf], 1) == nch - 1;
                    if (s.flag) {
                        __threadfence();
                        s.redo = __ldcg(&a.fb[mf]) != 0;   // any item of the matrix overflowed
                    }
                }
                tc::named_sync(2, 32 * kI8EpiWarps);
                if (!s.flag) continue;   // uniform: another CTA merges this matrix
                redo = s.redo != 0;
                __threadfence();
                const double* P0 = a.partial + (int64_t)a.info[mf].slot0 * TRI;
                for (int e = et; !redo && e < TRI; e += 32 * kI8EpiWarps) {
                    double acc = __ldcg(P0 + e);
                    for (int cI = 1; cI < nch; ++cI) acc += __ldcg(P0 + (int64_t)cI * TRI + e);
                    s.G[e] = acc;
                }
            } else {
                if (ovf && et == 0) a.fb[mf] = 1;
                redo = ovf != 0;
            }
            tc::named_sync(2, 32 * kI8EpiWarps);
            if (redo) continue;   // uniform: the fp64 leaf factors this matrix
            const bool good = i8_cholesky<RT>(s.G, s.diag, s.kc, r, et);
            if (!good) {
                if (et == 0) a.flags[mf] = 1;   // near-dependent columns: Householder TSQR
                continue;
            }
            float* out = (factor == 0 ? a.R_B : a.R_A) + (size_t)(mf >> 1) * a.rs * a.rs;
            for (int e = et; e < a.rs * a.rs; e += 32 * kI8EpiWarps) {
                const int jr = e / a.rs, jc = e % a.rs;
                out[e] = (jr < r && jc < r && jc >= jr) ? (float)s.G[tri_off<RT>(jr, jc)] : 0.f;
            }
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, kI8TmemCols);
}

}  // namespace lf
