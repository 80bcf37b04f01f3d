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
// rows the copies cannot address (row or offset not 16-byte aligned).
//
// Data flow per CTA (persistent, one per SM, static round-robin over the work items,
// longest first):
//   warp 0        producer: 64-row fp32 stages into a kI8FStages ring, completion
//                 counted in bytes: B (row-major d_out x r) by one 1-D bulk copy per
//                 stage, A^T (A is r x d_in row-major) by two 2-D TMA copies per stage
//                 (boxes of 32 rows x r columns of A^T, 128-byte swizzle, no multicast)
//                 through the matrix's tensor map;
//   warp 1        MMA issuer (one thread): per 128-row digit stage, D1 += [P0;P1] x
//                 [P0;P1;P2;P3]^T (M 128, N 256) and D2 += [P2;P3] x [P2;P3]^T (M 128,
//                 N 128) in four K = 32 steps each, into 384 TMEM columns (plane p =
//                 byte 3 - p);
//   warps 2..17   converters: column scales, fp32 -> digit planes (K-major, 128-byte
//                 swizzle) and the planes' column sums, one 16-row chunk of one
//                 column per thread and digit stage;
//   warps 18..21  epilogue: int32 accumulators -> signed-digit corrections -> the
//                 item's fp64 Gram (packed upper triangle) in its own global slot.
// Operand rows interleave the planes of a column (row 2c: plane 0 or 2 of column c,
// row 2c + 1: plane 1 or 3), so both planes of column c sit in adjacent TMEM lanes of
// one warp and the epilogue combines them with one shuffle.  gram_i8_root_kernel then
// sums a matrix's item Grams in item order and takes the fp64 Cholesky, so the result
// does not depend on scheduling.
#pragma once
#include <cuda.h>   // CUtensorMap (type only)
#include <float.h>

#include "common.cuh"
#include "gram.cuh"
#include "tc.cuh"

namespace lf {

constexpr int kI8Rows = 128;         // rows (the MMA's K) per digit stage
constexpr int kI8FRows = 64;         // rows per fp32 stage (two per digit stage)
constexpr int kI8FStages = 5;
constexpr int kI8DStages = 3;
constexpr int kI8ConvWarps = 16;
constexpr int kI8EpiWarps = 4;
constexpr int kI8ConvWarp0 = 2;
constexpr int kI8EpiWarp0 = kI8ConvWarp0 + kI8ConvWarps;       // 18
constexpr int kI8Threads = 32 * (kI8EpiWarp0 + kI8EpiWarps);   // 704
constexpr int kI8HeadBits = 2;       // 2^E is 4x to 8x the largest value of the first 128 rows
// Rows per work item: the largest accumulator, 255^2 * rows, stays below 2^31, and the
// corrected top-digit product times 2^24 stays below 2^53 (exact in fp64).
constexpr int kI8MaxRows = 24576;
constexpr int kI8LdS = 65;           // fp64 row stride of the epilogue's row buffer
constexpr int kI8FStageFloats = kI8FRows * 64;   // 16 KB: B rows (stride r) or A^T as two swizzled halves
constexpr int kI8AHalfBytes = 64 * 128;          // one A^T half: up to 64 columns x 32 rows
constexpr uint32_t kI8TmemCols = 512;

struct GramI8Meta {
    int32_t colsum[4][64];   // column sums of the digit planes over the item (plane 0 = top byte)
    int32_t E[64];           // column exponents: every |x| of the column is below 2^E
    int32_t ovf;             // a value reached 2^E, or was not finite
};

struct GramI8Smem {
    uint8_t dig[kI8DStages][256 * 128];     // digit stages: 4 planes x 64 columns x 128 rows (1024-aligned)
    float f32[kI8FStages][kI8FStageFloats]; // 1024-aligned (128-byte swizzle atoms of the A^T stages)
    double W[64 * kI8LdS];                  // fp64 row i of the column pair (i, j) sums
    GramI8Meta meta[2];
    float cmax[8][64];
    uint64_t full_f[kI8FStages], empty_f[kI8FStages];
    uint64_t full_d[kI8DStages], empty_d[kI8DStages];
    uint64_t acc_full, acc_empty, drain;
    uint64_t meta_full[2], meta_empty[2];
    uint64_t cmax_full, cmax_empty;          // the column-maximum exchange of an item's first stage
    uint32_t tmem;
    int abort;
};

constexpr size_t gram_i8_smem() { return sizeof(GramI8Smem) + 1024; }

struct GramI8Args {
    const lf_module* mods;
    const float* B_base;
    const CUtensorMap* amaps;  // per module: tensor map of its A (dims d_in x r, box 32 x r, 128-byte swizzle)
    const TsqrWork* work;      // work items of <= kI8MaxRows rows, longest first; .slot = the item's Gram slot
    int32_t n_work;
    double* gram;              // slot s: packed Gram (tri_size<RT> doubles) of one item, scaled to the input
    int32_t* fb;               // per mf: set to 1 when the matrix is left to the fp64 leaf
};

// Operand row of plane p (0 = top byte) of column c in a digit stage: planes 0, 1 of
// the columns interleaved in rows 0..127, planes 2, 3 in rows 128..255.
__device__ __forceinline__ int i8_row(int p, int c) { return (p >> 1) * 128 + 2 * c + (p & 1); }

// max(a, b) that returns NaN when either operand is NaN (fmaxf would return the other).
__device__ __forceinline__ float fmax_nan(float a, float b) {
    float d;
    asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
    return d;
}

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
// rows at or past `nvalid` and columns at or past r read as zero.  B stages are
// row-major with row stride r; A^T stages are two halves of 32 rows (the second at
// 8 KB), each r rows of 128 bytes (one column of A^T per row) with 16-byte chunks
// XOR-swizzled by row % 8.
__device__ __forceinline__ void i8_load_unit(float (&x)[16], const float* st, int factor, int c, int qs, int r,
                                             int nvalid) {
    if (c >= r) {
#pragma unroll
        for (int e = 0; e < 16; ++e) x[e] = 0.f;
        return;
    }
    if (factor == 0) {
        if (nvalid >= 16) {   // every stage but a matrix's last: no row tests
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = st[(16 * qs + e) * r + c];
        } else {
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = e < nvalid ? st[(16 * qs + e) * r + c] : 0.f;
        }
    } else {
        const char* row = reinterpret_cast<const char*>(st) + (qs >> 1) * kI8AHalfBytes + c * 128;
        float4 f[4];
#pragma unroll
        for (int v = 0; v < 4; ++v) f[v] = *reinterpret_cast<const float4*>(row + ((((qs & 1) * 4 + v) ^ (c & 7)) << 4));
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            x[4 * v + 0] = f[v].x;
            x[4 * v + 1] = f[v].y;
            x[4 * v + 2] = f[v].z;
            x[4 * v + 3] = f[v].w;
        }
        if (nvalid < 16) {
#pragma unroll
            for (int e = 0; e < 16; ++e)
                if (e >= nvalid) x[e] = 0.f;
        }
    }
}

// Each thread of a warp reads, at three TMEM column addresses, 16 consecutive 32-bit
// columns of its own lane as integers, then waits for the loads (one asm statement, so
// no use of v can be scheduled before the wait).
__device__ __forceinline__ void tmem_ld16x3(uint32_t t0, uint32_t t1, uint32_t t2, int32_t (&v)[48]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%48];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%49];\n\t"
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47}, [%50];\n\t"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31]),
          "=r"(v[32]), "=r"(v[33]), "=r"(v[34]), "=r"(v[35]), "=r"(v[36]), "=r"(v[37]), "=r"(v[38]), "=r"(v[39]),
          "=r"(v[40]), "=r"(v[41]), "=r"(v[42]), "=r"(v[43]), "=r"(v[44]), "=r"(v[45]), "=r"(v[46]), "=r"(v[47])
        : "r"(t0), "r"(t1), "r"(t2)
        : "memory");
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
        mbar_init(&s.cmax_full, kI8ConvWarps);
        mbar_init(&s.cmax_empty, kI8ConvWarps);
        s.abort = 0;
        fence_barrier_init();
    }
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
            const float* X = a.B_base + md.B_off;
            const CUtensorMap* amap = a.amaps + (w.mf >> 1);
            const int nf = 2 * (int)cdiv(w.nrows, kI8Rows);
            for (int f = 0; f < nf; ++f, ++g) {
                const int slot = g % kI8FStages;
                if (g >= kI8FStages) ok = wait(&s.empty_f[slot], (uint32_t)((g / kI8FStages - 1) & 1));
                if (!ok) break;
                const int rows = max(0, min(kI8FRows, w.nrows - kI8FRows * f));
                const int64_t row = (int64_t)w.row0 + (int64_t)kI8FRows * f;
                if (lane == 0) {
                    if (rows == 0) {
                        mbar_arrive1(&s.full_f[slot]);   // an empty second half of the last digit stage
                    } else if (factor == 0) {
                        const uint32_t bytes = (uint32_t)rows * (uint32_t)r * 4u;
                        mbar_arrive_expect_tx(&s.full_f[slot], bytes);
                        bulk_g2s(s.f32[slot], X + row * r, bytes, &s.full_f[slot]);
                    } else {
                        // one or two boxes of 32 rows of A^T (rows past d_in read as zeros)
                        const uint32_t nbox = rows > 32 ? 2u : 1u;
                        mbar_arrive_expect_tx(&s.full_f[slot], nbox * 32u * (uint32_t)r * 4u);
                        tc::tma_load_2d(s.f32[slot], amap, (int)row, 0, &s.full_f[slot]);
                        if (nbox == 2)
                            tc::tma_load_2d(reinterpret_cast<char*>(s.f32[slot]) + kI8AHalfBytes, amap, (int)row + 32,
                                            0, &s.full_f[slot]);
                    }
                }
                __syncwarp();
            }
        }
        // no copy of this warp may still be writing shared memory when the CTA leaves
        // (on the normal path these phases completed before their conversion)
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
            if (!ok) break;
            GramI8Meta& M = s.meta[ms];
            // this thread's column c and 16-row chunk q of every digit stage (chunk q in
            // fp32 stage q >> 2): B stages are read across columns (one row per load),
            // A^T stages across 8 columns of one chunk (16-byte loads, distinct swizzled chunks)
            const int c = factor == 0 ? 32 * (cw & 1) + lane : 8 * (cw & 7) + (lane & 7);
            const int q = factor == 0 ? (cw >> 1) : (lane >> 3) + 4 * (cw >> 3);
            for (int e = ct; e < 4 * 64; e += 32 * kI8ConvWarps) (&M.colsum[0][0])[e] = 0;
            if (ct == 0) M.ovf = 0;
            uint32_t cs[4] = {0u, 0u, 0u, 0u};
            bool vok = true;
            float mult = 0.f, lim = 0.f;
            for (int ds = 0; ds < nd; ++ds, g += 2, ++gd) {
                const int f0 = g % kI8FStages, f1 = (g + 1) % kI8FStages;
                ok = wait(&s.full_f[f0], (uint32_t)((g / kI8FStages) & 1)) &&
                     wait(&s.full_f[f1], (uint32_t)(((g + 1) / kI8FStages) & 1));
                if (!ok) break;
                const int rbase = kI8Rows * ds;
                // this thread's chunk into registers, then the fp32 stages go back to the
                // producer before any conversion work
                float xv[16];
                i8_load_unit(xv, s.f32[q < 4 ? f0 : f1], factor, c, q & 3, r, w.nrows - rbase - 16 * q);
                // the magnitude check reads every loaded value, and the empty asm pins it
                // before the release: the stage goes back to the producer only once this
                // thread's loads have returned (a shared-memory load still in flight at the
                // arrive could otherwise read the producer's next copy)
                float amax = 0.f;
#pragma unroll
                for (int e = 0; e < 16; ++e) amax = fmax_nan(amax, fabsf(xv[e]));   // a NaN stays in amax
                asm volatile("" ::"f"(amax));
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive1(&s.empty_f[f0]);
                    mbar_arrive1(&s.empty_f[f1]);
                }
                if (ds == 0) {
                    // column exponents from the item's first 128 rows
                    float mx = 0.f;
#pragma unroll
                    for (int e = 0; e < 16; ++e) mx = fmaxf(mx, fabsf(xv[e]));
                    // exchanged through mbarriers (bounded waits): the previous item's
                    // readers are done, every warp's maxima are in, then this warp is done
                    if (k >= 1) ok = wait(&s.cmax_empty, (uint32_t)((k - 1) & 1));
                    if (!ok) break;
                    s.cmax[q][c] = mx;
                    __threadfence_block();
                    __syncwarp();
                    if (lane == 0) mbar_arrive1(&s.cmax_full);
                    ok = wait(&s.cmax_full, (uint32_t)(k & 1));
                    if (!ok) break;
                    float m = s.cmax[0][c];
#pragma unroll
                    for (int h = 1; h < 8; ++h) m = fmaxf(m, s.cmax[h][c]);
                    asm volatile("" ::"f"(m));   // the reads have returned before the release
                    __syncwarp();
                    if (lane == 0) mbar_arrive1(&s.cmax_empty);
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
                    if (q == 0) M.E[c] = E;
                }
                if (gd >= kI8DStages) ok = wait(&s.empty_d[gd % kI8DStages], (uint32_t)((gd / kI8DStages - 1) & 1));
                if (!ok) break;
                uint8_t* dig = s.dig[gd % kI8DStages];
                uint32_t pw[4][4];
#pragma unroll
                for (int j4 = 0; j4 < 4; ++j4) {
                    uint32_t u[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        u[e] = (uint32_t)__float2int_rz(xv[4 * j4 + e] * mult);
                    }
                    uint32_t wd[4];
                    planes4(u, wd);
                    wd[0] ^= 0x80808080u;   // U = N + 2^31: the top byte's top bit, four rows at once
#pragma unroll
                    for (int p = 0; p < 4; ++p) {
                        pw[p][j4] = wd[p];
                        cs[p] = __dp4a(wd[p], 0x01010101u, cs[p]);
                    }
                }
                vok = vok && amax < lim;   // false for infinities and NaN as well
                // lanes 4..7 of each group of 8 (consecutive columns) store the other plane of
                // the pair (0 <-> 1, 2 <-> 3) than lanes 0..3, so the eight 16-byte stores of a
                // group land in eight different swizzled chunks (no bank conflict)
                const int flip = (lane >> 2) & 1;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int p = t ^ flip;
                    const int R = i8_row(p, c);   // operand row, 128 bytes
                    const uint4 val = flip ? make_uint4(pw[t ^ 1][0], pw[t ^ 1][1], pw[t ^ 1][2], pw[t ^ 1][3])
                                           : make_uint4(pw[t][0], pw[t][1], pw[t][2], pw[t][3]);
                    *reinterpret_cast<uint4*>(dig + R * 128 + ((q ^ (R & 7)) << 4)) = val;
                }
                tc::fence_proxy_async();   // the digit planes, to the tensor core's proxy
                __syncwarp();
                if (lane == 0) mbar_arrive1(&s.full_d[gd % kI8DStages]);
            }
            if (!ok) break;
#pragma unroll
            for (int p = 0; p < 4; ++p) atomicAdd(&M.colsum[p][c], (int)cs[p]);
            if (!vok) M.ovf = 1;
            __threadfence_block();   // every lane's sums and flag are in before its warp's arrive
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.meta_full[ms]);
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int et = tid - 32 * kI8EpiWarp0;   // 0..127
        const int lq = warp & 3;                 // the TMEM lane quarter this warp may read
        const int m = 32 * lq + lane;            // accumulator row: plane pair member m & 1 of column m >> 1
        const bool odd = (m & 1) != 0;           // planes 1 and 3 of column i (else planes 0 and 2)
        const int i = m >> 1;
        constexpr int TRI = tri_size<RT>();
        int k = 0;
        bool ok = true;
        for (int it = blockIdx.x; it < a.n_work && ok; it += gridDim.x, ++k) {
            const TsqrWork w = a.work[it];
            const int mf = w.mf;
            const int r = a.mods[mf >> 1].r;
            const int64_t Krows = (int64_t)cdiv(w.nrows, kI8Rows) * kI8Rows;   // zero rows included
            const int ms = k & 1;
            ok = wait(&s.acc_full, (uint32_t)(k & 1)) && wait(&s.meta_full[ms], (uint32_t)((k >> 1) & 1));
            ok = named_and(2, 32 * kI8EpiWarps, ok);
            if (!ok) break;
            tc::fence_after_sync();
            const GramI8Meta& M = s.meta[ms];
            // Row i of the column pairs (i, j): this lane's six products -> fp64 (exact
            // integer combination, then at most two roundings); D1 columns 2j, 2j+1:
            // planes 0, 1 of column j; 128 + 2j, +1: planes 2, 3; D2 (from column 256)
            // 2j, 2j+1: planes 2, 3.  The even lane (row planes 0 and 2) and the odd
            // lane (planes 1 and 3) of column i add their values in that order.
            const int64_t Si0 = M.colsum[0][i], Si1 = M.colsum[1][i];
            const uint32_t tb = tmem + ((uint32_t)(32 * lq) << 16);
            double* Wrow = s.W + i * kI8LdS;
            for (int jb = 0; jb < 8; ++jb) {
                int32_t v[48];
                tmem_ld16x3(tb + 16 * jb, tb + 128 + 16 * jb, tb + 256 + 16 * jb, v);
                double Wv[8];
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) {
                    const int j = 8 * jb + jj;
                    const int64_t p0 = v[2 * jj], p1 = v[2 * jj + 1], p2 = v[16 + 2 * jj], p3 = v[16 + 2 * jj + 1];
                    const int64_t p4 = v[32 + 2 * jj], p5 = v[32 + 2 * jj + 1];
                    double H, L;
                    if (!odd) {
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
                    const double Vo = __shfl_xor_sync(0xffffffffu, V, 1);
                    Wv[jj] = odd ? Vo + V : V + Vo;
                }
                // the even lane stores j = 8jb .. 8jb + 3, the odd lane 8jb + 4 .. 8jb + 7
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) Wrow[8 * jb + 4 * odd + jj] = odd ? Wv[4 + jj] : Wv[jj];
            }
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.acc_empty);   // the next item's MMAs may overwrite D
            tc::named_sync(2, 32 * kI8EpiWarps);
            // the item's Gram, packed upper triangle: G_ab = 2^(E_a + E_b - 62) (W_ab + W_ba)
            double* dst = a.gram + (int64_t)w.slot * TRI;
            for (int ra = 0; ra < RT; ++ra) {
                const int cb = ra + et;
                if (cb >= RT) continue;
                double gv = 0.0;
                if (cb < r) {
                    gv = ra == cb ? s.W[ra * kI8LdS + ra] : s.W[ra * kI8LdS + cb] + s.W[cb * kI8LdS + ra];
                    // times 2^(E_a + E_b - 62), exact (E in [-96, 127])
                    gv *= __longlong_as_double((long long)(M.E[ra] + M.E[cb] - 62 + 1023) << 52);
                }
                dst[tri_off<RT>(ra, cb)] = gv;
            }
            if (et == 0 && M.ovf) atomicExch(&a.fb[mf], 1);
            __syncwarp();
            if (lane == 0) mbar_arrive1(&s.meta_empty[ms]);
            tc::named_sync(2, 32 * kI8EpiWarps);   // W is rewritten by the next item
        }
    }
    tc::fence_before_sync();
    __syncthreads();
    if (warp == 1) tc::tmem_dealloc(tmem, kI8TmemCols);
}

// Root of the integer-Gram leaf: one warp per matrix (2 * module + factor).  The
// matrix's item Grams are summed in item order, then the fp64 Cholesky gives R (fp32
// output, zero past r); a rejected pivot marks the matrix for the Householder TSQR.
// Matrices the fp64 leaf takes (fb) are skipped.
struct GramI8RootArgs {
    const lf_module* mods;
    const TsqrInfo* info;      // per mf: item count and first slot
    const double* gram;
    const int32_t* fb;
    int32_t* flags;
    float* R_B;
    float* R_A;
    int32_t rs, n_mf;
};
constexpr int kI8RootWarps = 4;

template <int RT>
constexpr size_t gram_i8_root_smem() { return (size_t)kI8RootWarps * (tri_size<RT>() + RT) * sizeof(double); }

template <int RT>
__global__ void __launch_bounds__(32 * kI8RootWarps) gram_i8_root_kernel(GramI8RootArgs a) {
    constexpr int TRI = tri_size<RT>();
    extern __shared__ double root_sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double* Gw = root_sm + (size_t)warp * (TRI + RT);
    double* dg = Gw + TRI;
    const int mf = blockIdx.x * kI8RootWarps + warp;
    if (mf >= a.n_mf) return;
    if (a.fb[mf]) return;   // warp-uniform
    const TsqrInfo inf = a.info[mf];
    const double* P0 = a.gram + (int64_t)inf.slot0 * TRI;
    for (int e = lane; e < TRI; e += 32) {
        double acc = P0[e];
        for (int c = 1; c < inf.nchunks; ++c) acc += P0[(int64_t)c * TRI + e];
        Gw[e] = acc;
    }
    __syncwarp();
    const int r = a.mods[mf >> 1].r;
    if (!gram_cholesky<RT>(Gw, dg, r, lane)) {
        if (lane == 0) a.flags[mf] = 1;   // near-dependent columns: Householder TSQR
        return;
    }
    float* out = ((mf & 1) == 0 ? a.R_B : a.R_A) + (size_t)(mf >> 1) * a.rs * a.rs;
    for (int jr = 0; jr < a.rs; ++jr) {   // row jr of R: columns jr..r-1 of the packed row, zero elsewhere
        const double* gr = Gw + (tri_off<RT>(jr, jr) - jr);
        for (int jc = lane; jc < a.rs; jc += 32)
            out[(size_t)jr * a.rs + jc] = (jr < r && jc < r && jc >= jr) ? (float)gr[jc] : 0.f;
    }
}

}  // namespace lf
