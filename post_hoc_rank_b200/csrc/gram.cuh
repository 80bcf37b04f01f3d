// TSQR leaf by fp64 Gram accumulation on the fp64 tensor-core path.
//
// LoRAForge (kongchang.com), "FlashTSQR: An Accelerator for Batched Factor
// Construction": R of each tall-skinny factor comes from local work on row blocks
// followed by a merge, parallel across modules and row blocks.  Here the local
// product of a row block X_c is its Gram matrix G_c = X_c^T X_c, the merge is the
// fixed-order sum G = sum_c G_c (the Gram of the stacked blocks, exactly what the
// QR of [R_1; R_2; ...] preserves: R^T R = G), and the root takes R = chol(G), the
// unique upper-triangular factor with positive diagonal, i.e. the R of X = QR.
//
// Precision: every product of two fp32 inputs is exact in fp64, and the sums run in
// fp64, so G carries ~1e-16 relative error and R from the fp64 Cholesky has
// relative error ~1e-16 * kappa(X)^2.  A Cholesky pivot d_j at or below
// kGramPivotTol * G_jj (column j is numerically dependent on the earlier ones, a
// zero column, or a non-finite input) marks the matrix in `flags`; its R is then
// rebuilt by the structured-Householder TSQR kernel, which has no kappa^2 term.
//
// Work decomposition matches tsqr_kernel (the same TsqrWork / TsqrInfo lists):
// one warp owns one chunk of rows, streams it through a 4-stage cp.async ring of
// kGramTM-row stages, and accumulates the upper block triangle of G with
// mma.m8n8k4.f64 (fragments are read straight from the fp32 stage and widened in
// registers).  The last warp of a matrix (atomic counter) sums the chunk partials
// in chunk order, so the result does not depend on scheduling.
#pragma once
#include "common.cuh"
#include "tc.cuh"
#include "tsqr.cuh"

namespace lf {

constexpr int kGramTM = 16;        // rows per pipeline stage
constexpr int kGramStages = 4;
constexpr int kGramLdA = kGramTM + 4;   // column stride (floats) of an A^T stage
constexpr double kGramPivotTol = 1e-9;

// B stage: row-major, X[i][c] at i * (RT + 8) + c.  A^T stage: column-major,
// X[i][c] at c * kGramLdA + i.  Both strides make the fragment read of a warp
// (rows 4ks + lane%4, columns 8b + lane/4) hit 32 distinct banks.
template <int RT>
__host__ __device__ constexpr int gram_ldb() { return RT + 8; }
template <int RT>
__host__ __device__ constexpr int gram_stage_floats() {
    return kGramTM * gram_ldb<RT>() > RT * kGramLdA ? kGramTM * gram_ldb<RT>() : RT * kGramLdA;
}
// Bytes of one partial slot: the packed Gram (fp64) or the Householder partial R
// (fp32, RT x RT), whichever is larger; both kernels use the same slot buffer.
template <int RT>
__host__ __device__ constexpr size_t gram_slot_bytes() {
    return tri_size<RT>() * 8 > RT * RT * 4 ? (size_t)tri_size<RT>() * 8 : (size_t)RT * RT * 4;
}

struct GramArgs {
    const lf_module* mods;
    const float* B_base;
    const float* A_base;
    const TsqrWork* work;
    const int32_t* n_work;     // device scalar
    const TsqrInfo* info;      // per mf
    int32_t* counters;         // per mf, zero on entry
    double* partial;           // slot s at partial + s * slot_doubles: packed upper triangle of G_c
    int64_t slot_doubles;
    int32_t* flags;            // per mf, zero on entry; 1 = Cholesky rejected, R left to the Householder pass
    float* R_B;                // per module, rs x rs
    float* R_A;
    int32_t rs;
    const int32_t* only;       // per mf (nullable): zero = skip this matrix
    double* R64;               // nullable: per mf, rs x rs fp64 copy of R (mf = 2 * module + factor)
};

// D (8x8, two entries per lane) += A (8x4) * B (4x8), fp64, one warp.
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
    asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};"
        : "+d"(d[0]), "+d"(d[1])
        : "d"(a), "d"(b));
}

// 16-byte / 4-byte async copies that read src_bytes (<= the copy size) and fill the rest with zeros.
__device__ __forceinline__ void cp_async16_n(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async4_n(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}

// Copy rows i0 .. i0 + kGramTM - 1 of the chunk into one stage (rows past the chunk
// are zero-filled; columns >= r are never written and stay zero).
template <int RT, int FACTOR>
__device__ __forceinline__ void gram_issue(float* st, const float* X, int r, int d_in, int64_t rb, int nrem,
                                           bool vec, int lane) {
    constexpr int LDB = gram_ldb<RT>();
    if (vec) {
        if (FACTOR == 0) {   // B row-major d_out x r: stage row i <- X[(rb + i) * r .. + r)
            const int cpr = r >> 2;
            for (int q = lane; q < kGramTM * cpr; q += 32) {
                const int i = q / cpr, c4 = q - i * cpr;
                const bool ok = i < nrem;
                cp_async16_n(st + i * LDB + 4 * c4, ok ? X + (rb + i) * r + 4 * c4 : X, ok ? 16u : 0u);
            }
        } else {             // A row-major r x d_in: stage column c <- A[c][rb .. rb + TM)
            constexpr int cpc = kGramTM / 4;
            for (int q = lane; q < r * cpc; q += 32) {
                const int c = q / cpc, i4 = q - c * cpc;
                const int nv = min(4, max(0, nrem - 4 * i4));
                cp_async16_n(st + c * kGramLdA + 4 * i4, nv > 0 ? X + (int64_t)c * d_in + rb + 4 * i4 : X,
                             4u * (uint32_t)nv);
            }
        }
    } else {                 // unaligned rows: element copies
        for (int q = lane; q < kGramTM * r; q += 32) {
            const int i = q / r, c = q - i * r;
            const bool ok = i < nrem;
            if (FACTOR == 0)
                cp_async4_n(st + i * LDB + c, ok ? X + (rb + i) * r + c : X, ok ? 4u : 0u);
            else
                cp_async4_n(st + c * kGramLdA + i, ok ? X + (int64_t)c * d_in + rb + i : X, ok ? 4u : 0u);
        }
    }
}

// Accumulate the chunk's Gram: acc[p] holds block (bi, bj), bi <= bj, in the m8n8
// accumulator layout (row 8bi + lane/4, columns 8bj + 2(lane%4) + {0, 1}).
template <int RT, int FACTOR>
__device__ __forceinline__ void gram_chunk(double (&acc)[(RT / 8) * (RT / 8 + 1) / 2][2],
                                           float (*stage)[gram_stage_floats<RT>()], const float* X, int r,
                                           int d_in, int64_t row0, int nrows, bool vec, int lane) {
    constexpr int NB = RT / 8;
    constexpr int LDB = gram_ldb<RT>();
    constexpr int FSB = FACTOR == 0 ? 8 : 8 * kGramLdA;       // next 8-column block
    constexpr int FSK = FACTOR == 0 ? 4 * LDB : 4;            // next 4 rows
    const int fbase = FACTOR == 0 ? (lane & 3) * LDB + (lane >> 2) : (lane >> 2) * kGramLdA + (lane & 3);
    const int nst = (nrows + kGramTM - 1) / kGramTM;
#pragma unroll
    for (int s = 0; s < kGramStages - 1; ++s) {
        if (s < nst) gram_issue<RT, FACTOR>(stage[s], X, r, d_in, row0 + s * kGramTM, nrows - s * kGramTM, vec, lane);
        tc::cp_async_commit();
    }
    for (int t = 0; t < nst; ++t) {
        tc::cp_async_wait<kGramStages - 2>();
        __syncwarp();
        {
            const int tn = t + kGramStages - 1;
            if (tn < nst)
                gram_issue<RT, FACTOR>(stage[tn % kGramStages], X, r, d_in, row0 + tn * kGramTM,
                                       nrows - tn * kGramTM, vec, lane);
            tc::cp_async_commit();
        }
        const float* st = stage[t % kGramStages] + fbase;
#pragma unroll
        for (int ks = 0; ks < kGramTM / 4; ++ks) {
            double f[NB];
#pragma unroll
            for (int b = 0; b < NB; ++b) f[b] = (double)st[ks * FSK + b * FSB];
            int p = 0;
#pragma unroll
            for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                for (int bj = bi; bj < NB; ++bj) dmma_8x8x4(acc[p++], f[bi], f[bj]);
        }
    }
    tc::cp_async_wait<0>();
    __syncwarp();
}

// Right-looking Cholesky of the packed Gram G (r x r used) in place by one warp: row
// j of R overwrites row j of G.  Returns false (warp-uniform: every lane reads the same
// values) when a pivot falls to <= kGramPivotTol times its Gram diagonal.
template <int RT>
__device__ __forceinline__ bool gram_cholesky(double* G, double* s_diag, int r, int lane) {
    using C = Cols<RT>;
    for (int j = lane; j < r; j += 32) s_diag[j] = G[tri_off<RT>(j, j)];
    __syncwarp();
    for (int j = 0; j < r; ++j) {
        const int dj = tri_off<RT>(j, j);
        const double d = G[dj];
        if (!(d > kGramPivotTol * s_diag[j])) return false;
        const double rjj = sqrt(d);
        const double inv = 1.0 / rjj;   // one division per step; the row is scaled by it
        __syncwarp();
#pragma unroll
        for (int s = 0; s < C::NS; ++s) {
            const int c = C::col(lane, s);
            if (c > j && c < r) G[dj + (c - j)] *= inv;
        }
        if (lane == 0) G[dj] = rjj;
        __syncwarp();
        const double* rowj = G + (dj - j);   // rowj[k] = R_jk
#pragma unroll
        for (int s = 0; s < C::NS; ++s) {
            const int c = C::col(lane, s);
            if (c > j && c < r) {
                const double gjc = rowj[c];
                // column c, rows k = j+1..c; the packed offset of (k, c) grows by RT - k - 1
                // from k to k + 1.  Four rows per pass: loads first, then the stores.
                int k = j + 1;
                int p = tri_off<RT>(k, c);
                for (; k + 3 <= c; k += 4) {
                    const int p1 = p + (RT - k - 1), p2 = p1 + (RT - k - 2), p3 = p2 + (RT - k - 3);
                    const double a0 = rowj[k], a1 = rowj[k + 1], a2 = rowj[k + 2], a3 = rowj[k + 3];
                    const double g0 = G[p], g1 = G[p1], g2 = G[p2], g3 = G[p3];
                    G[p] = g0 - a0 * gjc;
                    G[p1] = g1 - a1 * gjc;
                    G[p2] = g2 - a2 * gjc;
                    G[p3] = g3 - a3 * gjc;
                    p = p3 + (RT - k - 4);
                }
                for (; k <= c; ++k) {
                    G[p] -= rowj[k] * gjc;
                    p += RT - k - 1;
                }
            }
        }
        __syncwarp();
    }
    return true;
}

template <int RT>
__global__ void __launch_bounds__(32, 8) gram_kernel(GramArgs a) {
    constexpr int NB = RT / 8;
    constexpr int NP = NB * (NB + 1) / 2;
    constexpr int TRI = tri_size<RT>();
    static_assert(TRI * 8 <= kGramStages * gram_stage_floats<RT>() * 4, "packed Gram must fit in the stages");
    __shared__ __align__(16) float stage[kGramStages][gram_stage_floats<RT>()];
    __shared__ double s_diag[RT];
    __shared__ int s_last;
    const int lane = threadIdx.x;
    if ((int)blockIdx.x >= *a.n_work) return;
    const TsqrWork w = a.work[blockIdx.x];
    const int mf = w.mf, factor = mf & 1;
    if (a.only && a.only[mf] == 0) return;
    const lf_module md = a.mods[mf >> 1];
    const int r = md.r;
    const float* X = factor == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
    const bool vec = factor == 0 ? ((md.B_off & 3) == 0 && (r & 3) == 0)
                                 : ((md.A_off & 3) == 0 && (md.d_in & 3) == 0);

    for (int e = lane; e < kGramStages * gram_stage_floats<RT>(); e += 32) (&stage[0][0])[e] = 0.f;
    __syncwarp();
    double acc[NP][2];
#pragma unroll
    for (int p = 0; p < NP; ++p) acc[p][0] = acc[p][1] = 0.0;
    if (factor == 0)
        gram_chunk<RT, 0>(acc, stage, X, r, md.d_in, w.row0, w.nrows, vec, lane);
    else
        gram_chunk<RT, 1>(acc, stage, X, r, md.d_in, w.row0, w.nrows, vec, lane);

    // packed upper triangle of this chunk's Gram -> dst (global partial slot or shared)
    auto store_acc = [&](double* dst) {
        const int m = lane >> 2, n2 = 2 * (lane & 3);
        int p = 0;
#pragma unroll
        for (int bi = 0; bi < NB; ++bi)
#pragma unroll
            for (int bj = bi; bj < NB; ++bj, ++p)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int row = 8 * bi + m, col = 8 * bj + n2 + e;
                    if (col >= row) dst[tri_off<RT>(row, col)] = acc[p][e];
                }
    };
    double* G = reinterpret_cast<double*>(&stage[0][0]);
    const TsqrInfo inf = a.info[mf];
    if (inf.nchunks > 1) {
        store_acc(a.partial + (int64_t)w.slot * a.slot_doubles);
        __threadfence();
        __syncwarp();
        if (lane == 0) s_last = (atomicAdd(&a.counters[mf], 1) == inf.nchunks - 1);
        __syncwarp();
        if (!s_last) return;
        __threadfence();
        const double* P0 = a.partial + (int64_t)inf.slot0 * a.slot_doubles;
        for (int e = lane; e < TRI; e += 32) {
            double s = __ldcg(P0 + e);
            for (int c = 1; c < inf.nchunks; ++c) s += __ldcg(P0 + (int64_t)c * a.slot_doubles + e);
            G[e] = s;
        }
    } else {
        store_acc(G);
    }
    __syncwarp();

    if (!gram_cholesky<RT>(G, s_diag, r, lane)) {
        if (lane == 0) a.flags[mf] = 1;
        return;
    }
    float* out = (factor == 0 ? a.R_B : a.R_A) + (size_t)(mf >> 1) * a.rs * a.rs;
    for (int e = lane; e < a.rs * a.rs; e += 32) {
        const int j = e / a.rs, c = e % a.rs;
        out[e] = (j < r && c < r && c >= j) ? (float)G[tri_off<RT>(j, c)] : 0.f;
    }
    if (a.R64) {
        double* o64 = a.R64 + (size_t)mf * a.rs * a.rs;
        for (int e = lane; e < a.rs * a.rs; e += 32) {
            const int j = e / a.rs, c = e % a.rs;
            o64[e] = (j < r && c < r && c >= j) ? G[tri_off<RT>(j, c)] : 0.0;
        }
    }
}

}  // namespace lf
