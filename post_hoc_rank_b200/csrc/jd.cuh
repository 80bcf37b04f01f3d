// Joint diagonalization of a LoRA collection (JD-Full) by eigenvalue iteration.
//
// "Compress then Serve" (academ.us/article/2407.00066), §3.1 eq. 1 and Appendix
// 8.1 (case 1) / 8.2: the n products B_i A_i of one module position share
// orthonormal bases U (d_out x r~) and V (d_in x r~), one full r~ x r~ Sigma_i each.
// One step of Appendix 8.2, with P_i = A_i V and Q_i = B_i^T U (r_i x r~):
//     S_i = P_i^T Q_i,   U_0 = sum_i w_i B_i (P_i S_i),   V_0 = sum_i w_i A_i^T (Q_i S_i^T),
//     U <- orthogonalize(U_0),   V <- orthogonalize(V_0),
// and Sigma_i = U^T B_i A_i V = Q_i^T P_i = S_i^T (eq. 6) at the final U, V.
//
// The state (U, V^T) of a problem has the layout of a LoRA module of rank r~ (U
// d_out x r~ row-major like B, V^T r~ x d_in row-major like A), so orthogonalize is
// the factor-construction TSQR on it followed by Q = X R^-1: the update kernel's
// epilogue forms the Gram of each finished 128-row tile (the TSQR leaf), the tiles are
// merged in order and the fp64 Cholesky is taken (the root), and Q = X R^-1 uses that
// fp64 R (orthonormal to ~kappa^2 u_64 + u_32).  A matrix whose pivot is rejected
// gets its R from the Householder TSQR kernel instead and a second pass (Gram leaf +
// Cholesky on Q_1, then Q = Q_1 R_2^-1: CholeskyQR2) restores orthonormality.
//
// Kernels of one step, all fp64 on the tensor-core path (mma.m8n8k4.f64: every
// product of two fp32 values is exact, sums are fp64):
//   jd_project_kernel  per (member, factor, row chunk): X_c^T Y_c with X the
//                      member's B (or A^T) and Y the problem's U (or V); chunk
//                      partials summed in chunk order by the last CTA -> Q_i, P_i.
//   jd_core_kernel     per member: S, W = w P S, Z = w Q S^T (and Sigma = S^T).
//   jd_update_kernel   per (problem, factor, 128-row tile): sum over members of
//                      X_tile W_i (or A_i^T Z_i) -> U_0 rows (or V_0^T columns).
//                      Its epilogue writes the tile's Gram.
//   jd_gram_sum_kernel per (problem, factor, slice of the Gram): tile Grams summed in order.
//   jd_chol_kernel     per (problem, factor): fp64 Cholesky of the summed Gram.
//   jd_rinv_kernel     per (problem, factor): R^-1 in fp64.
//   jd_qform_kernel    per (problem, factor, 128-row tile): Q = X R^-1 (fp64 tensor cores).
#pragma once
#include "common.cuh"
#include "tc.cuh"
#include "gram.cuh"

namespace lf {

constexpr int kJdChunk = 2048;   // rows per project work item
constexpr int kJdStages = 4;     // project cp.async ring depth (kGramTM rows per stage)
constexpr int kJdTR = 128;       // rows per update / Q-form CTA
constexpr int kJdLdM = kJdTR + 8;   // row stride (floats) of an A-like update stage

struct JdMember {
    int32_t mod;     // adapter module (index into the module table)
    int32_t prob;    // problem
    int32_t local;   // position of the adapter in its problem
    int32_t pad;
};

// Update / Q-form work item: rows row0 .. row0 + nrows of factor f of problem p.
struct JdTile {
    int32_t p, f, row0, nrows;
};

struct JdProbDev {
    int32_t g0, count;    // members g0 .. g0 + count
    int64_t sigma_off;
};

template <int R>
__host__ __device__ constexpr int jd_ldb() { return R + 8; }
template <int R>
__host__ __device__ constexpr int jd_stage_floats() {
    return kGramTM * jd_ldb<R>() > R * kGramLdA ? kGramTM * jd_ldb<R>() : R * kGramLdA;
}
template <int RY>
__host__ __device__ constexpr int jd_project_warps() { return RY == 64 ? 2 : 1; }

struct JdProjArgs {
    const lf_module* mods;
    const JdMember* members;
    const lf_module* basis;       // per problem: B_off -> U, A_off -> V^T, r = r~
    const float* B_base;
    const float* A_base;
    const float* U_base;
    const float* Vt_base;
    const TsqrWork* work;         // mf = 2 * member + factor
    const TsqrInfo* info;         // per mf
    int32_t* counters;            // per mf, zero on entry and on exit
    double* partial;              // slots of RX * RY doubles
    double* QP;                   // per mf: RX x RY (row = column of X, column = column of Y)
};

// Copy rows rb .. rb + kGramTM - 1 of a B-like (row-major d x r) or A-like
// (row-major r x d, staged column-major) matrix into one stage; rows past the
// chunk are zero-filled.  NT threads share the copies.
template <int R, int FACTOR, int NT>
__device__ __forceinline__ void jd_issue(float* st, const float* X, int r, int ld, int64_t rb, int nrem, bool vec,
                                         int tid) {
    constexpr int LDB = jd_ldb<R>();
    if (vec) {
        if (FACTOR == 0) {
            const int cpr = r >> 2;
            for (int q = tid; q < kGramTM * cpr; q += NT) {
                const int i = q / cpr, c4 = q - i * cpr;
                const bool ok = i < nrem;
                cp_async16_n(st + i * LDB + 4 * c4, ok ? X + (rb + i) * r + 4 * c4 : X, ok ? 16u : 0u);
            }
        } else {
            constexpr int cpc = kGramTM / 4;
            for (int q = tid; q < r * cpc; q += NT) {
                const int c = q / cpc, i4 = q - c * cpc;
                const int nv = min(4, max(0, nrem - 4 * i4));
                cp_async16_n(st + c * kGramLdA + 4 * i4, nv > 0 ? X + (int64_t)c * ld + rb + 4 * i4 : X,
                             4u * (uint32_t)nv);
            }
        }
    } else {
        for (int q = tid; q < kGramTM * r; q += NT) {
            const int i = q / r, c = q - i * r;
            const bool ok = i < nrem;
            if (FACTOR == 0)
                cp_async4_n(st + i * LDB + c, ok ? X + (rb + i) * r + c : X, ok ? 4u : 0u);
            else
                cp_async4_n(st + c * kGramLdA + i, ok ? X + (int64_t)c * ld + rb + i : X, ok ? 4u : 0u);
        }
    }
}

template <int RX, int RY, int FACTOR>
__device__ __forceinline__ void jd_project_chunk(double (&acc)[RX / 8][RY / 8 / jd_project_warps<RY>()][2],
                                                 float (*sx)[jd_stage_floats<RX>()],
                                                 float (*sy)[jd_stage_floats<RY>()], const float* X, int rx,
                                                 bool vx, const float* Y, int ry, bool vy, int ld, int64_t row0,
                                                 int nrows) {
    constexpr int NW = jd_project_warps<RY>();
    constexpr int NT = 32 * NW;
    constexpr int NBX = RX / 8, NBY = RY / 8 / NW;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int LX = jd_ldb<RX>(), LY = jd_ldb<RY>();
    // fragment bases: lane reads row 4ks + lane%4, column 8b + lane/4 of the stage
    const int fx = FACTOR == 0 ? (lane & 3) * LX + (lane >> 2) : (lane >> 2) * kGramLdA + (lane & 3);
    const int fy = FACTOR == 0 ? (lane & 3) * LY + (lane >> 2) : (lane >> 2) * kGramLdA + (lane & 3);
    constexpr int SKX = FACTOR == 0 ? 4 * LX : 4, SBX = FACTOR == 0 ? 8 : 8 * kGramLdA;
    constexpr int SKY = FACTOR == 0 ? 4 * LY : 4, SBY = FACTOR == 0 ? 8 : 8 * kGramLdA;
    const int by0 = warp * NBY;
    auto sync = [] {
        if (NW > 1) __syncthreads(); else __syncwarp();
    };
    auto issue = [&](int s, int t) {
        const int64_t rb = row0 + (int64_t)t * kGramTM;
        const int nrem = nrows - t * kGramTM;
        jd_issue<RX, FACTOR, NT>(sx[s], X, rx, ld, rb, nrem, vx, tid);
        jd_issue<RY, FACTOR, NT>(sy[s], Y, ry, ld, rb, nrem, vy, tid);
    };
    const int nst = (nrows + kGramTM - 1) / kGramTM;
#pragma unroll
    for (int s = 0; s < kJdStages - 1; ++s) {
        if (s < nst) issue(s, s);
        tc::cp_async_commit();
    }
    for (int t = 0; t < nst; ++t) {
        tc::cp_async_wait<kJdStages - 2>();
        sync();
        {
            const int tn = t + kJdStages - 1;
            if (tn < nst) issue(tn % kJdStages, tn);
            tc::cp_async_commit();
        }
        const float* px = sx[t % kJdStages] + fx;
        const float* py = sy[t % kJdStages] + fy;
#pragma unroll
        for (int ks = 0; ks < kGramTM / 4; ++ks) {
            double a[NBX], b[NBY];
#pragma unroll
            for (int i = 0; i < NBX; ++i) a[i] = (double)px[ks * SKX + i * SBX];
#pragma unroll
            for (int j = 0; j < NBY; ++j) b[j] = (double)py[ks * SKY + (by0 + j) * SBY];
#pragma unroll
            for (int i = 0; i < NBX; ++i)
#pragma unroll
                for (int j = 0; j < NBY; ++j) dmma_8x8x4(acc[i][j], a[i], b[j]);
        }
    }
    tc::cp_async_wait<0>();
    sync();
}

template <int RX, int RY>
__global__ void __launch_bounds__(32 * jd_project_warps<RY>()) jd_project_kernel(JdProjArgs a) {
    constexpr int NW = jd_project_warps<RY>();
    constexpr int NT = 32 * NW;
    constexpr int NBX = RX / 8, NBY = RY / 8 / NW;
    __shared__ __align__(16) float sx[kJdStages][jd_stage_floats<RX>()];
    __shared__ __align__(16) float sy[kJdStages][jd_stage_floats<RY>()];
    __shared__ int s_last;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const TsqrWork w = a.work[blockIdx.x];
    const int g = w.mf >> 1, factor = w.mf & 1;
    const JdMember mb = a.members[g];
    const lf_module md = a.mods[mb.mod];
    const lf_module bs = a.basis[mb.prob];
    const float* X = factor == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
    const float* Y = factor == 0 ? a.U_base + bs.B_off : a.Vt_base + bs.A_off;
    const bool vx = factor == 0 ? ((md.B_off & 3) == 0 && (md.r & 3) == 0) : ((md.A_off & 3) == 0 && (md.d_in & 3) == 0);
    const bool vy = factor == 0 ? ((bs.B_off & 3) == 0 && (bs.r & 3) == 0) : ((bs.A_off & 3) == 0 && (bs.d_in & 3) == 0);

    for (int e = tid; e < kJdStages * jd_stage_floats<RX>(); e += NT) (&sx[0][0])[e] = 0.f;
    for (int e = tid; e < kJdStages * jd_stage_floats<RY>(); e += NT) (&sy[0][0])[e] = 0.f;
    __syncthreads();
    double acc[NBX][NBY][2];
#pragma unroll
    for (int i = 0; i < NBX; ++i)
#pragma unroll
        for (int j = 0; j < NBY; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    if (factor == 0)
        jd_project_chunk<RX, RY, 0>(acc, sx, sy, X, md.r, vx, Y, bs.r, vy, md.d_in, w.row0, w.nrows);
    else
        jd_project_chunk<RX, RY, 1>(acc, sx, sy, X, md.r, vx, Y, bs.r, vy, md.d_in, w.row0, w.nrows);

    auto store = [&](double* dst) {   // RX x RY row-major
        const int m = lane >> 2, n2 = 2 * (lane & 3);
#pragma unroll
        for (int i = 0; i < NBX; ++i)
#pragma unroll
            for (int j = 0; j < NBY; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) dst[(8 * i + m) * RY + 8 * (warp * NBY + j) + n2 + e] = acc[i][j][e];
    };
    double* out = a.QP + (int64_t)w.mf * RX * RY;
    const TsqrInfo inf = a.info[w.mf];
    if (inf.nchunks == 1) {
        store(out);
        return;
    }
    store(a.partial + (int64_t)w.slot * RX * RY);
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = (atomicAdd(&a.counters[w.mf], 1) == inf.nchunks - 1);
    __syncthreads();
    if (!s_last) return;
    __threadfence();
    const double* P0 = a.partial + (int64_t)inf.slot0 * RX * RY;
    for (int e = tid; e < RX * RY; e += NT) {
        double s = __ldcg(P0 + e);
        for (int c = 1; c < inf.nchunks; ++c) s += __ldcg(P0 + (int64_t)c * RX * RY + e);
        out[e] = s;
    }
    if (tid == 0) a.counters[w.mf] = 0;   // every chunk has arrived: ready for the next step
}

struct JdCoreArgs {
    const JdMember* members;
    const lf_module* mods;
    const lf_module* basis;
    const JdProbDev* probs;
    const double* QP;        // per mf: RX x RY
    const double* weights;   // per member (nullable = 1)
    float* WZ;               // per mf: W (mf even) / Z (mf odd), RX x RY fp32, rows >= r zero
    float* sigma;            // nullable: Sigma_i = S^T, r~ x r~ fp32 at probs[p].sigma_off + local r~^2
    int32_t write_wz;
};

// One CTA per member: S = P^T Q, W = w P S, Z = w Q S^T, Sigma = S^T.  Every output
// entry is one thread's fixed-order fp64 sum.
template <int RX, int RY>
__global__ void __launch_bounds__(256) jd_core_kernel(JdCoreArgs a) {
    extern __shared__ __align__(16) double js[];
    double* P = js;                  // RX x RY
    double* Q = P + RX * RY;
    double* S = Q + RX * RY;         // RY x (RY + 1): the padded stride keeps S[j][m] reads over j conflict-free
    constexpr int LS = RY + 1;
    const int g = blockIdx.x, tid = threadIdx.x;
    const JdMember mb = a.members[g];
    const int r = a.mods[mb.mod].r, rt = a.basis[mb.prob].r;
    const double* Qg = a.QP + (int64_t)(2 * g) * RX * RY;       // B^T U
    const double* Pg = a.QP + (int64_t)(2 * g + 1) * RX * RY;   // A V
    for (int e = tid; e < RX * RY; e += 256) {
        P[e] = Pg[e];
        Q[e] = Qg[e];
    }
    __syncthreads();
    for (int e = tid; e < rt * rt; e += 256) {
        const int i = e / rt, j = e - i * rt;
        double s = 0.0;
#pragma unroll 4
        for (int l = 0; l < r; ++l) s = fma(P[l * RY + i], Q[l * RY + j], s);
        S[i * LS + j] = s;
    }
    __syncthreads();
    if (a.sigma) {
        const JdProbDev pd = a.probs[mb.prob];
        float* out = a.sigma + pd.sigma_off + (int64_t)mb.local * rt * rt;
        for (int e = tid; e < rt * rt; e += 256) {
            const int i = e / rt, j = e - i * rt;
            out[e] = (float)S[j * LS + i];
        }
    }
    if (!a.write_wz) return;
    const double w = a.weights ? a.weights[g] : 1.0;
    float* W = a.WZ + (int64_t)(2 * g) * RX * RY;
    float* Z = a.WZ + (int64_t)(2 * g + 1) * RX * RY;
    for (int e = tid; e < RX * RY; e += 256) {
        const int l = e / RY, j = e - l * RY;
        double sw = 0.0, sz = 0.0;
        if (l < r && j < rt) {
#pragma unroll 4
            for (int m = 0; m < rt; ++m) {
                sw = fma(P[l * RY + m], S[m * LS + j], sw);
                sz = fma(Q[l * RY + m], S[j * LS + m], sz);
            }
        }
        W[e] = (float)(w * sw);
        Z[e] = (float)(w * sz);
    }
}

template <int RX, int RY>
__host__ __device__ constexpr size_t jd_core_smem() {
    return (size_t)(2 * RX * RY + RY * (RY + 1)) * sizeof(double);
}

template <int RX, int RY>
__host__ __device__ constexpr int jd_update_x_floats() {
    return kJdTR * (RX + 4) > RX * kJdLdM ? kJdTR * (RX + 4) : RX * kJdLdM;
}
template <int RX, int RY>
__host__ __device__ constexpr int jd_update_stage_floats() {
    return jd_update_x_floats<RX, RY>() + RX * (RY + 8);
}
// Epilogue buffers: the finished tile (fp32, [kJdTR][RY + 8]) and the packed Gram sum.
template <int RY>
__host__ __device__ constexpr size_t jd_epilogue_bytes() {
    return (size_t)kJdTR * (RY + 8) * sizeof(float) + (size_t)tri_size<RY>() * sizeof(double);
}
template <int RX, int RY>
__host__ __device__ constexpr size_t jd_update_smem() {
    return 2 * (size_t)jd_update_stage_floats<RX, RY>() * sizeof(float) > jd_epilogue_bytes<RY>()
               ? 2 * (size_t)jd_update_stage_floats<RX, RY>() * sizeof(float)
               : jd_epilogue_bytes<RY>();
}

struct JdUpdArgs {
    const lf_module* mods;
    const JdMember* members;
    const JdProbDev* probs;
    const lf_module* basis_ws;   // output layout (U_0 rows, V_0^T columns in the workspace)
    const float* B_base;
    const float* A_base;
    const float* WZ;
    const JdTile* tiles;
    float* U_ws;
    float* Vt_ws;
    double* gram;                // per tile: packed upper Gram of the finished (fp32) tile, tri_size<RY>()
};

// Stage the member's rows of X (kJdTR rows) and its W (or Z) (r x RY) into one buffer.
template <int RX, int RY, int FACTOR>
__device__ __forceinline__ void jd_update_issue(float* st, const float* X, int r, int d_in, int64_t row0, int nrows,
                                                bool vec, const float* Wm, int tid) {
    constexpr int LX = RX + 4;
    const int r4 = (r + 3) & ~3;
    if (FACTOR == 0) {   // B rows: stage [row][LX]
        if (vec) {
            const int cpr = r >> 2;
            for (int q = tid; q < kJdTR * cpr; q += 128) {
                const int i = q / cpr, c4 = q - i * cpr;
                const bool ok = i < nrows;
                cp_async16_n(st + i * LX + 4 * c4, ok ? X + (row0 + i) * r + 4 * c4 : X, ok ? 16u : 0u);
            }
        } else {
            for (int q = tid; q < kJdTR * r4; q += 128) {
                const int i = q / r4, c = q - i * r4;
                const bool ok = i < nrows && c < r;
                cp_async4_n(st + i * LX + c, ok ? X + (row0 + i) * r + c : X, ok ? 4u : 0u);
            }
        }
    } else {             // A columns row0 .. row0 + kJdTR of rows j < r: stage [j][kJdLdM]
        if (vec) {
            constexpr int cpj = kJdTR / 4;
            for (int q = tid; q < r4 * cpj; q += 128) {
                const int j = q / cpj, i4 = q - j * cpj;
                const int nv = j < r ? min(4, max(0, nrows - 4 * i4)) : 0;
                cp_async16_n(st + j * kJdLdM + 4 * i4, nv > 0 ? X + (int64_t)j * d_in + row0 + 4 * i4 : X,
                             4u * (uint32_t)nv);
            }
        } else {
            for (int q = tid; q < r4 * kJdTR; q += 128) {
                const int j = q / kJdTR, i = q - j * kJdTR;
                const bool ok = j < r && i < nrows;
                cp_async4_n(st + j * kJdLdM + i, ok ? X + (int64_t)j * d_in + row0 + i : X, ok ? 4u : 0u);
            }
        }
    }
    // W / Z rows j < r4 (rows r .. r4 - 1 are zero in the buffer), RY columns
    float* sw = st + jd_update_x_floats<RX, RY>();
    constexpr int cpw = RY / 4;
    for (int q = tid; q < r4 * cpw; q += 128) {
        const int j = q / cpw, c4 = q - j * cpw;
        cp_async16_n(sw + j * (RY + 8) + 4 * c4, Wm + j * RY + 4 * c4, 16u);
    }
}

// CTA (problem, factor, 128-row tile), 4 warps of 32 rows: out rows = sum over the
// problem's members of X_rows (kJdTR x r_i) times W_i (r_i x r~), members in order.
template <int RX, int RY>
__global__ void __launch_bounds__(128) jd_update_kernel(JdUpdArgs a) {
    extern __shared__ __align__(16) float us[];
    constexpr int NBN = RY / 8;
    constexpr int LX = RX + 4, LW = RY + 8;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const JdTile tl = a.tiles[blockIdx.x];
    const JdProbDev pd = a.probs[tl.p];
    const lf_module bw = a.basis_ws[tl.p];
    double acc[4][NBN][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NBN; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

    auto member_src = [&](int gi, const float*& X, int& r, bool& vec, const float*& Wm) {
        const lf_module md = a.mods[a.members[pd.g0 + gi].mod];
        r = md.r;
        if (tl.f == 0) {
            X = a.B_base + md.B_off;
            vec = (md.B_off & 3) == 0 && (r & 3) == 0;
        } else {
            X = a.A_base + md.A_off;
            vec = (md.A_off & 3) == 0 && (md.d_in & 3) == 0;
        }
        Wm = a.WZ + (int64_t)(2 * (pd.g0 + gi) + tl.f) * RX * RY;
    };
    auto issue = [&](int gi, float* st) {
        const float* X;
        const float* Wm;
        int r;
        bool vec;
        member_src(gi, X, r, vec, Wm);
        const int d_in = a.mods[a.members[pd.g0 + gi].mod].d_in;
        if (tl.f == 0)
            jd_update_issue<RX, RY, 0>(st, X, r, d_in, tl.row0, tl.nrows, vec, Wm, tid);
        else
            jd_update_issue<RX, RY, 1>(st, X, r, d_in, tl.row0, tl.nrows, vec, Wm, tid);
    };
    constexpr int SF = jd_update_stage_floats<RX, RY>();
    if (pd.count > 0) issue(0, us);
    tc::cp_async_commit();
    for (int gi = 0; gi < pd.count; ++gi) {
        if (gi + 1 < pd.count) issue(gi + 1, us + ((gi + 1) & 1) * SF);
        tc::cp_async_commit();
        tc::cp_async_wait<1>();
        __syncthreads();
        const float* st = us + (gi & 1) * SF;
        const float* sw = st + jd_update_x_floats<RX, RY>();
        const int r = a.mods[a.members[pd.g0 + gi].mod].r;
        const int nks = (r + 3) >> 2;
        // A operand: X[row 32 warp + 8 bm + lane/4][j = 4 ks + lane%4]
        const int rl = 32 * warp + (lane >> 2), jl = lane & 3;
        for (int ks = 0; ks < nks; ++ks) {
            const int j = 4 * ks + jl;
            double xa[4], wb[NBN];
#pragma unroll
            for (int bm = 0; bm < 4; ++bm)
                xa[bm] = tl.f == 0 ? (double)st[(rl + 8 * bm) * LX + j] : (double)st[j * kJdLdM + rl + 8 * bm];
#pragma unroll
            for (int bn = 0; bn < NBN; ++bn) wb[bn] = (double)sw[j * LW + 8 * bn + (lane >> 2)];
#pragma unroll
            for (int bm = 0; bm < 4; ++bm)
#pragma unroll
                for (int bn = 0; bn < NBN; ++bn) dmma_8x8x4(acc[bm][bn], xa[bm], wb[bn]);
        }
        __syncthreads();   // the buffer is refilled by the next iteration's issue
    }
    tc::cp_async_wait<0>();
    __syncthreads();
    // epilogue: round the tile to fp32 in shared memory, store it, and form its Gram
    // (the first, row-tile level of the orthogonalize TSQR) from the stored values
    constexpr int LT = RY + 8;
    float* tile = us;
    const int rt = bw.r;
#pragma unroll
    for (int bm = 0; bm < 4; ++bm) {
        const int row = 32 * warp + 8 * bm + (lane >> 2);
#pragma unroll
        for (int bn = 0; bn < NBN; ++bn)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int c = 8 * bn + 2 * (lane & 3) + e;
                tile[row * LT + c] = (row < tl.nrows && c < rt) ? (float)acc[bm][bn][e] : 0.f;
            }
    }
    __syncthreads();
    if (tl.f == 0) {
        float* out = a.U_ws + bw.B_off + (int64_t)tl.row0 * rt;
        for (int i = tid; i < tl.nrows * rt; i += 128) {
            const int row = i / rt, c = i - row * rt;
            out[i] = tile[row * LT + c];
        }
    } else {
        for (int i = tid; i < rt * tl.nrows; i += 128) {
            const int c = i / tl.nrows, row = i - c * tl.nrows;
            a.Vt_ws[bw.A_off + (int64_t)c * bw.d_in + tl.row0 + row] = tile[row * LT + c];
        }
    }
    constexpr int NB = RY / 8, NP = NB * (NB + 1) / 2;
    double g[NP][2];
#pragma unroll
    for (int q = 0; q < NP; ++q) g[q][0] = g[q][1] = 0.0;
    const float* fb = tile + (32 * warp + (lane & 3)) * LT + (lane >> 2);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
        double f[NB];
#pragma unroll
        for (int b = 0; b < NB; ++b) f[b] = (double)fb[ks * 4 * LT + 8 * b];
        int q = 0;
#pragma unroll
        for (int bi = 0; bi < NB; ++bi)
#pragma unroll
            for (int bj = bi; bj < NB; ++bj) dmma_8x8x4(g[q++], f[bi], f[bj]);
    }
    double* red = reinterpret_cast<double*>(tile + kJdTR * LT);
    for (int w = 0; w < 4; ++w) {   // the four warps' row blocks, summed in order
        if (warp == w) {
            const int m = lane >> 2, n2 = 2 * (lane & 3);
            int q = 0;
#pragma unroll
            for (int bi = 0; bi < NB; ++bi)
#pragma unroll
                for (int bj = bi; bj < NB; ++bj, ++q)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int row = 8 * bi + m, col = 8 * bj + n2 + e;
                        if (col >= row) {
                            const int o = tri_off<RY>(row, col);
                            red[o] = (w == 0 ? 0.0 : red[o]) + g[q][e];
                        }
                    }
        }
        __syncthreads();
    }
    double* slot = a.gram + (int64_t)blockIdx.x * tri_size<RY>();
    for (int e = tid; e < tri_size<RY>(); e += 128) slot[e] = red[e];
}

// Per (problem, factor): the tile Grams summed in tile order (one thread per packed
// entry, CTAs over slices of the triangle).
struct JdGramSumArgs {
    const int32_t* tile0;    // per mf: first tile (tiles of one mf are consecutive)
    const int32_t* ntiles;   // per mf
    const double* gram;      // per tile
    double* G;               // per mf: packed Gram
};

template <int RT>
__global__ void __launch_bounds__(128) jd_gram_sum_kernel(JdGramSumArgs a) {
    constexpr int TRI = tri_size<RT>();
    const int mf = blockIdx.x, e = blockIdx.y * 128 + threadIdx.x;
    if (e >= TRI) return;
    const int nt = a.ntiles[mf];
    const double* src = a.gram + (int64_t)a.tile0[mf] * TRI + e;
    double s = 0.0;
#pragma unroll 8
    for (int t = 0; t < nt; ++t) s += src[(int64_t)t * TRI];
    a.G[(int64_t)mf * TRI + e] = s;
}

// Upper-triangular inverse of the r x r R held in the upper triangle of `A` (dense,
// stride RT + 1), by rows from the last: row i of R^-1 needs only rows > i.  Entry
// (l, j), l < j, is written to A[j][l] (the unused lower triangle), the diagonal to
// `dinv`.  Called by all `nt` threads of the block; columns j >= bad are zero.
// Four threads share each entry's dot product (strided terms, combined by shuffles in a
// fixed order); nt must be a multiple of 128.
template <int RT>
__device__ __forceinline__ void jd_upper_inverse(double (*A)[RT + 1], double* dinv, int r, int bad, int tid, int nt) {
    const int part = tid & 3;
    for (int i = r - 1; i >= 0; --i) {
        for (int j0 = i; j0 < i + RT; j0 += nt / 4) {   // uniform trip count: shuffles stay converged
            const int j = j0 + (tid >> 2);
            const bool live = j < r;
            double v = 0.0;
            if (live && j > i && j < bad) {
                if (part == 0) v = A[i][j] * dinv[j];   // l = j term
                for (int l = i + 1 + part; l < j; l += 4) v = fma(A[i][l], A[j][l], v);
            }
            v += __shfl_xor_sync(0xffffffffu, v, 1);
            v += __shfl_xor_sync(0xffffffffu, v, 2);
            if (live && part == 0) {
                if (j >= bad) {
                    if (j == i) dinv[i] = 0.0;
                    else A[j][i] = 0.0;
                } else if (j == i) {
                    dinv[i] = 1.0 / A[i][i];
                } else {
                    A[j][i] = -v / A[i][i];
                }
            }
        }
        __syncthreads();
    }
}

template <int RT>
__device__ __forceinline__ void jd_store_inverse(const double (*A)[RT + 1], const double* dinv, int r, double* out,
                                                 int rs, int tid, int nt) {
    for (int e = tid; e < rs * rs; e += nt) {
        const int l = e / rs, j = e - l * rs;
        out[e] = (l < r && j < r && j >= l) ? (j == l ? dinv[l] : A[j][l]) : 0.0;
    }
}

// Per (problem, factor), 256 threads: G = R^T R by fp64 Cholesky (the TSQR root; the
// same pivot rule as the Gram leaf), then R^-1.  A rejected pivot marks the matrix in
// `flags`; its R then comes from the Householder TSQR and jd_rinv_kernel inverts it.
struct JdCholArgs {
    const lf_module* basis;
    const double* G;         // per mf: packed Gram
    double* Rinv;            // per mf: rs x rs
    int32_t* flags;          // per mf, zero on entry
    int32_t rs;
};

template <int RT>
__global__ void __launch_bounds__(256) jd_chol_kernel(JdCholArgs a) {
    __shared__ double A[RT][RT + 1];
    __shared__ double s_diag[RT];
    __shared__ double dinv[RT];
    __shared__ int s_fail;
    const int mf = blockIdx.x, tid = threadIdx.x;
    const int r = a.basis[mf >> 1].r;
    const double* Gp = a.G + (int64_t)mf * tri_size<RT>();
    for (int e = tid; e < RT * RT; e += 256) {
        const int j = e / RT, c = e - j * RT;
        if (c >= j) A[j][c] = Gp[tri_off<RT>(j, c)];
    }
    if (tid < RT) s_diag[tid] = Gp[tri_off<RT>(tid, tid)];
    if (tid == 0) s_fail = 0;
    __syncthreads();
    for (int j = 0; j < r; ++j) {
        if (tid == 0) {
            const double d = A[j][j];
            if (!(d > kGramPivotTol * s_diag[j])) s_fail = 1;
            else A[j][j] = sqrt(d);
        }
        __syncthreads();
        if (s_fail) {
            if (tid == 0) a.flags[mf] = 1;
            return;
        }
        const double rjj = A[j][j];
        for (int c = j + 1 + tid; c < r; c += 256) A[j][c] /= rjj;
        __syncthreads();
        // trailing update of rows k > j: 8 warps over rows, lanes over columns
        for (int k = j + 1 + (tid >> 5); k < r; k += 8) {
            const double gjk = A[j][k];
            for (int c = k + (tid & 31); c < r; c += 32) A[k][c] -= gjk * A[j][c];
        }
        __syncthreads();
    }
    jd_upper_inverse<RT>(A, dinv, r, r, tid, 256);
    jd_store_inverse<RT>(A, dinv, r, a.Rinv + (int64_t)mf * a.rs * a.rs, a.rs, tid, 256);
}

// Per (problem, factor) whose R comes from elsewhere: R^-1 of the Householder TSQR's
// fp32 R (use32[mf] set) or of an fp64 R.  A diagonal entry that is not positive and
// finite (the update is numerically rank deficient) latches LF_ERR_NUMERIC; the columns
// from there on are zero.
struct JdRinvArgs {
    const lf_module* basis;
    const int32_t* only;     // per mf (nullable): zero = skip
    const int32_t* use32;    // per mf
    const double* R64;       // per mf, rs x rs
    const float* R_B;        // per problem, rs x rs
    const float* R_A;
    double* Rinv;            // per mf, rs x rs
    int32_t rs;
};

template <int RT>
__global__ void __launch_bounds__(128) jd_rinv_kernel(JdRinvArgs a) {
    __shared__ double A[RT][RT + 1];
    __shared__ double dinv[RT];
    const int mf = blockIdx.x, tid = threadIdx.x;
    if (a.only && a.only[mf] == 0) return;
    const int r = a.basis[mf >> 1].r;
    for (int e = tid; e < r * r; e += 128) {
        const int j = e / r, c = e - j * r;
        if (c >= j)
            A[j][c] = a.use32[mf] ? (double)((mf & 1) == 0 ? a.R_B : a.R_A)[(int64_t)(mf >> 1) * a.rs * a.rs + j * a.rs + c]
                                  : a.R64[(int64_t)mf * a.rs * a.rs + j * a.rs + c];
    }
    __syncthreads();
    int bad = r;
    for (int j = 0; j < r; ++j)
        if (!(A[j][j] > 0.0) || !isfinite(A[j][j])) {
            bad = j;
            break;
        }
    if (bad < r && tid == 0) latch_error(LF_ERR_NUMERIC);
    jd_upper_inverse<RT>(A, dinv, r, bad, tid, 128);
    jd_store_inverse<RT>(A, dinv, r, a.Rinv + (int64_t)mf * a.rs * a.rs, a.rs, tid, 128);
}

struct JdQArgs {
    const lf_module* src;    // per problem: B_off / A_off of X in src_U / src_Vt
    const float* src_U;
    const float* src_Vt;
    const lf_module* dst;    // per problem: where Q goes
    float* dst_U;
    float* dst_Vt;
    const lf_module* alt;    // per problem: where Q goes when route[mf] != 0
    float* alt_U;
    float* alt_Vt;
    const int32_t* route;    // per mf (nullable)
    const int32_t* only;     // per mf (nullable): zero = leave this matrix alone
    const double* Rinv;      // per mf, rs x rs
    int32_t rs;
    const JdTile* tiles;
};

template <int RT>
__host__ __device__ constexpr size_t jd_qform_smem() {
    return (size_t)kJdTR * (RT + 4) * sizeof(float) + (size_t)RT * (RT + 8) * sizeof(double);
}

// Q = X R^-1 on one 128-row tile: a fp64 tensor-core product of the staged fp32 tile
// with the fp64 R^-1, 4 warps of 32 rows.
template <int RT>
__global__ void __launch_bounds__(kJdTR) jd_qform_kernel(JdQArgs a) {
    extern __shared__ __align__(16) double qs[];
    constexpr int LX = RT + 4, LR = RT + 8, NBN = RT / 8;
    double* sRi = qs;                                           // RT x LR
    float* sx = reinterpret_cast<float*>(qs + RT * LR);         // kJdTR x LX
    const JdTile tl = a.tiles[blockIdx.x];
    const int mf = 2 * tl.p + tl.f;
    if (a.only && a.only[mf] == 0) return;
    const lf_module s = a.src[tl.p];
    const bool to_alt = a.route && a.route[mf] != 0;
    const lf_module d = to_alt ? a.alt[tl.p] : a.dst[tl.p];
    float* dU = to_alt ? a.alt_U : a.dst_U;
    float* dVt = to_alt ? a.alt_Vt : a.dst_Vt;
    const int rt = s.r, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const double* Ri = a.Rinv + (int64_t)mf * a.rs * a.rs;
    for (int e = tid; e < RT * RT; e += kJdTR) {
        const int i = e / RT, j = e - i * RT;
        sRi[i * LR + j] = (i < rt && j < rt) ? Ri[i * a.rs + j] : 0.0;
    }
    if (tl.f == 0) {
        const float* x = a.src_U + s.B_off + (int64_t)tl.row0 * rt;
        for (int e = tid; e < kJdTR * RT; e += kJdTR) {
            const int i = e / RT, c = e - i * RT;
            sx[i * LX + c] = (i < tl.nrows && c < rt) ? x[i * rt + c] : 0.f;
        }
    } else {
        const float* x = a.src_Vt + s.A_off + tl.row0;
        for (int e = tid; e < kJdTR * RT; e += kJdTR) {
            const int c = e / kJdTR, i = e - c * kJdTR;
            sx[i * LX + c] = (i < tl.nrows && c < rt) ? x[(int64_t)c * s.d_in + i] : 0.f;
        }
    }
    __syncthreads();
    double acc[4][NBN][2];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NBN; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
    const int rl = 32 * warp + (lane >> 2);
#pragma unroll
    for (int ks = 0; ks < RT / 4; ++ks) {
        const int l = 4 * ks + (lane & 3);
        double xa[4], rb[NBN];
#pragma unroll
        for (int bm = 0; bm < 4; ++bm) xa[bm] = (double)sx[(rl + 8 * bm) * LX + l];
#pragma unroll
        for (int bn = 0; bn < NBN; ++bn) rb[bn] = sRi[l * LR + 8 * bn + (lane >> 2)];
#pragma unroll
        for (int bm = 0; bm < 4; ++bm)
#pragma unroll
            for (int bn = 0; bn < NBN; ++bn) dmma_8x8x4(acc[bm][bn], xa[bm], rb[bn]);
    }
#pragma unroll
    for (int bm = 0; bm < 4; ++bm) {
        const int row = rl + 8 * bm;
        if (row >= tl.nrows) continue;
        const int64_t grow = tl.row0 + row;
#pragma unroll
        for (int bn = 0; bn < NBN; ++bn)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int c = 8 * bn + 2 * (lane & 3) + e;
                if (c >= rt) continue;
                if (tl.f == 0)
                    dU[d.B_off + grow * rt + c] = (float)acc[bm][bn][e];
                else
                    dVt[d.A_off + (int64_t)c * d.d_in + grow] = (float)acc[bm][bn][e];
            }
    }
}

}  // namespace lf
