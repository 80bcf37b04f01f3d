// Batched tall-skinny QR (FlashTSQR-style) and the small fp64 SVD of R_B R_A^T.
//
// LoRAForge (kongchang.com), "FlashTSQR: An Accelerator for Batched Factor
// Construction": TSQR factors a tall-skinny matrix by local QR of row blocks and
// then merges; the parallelism runs across modules and across row tiles.
// "Compress then Serve" (academ.us/article/2407.00066), section 4, eq. 4: the
// per-module SVD of dW = B A, here taken in factor space as the SVD of
// M = R_B R_A^T (dW = Q_B M Q_A^T).
//
// Work decomposition: every (module, factor) matrix X (B: d_out x r, or A^T:
// d_in x r) is cut into chunks of at most kTsqrChunk rows; one CTA owns one chunk
// and folds its row tiles into a running R by structured Householder reflections
// of [R; tile].  Chunk results are merged by the last CTA of the matrix to finish
// (atomic counter, no waiting), always in chunk order, so the result does not
// depend on scheduling.
#pragma once
#include "common.cuh"

namespace lf {

constexpr int kTsqrChunk = 2048;   // rows per work item
constexpr int kTsqrTM = 128;       // rows per smem tile
constexpr int kTsqrThreads = 256;

struct TsqrWork {
    int32_t mf;      // 2 * local module index + factor (0 = B, 1 = A^T)
    int32_t row0;    // first row of the chunk
    int32_t nrows;   // rows in the chunk
    int32_t slot;    // partial-R slot (-1 when the matrix has one chunk)
};
struct TsqrInfo {
    int32_t nchunks;
    int32_t slot0;
};

template <typename T>
struct TsqrArgs {
    const lf_module* mods;      // device copy of the module table
    const int32_t* mod_ids;     // local -> global module index (nullptr = identity)
    const float* B_base;
    const float* A_base;
    const TsqrWork* work;
    const int32_t* n_work;      // device scalar
    const TsqrInfo* info;       // per local mf
    int32_t* counters;          // per local mf, zero on entry
    T* partial;                 // slots x RT x RT
    T* R_B;                     // per local module, rs x rs
    T* R_A;
    int32_t rs;
};

template <typename T, int RT, int TM>
struct TsqrSmem {
    T R[RT][RT + 1];
    T tile[TM][RT + 1];
    T v[TM];
    T scal[2];
    int flag;
};

// Structured Householder QR of the stacked [R (RT x RT upper); tile (TM x RT)],
// columns 0..ncols-1; R is overwritten with the new triangle, the tile is consumed.
// Reflector j touches row j of R and every tile row (LAPACK tpqrt-style).
template <typename T, int RT, int TM, int NT>
__device__ void absorb_tile(TsqrSmem<T, RT, TM>& s, int ncols) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = NT / 32;
    for (int j = 0; j < ncols; ++j) {
        if (warp == 0) {
            T ss = 0;
            for (int i = lane; i < TM; i += 32) {
                T x = s.tile[i][j];
                ss += x * x;
            }
            ss = warp_sum(ss);
            if (lane == 0) {
                T x0 = s.R[j][j];
                T tau = 0, scale = 0;
                if (ss > T(0)) {
                    T nrm = sqrt(x0 * x0 + ss);
                    T beta = x0 >= T(0) ? -nrm : nrm;
                    tau = (beta - x0) / beta;
                    scale = T(1) / (x0 - beta);
                    s.R[j][j] = beta;
                }
                s.scal[0] = tau;
                s.scal[1] = scale;
            }
        }
        __syncthreads();
        const T tau = s.scal[0];
        const T scale = s.scal[1];
        if (tau == T(0)) {
            __syncthreads();
            continue;
        }
        for (int i = tid; i < TM; i += NT) s.v[i] = s.tile[i][j] * scale;
        __syncthreads();
        for (int c = j + 1 + warp; c < ncols; c += NW) {
            T d = 0;
            for (int i = lane; i < TM; i += 32) d += s.v[i] * s.tile[i][c];
            d = warp_sum(d);
            const T w = (s.R[j][c] + d) * tau;
            __syncwarp();
            if (lane == 0) s.R[j][c] -= w;
            for (int i = lane; i < TM; i += 32) s.tile[i][c] -= w * s.v[i];
        }
        __syncthreads();
    }
}

template <typename T, int RT, int TM, int NT>
__device__ void load_tile(TsqrSmem<T, RT, TM>& s, const float* __restrict__ X, int factor,
                          int64_t row_base, int nr, int r, int ld) {
    // factor 0: X = B (row-major, ld = r);  factor 1: X = A^T, A row-major (ld = d_in)
    if (factor == 0) {
        for (int e = threadIdx.x; e < TM * RT; e += NT) {
            const int i = e / RT, c = e % RT;
            T v = 0;
            if (i < nr && c < r) v = (T)__ldg(X + (row_base + i) * (int64_t)r + c);
            s.tile[i][c] = v;
        }
    } else {
        for (int e = threadIdx.x; e < TM * RT; e += NT) {
            const int c = e / TM, i = e % TM;
            T v = 0;
            if (i < nr && c < r) v = (T)__ldg(X + (int64_t)c * ld + row_base + i);
            s.tile[i][c] = v;
        }
    }
}

template <typename T, int RT, int TM, int NT>
__device__ void write_final(TsqrSmem<T, RT, TM>& s, T* out, int r, int rs) {
    // canonical sign: diag(R) >= 0 (flip whole rows)
    for (int e = threadIdx.x; e < rs * rs; e += NT) {
        const int j = e / rs, c = e % rs;
        T v = 0;
        if (j < r && c < r && c >= j) {
            v = s.R[j][c];
            if (s.R[j][j] < T(0)) v = -v;
        }
        out[e] = v;
    }
}

template <typename T, int RT, int TM, int NT>
__global__ void __launch_bounds__(NT) tsqr_kernel(TsqrArgs<T> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& s = *reinterpret_cast<TsqrSmem<T, RT, TM>*>(smem_raw);
    const int wi = blockIdx.x;
    if (wi >= *a.n_work) return;
    const TsqrWork w = a.work[wi];
    const int local = w.mf >> 1, factor = w.mf & 1;
    const int gm = a.mod_ids ? a.mod_ids[local] : local;
    const lf_module md = a.mods[gm];
    const int r = md.r;
    const float* X = factor == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
    const int ld = factor == 0 ? r : md.d_in;

    for (int e = threadIdx.x; e < RT * (RT + 1); e += NT) (&s.R[0][0])[e] = T(0);
    for (int t0 = 0; t0 < w.nrows; t0 += TM) {
        const int nr = min(TM, w.nrows - t0);
        __syncthreads();
        load_tile<T, RT, TM, NT>(s, X, factor, (int64_t)w.row0 + t0, nr, r, ld);
        __syncthreads();
        absorb_tile<T, RT, TM, NT>(s, r);
    }
    __syncthreads();

    T* out = (factor == 0 ? a.R_B : a.R_A) + (size_t)local * a.rs * a.rs;
    const TsqrInfo inf = a.info[w.mf];
    if (inf.nchunks == 1) {
        write_final<T, RT, TM, NT>(s, out, r, a.rs);
        return;
    }
    T* P = a.partial + (size_t)w.slot * RT * RT;
    for (int e = threadIdx.x; e < RT * RT; e += NT) P[e] = s.R[e / RT][e % RT];
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const int prev = atomicAdd(&a.counters[w.mf], 1);
        s.flag = (prev == inf.nchunks - 1);
    }
    __syncthreads();
    if (!s.flag) return;
    __threadfence();
    // fold the chunk triangles in chunk order: R = R_0, then R <- R([R; R_c])
    const T* P0 = a.partial + (size_t)inf.slot0 * RT * RT;
    for (int e = threadIdx.x; e < RT * RT; e += NT) s.R[e / RT][e % RT] = __ldcg(P0 + e);
    for (int c = 1; c < inf.nchunks; ++c) {
        const T* Pc = a.partial + (size_t)(inf.slot0 + c) * RT * RT;
        __syncthreads();
        for (int e = threadIdx.x; e < TM * RT; e += NT) {
            const int i = e / RT, col = e % RT;
            s.tile[i][col] = i < RT ? __ldcg(Pc + i * RT + col) : T(0);
        }
        __syncthreads();
        absorb_tile<T, RT, TM, NT>(s, r);
    }
    __syncthreads();
    write_final<T, RT, TM, NT>(s, out, r, a.rs);
}

// ----------------------------------------------------------------------------
// Small SVD: M = R_B R_A^T (r x r, fp64), one-sided Jacobi on the rows of M.
// Rotating rows p, q of M by the same plane rotation that is applied to columns
// p, q of U (U starts at I) keeps M = U M'; at convergence the rows of M' are
// orthogonal, sigma_p = |m'_p|, and row p of M' is sigma_p v_p^T.
// ----------------------------------------------------------------------------
constexpr int kSvdThreads = 128;

template <typename TIN>
struct SvdArgs {
    const lf_module* mods;
    const int32_t* mod_ids;   // local -> global (nullptr = identity)
    const int32_t* n;         // device scalar: number of local modules
    const TIN* R_B;
    const TIN* R_A;
    double* sigma;            // per local module, rs
    double* U;                // per local module, rs x rs (may be nullptr)
    double* V;                // per local module, rs x rs (may be nullptr)
    int32_t rs;
    int32_t max_sweeps;
};

template <int RT>
struct SvdSmem {
    double M[RT][RT + 1];
    double Ut[RT][RT + 1];
    double sig[RT];
    int perm[RT];
    int rot;
};

template <typename TIN, int RT>
__global__ void __launch_bounds__(kSvdThreads) svd_kernel(SvdArgs<TIN> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    auto& s = *reinterpret_cast<SvdSmem<RT>*>(smem_raw);
    const int local = blockIdx.x;
    if (local >= *a.n) return;
    const int gm = a.mod_ids ? a.mod_ids[local] : local;
    const int r = a.mods[gm].r;
    const int rs = a.rs;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    constexpr int NW = kSvdThreads / 32;
    const TIN* RB = a.R_B + (size_t)local * rs * rs;
    const TIN* RA = a.R_A + (size_t)local * rs * rs;

    // M[i][j] = sum_{l >= max(i,j)} R_B[i][l] R_A[j][l]
    for (int e = tid; e < r * r; e += kSvdThreads) {
        const int i = e / r, j = e % r;
        double acc = 0.0;
        for (int l = max(i, j); l < r; ++l) acc += (double)RB[i * rs + l] * (double)RA[j * rs + l];
        s.M[i][j] = acc;
    }
    for (int e = tid; e < r * r; e += kSvdThreads) {
        const int i = e / r, j = e % r;
        s.Ut[i][j] = i == j ? 1.0 : 0.0;
    }
    __syncthreads();

    const int rp = (r + 1) & ~1;  // even number of players (index r is a bye when r is odd)
    const double tol = 1e-15;
    for (int sweep = 0; sweep < a.max_sweeps; ++sweep) {
        if (tid == 0) s.rot = 0;
        __syncthreads();
        for (int t = 0; t < rp - 1; ++t) {
            for (int pi = warp; pi < rp / 2; pi += NW) {
                int p, q;
                if (pi == 0) {
                    p = rp - 1;
                    q = t;
                } else {
                    p = (t + pi) % (rp - 1);
                    q = (t - pi + rp - 1) % (rp - 1);
                }
                if (p >= r || q >= r) continue;
                double al = 0, be = 0, ga = 0;
                for (int l = lane; l < r; l += 32) {
                    const double x = s.M[p][l], y = s.M[q][l];
                    al += x * x;
                    be += y * y;
                    ga += x * y;
                }
                al = warp_sum(al);
                be = warp_sum(be);
                ga = warp_sum(ga);
                if (ga == 0.0 || fabs(ga) <= tol * sqrt(al * be)) continue;
                const double zeta = (be - al) / (2.0 * ga);
                const double tt = (zeta >= 0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                const double c = 1.0 / sqrt(1.0 + tt * tt);
                const double sn = c * tt;
                for (int l = lane; l < r; l += 32) {
                    const double x = s.M[p][l], y = s.M[q][l];
                    s.M[p][l] = c * x - sn * y;
                    s.M[q][l] = sn * x + c * y;
                    const double u = s.Ut[p][l], v = s.Ut[q][l];
                    s.Ut[p][l] = c * u - sn * v;
                    s.Ut[q][l] = sn * u + c * v;
                }
                if (lane == 0) s.rot = 1;
            }
            __syncthreads();
        }
        const int any = s.rot;
        __syncthreads();
        if (!any) break;
    }

    for (int p = warp; p < r; p += NW) {
        double nn = 0;
        for (int l = lane; l < r; l += 32) nn += s.M[p][l] * s.M[p][l];
        nn = warp_sum(nn);
        if (lane == 0) s.sig[p] = sqrt(nn);
    }
    __syncthreads();
    // descending order, ties by index
    for (int p = tid; p < r; p += kSvdThreads) {
        const double sp = s.sig[p];
        int rank = 0;
        for (int q = 0; q < r; ++q) {
            const double sq = s.sig[q];
            rank += (sq > sp) || (sq == sp && q < p);
        }
        s.perm[rank] = p;
        if (!isfinite(sp)) latch_error(LF_ERR_NUMERIC);
    }
    __syncthreads();
    double* sg = a.sigma + (size_t)local * rs;
    for (int j = tid; j < rs; j += kSvdThreads) sg[j] = j < r ? s.sig[s.perm[j]] : 0.0;
    if (a.U) {
        double* Uo = a.U + (size_t)local * rs * rs;
        for (int e = tid; e < rs * rs; e += kSvdThreads) {
            const int row = e / rs, j = e % rs;
            Uo[e] = (row < r && j < r) ? s.Ut[s.perm[j]][row] : 0.0;
        }
    }
    if (a.V) {
        double* Vo = a.V + (size_t)local * rs * rs;
        for (int e = tid; e < rs * rs; e += kSvdThreads) {
            const int row = e / rs, j = e % rs;
            double v = 0.0;
            if (row < r && j < r) {
                const int p = s.perm[j];
                const double sp = s.sig[p];
                v = sp > 0.0 ? s.M[p][row] / sp : 0.0;
            }
            Vo[e] = v;
        }
    }
}

}  // namespace lf
