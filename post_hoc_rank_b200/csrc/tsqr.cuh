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
// d_in x r) is cut into chunks of at most kTsqrChunk rows; one warp owns one chunk
// and folds its 32-row register tiles into a running R by structured Householder
// reflections of [R; tile].  Chunk results are merged by the last warp of the
// matrix to finish (atomic counter, no waiting), always in chunk order, so the
// result does not depend on scheduling.
#pragma once
#include "common.cuh"

#include <type_traits>

namespace lf {

constexpr int kTsqrChunk = 2048;   // rows per work item (one warp)
constexpr int kTsqrTM = 32;        // rows per register tile
// warps (independent work items) per CTA: the packed R of every warp lives in static
// shared memory (fp32 RT=64: 8.3 KB per warp; fp64: 16.6 KB).  fp32 uses one warp
// per CTA so a short chunk never holds a finished warp resident.
template <typename T>
__host__ __device__ constexpr int tsqr_warps() { return sizeof(T) == 8 ? 2 : 1; }

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
    int32_t* counters;          // per local mf (tree: per slot), zero on entry
    T* partial;                 // slots x RT x RT (tree: slots x packed triangle)
    T* R_B;                     // per local module, rs x rs
    T* R_A;
    int32_t rs;
    const int32_t* only;        // per local mf (nullable): nonzero = factor this matrix, zero = skip it
    // 0: the last chunk of a matrix to finish folds every chunk R in chunk order (dense
    //    RT x RT slots, counters per mf);
    // 1: binary merge tree over the chunks (packed triangle slots, one slot and one
    //    counter per tree node: see tree_slots)
    int32_t tree;
};

// Nodes of the binary merge tree over n chunks, every level included: level 0 holds
// the n chunks, level l + 1 the ceil(n_l / 2) merges of level l, up to one root.  Node
// i of level l has slot (and counter) slot0 + (nodes below level l) + i.
__host__ __device__ inline int tree_slots(int n) {
    int t = 0;
    for (int m = n; ; m = (m + 1) >> 1) {
        t += m;
        if (m == 1) break;
    }
    return t;
}

// Packed upper triangle of an RT x RT matrix, row-major: row j holds columns j..RT-1.
template <int RT>
__device__ __forceinline__ int tri_off(int j, int c) { return j * RT - (j * (j - 1)) / 2 + (c - j); }
template <int RT>
__host__ __device__ constexpr int tri_size() { return RT * (RT + 1) / 2; }

// Column ownership inside a warp: RT = 64 -> lane l owns columns l and 63 - l
// (keeps the shrinking trailing triangle spread over the most lanes); RT <= 32 ->
// lane l owns column l.
template <int RT>
struct Cols {
    static constexpr int NS = RT > 32 ? 2 : 1;
    __device__ static int col(int lane, int s) { return s == 0 ? lane : RT - 1 - lane; }
    __device__ static int owner(int j) { return (RT > 32 && j >= 32) ? RT - 1 - j : j; }
    __device__ static int slot(int j) { return (RT > 32 && j >= 32) ? 1 : 0; }
};

// One warp folds a TM x RT tile (registers x[s][i] = X[i][col(lane, s)]) into the
// running triangle Rp (packed, shared memory) by structured Householder reflections
// of [R; tile]: reflector j involves row j of R and every tile row, so
//   beta_j = -sign(R_jj) ||[R_jj; X_:j]||,  tau = (beta - R_jj) / beta,
//   v = [1; X_:j / (R_jj - beta)],  w_c = tau (R_jc + v^T X_:c),
//   R_jc -= w_c,  X_:c -= w_c v   for c > j.
// All dot products are over the lane's own rows; the reflector column is published
// once through shared memory.
template <typename T>
__device__ __forceinline__ T quick_div(T a, T b) { return a / b; }
template <>
__device__ __forceinline__ float quick_div<float>(float a, float b) { return __fdividef(a, b); }

template <typename T, int RT>
__device__ __forceinline__ void warp_absorb(T (&x)[Cols<RT>::NS][kTsqrTM], T* Rp, T* vbuf, int r) {
    const int lane = threadIdx.x & 31;
    using C = Cols<RT>;
    constexpr int VW = 16 / sizeof(T);   // elements per 16-byte vector
    using V = typename std::conditional<sizeof(T) == 4, float4, double2>::type;
    for (int j = 0; j < r; ++j) {
        const int own = C::owner(j), sl = C::slot(j);
        if (lane == own) {   // publish column j (16-byte stores)
            V* dst = reinterpret_cast<V*>(vbuf);
            if (sl == 0) {
#pragma unroll
                for (int i = 0; i < kTsqrTM; i += VW) dst[i / VW] = *reinterpret_cast<const V*>(&x[0][i]);
            } else {
#pragma unroll
                for (int i = 0; i < kTsqrTM; i += VW) dst[i / VW] = *reinterpret_cast<const V*>(&x[C::NS - 1][i]);
            }
        }
        __syncwarp();
        T v[kTsqrTM];
#pragma unroll
        for (int i = 0; i < kTsqrTM; i += VW) *reinterpret_cast<V*>(&v[i]) = reinterpret_cast<const V*>(vbuf)[i / VW];
        const T x0 = Rp[tri_off<RT>(j, j)];
        __syncwarp();
        T s4[4] = {0, 0, 0, 0};   // every lane forms the column norm from its copy of v
#pragma unroll
        for (int i = 0; i < kTsqrTM; ++i) s4[i & 3] = fma(v[i], v[i], s4[i & 3]);
        const T ss = (s4[0] + s4[1]) + (s4[2] + s4[3]);
        if (ss == T(0)) continue;  // column already zero below R_jj: H = I (warp-uniform)
        const T nrm = sqrt(fma(x0, x0, ss));
        const T beta = x0 >= T(0) ? -nrm : nrm;
        const T tau = quick_div(beta - x0, beta);
        const T scale = quick_div(T(1), x0 - beta);
        if (lane == 0) Rp[tri_off<RT>(j, j)] = beta;
#pragma unroll
        for (int s = 0; s < C::NS; ++s) {
            const int c = C::col(lane, s);
            if (c > j && c < r) {
                T d4[4] = {0, 0, 0, 0};
#pragma unroll
                for (int i = 0; i < kTsqrTM; ++i) d4[i & 3] = fma(v[i], x[s][i], d4[i & 3]);
                const T d = (d4[0] + d4[1]) + (d4[2] + d4[3]);
                const int o = tri_off<RT>(j, c);
                const T w = tau * fma(scale, d, Rp[o]);
                Rp[o] -= w;
                const T a = w * scale;
#pragma unroll
                for (int i = 0; i < kTsqrTM; ++i) x[s][i] = fma(-a, v[i], x[s][i]);
            }
        }
        __syncwarp();
    }
}

template <typename T, int RT>
__device__ __forceinline__ void load_rows(T (&x)[Cols<RT>::NS][kTsqrTM], const float* __restrict__ X, int factor,
                                          int64_t row_base, int nr, int r, int ld) {
    const int lane = threadIdx.x & 31;
    using C = Cols<RT>;
#pragma unroll
    for (int s = 0; s < C::NS; ++s) {
        const int c = C::col(lane, s);
        const bool okc = c < r;
        if (factor == 0) {  // X = B, row-major d_out x r: X[i][c] = B[(row_base+i)*r + c]
            const float* p = X + row_base * (int64_t)r + c;
#pragma unroll
            for (int i = 0; i < kTsqrTM; ++i) x[s][i] = (okc && i < nr) ? (T)__ldg(p + (int64_t)i * r) : T(0);
        } else {            // X = A^T, A row-major r x d_in: X[i][c] = A[c*ld + row_base + i]
            const float* p = X + (int64_t)c * ld + row_base;
#pragma unroll
            for (int i = 0; i < kTsqrTM; ++i) x[s][i] = (okc && i < nr) ? (T)__ldg(p + i) : T(0);
        }
    }
}

template <typename T, int RT>
__device__ __forceinline__ void load_tri_rows(T (&x)[Cols<RT>::NS][kTsqrTM], const T* P, int i0) {
    // rows i0..i0+TM-1 of a dense RT x RT (upper-triangular) partial R
    const int lane = threadIdx.x & 31;
    using C = Cols<RT>;
#pragma unroll
    for (int s = 0; s < C::NS; ++s) {
        const int c = C::col(lane, s);
#pragma unroll
        for (int i = 0; i < kTsqrTM; ++i) {
            const int row = i0 + i;
            x[s][i] = (c < RT && row < RT) ? __ldcg(P + row * RT + c) : T(0);
        }
    }
}

template <typename T, int RT>
__device__ __forceinline__ void load_packed_rows(T (&x)[Cols<RT>::NS][kTsqrTM], const T* P, int i0) {
    // rows i0..i0+TM-1 of a packed upper triangle (zero below the diagonal)
    const int lane = threadIdx.x & 31;
    using C = Cols<RT>;
#pragma unroll
    for (int s = 0; s < C::NS; ++s) {
        const int c = C::col(lane, s);
#pragma unroll
        for (int i = 0; i < kTsqrTM; ++i) {
            const int row = i0 + i;
            x[s][i] = (c < RT && row <= c) ? __ldcg(P + tri_off<RT>(row, c)) : T(0);
        }
    }
}

template <typename T, int RT>
__device__ __forceinline__ void tsqr_item(const TsqrArgs<T>& a, int wi, T* Rp, T* vbuf, int* s_last, int lane) {
    const TsqrWork w = a.work[wi];
    if (a.only && a.only[w.mf] == 0) return;   // warp-uniform
    const int local = w.mf >> 1, factor = w.mf & 1;
    const int gm = a.mod_ids ? a.mod_ids[local] : local;
    const lf_module md = a.mods[gm];
    const int r = md.r;
    const float* X = factor == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
    const int ld = factor == 0 ? r : md.d_in;

    for (int e = lane; e < tri_size<RT>(); e += 32) Rp[e] = T(0);
    __syncwarp();
    T x[Cols<RT>::NS][kTsqrTM];
    for (int t0 = 0; t0 < w.nrows; t0 += kTsqrTM) {
        load_rows<T, RT>(x, X, factor, (int64_t)w.row0 + t0, min(kTsqrTM, w.nrows - t0), r, ld);
        warp_absorb<T, RT>(x, Rp, vbuf, r);
    }

    T* out = (factor == 0 ? a.R_B : a.R_A) + (size_t)local * a.rs * a.rs;
    const TsqrInfo inf = a.info[w.mf];
    if (inf.nchunks > 1 && a.tree) {
        // Each node of the tree is qr([R_left; R_right]) of its two children, formed by
        // the second child to finish (the fixed left-right order keeps the result
        // independent of scheduling); a node with one child passes its R up unchanged.
        constexpr int TRI = tri_size<RT>();
        int node = w.slot - inf.slot0, nl = inf.nchunks, off = 0;
        while (nl > 1) {
            const int parent = node >> 1, offp = off + nl;
            if ((node ^ 1) < nl) {
                T* P = a.partial + (size_t)(inf.slot0 + off + node) * TRI;
                for (int e = lane; e < TRI; e += 32) P[e] = Rp[e];
                __threadfence();
                __syncwarp();
                if (lane == 0) *s_last = (atomicAdd(&a.counters[inf.slot0 + offp + parent], 1) == 1);
                __syncwarp();
                if (!*s_last) return;
                __threadfence();
                const int left = node & ~1;
                const T* PL = a.partial + (size_t)(inf.slot0 + off + left) * TRI;
                const T* PR = PL + TRI;
                if (node != left)
                    for (int e = lane; e < TRI; e += 32) Rp[e] = __ldcg(PL + e);
                __syncwarp();
                for (int i0 = 0; i0 < r; i0 += kTsqrTM) {
                    load_packed_rows<T, RT>(x, PR, i0);
                    warp_absorb<T, RT>(x, Rp, vbuf, r);
                }
            }
            node = parent;
            nl = (nl + 1) >> 1;
            off = offp;
        }
    } else if (inf.nchunks > 1) {
        T* P = a.partial + (size_t)w.slot * RT * RT;
        for (int e = lane; e < RT * RT; e += 32) {
            const int j = e / RT, c = e % RT;
            P[e] = c >= j ? Rp[tri_off<RT>(j, c)] : T(0);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) *s_last = (atomicAdd(&a.counters[w.mf], 1) == inf.nchunks - 1);
        __syncwarp();
        if (!*s_last) return;
        __threadfence();
        // fold the chunk triangles in chunk order: R = R_0, then R <- R([R; R_c])
        const T* P0 = a.partial + (size_t)inf.slot0 * RT * RT;
        for (int e = lane; e < RT * RT; e += 32) {
            const int j = e / RT, c = e % RT;
            if (c >= j) Rp[tri_off<RT>(j, c)] = __ldcg(P0 + e);
        }
        __syncwarp();
        for (int c = 1; c < inf.nchunks; ++c) {
            const T* Pc = a.partial + (size_t)(inf.slot0 + c) * RT * RT;
            for (int i0 = 0; i0 < r; i0 += kTsqrTM) {
                load_tri_rows<T, RT>(x, Pc, i0);
                warp_absorb<T, RT>(x, Rp, vbuf, r);
            }
        }
    }
    // canonical sign: diag(R) >= 0 (flip whole rows); zero past r
    for (int e = lane; e < a.rs * a.rs; e += 32) {
        const int j = e / a.rs, c = e % a.rs;
        T v = 0;
        if (j < r && c < r && c >= j) {
            v = Rp[tri_off<RT>(j, c)];
            if (Rp[tri_off<RT>(j, j)] < T(0)) v = -v;
        }
        out[e] = v;
    }
}

// One warp per work item; a bounded grid strides over the device-side item count
// (warps are independent: no block-level barriers).
template <typename T, int RT>
__global__ void __launch_bounds__(32 * tsqr_warps<T>(), sizeof(T) == 4 ? 16 : 1) tsqr_kernel(TsqrArgs<T> a) {
    constexpr int W = tsqr_warps<T>();
    __shared__ T s_R[W][tri_size<RT>()];
    __shared__ __align__(16) T s_v[W][kTsqrTM];
    __shared__ int s_last[W];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int wi = blockIdx.x * W + warp; wi < *a.n_work; wi += gridDim.x * W) {
        tsqr_item<T, RT>(a, wi, s_R[warp], s_v[warp], &s_last[warp], lane);
        __syncwarp();
    }
}

// ----------------------------------------------------------------------------
// Small SVD: M = R_B R_A^T (r x r), one-sided Jacobi on the rows of M.
// Rotating rows p, q of M by the plane rotation that is also applied to columns
// p, q of U (U starts at I) keeps M = U M'; at convergence the rows of M' are
// orthogonal, sigma_p = |m'_p| and row p of M' is sigma_p v_p^T.
// One warp per module; in each round of the round-robin ordering every lane owns
// one of the r/2 disjoint pairs and forms its three dot products alone, so a round
// needs no reductions.  T = float for the main path (the retained directions and
// the energies near the S boundary are accurate to ~1e-6), T = double for the
// boundary refinement.
// ----------------------------------------------------------------------------
template <typename TIN, typename T>
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

template <typename T, int RT>
struct alignas(16) SvdSmem {
    static constexpr int LD = RT + 16 / (int)sizeof(T);   // 16-byte aligned rows, 4-bank shift per row
    T M[RT][LD];
    // Ut[p] = column p of U, accumulated by the fp64 refinement only (the fp32 path forms
    // U at the end and stages R_A here during setup only when it has room: see svd_kernel)
    T Ut[sizeof(T) == 8 ? RT : 1][LD];
    T sig[RT];
    int perm[RT];
};

// Four consecutive elements from / to a 16-byte aligned address in shared memory.
__device__ __forceinline__ void ld4(const float* p, float (&v)[4]) {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
__device__ __forceinline__ void ld4(const double* p, double (&v)[4]) {
    const double2 a = reinterpret_cast<const double2*>(p)[0], b = reinterpret_cast<const double2*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}
__device__ __forceinline__ void st4(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st4(double* p, const double (&v)[4]) {
    reinterpret_cast<double2*>(p)[0] = make_double2(v[0], v[1]);
    reinterpret_cast<double2*>(p)[1] = make_double2(v[2], v[3]);
}

// One warp (one module) per CTA: a finished module frees its shared memory at once.
template <typename T>
__host__ __device__ constexpr int svd_warps() { return 1; }
// Rotation threshold |gamma| > tol * sqrt(alpha beta): r * eps of the working type
// (a tighter threshold cannot be met by rotations computed in that type).
template <typename T>
__device__ __forceinline__ T svd_tol(int r) { return T(r) * (sizeof(T) == 8 ? T(2.220446049250313e-16) : T(1.1920929e-7)); }

// One Jacobi rotation of rows p, q of M and of columns p, q of U (fp64 refinement):
// returns whether the pair was rotated.
template <typename T, int RT, bool ACC>
__device__ __forceinline__ bool svd_rotate_acc(SvdSmem<T, RT>& s, int p, int q, int r, T tol) {
    T al[4] = {0, 0, 0, 0}, be[4] = {0, 0, 0, 0}, ga[4] = {0, 0, 0, 0};
    const T* mp = s.M[p];
    const T* mq = s.M[q];
    int l = 0;
#pragma unroll 4
    for (; l + 3 < r; l += 4) {   // four independent chains per sum, 16-byte loads
        T xv[4], yv[4];
        ld4(mp + l, xv);
        ld4(mq + l, yv);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            al[u] = fma(xv[u], xv[u], al[u]);
            be[u] = fma(yv[u], yv[u], be[u]);
            ga[u] = fma(xv[u], yv[u], ga[u]);
        }
    }
    for (; l < r; ++l) {
        const T x = mp[l], y = mq[l];
        al[0] = fma(x, x, al[0]);
        be[0] = fma(y, y, be[0]);
        ga[0] = fma(x, y, ga[0]);
    }
    const T alpha = (al[0] + al[1]) + (al[2] + al[3]);
    const T beta_ = (be[0] + be[1]) + (be[2] + be[3]);
    const T gamma = (ga[0] + ga[1]) + (ga[2] + ga[3]);
    if (!(gamma != T(0) && fabs(gamma) > tol * sqrt(alpha * beta_))) return false;
    const T zeta = (beta_ - alpha) / (T(2) * gamma);
    const T tt = (zeta >= T(0) ? T(1) : T(-1)) / (fabs(zeta) + sqrt(T(1) + zeta * zeta));
    const T c = T(1) / sqrt(T(1) + tt * tt);
    const T sn = c * tt;
    T* Mp = s.M[p];
    T* Mq = s.M[q];
    T* Up = s.Ut[p];
    T* Uq = s.Ut[q];
    int k = 0;
    if constexpr (!ACC) {   // singular values only: rows of M alone
#pragma unroll 2
        for (; k + 3 < r; k += 4) {
            T x[4], y[4], x2[4], y2[4];
            ld4(Mp + k, x); ld4(Mq + k, y);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x2[e] = c * x[e] - sn * y[e];
                y2[e] = sn * x[e] + c * y[e];
            }
            st4(Mp + k, x2); st4(Mq + k, y2);
        }
        for (; k < r; ++k) {
            const T x = Mp[k], y = Mq[k];
            Mp[k] = c * x - sn * y;
            Mq[k] = sn * x + c * y;
        }
    } else {
#pragma unroll 2
        for (; k + 3 < r; k += 4) {   // 16-byte loads and stores of four columns
            T x[4], y[4], u[4], v[4], x2[4], y2[4], u2[4], v2[4];
            ld4(Mp + k, x); ld4(Mq + k, y); ld4(Up + k, u); ld4(Uq + k, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                x2[e] = c * x[e] - sn * y[e];
                y2[e] = sn * x[e] + c * y[e];
                u2[e] = c * u[e] - sn * v[e];
                v2[e] = sn * u[e] + c * v[e];
            }
            st4(Mp + k, x2); st4(Mq + k, y2); st4(Up + k, u2); st4(Uq + k, v2);
        }
        for (; k < r; ++k) {
            const T x = Mp[k], y = Mq[k], u = Up[k], v = Uq[k];
            Mp[k] = c * x - sn * y;
            Mq[k] = sn * x + c * y;
            Up[k] = c * u - sn * v;
            Uq[k] = sn * u + c * v;
        }
    }
    return true;
}

// One Jacobi rotation of rows p, q of M only (fp32 main path): both rows are read once
// into registers (16-byte chunks; the row padding past r is zero), the three dot
// products and the rotation run there on packed fp32 pairs (each component rounds as
// fmaf), and the rows are written back once.  Each sum keeps four partial chains,
// element e of a chunk in chain e, added as (0 + 1) + (2 + 3).
template <typename T, int RT>
__device__ __forceinline__ bool svd_rotate_rows(SvdSmem<T, RT>& s, int p, int q, int r, T tol) {
    static_assert(sizeof(T) == 4, "register path is fp32");
    constexpr int NC = RT / 4;
    float4 x[NC], y[NC];
    float2 al01 = make_float2(0.f, 0.f), al23 = al01, be01 = al01, be23 = al01, ga01 = al01, ga23 = al01;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        if (4 * c < r) {
            x[c] = *reinterpret_cast<const float4*>(&s.M[p][4 * c]);
            y[c] = *reinterpret_cast<const float4*>(&s.M[q][4 * c]);
        } else {
            x[c] = y[c] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        const float2 x01 = make_float2(x[c].x, x[c].y), x23 = make_float2(x[c].z, x[c].w);
        const float2 y01 = make_float2(y[c].x, y[c].y), y23 = make_float2(y[c].z, y[c].w);
        al01 = __ffma2_rn(x01, x01, al01);
        al23 = __ffma2_rn(x23, x23, al23);
        be01 = __ffma2_rn(y01, y01, be01);
        be23 = __ffma2_rn(y23, y23, be23);
        ga01 = __ffma2_rn(x01, y01, ga01);
        ga23 = __ffma2_rn(x23, y23, ga23);
    }
    const float alpha = (al01.x + al01.y) + (al23.x + al23.y);
    const float beta_ = (be01.x + be01.y) + (be23.x + be23.y);
    const float gamma = (ga01.x + ga01.y) + (ga23.x + ga23.y);
    if (!(gamma != 0.f && fabsf(gamma) > tol * sqrtf(alpha * beta_))) return false;
    const float zeta = (beta_ - alpha) / (2.f * gamma);
    const float tt = (zeta >= 0.f ? 1.f : -1.f) / (fabsf(zeta) + sqrtf(1.f + zeta * zeta));
    const float cs = 1.f / sqrtf(1.f + tt * tt);
    const float sn = cs * tt;
    const float2 c2 = make_float2(cs, cs), s2 = make_float2(sn, sn), ms2 = make_float2(-sn, -sn);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        if (4 * c < r) {
            const float2 a01 = make_float2(x[c].x, x[c].y), a23 = make_float2(x[c].z, x[c].w);
            const float2 b01 = make_float2(y[c].x, y[c].y), b23 = make_float2(y[c].z, y[c].w);
            // x' = cs a - sn b,  y' = sn a + cs b  (the product with b rounded first)
            const float2 xp01 = __ffma2_rn(c2, a01, __fmul2_rn(ms2, b01));
            const float2 xp23 = __ffma2_rn(c2, a23, __fmul2_rn(ms2, b23));
            const float2 yp01 = __ffma2_rn(s2, a01, __fmul2_rn(c2, b01));
            const float2 yp23 = __ffma2_rn(s2, a23, __fmul2_rn(c2, b23));
            *reinterpret_cast<float4*>(&s.M[p][4 * c]) = make_float4(xp01.x, xp01.y, xp23.x, xp23.y);
            *reinterpret_cast<float4*>(&s.M[q][4 * c]) = make_float4(yp01.x, yp01.y, yp23.x, yp23.y);
        }
    }
    return true;
}

template <typename TIN, typename T, int RT>
__global__ void __launch_bounds__(32 * svd_warps<T>()) svd_kernel(SvdArgs<TIN, T> a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    auto& s = reinterpret_cast<SvdSmem<T, RT>*>(smem_raw)[warp];
    const int local = blockIdx.x * svd_warps<T>() + warp;
    if (local >= *a.n) return;   // warp-uniform; no block barriers below
    const int gm = a.mod_ids ? a.mod_ids[local] : local;
    const int r = a.mods[gm].r;
    const int rs = a.rs;
    const TIN* RB = a.R_B + (size_t)local * rs * rs;
    const TIN* RA = a.R_A + (size_t)local * rs * rs;

    // fp64 (refinement): U accumulates the rotations when U is wanted (the refinement
    // itself needs sigma only).  fp32 (main path): rows of M only
    // are rotated, and U = M_0 M'^T Sigma^-2 is formed at the end from M_0, which is
    // parked in the module's U output block meanwhile.
    constexpr bool kAccU = sizeof(T) == 8;
    if constexpr (kAccU) {
        // stage R_A in Ut, then M[i][j] = sum_{l >= max(i,j)} R_B[i][l] R_A[j][l] (one row per lane)
        for (int e = lane; e < r * r; e += 32) {
            const int i = e / r, l = e % r;
            s.Ut[i][l] = (T)RA[i * rs + l];
        }
        __syncwarp();
        for (int i = lane; i < r; i += 32) {
            const TIN* rb = RB + (size_t)i * rs;
            for (int j0 = 0; j0 < r; j0 += 4) {   // four columns of M at a time (independent chains)
                T acc[4] = {0, 0, 0, 0};
                for (int l = i; l < r; ++l) {
                    const T b = (T)rb[l];
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        if (j0 + q < r && l >= j0 + q) acc[q] = fma(b, s.Ut[j0 + q][l], acc[q]);
                }
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (j0 + q < r) s.M[i][j0 + q] = acc[q];
            }
        }
        __syncwarp();
        for (int e = lane; e < RT * SvdSmem<T, RT>::LD; e += 32) {
            const int i = e / SvdSmem<T, RT>::LD, l = e % SvdSmem<T, RT>::LD;
            if (i < r && l >= r) s.M[i][l] = T(0);
            s.Ut[i][l] = (i == l && i < r) ? T(1) : T(0);
        }
    } else {
        // M[i][j] = R_B[i] . R_A[j] (both R are zero below the diagonal and past r): lane j
        // holds rows j and j + 32 of R_A, row i of R_B is broadcast to the warp
        constexpr int NC = RT / 4;
        // 16-byte loads when every row starts on a 16-byte boundary (rs % 4 == 0: a chunk
        // that starts below r then ends inside the row); element loads otherwise
        const bool vec = (rs & 3) == 0 && ((reinterpret_cast<uintptr_t>(RA) | reinterpret_cast<uintptr_t>(RB)) & 15) == 0;
        auto ld_chunk = [&](const float* row, int c) -> float4 {
            if (4 * c >= r) return make_float4(0.f, 0.f, 0.f, 0.f);
            if (vec) return *reinterpret_cast<const float4*>(row + 4 * c);
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = 4 * c + u < r ? row[4 * c + u] : 0.f;
            return make_float4(v[0], v[1], v[2], v[3]);
        };
        float4 ra[2][NC];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int j = lane + 32 * h;
#pragma unroll
            for (int c = 0; c < NC; ++c)
                ra[h][c] = j < r ? ld_chunk(RA + (size_t)j * rs, c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        double* M0 = a.U ? a.U + (size_t)local * rs * rs : nullptr;
        for (int i = 0; i < r; ++i) {
            float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                if (4 * c < r) {
                    const float4 b = ld_chunk(RB + (size_t)i * rs, c);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        acc[h][0] = fmaf(b.x, ra[h][c].x, acc[h][0]);
                        acc[h][1] = fmaf(b.y, ra[h][c].y, acc[h][1]);
                        acc[h][2] = fmaf(b.z, ra[h][c].z, acc[h][2]);
                        acc[h][3] = fmaf(b.w, ra[h][c].w, acc[h][3]);
                    }
                }
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int j = lane + 32 * h;
                if (j < r) {
                    const float m = (acc[h][0] + acc[h][1]) + (acc[h][2] + acc[h][3]);
                    s.M[i][j] = m;
                    if (M0) M0[(size_t)i * rs + j] = (double)m;
                }
            }
        }
        for (int e = lane; e < RT * SvdSmem<T, RT>::LD; e += 32) {
            const int i = e / SvdSmem<T, RT>::LD, l = e % SvdSmem<T, RT>::LD;
            if (i < r && l >= r) s.M[i][l] = T(0);   // zero padding: whole 16-byte chunks are read
        }
    }
    __syncwarp();

    const int rp = (r + 1) & ~1;  // even number of players (index r is a bye when r is odd)
    const T tol = svd_tol<T>(r);
    for (int sweep = 0; sweep < a.max_sweeps; ++sweep) {
        bool rot = false;
        for (int t = 0; t < rp - 1; ++t) {
            if (lane < rp / 2) {
                int p, q;
                if (lane == 0) {
                    p = rp - 1;
                    q = t;
                } else {   // (t + lane) mod (rp - 1) and (t - lane) mod (rp - 1), both in range
                    p = t + lane;
                    if (p >= rp - 1) p -= rp - 1;
                    q = t - lane;
                    if (q < 0) q += rp - 1;
                }
                if (p < r && q < r) {
                    if constexpr (kAccU) {
                        rot |= a.U ? svd_rotate_acc<T, RT, true>(s, p, q, r, tol)
                                   : svd_rotate_acc<T, RT, false>(s, p, q, r, tol);
                    } else {
                        rot |= svd_rotate_rows<T, RT>(s, p, q, r, tol);
                    }
                }
            }
            __syncwarp();
        }
        if (!__any_sync(0xffffffffu, rot)) break;
    }

    for (int p = lane; p < r; p += 32) {
        T nn = 0;
        for (int l = 0; l < r; ++l) nn = fma(s.M[p][l], s.M[p][l], nn);
        s.sig[p] = sqrt(nn);
    }
    __syncwarp();
    for (int p = lane; p < r; p += 32) {  // descending, ties by index
        const T sp = s.sig[p];
        int rank = 0;
        for (int q = 0; q < r; ++q) {
            const T sq = s.sig[q];
            rank += (sq > sp) || (sq == sp && q < p);
        }
        s.perm[rank] = p;
        if (!isfinite((double)sp)) latch_error(LF_ERR_NUMERIC);
    }
    __syncwarp();
    double* sg = a.sigma + (size_t)local * rs;
    for (int j = lane; j < rs; j += 32) sg[j] = j < r ? (double)s.sig[s.perm[j]] : 0.0;
    if (a.U) {
        double* Uo = a.U + (size_t)local * rs * rs;
        if constexpr (kAccU) {
            for (int e = lane; e < rs * rs; e += 32) {
                const int row = e / rs, j = e % rs;
                Uo[e] = (row < r && j < r) ? (double)s.Ut[s.perm[j]][row] : 0.0;
            }
        } else {   // column j of U = M_0 m'_p / sigma_p^2 (p = perm[j]); zero where sigma_p = 0
            for (int row = lane; row < rs; row += 32) {
                float m0[RT];
#pragma unroll
                for (int l = 0; l < RT; ++l) m0[l] = (row < r && l < r) ? (float)Uo[(size_t)row * rs + l] : 0.f;
                for (int j = 0; j < rs; ++j) {
                    double u = 0.0;
                    if (row < r && j < r) {
                        const int pj = s.perm[j];
                        const T sp = s.sig[pj];
                        float d0 = 0.f, d1 = 0.f, d2 = 0.f, d3 = 0.f;
#pragma unroll
                        for (int c = 0; c < RT / 4; ++c) {
                            if (4 * c < r) {
                                const float4 mp = *reinterpret_cast<const float4*>(&s.M[pj][4 * c]);
                                d0 = fmaf(m0[4 * c], mp.x, d0);
                                d1 = fmaf(m0[4 * c + 1], mp.y, d1);
                                d2 = fmaf(m0[4 * c + 2], mp.z, d2);
                                d3 = fmaf(m0[4 * c + 3], mp.w, d3);
                            }
                        }
                        const double dot = (double)((d0 + d1) + (d2 + d3));
                        u = sp > T(0) ? dot / ((double)sp * (double)sp) : 0.0;
                    }
                    Uo[(size_t)row * rs + j] = u;   // row `row` of M_0 is in registers already
                }
            }
        }
    }
    if (a.V) {
        double* Vo = a.V + (size_t)local * rs * rs;
        for (int e = lane; e < rs * rs; e += 32) {
            const int row = e / rs, j = e % rs;
            double v = 0.0;
            if (row < r && j < r) {
                const int p = s.perm[j];
                const double sp = (double)s.sig[p];
                v = sp > 0.0 ? (double)s.M[p][row] / sp : 0.0;
            }
            Vo[e] = v;
        }
    }
}

}  // namespace lf
