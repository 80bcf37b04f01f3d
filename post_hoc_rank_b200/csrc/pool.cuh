// Pool-wide shared subspace of a LoRA pool's stacked factors (LoRASpace).
//
// LoRASpace (the arXiv listing's abstract, "LoRASpace: A Pool-Wide Shared Substrate for
// Static and Dynamic Multi-LoRA Composition"): the stacked low-rank factors of a pool
// need far fewer directions than their summed ranks; the SVD of the stack gives the
// minimal subspace that keeps 99 % of the factor energy, computed once per pool.
//
// The stack S (R stack vectors of length d: the rows A_i of the row factors, or the
// columns of the column factors B_i) has the Gram matrix G = S S^T (R x R), formed in
// fp64 from the fp32 inputs (every product exact).  G = U diag(lambda) U^T with
// lambda_j = sigma_j^2, the squared singular values of S, and the directions of the
// subspace are the rows of Sigma^-1 U^T S (the right singular vectors of the stack of
// vectors).  U comes from a one-sided Jacobi iteration on G: pairs of columns of X = G J
// are rotated until they are orthogonal, J accumulating the rotations; then X = U diag
// (lambda) and J = U (up to the order of the columns).  Pairs follow the round-robin
// (circle) schedule, R/2 disjoint pairs per round, one warp per pair, so a round has
// no data dependence between warps; the CTAs of a cooperative launch meet at a grid
// barrier between rounds (a bounded spin: a barrier that does not complete latches
// LF_ERR_TIMEOUT and every CTA leaves).
#pragma once
#include "common.cuh"

namespace lf {

constexpr int kPoolMaxRank = LF_POOL_MAX_RANK;
constexpr int kPoolThreads = 256;
constexpr int kPoolMaxSweeps = 40;

struct PoolArgs {
    int32_t R, d, num, den;
    const float* base;
    const int64_t* row_off;   // per stack vector: element offset of its first entry
    const int32_t* row_step;  // per stack vector: element step between its entries
    float* Sv;                // R x d fp32: the gathered stack
    double* X;                // R x R, column j at X + j * R (G, then G J)
    double* V;                // R x R, column j at V + j * R (J)
    double* lam;              // R: |X_j| after the iteration
    int32_t* order;           // R: column of the j-th largest lambda
    uint32_t* bar;            // [0] count, [1] generation, [2] abort, [3..5] rotation flags of sweeps (mod 3)
    int32_t* k_out;
    double* sigma;            // R, descending
    float* basis;             // R x d, row j = direction j
    float* coef;              // R x R: coef[a][j] = stack vector a . direction j
    double* resid_part;       // R: per stack vector, sum over j >= k of coef^2
    double* resid;            // 1
};

// Stack vector a, entries x .. of the pool (row factors: a row of some A_i, step 1; column
// factors: a column of some B_i, step r_i); a non-finite value latches LF_ERR_NUMERIC.
__global__ void pool_gather_kernel(PoolArgs a) {
    const int row = blockIdx.y;
    const int64_t off = a.row_off[row];
    const int step = a.row_step[row];
    for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < a.d; x += gridDim.x * blockDim.x) {
        float v = a.base[off + (int64_t)x * step];
        if (!isfinite(v)) {
            latch_error(LF_ERR_NUMERIC);
            v = 0.f;
        }
        a.Sv[(int64_t)row * a.d + x] = v;
    }
}

// G[r1][r2] = sum_x Sv[r1][x] Sv[r2][x] in fp64, x ascending (so G[r1][r2] and G[r2][r1]
// are the same bits); CTA = 32 x 32 tile, 256 threads, 4 entries each; X = G, V = I.
constexpr int kPoolTile = 32;
__global__ void __launch_bounds__(kPoolThreads) pool_gram_kernel(PoolArgs a) {
    __shared__ float sa[kPoolTile][kPoolTile + 1];
    __shared__ float sb[kPoolTile][kPoolTile + 1];
    const int r0 = blockIdx.y * kPoolTile, c0 = blockIdx.x * kPoolTile;
    const int tid = threadIdx.x;
    const int tr = tid / 8, tc = (tid % 8) * 4;   // entry rows tr, columns tc .. tc + 3
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int x0 = 0; x0 < a.d; x0 += kPoolTile) {
        for (int e = tid; e < kPoolTile * kPoolTile; e += kPoolThreads) {
            const int i = e / kPoolTile, x = e % kPoolTile;
            const bool okx = x0 + x < a.d;
            sa[i][x] = (r0 + i < a.R && okx) ? a.Sv[(int64_t)(r0 + i) * a.d + x0 + x] : 0.f;
            sb[i][x] = (c0 + i < a.R && okx) ? a.Sv[(int64_t)(c0 + i) * a.d + x0 + x] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int x = 0; x < kPoolTile; ++x) {
            const double u = sa[tr][x];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fma(u, (double)sb[tc + q][x], acc[q]);
        }
        __syncthreads();
    }
    const int rr = r0 + tr;
    if (rr < a.R)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int cc = c0 + tc + q;
            if (cc < a.R) {
                a.X[(int64_t)cc * a.R + rr] = acc[q];
                a.V[(int64_t)cc * a.R + rr] = rr == cc ? 1.0 : 0.0;
            }
        }
}

// Grid barrier of a cooperative launch (every CTA resident): the last CTA to arrive
// resets the count and advances the generation.  The wait gives up after about a
// second, latches LF_ERR_TIMEOUT and sets the abort word.  Returns false on abort.
__device__ __forceinline__ bool pool_grid_sync(uint32_t* bar) {
    __syncthreads();
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        volatile uint32_t* vb = bar;
        const uint32_t gen = vb[1];
        __threadfence();
        if (atomicAdd(&bar[0], 1u) == gridDim.x - 1) {
            bar[0] = 0;
            __threadfence();
            atomicAdd(&bar[1], 1u);
        } else {
            const long long t0 = clock64();
            for (int i = 0; vb[1] == gen; ++i) {
                __nanosleep(64);
                if (vb[2] || ((i & 255) == 255 && clock64() - t0 > 2000000000ll)) {
                    if (!vb[2]) latch_error(LF_ERR_TIMEOUT);
                    atomicExch(&bar[2], 1u);
                    break;
                }
            }
        }
        __threadfence();
        s_ok = vb[2] == 0;
    }
    __syncthreads();
    return s_ok != 0;
}

// Player at position pos of round t of the circle schedule over P (even) players.
__device__ __forceinline__ int pool_player(int pos, int t, int P) {
    return pos == 0 ? 0 : 1 + (pos - 1 + t) % (P - 1);
}

// One-sided Jacobi on the columns of X (= G J), accumulating J in V.  Cooperative launch.
__global__ void __launch_bounds__(kPoolThreads) pool_jacobi_kernel(PoolArgs a) {
    const int R = a.R, P = (R + 1) & ~1;
    const int lane = threadIdx.x & 31;
    const int gw = blockIdx.x * (kPoolThreads / 32) + (threadIdx.x >> 5);
    const int nw = gridDim.x * (kPoolThreads / 32);
    volatile uint32_t* vb = a.bar;
    for (int sweep = 0; sweep < kPoolMaxSweeps; ++sweep) {
        if (blockIdx.x == 0 && threadIdx.x == 0) vb[3 + (sweep + 1) % 3] = 0;   // flag of the next sweep
        for (int t = 0; t < P - 1; ++t) {
            for (int i = gw; i < P / 2; i += nw) {
                int p = pool_player(i, t, P), q = pool_player(P - 1 - i, t, P);
                if (p >= R || q >= R) continue;   // the extra player of an odd R
                if (p > q) {
                    const int tmp = p;
                    p = q;
                    q = tmp;
                }
                double* xp = a.X + (int64_t)p * R;
                double* xq = a.X + (int64_t)q * R;
                double al = 0.0, be = 0.0, ga = 0.0;
                for (int e = lane; e < R; e += 32) {
                    const double u = xp[e], v = xq[e];
                    al = fma(u, u, al);
                    be = fma(v, v, be);
                    ga = fma(u, v, ga);
                }
                al = warp_sum(al);
                be = warp_sum(be);
                ga = warp_sum(ga);   // every lane holds the same three values
                // orthogonal to working precision (tolerance R u, u = 2^-53): no rotation
                if (!(fabs(ga) > (double)R * 0x1p-52 * sqrt(al * be)) || al == 0.0 || be == 0.0) continue;
                const double zeta = (be - al) / (2.0 * ga);
                const double tt = (zeta >= 0.0 ? 1.0 : -1.0) / (fabs(zeta) + sqrt(1.0 + zeta * zeta));
                const double c = 1.0 / sqrt(1.0 + tt * tt), s = c * tt;
                for (int e = lane; e < R; e += 32) {
                    const double u = xp[e], v = xq[e];
                    xp[e] = c * u - s * v;
                    xq[e] = s * u + c * v;
                }
                double* vp = a.V + (int64_t)p * R;
                double* vq = a.V + (int64_t)q * R;
                for (int e = lane; e < R; e += 32) {
                    const double u = vp[e], v = vq[e];
                    vp[e] = c * u - s * v;
                    vq[e] = s * u + c * v;
                }
                if (lane == 0) vb[3 + sweep % 3] = 1;
            }
            if (!pool_grid_sync(a.bar)) return;
        }
        if (vb[3 + sweep % 3] == 0) return;   // no rotation in a whole sweep: converged
    }
}

// lambda_j = |X_j|, the order of the columns by lambda (descending; equal values by
// column index), sigma = sqrt(lambda) in that order, and k: the smallest k >= 1 with
// den * sum_{j<k} lambda_j >= num * sum_j lambda_j (sums in order; a zero stack keeps 1).
__global__ void __launch_bounds__(kPoolMaxRank) pool_order_kernel(PoolArgs a) {
    __shared__ double s_lam[kPoolMaxRank];
    const int R = a.R, j = threadIdx.x;
    if (j < R) {
        const double* xj = a.X + (int64_t)j * R;
        double s = 0.0;
        for (int e = 0; e < R; ++e) s = fma(xj[e], xj[e], s);
        s_lam[j] = sqrt(s);
        a.lam[j] = s_lam[j];
    }
    __syncthreads();
    if (j < R) {
        const double lj = s_lam[j];
        int rank = 0;
        for (int e = 0; e < R; ++e) {
            const double le = s_lam[e];
            rank += (le > lj) || (le == lj && e < j);
        }
        a.order[rank] = j;
        a.sigma[rank] = sqrt(lj);
    }
    __syncthreads();
    if (j == 0) {
        double tot = 0.0;
        for (int e = 0; e < R; ++e) tot += s_lam[a.order[e]];
        int k = R;
        double cum = 0.0;
        if (tot > 0.0) {
            for (int e = 0; e < R; ++e) {
                cum += s_lam[a.order[e]];
                if ((double)a.den * cum >= (double)a.num * tot) {
                    k = e + 1;
                    break;
                }
            }
        } else {
            k = 1;
        }
        *a.k_out = k;
    }
}

// basis[j][x] = (sum_a Sv[a][x] V[a][order[j]]) / sigma_j (fp64 sums in a order).  A
// direction whose sigma_j is at most kPoolResolve sigma_1 is not resolved by the Gram
// (its lambda_j is within the rounding of lambda_1 times R) and gets a zero row.
// CTA: 32 directions x 256 positions x.
constexpr double kPoolResolve = 1e-6;
__global__ void __launch_bounds__(kPoolThreads) pool_basis_kernel(PoolArgs a) {
    const int R = a.R;
    const int x = blockIdx.x * kPoolThreads + threadIdx.x;
    const int j0 = blockIdx.y * kPoolTile;
    __shared__ double sv[kPoolTile][kPoolTile];   // V[a][order[j0 + jj]] for a block of a
    double acc[kPoolTile];
#pragma unroll
    for (int jj = 0; jj < kPoolTile; ++jj) acc[jj] = 0.0;
    for (int a0 = 0; a0 < R; a0 += kPoolTile) {
        for (int e = threadIdx.x; e < kPoolTile * kPoolTile; e += kPoolThreads) {
            const int ai = e / kPoolTile, jj = e % kPoolTile;
            sv[ai][jj] = (a0 + ai < R && j0 + jj < R) ? a.V[(int64_t)a.order[j0 + jj] * R + a0 + ai] : 0.0;
        }
        __syncthreads();
        if (x < a.d) {
            for (int ai = 0; ai < kPoolTile && a0 + ai < R; ++ai) {
                const double sx = a.Sv[(int64_t)(a0 + ai) * a.d + x];
#pragma unroll
                for (int jj = 0; jj < kPoolTile; ++jj) acc[jj] = fma(sx, sv[ai][jj], acc[jj]);
            }
        }
        __syncthreads();
    }
    if (x < a.d)
#pragma unroll
        for (int jj = 0; jj < kPoolTile; ++jj) {
            const int j = j0 + jj;
            if (j < R) {
                const double sg = a.sigma[j];
                a.basis[(int64_t)j * a.d + x] = sg > kPoolResolve * a.sigma[0] ? (float)(acc[jj] / sg) : 0.f;
            }
        }
}

// coef[r1][j] = sum_x Sv[r1][x] basis[j][x] (fp64, x ascending) as in pool_gram_kernel
// with the basis as the second operand; resid_part[r1] = sum_{j >= k} coef[r1][j]^2.
__global__ void __launch_bounds__(kPoolThreads) pool_coef_kernel(PoolArgs a) {
    __shared__ float sa[kPoolTile][kPoolTile + 1];
    __shared__ float sb[kPoolTile][kPoolTile + 1];
    const int r0 = blockIdx.y * kPoolTile, c0 = blockIdx.x * kPoolTile;
    const int tid = threadIdx.x;
    const int tr = tid / 8, tc = (tid % 8) * 4;
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int x0 = 0; x0 < a.d; x0 += kPoolTile) {
        for (int e = tid; e < kPoolTile * kPoolTile; e += kPoolThreads) {
            const int i = e / kPoolTile, x = e % kPoolTile;
            const bool okx = x0 + x < a.d;
            sa[i][x] = (r0 + i < a.R && okx) ? a.Sv[(int64_t)(r0 + i) * a.d + x0 + x] : 0.f;
            sb[i][x] = (c0 + i < a.R && okx) ? a.basis[(int64_t)(c0 + i) * a.d + x0 + x] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int x = 0; x < kPoolTile; ++x) {
            const double u = sa[tr][x];
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] = fma(u, (double)sb[tc + q][x], acc[q]);
        }
        __syncthreads();
    }
    const int rr = r0 + tr;
    if (rr < a.R)
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const int cc = c0 + tc + q;
            if (cc < a.R) a.coef[(int64_t)rr * a.R + cc] = (float)acc[q];
        }
}

// resid = sum over stack vectors (in order) of sum_{j >= k} coef^2 (each row's sum in j
// order, one thread per row, then the rows in order by one thread).
__global__ void __launch_bounds__(kPoolMaxRank) pool_resid_kernel(PoolArgs a) {
    __shared__ double part[kPoolMaxRank];
    const int R = a.R, r1 = threadIdx.x;
    const int k = *a.k_out;
    if (r1 < R) {
        double s = 0.0;
        for (int j = k; j < R; ++j) {
            const double c = a.coef[(int64_t)r1 * R + j];
            s = fma(c, c, s);
        }
        part[r1] = s;
    }
    __syncthreads();
    if (r1 == 0) {
        double s = 0.0;
        for (int e = 0; e < R; ++e) s += part[e];
        *a.resid = s;
    }
}

}  // namespace lf
