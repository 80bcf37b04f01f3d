// Retained-rank allocation (LoRAForge-U / LoRAForge-S) and factor export.
//
// LoRAForge abstract (mlinfo.pages.dev, arXiv 2611.01256) and LoRAForge
// (kongchang.com), "LoRAForge's Core Design: Explicit Retained-Rank
// Representation and Dual Strategies": U keeps one ratio everywhere; S spends a
// rank budget along each module's spectral-energy accumulation curve (energy =
// sum of squared singular values), with a rank floor.  The budget is taken per
// adapter (module group) in rank units: K = floor(num * sum r / den); the extra
// K - floor * M slots go to the largest normalised energies
// e_ij = sigma_ij^2 / sum_j sigma_ij^2 (j >= floor, e > 0), ties to the lower
// module, then the lower j.
//
// "Compress then Serve" (academ.us/article/2407.00066), section 4, eq. 4: the
// retained factors are the truncated SVD, with S_k V_k^T kept as one matrix:
//   B'^T = (R_A^T V_k S_k^-1)^T B^T,   A' = (U_k^T R_B) A.
#pragma once
#include "common.cuh"

namespace lf {

constexpr int kSelThreads = 256;

struct SelArgs {
    const lf_module* mods;
    const int32_t* grp_ptr;    // n_groups + 1
    const int32_t* grp_mods;   // module indices, ascending inside each group
    const double* sigma;       // n x rs
    double* energy;            // n x rs scratch (normalised energies)
    int32_t rs;
    lf_policy pol;
    int32_t* ranks;            // n
    // boundary band (refinement); flag_list == nullptr disables flagging
    double band;
    int32_t* flag_list;
    int32_t* flag_count;
};

__device__ __forceinline__ int64_t block_sum_i64(int64_t v, int64_t* red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    v = warp_sum(v);
    __syncthreads();
    if (lane == 0) red[warp] = v;
    __syncthreads();
    int64_t t = 0;
    if (threadIdx.x < 32) {
        t = threadIdx.x < (int)(blockDim.x >> 5) ? red[threadIdx.x] : 0;
        t = warp_sum(t);
        if (threadIdx.x == 0) red[0] = t;
    }
    __syncthreads();
    return red[0];
}

// number of candidates (j >= floor, e > 0) with e >= t  (t >= smallest positive double)
__device__ int64_t count_ge(const SelArgs& a, int m0, int M, double t, int64_t* red) {
    int64_t c = 0;
    const int fl = a.pol.floor;
    for (int q = threadIdx.x; q < M * a.rs; q += blockDim.x) {
        const int mi = q / a.rs, j = q % a.rs;
        const int i = a.grp_mods[m0 + mi];
        if (j < fl || j >= a.mods[i].r) continue;
        const double e = a.energy[(size_t)i * a.rs + j];
        c += (e > 0.0 && e >= t);
    }
    return block_sum_i64(c, red);
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelArgs a) {
    __shared__ int64_t red[32];
    __shared__ int64_t s_take_eq;
    __shared__ double s_theta;
    const int g = blockIdx.x;
    const int m0 = a.grp_ptr[g], m1 = a.grp_ptr[g + 1], M = m1 - m0;
    const int fl = a.pol.floor;

    if (a.pol.kind == 0) {  // LoRAForge-U
        for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            int k = (a.pol.ratio_num * r + a.pol.ratio_den / 2) / a.pol.ratio_den;
            a.ranks[i] = min(r, max(fl, k));
        }
        return;
    }
    // energies, one module per thread, summed in j order
    int64_t rsum = 0;
    for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
        const int i = a.grp_mods[m0 + mi];
        const int r = a.mods[i].r;
        rsum += r;
        const double* sg = a.sigma + (size_t)i * a.rs;
        double tot = 0.0;
        for (int j = 0; j < r; ++j) {
            const double sq = sg[j] * sg[j];
            tot += sq;
            if (j + 1 < r && sg[j + 1] > sg[j]) latch_error(LF_ERR_INVALID_ARG);  // rows must descend
        }
        if (!isfinite(tot)) latch_error(LF_ERR_NUMERIC);
        double* en = a.energy + (size_t)i * a.rs;
        for (int j = 0; j < a.rs; ++j) {
            double e = 0.0;
            if (j < r && tot > 0.0) {
                const double sq = sg[j] * sg[j];
                e = __ddiv_rn(sq, tot);
            }
            en[j] = e;
        }
        a.ranks[i] = fl;
    }
    rsum = block_sum_i64(rsum, red);
    const int64_t K = ((int64_t)a.pol.ratio_num * rsum) / a.pol.ratio_den;
    const int64_t extra = K - (int64_t)fl * M;
    if (extra <= 0) return;  // ranks stay at the floor

    const double tiny = __longlong_as_double(1ll);
    const int64_t npos = count_ge(a, m0, M, tiny, red);
    double theta;
    int64_t take_eq;
    if (npos <= extra) {
        theta = tiny;  // take every positive candidate
        take_eq = INT64_MAX;
    } else {
        // largest bit pattern t with count(e >= t) >= extra (bisection on the ordered bits)
        long long lo = 1, hi = 0x7FF0000000000000ll;
        while (lo < hi) {
            const long long mid = lo + (hi - lo + 1) / 2;
            const int64_t c = count_ge(a, m0, M, __longlong_as_double(mid), red);
            if (c >= extra) lo = mid; else hi = mid - 1;
        }
        theta = __longlong_as_double(lo);
        const int64_t n_gt = count_ge(a, m0, M, __longlong_as_double(lo + 1), red);
        take_eq = extra - n_gt;
    }
    if (threadIdx.x == 0) {
        s_theta = theta;
        s_take_eq = take_eq;
    }
    __syncthreads();
    theta = s_theta;
    take_eq = s_take_eq;
    // per module: all e > theta, then the first take_eq candidates equal to theta in
    // (module, j) order.  The equal-candidate prefix over modules is taken serially.
    if (threadIdx.x == 0) {
        int64_t left = take_eq;
        for (int mi = 0; mi < M; ++mi) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            const double* en = a.energy + (size_t)i * a.rs;
            int k = fl;
            for (int j = fl; j < r; ++j) {
                const double e = en[j];
                if (!(e > 0.0)) break;
                if (e > theta) {
                    ++k;
                } else if (e == theta && left > 0) {
                    ++k;
                    --left;
                } else {
                    break;
                }
            }
            a.ranks[i] = k;
        }
    }
    if (a.flag_list && npos > extra) {
        for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            const double* en = a.energy + (size_t)i * a.rs;
            bool f = false;
            for (int j = fl; j < r; ++j) {
                const double e = en[j];
                if (e > 0.0 && fabs(e - theta) <= a.band * theta) f = true;
            }
            if (f) {
                const int slot = atomicAdd(a.flag_count, 1);
                a.flag_list[slot] = i;
            }
        }
    }
}

// off_A[i+1] = off_A[i] + ranks[i] * d_in, off_Bt likewise with d_out (one CTA).
__global__ void __launch_bounds__(1024) offsets_kernel(const lf_module* mods, int n, const int32_t* ranks,
                                                       int64_t* off_A, int64_t* off_Bt, int64_t cap_A,
                                                       int64_t cap_Bt) {
    __shared__ int64_t sa[1024], sb[1024];
    const int tid = threadIdx.x;
    const int per = (n + 1023) / 1024;
    const int i0 = min(n, tid * per), i1 = min(n, i0 + per);
    int64_t ta = 0, tb = 0;
    for (int i = i0; i < i1; ++i) {
        ta += (int64_t)ranks[i] * mods[i].d_in;
        tb += (int64_t)ranks[i] * mods[i].d_out;
    }
    sa[tid] = ta;
    sb[tid] = tb;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {  // Hillis-Steele inclusive scan
        int64_t xa = tid >= o ? sa[tid - o] : 0, xb = tid >= o ? sb[tid - o] : 0;
        __syncthreads();
        sa[tid] += xa;
        sb[tid] += xb;
        __syncthreads();
    }
    int64_t ca = sa[tid] - ta, cb = sb[tid] - tb;
    if (tid == 0) {
        off_A[0] = 0;
        off_Bt[0] = 0;
    }
    for (int i = i0; i < i1; ++i) {
        ca += (int64_t)ranks[i] * mods[i].d_in;
        cb += (int64_t)ranks[i] * mods[i].d_out;
        off_A[i + 1] = ca;
        off_Bt[i + 1] = cb;
    }
    if (tid == 1023 && (sa[1023] > cap_A || sb[1023] > cap_Bt)) latch_error(LF_ERR_WORKSPACE);
}

// Replace sigma rows of refined modules: sig_out[mod_ids[l]] = sig_ref[l].
__global__ void scatter_sigma_kernel(const int32_t* mod_ids, const int32_t* n, const double* sig_ref,
                                     double* sig_out, int rs) {
    const int l = blockIdx.x;
    if (l >= *n) return;
    const int i = mod_ids[l];
    for (int j = threadIdx.x; j < rs; j += blockDim.x) sig_out[(size_t)i * rs + j] = sig_ref[(size_t)l * rs + j];
}

// Build the fp64 refinement work list on the device from the flagged modules.
__global__ void refine_plan_kernel(const lf_module* mods, const int32_t* flag_list, const int32_t* flag_count,
                                   TsqrWork* work, int32_t* n_work, TsqrInfo* info, int chunk) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const int nf = *flag_count;
    int w = 0, slot = 0;
    for (int l = 0; l < nf; ++l) {
        const lf_module md = mods[flag_list[l]];
        for (int f = 0; f < 2; ++f) {
            const int rows = f == 0 ? md.d_out : md.d_in;
            const int nch = (rows + chunk - 1) / chunk;
            const int mf = 2 * l + f;
            info[mf].nchunks = nch;
            info[mf].slot0 = nch > 1 ? slot : -1;
            for (int c = 0; c < nch; ++c) {
                work[w].mf = mf;
                work[w].row0 = c * chunk;
                work[w].nrows = min(chunk, rows - c * chunk);
                work[w].slot = nch > 1 ? slot + c : -1;
                ++w;
            }
            if (nch > 1) slot += nch;
        }
    }
    *n_work = w;
}

// ---------------------------------------------------------------------------
// Export.  Coefficients (fp64 -> fp32), one CTA per module:
//   C_A [j][l] = sum_{a<=l} U[a][j] R_B[a][l]                 (k x r)
//   C_Bt[j][l] = (sum_{a<=l} R_A[a][l] V[a][j]) / sigma_j     (k x r), 0 if sigma_j = 0
// ---------------------------------------------------------------------------
__global__ void export_coef_kernel(const lf_module* mods, const int32_t* ranks, const float* R_B,
                                   const float* R_A, const double* sigma, const double* U, const double* V,
                                   int rs, float* C_A, float* C_Bt) {
    const int i = blockIdx.x;
    const int r = mods[i].r, k = ranks[i];
    const size_t b = (size_t)i * rs * rs;
    for (int e = threadIdx.x; e < k * r; e += blockDim.x) {
        const int j = e / r, l = e % r;
        double ca = 0.0, cb = 0.0;
        for (int q = 0; q <= l; ++q) {
            ca += U[b + (size_t)q * rs + j] * (double)R_B[b + (size_t)q * rs + l];
            cb += (double)R_A[b + (size_t)q * rs + l] * V[b + (size_t)q * rs + j];
        }
        const double sj = sigma[(size_t)i * rs + j];
        C_A[b + (size_t)j * rs + l] = (float)ca;
        C_Bt[b + (size_t)j * rs + l] = sj > 0.0 ? (float)(cb / sj) : 0.0f;
    }
}

struct ExportWork {
    int32_t mod;
    int32_t part;   // 0 = B rows -> B'^T columns, 1 = A columns -> A' columns
    int32_t start;
    int32_t len;
};

struct ExportArgs {
    const lf_module* mods;
    const ExportWork* work;
    const float* B_base;
    const float* A_base;
    const int32_t* ranks;
    const int64_t* off_A;
    const int64_t* off_Bt;
    const float* C_A;
    const float* C_Bt;
    int32_t rs;
    float* A_pool;
    float* Bt_pool;
    __nv_bfloat16* A_pool16;
    __nv_bfloat16* Bt_pool16;
    int64_t cap_A, cap_Bt;
};

constexpr int kExpThreads = 256;   // 8 warps
constexpr int kExpJ = 16;          // retained directions per accumulator pass

// B part: lane owns one row e of B (r fp32 = 16 float4 loads issued together) and
// writes B'^T[j][e] = sum_l C_Bt[j][l] B[e][l] for j < k (coalesced across lanes).
__device__ void export_b_rows(const ExportArgs& a, const lf_module& md, int k, const float* cB, int64_t obt,
                              int start, int len) {
    const int r = md.r, tid = threadIdx.x;
    const float* B = a.B_base + md.B_off;
    for (int e0 = start; e0 < start + len; e0 += kExpThreads) {
        const int e = e0 + tid;
        if (e >= start + len) break;
        float x[kMaxRank];
        if (r == kMaxRank) {
            const float4* src = reinterpret_cast<const float4*>(B + (int64_t)e * kMaxRank);
#pragma unroll
            for (int q = 0; q < kMaxRank / 4; ++q) {
                const float4 v = __ldg(src + q);
                x[4 * q] = v.x; x[4 * q + 1] = v.y; x[4 * q + 2] = v.z; x[4 * q + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int l = 0; l < kMaxRank; ++l) x[l] = l < r ? __ldg(B + (int64_t)e * r + l) : 0.f;
        }
        for (int j0 = 0; j0 < k; j0 += kExpJ) {
            float acc[kExpJ];
#pragma unroll
            for (int jj = 0; jj < kExpJ; ++jj) {
                float t = 0.f;
                if (j0 + jj < k) {
                    const float* cr = cB + (j0 + jj) * kMaxRank;
#pragma unroll
                    for (int l = 0; l < kMaxRank; ++l) t = fmaf(cr[l], x[l], t);
                }
                acc[jj] = t;
            }
#pragma unroll
            for (int jj = 0; jj < kExpJ; ++jj) {
                if (j0 + jj < k) {
                    const int64_t o = obt + (int64_t)(j0 + jj) * md.d_out + e;
                    a.Bt_pool[o] = acc[jj];
                    if (a.Bt_pool16) a.Bt_pool16[o] = __float2bfloat16_rn(acc[jj]);
                }
            }
        }
    }
}

// A part: thread owns 4 consecutive columns d..d+3 of A (r x d_in) and writes
// A'[j][d..d+3] = sum_l C_A[j][l] A[l][d..d+3].
__device__ void export_a_cols(const ExportArgs& a, const lf_module& md, int k, const float* cA, int64_t oa,
                              int start, int len) {
    const int r = md.r;
    const float* A = a.A_base + md.A_off;
    const bool vec = (md.d_in % 4 == 0) && (start % 4 == 0);
    for (int d = start + 4 * threadIdx.x; d < start + len; d += 4 * kExpThreads) {
        const int nd = min(4, start + len - d);
        for (int j0 = 0; j0 < k; j0 += kExpJ) {
            float acc[kExpJ][4];
#pragma unroll
            for (int jj = 0; jj < kExpJ; ++jj)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[jj][c] = 0.f;
#pragma unroll 16
            for (int l = 0; l < r; ++l) {
                float4 v;
                const float* src = A + (int64_t)l * md.d_in + d;
                if (vec && nd == 4) {
                    v = __ldg(reinterpret_cast<const float4*>(src));
                } else {
                    v.x = __ldg(src);
                    v.y = nd > 1 ? __ldg(src + 1) : 0.f;
                    v.z = nd > 2 ? __ldg(src + 2) : 0.f;
                    v.w = nd > 3 ? __ldg(src + 3) : 0.f;
                }
#pragma unroll
                for (int jj = 0; jj < kExpJ; ++jj) {
                    if (j0 + jj < k) {
                        const float cj = cA[(j0 + jj) * kMaxRank + l];
                        acc[jj][0] = fmaf(cj, v.x, acc[jj][0]);
                        acc[jj][1] = fmaf(cj, v.y, acc[jj][1]);
                        acc[jj][2] = fmaf(cj, v.z, acc[jj][2]);
                        acc[jj][3] = fmaf(cj, v.w, acc[jj][3]);
                    }
                }
            }
#pragma unroll
            for (int jj = 0; jj < kExpJ; ++jj) {
                if (j0 + jj < k) {
                    const int64_t o = oa + (int64_t)(j0 + jj) * md.d_in + d;
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        if (c < nd) {
                            a.A_pool[o + c] = acc[jj][c];
                            if (a.A_pool16) a.A_pool16[o + c] = __float2bfloat16_rn(acc[jj][c]);
                        }
                    }
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kExpThreads) export_kernel(ExportArgs a) {
    __shared__ __align__(16) float coef[kMaxRank * kMaxRank];   // k x r, row stride kMaxRank, zero past r
    const ExportWork w = a.work[blockIdx.x];
    const lf_module md = a.mods[w.mod];
    const int k = a.ranks[w.mod];
    const int r = md.r;
    if (k <= 0) return;
    const int64_t oa = a.off_A[w.mod], obt = a.off_Bt[w.mod];
    if (w.part == 0) {
        if (obt + (int64_t)k * md.d_out > a.cap_Bt) return;
    } else {
        if (oa + (int64_t)k * md.d_in > a.cap_A) return;
    }
    const float* C = (w.part == 0 ? a.C_Bt : a.C_A) + (size_t)w.mod * a.rs * a.rs;
    for (int e = threadIdx.x; e < k * kMaxRank; e += kExpThreads) {
        const int j = e / kMaxRank, l = e % kMaxRank;
        coef[e] = l < r ? C[j * a.rs + l] : 0.f;
    }
    __syncthreads();
    if (w.part == 0) export_b_rows(a, md, k, coef, obt, w.start, w.len);
    else export_a_cols(a, md, k, coef, oa, w.start, w.len);
}

}  // namespace lf
