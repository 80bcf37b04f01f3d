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
#include "tc.cuh"

namespace lf {

constexpr int kSelThreads = 1024;
constexpr int kSelMaxCand = 26624;   // candidates a group keeps in shared memory (208 KB of fp64)

struct SelArgs {
    const lf_module* mods;
    const int32_t* grp_ptr;    // n_groups + 1
    const int32_t* grp_mods;   // module indices, ascending inside each group
    const double* sigma;       // n x rs
    double* energy;            // n x rs scratch (energies: normalised, or absolute for kind 2)
    int32_t rs;
    lf_policy pol;
    int32_t* ranks;            // n
    // boundary band (refinement); flag_list == nullptr disables flagging
    double band;
    int32_t* flag_list;
    int32_t* flag_count;
    int32_t cand_cap;          // capacity of the shared-memory candidate list (dynamic shared memory / 8)
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

// largest candidate energy (j >= floor, e > 0) strictly below t, 0 if there is none
__device__ double max_below(const SelArgs& a, int m0, int M, double t, double* dred) {
    double b = 0.0;
    const int fl = a.pol.floor;
    for (int q = threadIdx.x; q < M * a.rs; q += blockDim.x) {
        const int mi = q / a.rs, j = q % a.rs;
        const int i = a.grp_mods[m0 + mi];
        if (j < fl || j >= a.mods[i].r) continue;
        const double e = a.energy[(size_t)i * a.rs + j];
        if (e > 0.0 && e < t) b = fmax(b, e);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b = fmax(b, __shfl_xor_sync(0xffffffffu, b, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) dred[threadIdx.x >> 5] = b;
    __syncthreads();
    double m = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, dred[w]);
    return m;
}

// The same two counts over the group's candidate list in shared memory (`nc` energies,
// each > 0), when the whole list fits.
__device__ int64_t count_ge_s(const double* c, int nc, double t, int64_t* red) {
    int64_t n = 0;
    for (int q = threadIdx.x; q < nc; q += blockDim.x) n += (c[q] >= t);
    return block_sum_i64(n, red);
}

__device__ double max_below_s(const double* c, int nc, double t, double* dred) {
    double b = 0.0;
    for (int q = threadIdx.x; q < nc; q += blockDim.x)
        if (c[q] < t) b = fmax(b, c[q]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) b = fmax(b, __shfl_xor_sync(0xffffffffu, b, o));
    __syncthreads();
    if ((threadIdx.x & 31) == 0) dred[threadIdx.x >> 5] = b;
    __syncthreads();
    double m = 0.0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) m = fmax(m, dred[w]);
    return m;
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelArgs a) {
    extern __shared__ double s_cand[];   // a.cand_cap entries
    __shared__ int s_nc;
    __shared__ int64_t red[32];
    __shared__ double dred[32];
    __shared__ int64_t s_take_eq, s_n_eq;
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
    if (a.pol.kind == 3) {  // energy fraction: smallest k >= floor with den * sum_{j<k} s_j^2 >= num * sum_j s_j^2
        for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            const double* sg = a.sigma + (size_t)i * a.rs;
            double tot = 0.0;
            for (int j = 0; j < r; ++j) {
                tot += sg[j] * sg[j];
                if (j + 1 < r && sg[j + 1] > sg[j]) latch_error(LF_ERR_INVALID_ARG);  // rows must descend
            }
            if (!isfinite(tot)) latch_error(LF_ERR_NUMERIC);
            int k = fl;
            bool near = false;
            if (tot > 0.0) {
                const double rhs = (double)a.pol.ratio_num * tot;
                double cum = 0.0;
                int found = 0;
                for (int j = 0; j < r; ++j) {
                    cum += sg[j] * sg[j];
                    if (j + 1 < fl) continue;
                    const double lhs = (double)a.pol.ratio_den * cum;
                    if (!found && lhs >= rhs) found = j + 1;
                    if (rhs > 0.0 && fabs(lhs - rhs) <= a.band * rhs) near = true;   // within the fp32 SVD's reach
                }
                k = found ? found : r;
            }
            a.ranks[i] = min(r, max(fl, k));
            if (a.flag_list && near) {
                const int slot = atomicAdd(a.flag_count, 1);
                a.flag_list[slot] = i;
            }
        }
        return;
    }
    // energies, one module per thread, summed in j order; the candidates (j >= floor,
    // e > 0) are also copied to shared memory when the group's list fits
    if (threadIdx.x == 0) s_nc = 0;
    __syncthreads();
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
                e = a.pol.kind == 2 ? sq : __ddiv_rn(sq, tot);   // kind 2: absolute energy
            }
            en[j] = e;
        }
        int nv = 0;
        for (int j = fl; j < r; ++j) nv += en[j] > 0.0;
        const int b = atomicAdd(&s_nc, nv);
        if (b + nv <= a.cand_cap)
            for (int j = fl, q = b; j < r; ++j)
                if (en[j] > 0.0) s_cand[q++] = en[j];
        a.ranks[i] = fl;
    }
    rsum = block_sum_i64(rsum, red);   // (synchronises the block: s_nc and s_cand are complete)
    const int nc = s_nc;
    const bool in_smem = nc <= a.cand_cap;
#define LF_COUNT_GE(t) (in_smem ? count_ge_s(s_cand, nc, (t), red) : count_ge(a, m0, M, (t), red))
    const int64_t K = ((int64_t)a.pol.ratio_num * rsum) / a.pol.ratio_den;
    const int64_t extra = K - (int64_t)fl * M;
    if (extra <= 0) return;  // ranks stay at the floor

    const double tiny = __longlong_as_double(1ll);
    const int64_t npos = LF_COUNT_GE(tiny);
    double theta;
    int64_t take_eq, n_eq = 0;
    if (npos <= extra) {
        theta = tiny;  // take every positive candidate
        take_eq = INT64_MAX;
    } else {
        // largest bit pattern t with count(e >= t) >= extra (bisection on the ordered bits)
        long long lo = 1, hi = 0x7FF0000000000000ll;
        while (lo < hi) {
            const long long mid = lo + (hi - lo + 1) / 2;
            const int64_t c = LF_COUNT_GE(__longlong_as_double(mid));
            if (c >= extra) lo = mid; else hi = mid - 1;
        }
        theta = __longlong_as_double(lo);
        const int64_t n_gt = LF_COUNT_GE(__longlong_as_double(lo + 1));
        take_eq = extra - n_gt;
        n_eq = LF_COUNT_GE(theta) - n_gt;
    }
    if (threadIdx.x == 0) {
        s_theta = theta;
        s_take_eq = take_eq;
        s_n_eq = n_eq;
    }
    __syncthreads();
    theta = s_theta;
    take_eq = s_take_eq;
    n_eq = s_n_eq;
    // per module: all e > theta, then the first take_eq candidates equal to theta in
    // (module, j) order.  When every candidate equal to theta is taken (the usual case)
    // each module counts its e >= theta on its own; a tie cut by the budget takes the
    // equal-candidate prefix over modules serially.
    if (take_eq >= n_eq) {
        for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            const double* en = a.energy + (size_t)i * a.rs;
            int k = fl;
            for (int j = fl; j < r; ++j) {
                const double e = en[j];
                if (e > 0.0 && e >= theta) ++k;
                else break;
            }
            a.ranks[i] = k;
        }
    } else if (threadIdx.x == 0) {
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
        // The selection can differ from the exact one only if the boundary is a near tie:
        // the last selected energy theta and the first one left out (a candidate equal to
        // theta that the tie order leaves out, else the largest below theta) closer than
        // twice the band, the band being far above the main path's energy error.  Then
        // the modules holding a candidate within the band of theta are refined in fp64.
        const double below = in_smem ? max_below_s(s_cand, nc, theta, dred) : max_below(a, m0, M, theta, dred);
        const bool tie_out = n_eq > take_eq;
        if (!tie_out && theta - below > 2.0 * a.band * theta) return;
        for (int mi = threadIdx.x; mi < M; mi += blockDim.x) {
            const int i = a.grp_mods[m0 + mi];
            const int r = a.mods[i].r;
            const double* en = a.energy + (size_t)i * a.rs;
            bool f = false;
            for (int j = fl; j < r; ++j) {
                const double e = en[j];
                if (e > 0.0 && fabs(e - theta) <= 2.0 * a.band * theta) f = true;
            }
            if (f) {
                const int slot = atomicAdd(a.flag_count, 1);
                a.flag_list[slot] = i;
            }
        }
    }
#undef LF_COUNT_GE
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
            info[mf].slot0 = nch > 1 ? slot : -1;   // nch > 1: the merge tree's nodes from slot0
            for (int c = 0; c < nch; ++c) {
                work[w].mf = mf;
                work[w].row0 = c * chunk;
                work[w].nrows = min(chunk, rows - c * chunk);
                work[w].slot = nch > 1 ? slot + c : -1;
                ++w;
            }
            if (nch > 1) slot += tree_slots(nch);
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
constexpr int kExpRows = 64;       // B part: rows per pipeline stage
constexpr int kExpStages = 3;
constexpr int kExpStageFloats = kExpRows * kMaxRank;   // 16 KB per stage
constexpr int kExpACols = 256;     // A part: columns per block (one per thread)
constexpr int kExpALRows = 16;     // A part: rows of A per stage (4 stages per column block)
constexpr int kExpAJ = 16;         // A part: retained directions per pass
constexpr size_t kExportSmem = (size_t)(kMaxRank * kMaxRank + kExpStages * kExpStageFloats) * sizeof(float);
static_assert(kExpACols * kExpALRows == kExpStageFloats, "A stage = B stage size");

__device__ __forceinline__ void exp_cp16(float* dst, const float* src, uint32_t n) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void exp_cp4(float* dst, const float* src, uint32_t n) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(n) : "memory");
}

// B stage: rows e0 .. e0+63 of B, 64 floats per row, 16-byte chunk c of row e stored at
// chunk position c ^ (e & 7) (whole 128-byte lines for the copies, distinct banks for
// the per-row reads).  Entries past the item or past r are zero-filled.
__device__ __forceinline__ void export_issue_b(float* st, const float* X, int r, int i0, int nrem, bool vec) {
    const int tid = threadIdx.x;
    if (vec) {
        for (int q = tid; q < kExpRows * 16; q += kExpThreads) {
            const int row = q >> 4, c4 = q & 15;
            const bool ok = row < nrem && 4 * c4 < r;
            exp_cp16(st + row * kMaxRank + 4 * (c4 ^ (row & 7)), ok ? X + (int64_t)(i0 + row) * r + 4 * c4 : X,
                     ok ? 16u : 0u);
        }
    } else {
        for (int q = tid; q < kExpRows * kMaxRank; q += kExpThreads) {
            const int row = q >> 6, c = q & 63;
            const bool ok = row < nrem && c < r;
            exp_cp4(st + row * kMaxRank + 4 * ((c >> 2) ^ (row & 7)) + (c & 3),
                    ok ? X + (int64_t)(i0 + row) * r + c : X, ok ? 4u : 0u);
        }
    }
}

// A stage: rows l0 .. l0+15 of A, columns c0 .. c0+255 (row-major, 1 KB per row).
// Rows past r and columns past the item are zero-filled.
__device__ __forceinline__ void export_issue_a(float* st, const float* X, int r, int64_t d_in, int l0, int c0,
                                               int ncols, bool vec) {
    const int tid = threadIdx.x;
    if (vec) {
        for (int q = tid; q < kExpALRows * (kExpACols / 4); q += kExpThreads) {
            const int l = q >> 6, c4 = q & 63;
            const int nv = (l0 + l < r) ? min(4, max(0, ncols - 4 * c4)) : 0;
            exp_cp16(st + l * kExpACols + 4 * c4, nv > 0 ? X + (int64_t)(l0 + l) * d_in + c0 + 4 * c4 : X,
                     4u * (uint32_t)nv);
        }
    } else {
        for (int q = tid; q < kExpALRows * kExpACols; q += kExpThreads) {
            const int l = q >> 8, c = q & 255;
            const bool ok = l0 + l < r && c < ncols;
            exp_cp4(st + l * kExpACols + c, ok ? X + (int64_t)(l0 + l) * d_in + c0 + c : X, ok ? 4u : 0u);
        }
    }
}

// One B stage: thread (row e = tid % 64, output group g = tid / 64) forms outputs
// j = g, g + 4, ... (< k) as dot products of its row with coefficient rows j (shared
// memory, broadcast within the warp):  B'^T[j][e] = sum_l C_Bt[j][l] B[e][l].
template <int NQ>
__device__ __forceinline__ void export_stage_b(const ExportArgs& a, const lf_module& md, int k, const float* coef,
                                               const float* st, int i0, int nrem, int64_t obase, int jbase) {
    const int tid = threadIdx.x, e = tid & (kExpRows - 1), g = tid >> 6;
    // outputs j = jbase + g + 4q of this thread; g is uniform over a warp, so the
    // directions past k are skipped without divergence (NQ covers the largest k)
    const int nq = min(NQ, max(0, (k - jbase - g + 3) / 4));
    if (nq == 0) return;
    // packed fp32 pairs: even and odd columns in two chains, added at the end
    float2 acc[NQ];
#pragma unroll
    for (int q = 0; q < NQ; ++q) acc[q] = make_float2(0.f, 0.f);
    const float* row = st + e * kMaxRank;
#pragma unroll 4
    for (int c = 0; c < 16; ++c) {
        const float4 x = *reinterpret_cast<const float4*>(row + 4 * (c ^ (e & 7)));
        const float2 x01 = make_float2(x.x, x.y), x23 = make_float2(x.z, x.w);
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
            if (q < nq) {
                const float4 cf = *reinterpret_cast<const float4*>(coef + (jbase + g + 4 * q) * kMaxRank + 4 * c);
                acc[q] = __ffma2_rn(make_float2(cf.x, cf.y), x01, acc[q]);
                acc[q] = __ffma2_rn(make_float2(cf.z, cf.w), x23, acc[q]);
            }
        }
    }
    if (e >= nrem) return;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
        const int j = jbase + g + 4 * q;
        if (j < k) {
            const float v = acc[q].x + acc[q].y;
            const int64_t o = obase + (int64_t)j * md.d_out + i0 + e;
            a.Bt_pool[o] = v;
            if (a.Bt_pool16) a.Bt_pool16[o] = __float2bfloat16_rn(v);
        }
    }
}

template <int NQ>
__device__ void export_item_b(const ExportArgs& a, const lf_module& md, int k, const float* coef, float* stages,
                              const float* X, int start, int len, int64_t obase, bool vec) {
    const int nst = (len + kExpRows - 1) / kExpRows;
#pragma unroll
    for (int s = 0; s < kExpStages - 1; ++s) {
        if (s < nst) export_issue_b(stages + s * kExpStageFloats, X, md.r, start + s * kExpRows, len - s * kExpRows, vec);
        tc::cp_async_commit();
    }
    for (int t = 0; t < nst; ++t) {
        tc::cp_async_wait<kExpStages - 2>();
        __syncthreads();   // stage t landed for every thread; stage t - 1 fully consumed
        const int tn = t + kExpStages - 1;
        if (tn < nst)
            export_issue_b(stages + (tn % kExpStages) * kExpStageFloats, X, md.r, start + tn * kExpRows,
                           len - tn * kExpRows, vec);
        tc::cp_async_commit();
        const float* st = stages + (t % kExpStages) * kExpStageFloats;
        export_stage_b<NQ>(a, md, k, coef, st, start + t * kExpRows, len - t * kExpRows, obase, 0);
        if (NQ == 8)   // k > 16: a second pass for j = 32 .. 63
            export_stage_b<NQ>(a, md, k, coef, st, start + t * kExpRows, len - t * kExpRows, obase, 32);
    }
    tc::cp_async_wait<0>();
}

// A part: the item's columns go in blocks of 256 (one column per thread); each block is
// four stages of 16 rows of A, accumulated in registers for kExpAJ retained directions
// at a time (further passes re-stream the block when k > kExpAJ):
//   A'[j][d] = sum_l C_A[j][l] A[l][d].
__device__ void export_item_a(const ExportArgs& a, const lf_module& md, int k, const float* coef, float* stages,
                              const float* X, int start, int len, int64_t obase, bool vec) {
    const int tid = threadIdx.x;
    const int nblk = (len + kExpACols - 1) / kExpACols;
    const int npass = (k + kExpAJ - 1) / kExpAJ;
    const int nst = npass * nblk * 4;
    auto issue = [&](int t) {
        const int lq = t & 3, blk = (t >> 2) % nblk;
        const int c0 = start + blk * kExpACols;
        export_issue_a(stages + (t % kExpStages) * kExpStageFloats, X, md.r, md.d_in, kExpALRows * lq, c0,
                       min(kExpACols, start + len - c0), vec);
    };
#pragma unroll
    for (int s = 0; s < kExpStages - 1; ++s) {
        if (s < nst) issue(s);
        tc::cp_async_commit();
    }
    float2 acc[kExpAJ / 2];   // packed pairs of retained directions (2p, 2p + 1)
    for (int t = 0; t < nst; ++t) {
        tc::cp_async_wait<kExpStages - 2>();
        __syncthreads();
        const int tn = t + kExpStages - 1;
        if (tn < nst) issue(tn);
        tc::cp_async_commit();
        const int lq = t & 3, blk = (t >> 2) % nblk, pass = t / (4 * nblk);
        const int j0 = pass * kExpAJ;
        if (lq == 0) {
#pragma unroll
            for (int jp = 0; jp < kExpAJ / 2; ++jp) acc[jp] = make_float2(0.f, 0.f);
        }
        const float* st = stages + (t % kExpStages) * kExpStageFloats;
        float x[kExpALRows];
#pragma unroll
        for (int l = 0; l < kExpALRows; ++l) x[l] = st[l * kExpACols + tid];
        const int nj = min(kExpAJ, k - j0);
        // coefficients pair-interleaved: float2 (C[2p][l], C[2p + 1][l]) at p * 64 + l
        const float4* cp4 = reinterpret_cast<const float4*>(coef);
#pragma unroll
        for (int jp = 0; jp < kExpAJ / 2; ++jp) {
            if (2 * jp < nj) {
                const int p = j0 / 2 + jp;
                float2 t2 = acc[jp];
#pragma unroll
                for (int l2 = 0; l2 < kExpALRows / 2; ++l2) {
                    const float4 cf = cp4[p * (kMaxRank / 2) + (kExpALRows * lq) / 2 + l2];
                    t2 = __ffma2_rn(make_float2(cf.x, cf.y), make_float2(x[2 * l2], x[2 * l2]), t2);
                    t2 = __ffma2_rn(make_float2(cf.z, cf.w), make_float2(x[2 * l2 + 1], x[2 * l2 + 1]), t2);
                }
                acc[jp] = t2;
            }
        }
        if (lq == 3) {
            const int d = start + blk * kExpACols + tid;
            if (d < start + len) {
#pragma unroll
                for (int jj = 0; jj < kExpAJ; ++jj) {
                    if (jj < nj) {
                        const float v = (jj & 1) ? acc[jj >> 1].y : acc[jj >> 1].x;
                        const int64_t o = obase + (int64_t)(j0 + jj) * md.d_in + d;
                        a.A_pool[o] = v;
                        if (a.A_pool16) a.A_pool16[o] = __float2bfloat16_rn(v);
                    }
                }
            }
        }
    }
    tc::cp_async_wait<0>();
}

// One CTA per work item (a run of up to 2048 rows of B or columns of A of one
// module), streamed through a kExpStages cp.async ring of 16 KB stages; every output
// element is one 64-term dot product with a row of the coefficients.
__global__ void __launch_bounds__(kExpThreads, 3) export_kernel(ExportArgs a) {
    extern __shared__ __align__(16) float exp_smem[];
    float* coef = exp_smem;                             // k x 64, row stride 64, zero past r and past k
    float* stages = exp_smem + kMaxRank * kMaxRank;
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
    const int kfill = w.part == 1 ? min(kMaxRank, ((k + kExpAJ - 1) / kExpAJ) * kExpAJ)
                                  : (k <= 4 ? 4 : (k <= 8 ? 8 : (k <= 16 ? 16 : kMaxRank)));   // rows the stages read
    for (int e = threadIdx.x; e < kfill * kMaxRank; e += kExpThreads) {
        const int j = e / kMaxRank, l = e % kMaxRank;
        const float v = (j < k && l < r) ? C[j * a.rs + l] : 0.f;
        if (w.part == 1)   // A part: pair-interleaved, float2 (C[2p][l], C[2p + 1][l]) at p * 64 + l
            coef[(j >> 1) * 2 * kMaxRank + 2 * l + (j & 1)] = v;
        else
            coef[e] = v;
    }
    const float* X = w.part == 0 ? a.B_base + md.B_off : a.A_base + md.A_off;
    // coefficient rows are read after the first barrier inside export_item_*
    if (w.part == 1) {
        export_item_a(a, md, k, coef, stages, X, w.start, w.len, oa, md.d_in % 4 == 0);
        return;
    }
    const bool vec = r % 4 == 0;
    if (k <= 4)
        export_item_b<1>(a, md, k, coef, stages, X, w.start, w.len, obt, vec);
    else if (k <= 8)
        export_item_b<2>(a, md, k, coef, stages, X, w.start, w.len, obt, vec);
    else if (k <= 16)
        export_item_b<4>(a, md, k, coef, stages, X, w.start, w.len, obt, vec);
    else
        export_item_b<8>(a, md, k, coef, stages, X, w.start, w.len, obt, vec);
}

}  // namespace lf
