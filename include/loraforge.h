/*
 * loraforge.h -- C ABI of libloraforge.so, the sm_100a hot path of LoRAForge-style
 * post-hoc LoRA compression and multi-LoRA serving.
 *
 * What the method computes (sources are named by page title and section):
 *  - "Compress then Serve" (academ.us/article/2407.00066), section 3: a module's
 *    LoRA update is dW = B A with B (d_out x r) and A (r x d_in); the adapted
 *    output is (W0 + B A) x.  Section 4, eq. 4: the per-module truncated SVD
 *    U_k S_k V_k^T is the best rank-k approximation (Eckart-Young), with S_k V_k^T
 *    stored as one matrix.
 *  - LoRAForge (kongchang.com), section "FlashTSQR: An Accelerator for Batched
 *    Factor Construction": factor construction runs a tall-skinny QR (local QR of
 *    row blocks, then merging) batched across modules and row tiles.
 *  - LoRAForge abstract (mlinfo.pages.dev, arXiv 2611.01256) and the kongchang.com
 *    section "LoRAForge's Core Design: Explicit Retained-Rank Representation and
 *    Dual Strategies": retained ranks come from a uniform ratio (LoRAForge-U) or a
 *    spectral-energy budget with a per-module floor (LoRAForge-S) and are carried
 *    as an explicit retained-rank table to rank-specialised kernels, never padded.
 *  - "Compress then Serve", section 13.4 "Punica": the side path is buffer = A x
 *    (fp32 buffer, rows selected per token by an adapter index), then
 *    y += scale * B buffer.
 *
 * Conventions shared by every entry point:
 *  - All pointers are DEVICE pointers unless marked [host].  Matrices are
 *    row-major.  The caller owns all memory; the library allocates nothing.
 *    Scratch memory ("workspace") is passed in; its size comes from the matching
 *    *_workspace_size query.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; 0 = legacy default).
 *    Argument errors are found on the host before any launch and returned as an
 *    lf_status; nothing is launched in that case.  Errors that only the device can
 *    see (an adapter id out of range, a non-finite value, a pool that is too small,
 *    a misaligned device offset) are latched into a per-device error word that
 *    lf_get_device_status() returns and clears.  Kernels never trap.
 *  - Results are bitwise reproducible from run to run: no floating-point atomics,
 *    fixed reduction orders.
 *  - Device pointers to fp32 data must be 16-byte aligned; factor offsets (in
 *    elements) must be multiples of 4; bf16 rows (x, y, pools) must be 16-byte
 *    aligned and d_in, d_out multiples of 8.  Violations return LF_ERR_ALIGNMENT.
 */
#ifndef LORAFORGE_H
#define LORAFORGE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* lf_stream_t; /* the same handle as cudaStream_t */

typedef enum {
    LF_OK = 0,
    LF_ERR_INVALID_ARG = 1, /* null pointer, negative count, bad policy fields      */
    LF_ERR_SHAPE = 2,       /* r < 1, r > 64, r > min(d_in, d_out), floor > r ...    */
    LF_ERR_BAD_INDEX = 3,   /* (device) adapter id < -1 or >= n_adapters             */
    LF_ERR_WORKSPACE = 4,   /* workspace or output pool smaller than required        */
    LF_ERR_NUMERIC = 5,     /* (device) non-finite input or singular value           */
    LF_ERR_TIMEOUT = 6,     /* (device) a bounded wait ran out                       */
    LF_ERR_CUDA = 7,        /* a CUDA runtime call failed                            */
    LF_ERR_ALIGNMENT = 8    /* pointer/offset/leading dimension not aligned          */
} lf_status;

/* One LoRA module (B: d_out x r, A: r x d_in), "Compress then Serve" section 3.
 * group = adapter id: the scope of the LoRAForge-S budget.
 * B_off / A_off = element offsets of B and A inside the B_base / A_base buffers. */
typedef struct {
    int32_t d_out, d_in, r, group;
    int64_t B_off, A_off;
} lf_module;

/* Allocation policy.  kind 0 = LoRAForge-U, kind 1 = LoRAForge-S, kind 2 =
 * spectral budget on absolute energies (variant of S), kind 3 = energy fraction.
 * ratio = ratio_num / ratio_den (exact integers, e.g. 1/4, 1/12); floor >= 1.
 *  U: k = clamp(floor(ratio_num*r/ratio_den + 1/2), floor, r).
 *  S: per group, K = floor(ratio_num * sum r / ratio_den); every module gets
 *     `floor`; the remaining K - floor*M slots go to the largest normalised
 *     energies e_ij = sigma_ij^2 / sum_j sigma_ij^2 (j >= floor, e_ij > 0),
 *     ties to the lower module index, then lower j.
 *  kind 2: as S with e_ij = sigma_ij^2 (the choice that minimises the group's
 *     summed squared Frobenius error sum_i ||dW_i - B'_i A'_i||^2 under the budget).
 *  kind 3: per module, the smallest k in [floor, r] whose leading directions keep
 *     ratio_num / ratio_den (<= 1) of its spectral energy,
 *     ratio_den * sum_{j<k} sigma_j^2 >= ratio_num * sum_j sigma_j^2 (LoRASpace's
 *     minimal subspace keeping 99 % of the energy, read per module); no group budget.
 *  Spectral kinds (1-3) recompute in fp64 the modules whose decision is a near tie
 *  (kinds 1-2: the last selected energy and the first left out closer than 2e-4 of the
 *  threshold; kind 3: a cumulative energy within 1e-4 of it), so ranks match an fp64
 *  reference.
 * The budget scope is the module `group`: one group per adapter gives per-adapter
 * budgets, one group over all modules a fleet-wide budget. */
typedef struct {
    int32_t kind, ratio_num, ratio_den, floor;
} lf_policy;

/* Largest r over the modules: the stride used by the per-module r x r outputs. */
int32_t lf_rank_stride(const lf_module* mods /*[host]*/, int32_t n);

/* ---- Factor construction (FlashTSQR + small SVD) -----------------------------
 * For every module i, with X_B = B_i (d_out x r) and X_A = A_i^T (d_in x r):
 *   R_B = R(X_B), R_A = R(X_A): the R factors of the thin QRs, upper triangular,
 *         diag >= 0, computed by a batched tall-skinny QR over row tiles of every
 *         module at once: each row tile (up to 24 576 rows) contributes its Gram,
 *         tile Grams are summed in a fixed order and R = chol(X^T X) in fp64
 *         (R^T R = X^T X defines the same R as the QR).  The tile Gram is exact for
 *         the 32-bit fixed-point image of the tile (each column scaled by a power of
 *         two from its first 128 rows and truncated: a columnwise error below 2^-27
 *         of the column's largest value), formed on the int8 tensor cores from its
 *         four byte planes.  A matrix whose rows or offset are not 16-byte aligned,
 *         or with a value at or above its column's scale, takes an fp64 Gram of the
 *         fp32 products instead.  A matrix whose Cholesky pivot falls to <= 1e-9 of
 *         its Gram diagonal (numerically rank-deficient, a zero column, non-finite
 *         input) is factored by structured Householder reflections of [R; tile]
 *         over row chunks, merged in chunk order;
 *   M = R_B R_A^T (r x r) and its SVD M = U S V^T (one-sided Jacobi in fp32,
 *   outputs stored as fp64):
 *   sigma (descending) are the singular values of dW = B A, Q_B U its left and
 *   Q_A V its right singular vectors.
 * Outputs (rs = lf_rank_stride):
 *   R_B, R_A : n x rs x rs fp32, entries past r_i are zero.
 *   sigma    : n x rs fp64, descending, zero past r_i.
 *   U, V     : n x rs x rs fp64; column j of U[i] / V[i] pairs with sigma[i][j];
 *              U and V columns with sigma = 0 are zero.  The Jacobi sweeps rotate
 *              the rows of M only (rows end as sigma_j v_j^T); column j of U is
 *              M v_j / sigma_j, accurate to about 1e-7 sigma_1 / sigma_j, so the
 *              leading (retained) directions are the accurate ones.  U may be null;
 *              when it is not, its block also serves as scratch during the call.
 * Workspace: lf_tsqr_workspace_size(mods, n) bytes.  B_base and A_base are fp32. */
size_t lf_tsqr_workspace_size(const lf_module* mods /*[host]*/, int32_t n);
lf_status lf_tsqr_batched(const lf_module* mods /*[host]*/, int32_t n,
                          const float* B_base, const float* A_base,
                          float* R_B, float* R_A, double* sigma, double* U, double* V,
                          void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Rank allocation alone (LoRAForge-U / -S) --------------------------------
 * ranks[i] from sigma (n x rs fp64, rows descending) under `pol`; off_A / off_Bt
 * are n+1 prefix sums of ranks[i]*d_in and ranks[i]*d_out (pool element offsets).
 * A row that is not in descending order latches LF_ERR_INVALID_ARG on the device.
 * Workspace: lf_select_workspace_size(mods, n). */
size_t lf_select_workspace_size(const lf_module* mods /*[host]*/, int32_t n);
lf_status lf_select_ranks(const lf_module* mods /*[host]*/, int32_t n, lf_policy pol,
                          const double* sigma, int32_t* ranks, int64_t* off_A, int64_t* off_Bt,
                          void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Truncation + export -----------------------------------------------------
 * Allocates ranks as lf_select_ranks does.  For the spectral policies, in a group
 * whose selection boundary is a near tie (the last selected energy theta and the first
 * one left out closer than 2e-4 theta), the modules holding a candidate within 2e-4
 * theta of theta get their spectrum recomputed in fp64 from B and A before the final
 * choice, so ranks match an fp64 computation; more such modules than the workspace's
 * refinement capacity (8 per group + 64) latch LF_ERR_WORKSPACE.  Then, per module with k = ranks[i]:
 *   B'^T = (R_A^T V_k S_k^-1)^T B^T   (k x d_out, rows of the retained left
 *                                      singular vectors of dW)
 *   A'   = (U_k^T R_B) A               (k x d_in, = S_k V_k^T Q_A^T)
 * so that B' A' is the rank-k truncated SVD of dW.  Directions with sigma = 0
 * export as zero rows.  Pools are packed with no padding: module i occupies
 * A_pool[off_A[i] .. off_A[i+1]) and Bt_pool[off_Bt[i] .. off_Bt[i+1]).
 * pool_cap_A / pool_cap_Bt = pool capacities in elements; a larger total latches
 * LF_ERR_WORKSPACE and writes nothing past the capacity (lf_export_pool_bound gives
 * a safe capacity).  A_pool_bf16 / Bt_pool_bf16 (same offsets, at least the same
 * capacities) may be NULL. */
size_t lf_export_workspace_size(const lf_module* mods /*[host]*/, int32_t n);
void lf_export_pool_bound(const lf_module* mods /*[host]*/, int32_t n, lf_policy pol,
                          int64_t* cap_A /*[host]*/, int64_t* cap_Bt /*[host]*/);
lf_status lf_truncate_export(const lf_module* mods /*[host]*/, int32_t n, lf_policy pol,
                             const float* B_base, const float* A_base,
                             const float* R_B, const float* R_A, const double* sigma,
                             const double* U, const double* V,
                             int32_t* ranks, int64_t* off_A, int64_t* off_Bt,
                             float* A_pool, float* Bt_pool,
                             void* A_pool_bf16, void* Bt_pool_bf16,
                             int64_t pool_cap_A, int64_t pool_cap_Bt,
                             void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Multi-LoRA shrink / expand (one projection) -----------------------------
 * For every token t with a = ids[t] >= 0:
 *   t_vec = A'_a x_t              (k_a values, fp32, never rounded)
 *   y_t   = bf16( y_t + scale * B'_a t_vec )   (one rounding, RN-even)
 * x: T x d_in bf16, y: T x d_out bf16 (in place), ids: T int32 (-1 = no adapter,
 * row left bit-for-bit unchanged; an id >= n_adapters or < -1 latches
 * LF_ERR_BAD_INDEX and leaves that token untouched).
 * ranks / off_A / off_Bt: per adapter, this projection's retained rank and element
 * offsets of its A' (k x d_in) and B'^T (k x d_out) inside the bf16 pools, which
 * hold pool_elems_A / pool_elems_Bt elements; an adapter whose rows would reach
 * past a pool (or whose offset is not a multiple of 8, or k > 64) latches an error
 * on the device and its tokens are left untouched.
 * A batch with few tokens per resident adapter (T <= 8 * n_adapters) is applied
 * token by token with each token's own adapter index (no sort).  Other batches are
 * routed by a stable sort on the adapter id into segments (adapter, start, length)
 * over a permutation of token indices; segments of 64 or more tokens run on tcgen05
 * tensor cores (every adapter's k rows read once per 128-token tile), the other
 * tokens on the token-parallel kernel in routing order; k is never padded.  On the tensor-core path a 128-token tile whose tokens are consecutive rows
 * of x and y (a prefill request) moves x and y by TMA tiles; a tile of scattered
 * tokens gathers its rows one by one (same results, bit for bit).  If seg_out is
 * not NULL it receives the routing, as int32: [n_seg,
 * n_valid, then 3*n_seg (adapter,start,len), then n_valid token indices]; it must
 * hold 2 + 3*min(T,n_adapters) + T ints.
 * Workspace: lf_apply_workspace_size(T, n_adapters).  The same as a one-slice
 * lf_lora_shrink_expand_slices call with y_ld = d_out. */
size_t lf_apply_workspace_size(int32_t T, int32_t n_adapters);
lf_status lf_lora_shrink_expand(int32_t T, int32_t d_in, int32_t d_out,
                                const void* x, void* y, const int32_t* ids,
                                int32_t n_adapters, const int32_t* ranks,
                                const int64_t* off_A, const int64_t* off_Bt,
                                const void* A_pool, const void* Bt_pool,
                                int64_t pool_elems_A, int64_t pool_elems_Bt, float scale,
                                int32_t* seg_out, void* ws, size_t ws_bytes,
                                lf_stream_t stream);

/* ---- Multi-LoRA shrink / expand over output slices sharing x ------------------
 * LoRAForge's serving side runs the projections that read the same input (q/k/v,
 * gate/up) together: one call applies up to 4 output slices, each a projection
 * with its own factor pools, ranks and place in y.  For every token t with
 * a = ids[t] >= 0 and every slice s:
 *   t_s    = A'_{s,a} x_t                                    (k_{s,a} fp32 values)
 *   y_t[y_offset_s .. y_offset_s + d_out_s) =
 *            bf16( y_t[...] + scale_a * B'_{s,a} t_s )       (one rounding)
 * with scale_a = adapter_scale[a] when adapter_scale (device, n_adapters floats)
 * is not NULL, else `scale`.  y has T rows of y_ld elements; slices must not
 * overlap in y (overlapping slices race).  The routing is computed once for all
 * slices, and on the tensor-core path x is read once: the shrink contracts x with
 * the slices' A' rows concatenated (N = sum of ranks).  Argument rules as for
 * lf_lora_shrink_expand, plus: 1 <= n_slices <= 4, d_out_s, y_offset_s and y_ld
 * multiples of 8, y_offset_s + d_out_s <= y_ld; errors per (adapter, slice) leave
 * that slice of the adapter's tokens untouched.
 * Workspace: lf_apply_slices_workspace_size(T, n_adapters, n_slices). */
typedef struct {
    int32_t d_out;              /* output columns of the slice */
    int32_t max_rank;           /* 0, or an upper bound (1..64) of every adapter's rank in this slice:
                                   a launch may then leave out kernels sized for larger ranks (on the
                                   tensor-core path a bound <= 16 keeps only the rank-16 expand); an
                                   adapter whose rank exceeds it latches LF_ERR_SHAPE and its tokens
                                   are left untouched in this slice */
    int64_t y_offset;           /* first column of the slice in each row of y */
    const int32_t* ranks;       /* per adapter: retained rank of this slice's module */
    const int64_t* off_A;       /* per adapter: element offset of A' (k x d_in) in A_pool */
    const int64_t* off_Bt;      /* per adapter: element offset of B'^T (k x d_out) in Bt_pool */
    const void* A_pool;         /* bf16 */
    const void* Bt_pool;        /* bf16 */
    int64_t pool_elems_A, pool_elems_Bt;
} lf_slice;
size_t lf_apply_slices_workspace_size(int32_t T, int32_t n_adapters, int32_t n_slices);
lf_status lf_lora_shrink_expand_slices(int32_t T, int32_t d_in, const void* x, void* y, int64_t y_ld,
                                       const int32_t* ids, int32_t n_adapters,
                                       const lf_slice* slices /*[host]*/, int32_t n_slices,
                                       float scale, const float* adapter_scale, int32_t* seg_out,
                                       void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Several projections of one batch in one call -----------------------------
 * A decode step applies every adapted projection of a layer to the same tokens
 * ("Compress then Serve", section 13.4: the side path per token, indexed by the
 * token's adapter).  This call takes up to LF_MAX_PROJECTIONS projections, each
 * with its own input x (T x d_in bf16, row-major), its own y (T rows of y_ld bf16)
 * and its own factor tables (the lf_slice fields: d_out, y_offset, ranks, offsets,
 * pools), and for every token t with a = ids[t] >= 0 and every projection p:
 *   t_p    = A'_{p,a} x_{p,t}                                 (k_{p,a} fp32 values)
 *   y_{p,t}[y_offset_p .. y_offset_p + d_out_p) =
 *            bf16( y_{p,t}[...] + scale_a * B'_{p,a} t_p )    (one rounding)
 * with scale_a as for lf_lora_shrink_expand_slices.  In the decode regime
 * (T <= 8 n_adapters) every projection goes in one launch of the token-parallel
 * kernel, and ws is not used (it may be NULL with ws_bytes 0).  Otherwise the
 * projections are applied one after the other on the routed path: the first routes
 * the batch into ws and the others reuse its tables, so ws must then hold
 * lf_apply_workspace_size(T, n_adapters) bytes.  Projections must not write
 * overlapping parts of any y, and no y may overlap an x of the same call.
 * Per projection the argument rules of lf_lora_shrink_expand_slices with one slice
 * apply (the projection's reserved field 0); host errors are returned before anything is launched,
 * and device-side errors latch as there, per (adapter, projection). */
#define LF_MAX_PROJECTIONS 8
typedef struct {
    const void* x;              /* T x d_in bf16 */
    void* y;                    /* T rows of y_ld bf16, updated in place */
    int32_t d_in;
    int32_t reserved;           /* 0 */
    int64_t y_ld;               /* row stride of y (elements), multiple of 8 */
    lf_slice slice;             /* where in y, and with which factors */
} lf_projection;
lf_status lf_lora_shrink_expand_projections(int32_t T, const int32_t* ids, int32_t n_adapters,
                                            const lf_projection* projs /*[host]*/, int32_t n_proj,
                                            float scale, const float* adapter_scale,
                                            void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Routing once per batch ---------------------------------------------------
 * Every projection of a forward pass sees the same token ids, so the routing (the
 * stable sort of tokens by adapter, the segment table and the work items) can be
 * computed once: lf_route_tokens writes it into `ws`, and
 * lf_lora_shrink_expand_slices_routed then applies any projection of the batch
 * (same T, ids and n_adapters, any n_slices) from those tables without a routing
 * pass.  ws must be sized for the largest n_slices used with it
 * (lf_apply_slices_workspace_size); the tables in ws are those of the most recent
 * routing pass on it (lf_route_tokens or any unrouted apply call).  A routed call on
 * a workspace whose tables were written for another T or n_adapters (or never)
 * applies nothing and latches LF_ERR_INVALID_ARG.  In the decode regime
 * (T <= 8 n_adapters) the side path reads ids directly and the tables are not used.
 * Host errors as for lf_lora_shrink_expand_slices. */
lf_status lf_route_tokens(int32_t T, const int32_t* ids, int32_t n_adapters, void* ws, size_t ws_bytes,
                          lf_stream_t stream);
lf_status lf_lora_shrink_expand_slices_routed(int32_t T, int32_t d_in, const void* x, void* y, int64_t y_ld,
                                              const int32_t* ids, int32_t n_adapters,
                                              const lf_slice* slices /*[host]*/, int32_t n_slices,
                                              float scale, const float* adapter_scale,
                                              void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Sigma-sandwich serving (jointly compressed adapters) ---------------------
 * "Compress then Serve" (academ.us/article/2407.00066), sections 3.1 and 11: the
 * adapters of one module share U (d_out x rank) and V (d_in x rank) and keep a
 * small Sigma_a each, B_a A_a ~ U Sigma_a V^T; serving applies, for every token t
 * with a = ids[t] >= 0,
 *   y_t = bf16( y_t + scale * U (Sigma_a (V^T x_t)) )     (fp32 intermediates, one rounding)
 * Vt = V^T (rank x d_in bf16), Ut = U^T (rank x d_out bf16), both shared by all
 * adapters; sigma (device fp32): sigma_diag = 1 -> n_adapters x rank (diagonal
 * Sigma_a), sigma_diag = 0 -> n_adapters x rank x rank row-major (full Sigma_a).
 * Same routing, regimes, id rules and workspace as lf_lora_shrink_expand
 * (lf_apply_workspace_size(T, n_adapters)); 1 <= rank <= 64. */
lf_status lf_lora_sigma_sandwich(int32_t T, int32_t d_in, int32_t d_out, const void* x, void* y,
                                 const int32_t* ids, int32_t n_adapters, int32_t rank,
                                 const void* Vt, const void* Ut, const float* sigma, int32_t sigma_diag,
                                 float scale, void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Joint diagonalization (JD-Full) by eigenvalue iteration ------------------
 * "Compress then Serve" (academ.us/article/2407.00066), section 3.1 eq. 1 and
 * Appendix 8.1 (case 1, eqs. 6-7) / 8.2.  A problem is one module position shared
 * by `count` LoRAs (modules mods[members[first + j]], all of the problem's d_out x
 * d_in, ranks r_i <= 64): find U (d_out x rank) and V (d_in x rank) with
 * orthonormal columns and one full rank x rank Sigma_i per LoRA such that
 * B_i A_i ~ U Sigma_i V^T.  Each of `iters` steps updates both bases from the
 * previous iterate, with P_i = A_i V and Q_i = B_i^T U:
 *     U <- orthogonalize(sum_i w_i B_i (P_i (P_i^T Q_i))),
 *     V <- orthogonalize(sum_i w_i A_i^T (Q_i (Q_i^T P_i))),
 * orthogonalize = the Q of the thin QR with positive diag(R): the factor-
 * construction TSQR's Gram leaf and fp64 Cholesky give R, then Q = X R^-1; a matrix
 * whose pivot is rejected takes the Householder TSQR and a second pass on Q.
 * Afterwards, if `sigma` is not null, Sigma_i = U^T B_i A_i V (eq. 6) at the final U, V.
 * Contractions run on the fp64 tensor-core path (fp32 inputs, exact products,
 * fp64 sums); U, V and Sigma are stored fp32.
 * State: U of problem p at U_base + U_off (d_out x rank fp32, row-major), V^T at
 * Vt_base + Vt_off (rank x d_in fp32, row-major): the layout of a rank-`rank`
 * LoRA module (B = U, A = V^T) and of lf_lora_sigma_sandwich's V^T.  On entry
 * they hold the starting bases (used as given; they need not be orthonormal),
 * on return the bases after `iters` steps (unchanged when iters = 0).
 * Sigma_i of the problem's j-th LoRA: rank x rank fp32 row-major at
 * sigma + sigma_off + j * rank * rank (the layout of lf_lora_sigma_sandwich's
 * full Sigma).  weights (nullable = all 1): fp64, one per entry of `members`;
 * the pages' unit-Frobenius normalisation is w_i = 1 / ||B_i A_i||_F^2 (the sum
 * of sigma^2 from lf_tsqr_batched).
 * Errors: LF_ERR_INVALID_ARG (null pointers, iters < 0, member index out of
 * range, count < 1), LF_ERR_SHAPE (rank outside 1..min(64, d_out, d_in), a
 * member whose d_out / d_in differ from the problem's, r_i outside 1..64),
 * LF_ERR_ALIGNMENT (a base pointer not 16-byte aligned), LF_ERR_WORKSPACE.
 * Device-side: LF_ERR_NUMERIC when an update is numerically rank deficient
 * (orthogonalize meets R_jj <= 0; the columns from there on are zeroed). */
typedef struct {
    int32_t d_out, d_in, rank;
    int32_t first, count;      /* members[first .. first + count): module indices */
    int64_t U_off, Vt_off;     /* element offsets of U and V^T */
    int64_t sigma_off;         /* element offset of the problem's Sigma block */
} lf_jd_problem;
size_t lf_jd_workspace_size(const lf_module* mods /*[host]*/, int32_t n_mods,
                            const int32_t* members /*[host]*/, int32_t n_members,
                            const lf_jd_problem* probs /*[host]*/, int32_t n_probs);
lf_status lf_jd_full(const lf_module* mods /*[host]*/, int32_t n_mods,
                     const int32_t* members /*[host]*/, int32_t n_members,
                     const lf_jd_problem* probs /*[host]*/, int32_t n_probs,
                     const float* B_base, const float* A_base, const double* weights,
                     int32_t iters, float* U_base, float* Vt_base, float* sigma,
                     void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Pool-wide shared subspace (LoRASpace) ------------------------------------
 * LoRASpace (the arXiv listing's abstract, "LoRASpace: A Pool-Wide Shared Substrate
 * for Static and Dynamic Multi-LoRA Composition"): the stacked factors of a LoRA pool
 * need far fewer directions than their summed ranks; the SVD of the stack gives the
 * minimal subspace that keeps 99 % of the factor energy.
 * side 0: the row factors A_i (r_i x d, row-major, element offset offs[i] of base) are
 *   stacked as rows, S = [A_1; A_2; ...] (R x d);
 * side 1: the column factors B_i (d x r_i, row-major, element offset offs[i]) are put
 *   side by side, S = [B_1 B_2 ...] (d x R).
 * R = sum r_i, at most LF_POOL_MAX_RANK and at most d.  "Stack vector" a is row a of S
 * (side 0) or column a (side 1), in the order of the factors.
 * Outputs (device): k (1 int): the smallest k >= 1 whose leading directions hold
 *   num/den of the energy sum_j sigma_j^2 (sums in order); sigma (R doubles): the
 *   singular values of S, descending; basis (R x d fp32, row-major): row j = direction j
 *   (orthonormal; the right singular vectors of the stacked rows, or the left ones of
 *   the side-by-side columns); a direction with sigma_j <= 1e-6 sigma_1, which the
 *   fp64 Gram does not resolve, has a zero row; coef (R x R fp32):
 *   coef[a][j] = (stack vector a) . (direction j), so factor i is approximated by its
 *   rows' first k coefficients times the first k directions; resid (1 double): the
 *   energy outside the subspace, sum_a sum_{j >= k} coef[a][j]^2.
 * Computed as the eigen-decomposition of the fp64 Gram S S^T (S^T S for side 1) by a
 * one-sided Jacobi iteration across the GPU (cooperative launch).  All memory is the
 * caller's; workspace: lf_pool_workspace_size (0 for invalid arguments).
 * Errors: LF_ERR_INVALID_ARG (side, counts, ranks < 1, negative offsets, num/den not a
 * fraction, null pointers), LF_ERR_SHAPE (R > LF_POOL_MAX_RANK or R > d),
 * LF_ERR_WORKSPACE.  Device-side: LF_ERR_NUMERIC for a non-finite input (read as 0),
 * LF_ERR_TIMEOUT when a grid barrier does not complete. */
#define LF_POOL_MAX_RANK 512
size_t lf_pool_workspace_size(int32_t side, int32_t n_lora, const int32_t* ranks /*[host]*/,
                              const int64_t* offs /*[host]*/, int32_t d);
lf_status lf_pool_subspace(int32_t side, int32_t n_lora, const int32_t* ranks /*[host]*/,
                           const int64_t* offs /*[host]*/, int32_t d, const float* base,
                           int32_t num, int32_t den, int32_t* k, double* sigma, float* basis,
                           float* coef, double* resid, void* ws, size_t ws_bytes, lf_stream_t stream);

/* ---- Shrink / expand with library-owned scratch -------------------------------
 * This entry point has no counterpart in the paper; it exists for callers that
 * cannot call cudaMalloc.  Examples: a serving loop that reserved all device memory
 * when it started and may not allocate afterwards, or a latency-critical path where
 * cudaMalloc's implicit synchronisation and unbounded cost are not acceptable.
 * Such a caller still passes x, y, ids, the rank table and the pools, but no
 * workspace: the routing scratch lives in a fixed array inside the library
 * (a file-scope __device__ array sized for LF_NOALLOC_MAX_TOKENS tokens and
 * LF_NOALLOC_MAX_ADAPTERS adapters, 4 407 808 bytes, held on every GPU that loads the
 * library until the process exits).
 *  - Same arguments and device-side errors as lf_lora_shrink_expand, minus the
 *    workspace; the results agree with it within the apply tolerance (it always
 *    runs the GEMV kernels, so the bf16 rounding of y may differ).
 *    T > LF_NOALLOC_MAX_TOKENS or n_adapters > LF_NOALLOC_MAX_ADAPTERS returns
 *    LF_ERR_WORKSPACE without launching anything.
 *  - Runs on the device that is current when it is called; `stream` must belong
 *    to that device.  The first call on each device looks up the array's device
 *    address (cudaGetSymbolAddress) and keeps it until the process exits; make that
 *    first call before any stream capture.  Resetting a device (cudaDeviceReset)
 *    while the library is loaded is not supported: the array may come back at
 *    another address.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *  - All calls on one device share the one array and every call overwrites what it
 *    reads before reading it (nothing in it has to start at zero).  Two calls whose
 *    work overlaps on the GPU (for instance on two streams) race on the array and
 *    give wrong results: serialise them, e.g. on one stream. */
#define LF_NOALLOC_MAX_TOKENS 16384
#define LF_NOALLOC_MAX_ADAPTERS 4096
lf_status lf_lora_shrink_expand_noalloc(int32_t T, int32_t d_in, int32_t d_out,
                                        const void* x, void* y, const int32_t* ids,
                                        int32_t n_adapters, const int32_t* ranks,
                                        const int64_t* off_A, const int64_t* off_Bt,
                                        const void* A_pool, const void* Bt_pool,
                                        int64_t pool_elems_A, int64_t pool_elems_Bt,
                                        float scale, int32_t* seg_out, lf_stream_t stream);

/* ---- Tracing (no counterpart on the pages: measurement support) --------------
 * Every kernel launch of the library is counted.  With timing enabled, each
 * launch is also bracketed by CUDA events recorded on its own stream and its
 * device time is added to a named phase ("tsqr_gram_leaf", "svd_jacobi",
 * "select", "export_stream", "shrink_expand_gemv", ...).  lf_profile_read waits
 * for the pending events, then copies up to max_phases entries into `out`
 * [host] and returns the number of phases.  Process-wide state, not thread-safe. */
typedef struct {
    char name[32];
    double total_ms;
    int64_t launches;
} lf_phase_time;
void lf_profile_enable(int on);
void lf_profile_reset(void);
int32_t lf_profile_read(lf_phase_time* out /*[host]*/, int32_t max_phases);
int64_t lf_launch_count(void);

/* ---- Failure detection check (no counterpart on the pages) --------------------
 * Launches one thread that waits, through the same bounded mbarrier wait every
 * pipeline of the library uses, on a barrier nothing arrives at, giving up after
 * `polls` polls (0 .. 2^20).  The wait runs out, LF_ERR_TIMEOUT is latched and the
 * kernel returns, so the context stays usable: lf_get_device_status then reports
 * LF_ERR_TIMEOUT.  Nothing else is in flight in that kernel (no copy, no MMA).
 * Returns LF_ERR_INVALID_ARG for polls outside the range. */
lf_status lf_check_bounded_wait(int32_t polls, lf_stream_t stream);

/* ---- Status ------------------------------------------------------------------ */
const char* lf_status_string(lf_status s);
/* Synchronises `stream`, returns the first device-side error latched since the
 * last call (LF_OK if none) and clears it; LF_ERR_CUDA if the stream reports a
 * CUDA error. */
lf_status lf_get_device_status(lf_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* LORAFORGE_H */
