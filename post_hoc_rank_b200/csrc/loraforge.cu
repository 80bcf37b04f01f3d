// libloraforge: host planner + C ABI (see include/loraforge.h for the contract).
// One translation unit: the kernel headers are included here so the device error
// word needs no relocatable device code.
#include <algorithm>
#include <climits>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"
#include "tsqr.cuh"
#include "gram.cuh"
#include "gram_i8.cuh"
#include "select_export.cuh"
#include "apply.cuh"
#include "jd.cuh"
#include "pool.cuh"

namespace lf {

// ------------------------------------------------------------- tracing/timing
// Every kernel launch goes through LF_LAUNCH, which counts it and, when timing is
// on, brackets it with CUDA events recorded on the launching stream.
struct ProfState {
    bool on = false;
    int64_t launches = 0;
    struct Rec {
        int phase;
        cudaEvent_t a, b;
    };
    std::vector<Rec> pending;
    std::vector<cudaEvent_t> free_events;
    std::vector<std::string> names;
    std::vector<double> ms;
    std::vector<int64_t> count;
};
static ProfState g_prof;

static int phase_id(const char* name) {
    for (size_t i = 0; i < g_prof.names.size(); ++i)
        if (g_prof.names[i] == name) return (int)i;
    g_prof.names.push_back(name);
    g_prof.ms.push_back(0.0);
    g_prof.count.push_back(0);
    return (int)g_prof.names.size() - 1;
}

static cudaEvent_t take_event() {
    if (!g_prof.free_events.empty()) {
        cudaEvent_t e = g_prof.free_events.back();
        g_prof.free_events.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
}

struct PhaseScope {
    int phase = -1;
    cudaEvent_t a = nullptr;
    cudaStream_t s;
    PhaseScope(const char* name, cudaStream_t st) : s(st) {
        ++g_prof.launches;
        if (!g_prof.on) return;
        phase = phase_id(name);
        a = take_event();
        cudaEventRecord(a, s);
    }
    ~PhaseScope() {
        if (phase < 0) return;
        cudaEvent_t b = take_event();
        cudaEventRecord(b, s);
        g_prof.pending.push_back(ProfState::Rec{phase, a, b});
    }
};

#define LF_LAUNCH(name, kernel, grid, block, smem, stream, ...)            \
    do {                                                                   \
        PhaseScope ps_(name, stream);                                      \
        kernel<<<grid, block, smem, stream>>>(__VA_ARGS__);                \
    } while (0)

// ----------------------------------------------------------------- validation
static lf_status check_mods(const lf_module* mods, int32_t n) {
    if (n < 0) return LF_ERR_INVALID_ARG;
    if (n > 0 && !mods) return LF_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        const lf_module& m = mods[i];
        if (m.d_out < 1 || m.d_in < 1 || m.r < 1 || m.r > kMaxRank || m.r > m.d_out || m.r > m.d_in)
            return LF_ERR_SHAPE;
        if (m.group < 0 || m.B_off < 0 || m.A_off < 0) return LF_ERR_INVALID_ARG;
        if ((m.B_off & 3) || (m.A_off & 3)) return LF_ERR_ALIGNMENT;
    }
    return LF_OK;
}

static lf_status check_policy(const lf_module* mods, int32_t n, lf_policy p) {
    if (p.kind < 0 || p.kind > 3) return LF_ERR_INVALID_ARG;
    if (p.ratio_num < 0 || p.ratio_den <= 0 || p.floor < 1) return LF_ERR_INVALID_ARG;
    if (p.kind == 3 && p.ratio_num > p.ratio_den) return LF_ERR_INVALID_ARG;   // a fraction of the energy
    for (int32_t i = 0; i < n; ++i)
        if (p.floor > mods[i].r) return LF_ERR_SHAPE;
    return LF_OK;
}

static int rank_stride(const lf_module* mods, int32_t n) {
    int rs = 0;
    for (int32_t i = 0; i < n; ++i) rs = std::max(rs, (int)mods[i].r);
    return rs;
}

static int rt_bucket(int rs) { return rs <= 16 ? 16 : (rs <= 32 ? 32 : 64); }

// Host staging: pieces laid out exactly as the Carver lays them out on the device,
// so one cudaMemcpyAsync uploads all of them.
struct Staging {
    std::vector<char> buf;
    size_t off = 0;
    template <typename T>
    size_t put(const T* src, size_t count) {
        off = (size_t)align_up((int64_t)off, 256);
        const size_t at = off;
        off += count * sizeof(T);
        if (buf.size() < off) buf.resize(off);
        if (count) std::memcpy(buf.data() + at, src, count * sizeof(T));
        return at;
    }
};

// ------------------------------------------------------------------ TSQR plan
struct TsqrPlan {
    std::vector<TsqrWork> work;
    std::vector<TsqrInfo> info;
    int32_t slots = 0;
    int rs = 0, RT = 16;
};

static void plan_tsqr(const lf_module* mods, int32_t n, TsqrPlan& p) {
    p.rs = rank_stride(mods, n);
    p.RT = rt_bucket(p.rs);
    p.info.resize((size_t)2 * n);
    p.work.clear();
    for (int32_t i = 0; i < n; ++i)
        for (int f = 0; f < 2; ++f) {
            const int rows = f == 0 ? mods[i].d_out : mods[i].d_in;
            const int nch = (int)cdiv(rows, kTsqrChunk);
            const int mf = 2 * i + f;
            p.info[mf] = TsqrInfo{nch, nch > 1 ? p.slots : -1};
            for (int c = 0; c < nch; ++c)
                p.work.push_back(TsqrWork{mf, c * kTsqrChunk, std::min(kTsqrChunk, rows - c * kTsqrChunk),
                                          nch > 1 ? p.slots + c : -1});
            if (nch > 1) p.slots += nch;
        }
    // longest chunks first: single-warp CTAs of similar length finish together
    std::stable_sort(p.work.begin(), p.work.end(),
                     [](const TsqrWork& a, const TsqrWork& b) { return a.nrows > b.nrows; });
}

// Work list of the integer-Gram leaf: every matrix whose rows the copies can address
// (16-byte aligned rows and offsets) in items of at most kI8MaxRows rows, longest first;
// each item has its own Gram slot, a matrix's slots consecutive in row order.  fb (per
// matrix) starts at 1 for the others, which the fp64 leaf takes.
struct I8Plan {
    std::vector<TsqrWork> work;
    std::vector<TsqrInfo> info;
    std::vector<int32_t> fb;
    int32_t slots = 0;
};

static bool i8_eligible(const lf_module& m, int factor) {
    return factor == 0 ? ((m.r & 3) == 0 && (m.B_off & 3) == 0) : ((m.d_in & 3) == 0 && (m.A_off & 3) == 0);
}

static void plan_i8(const lf_module* mods, int32_t n, I8Plan& p) {
    p.work.clear();
    p.info.assign((size_t)2 * n, TsqrInfo{0, -1});
    p.fb.assign((size_t)2 * n, 1);
    p.slots = 0;
    for (int32_t i = 0; i < n; ++i)
        for (int f = 0; f < 2; ++f) {
            if (!i8_eligible(mods[i], f)) continue;
            const int rows = f == 0 ? mods[i].d_out : mods[i].d_in;
            const int nch = (int)cdiv(rows, kI8MaxRows);
            const int mf = 2 * i + f;
            p.info[mf] = TsqrInfo{nch, p.slots};
            p.fb[mf] = 0;
            for (int c = 0; c < nch; ++c)
                p.work.push_back(TsqrWork{mf, c * kI8MaxRows, std::min(kI8MaxRows, rows - c * kI8MaxRows), p.slots + c});
            p.slots += nch;
        }
    std::stable_sort(p.work.begin(), p.work.end(),
                     [](const TsqrWork& a, const TsqrWork& b) { return a.nrows > b.nrows; });
}

static size_t i8_slot_bytes(int RT) {
    return sizeof(double) * (size_t)(RT == 16 ? tri_size<16>() : (RT == 32 ? tri_size<32>() : tri_size<64>()));
}

struct TsqrLayout {
    size_t mods, work, nwork, info, n_dev, counters, partial, i8work, i8info, fb, amaps, i8gram, total;
};

// Partial-slot bytes: the fp64 packed Gram of the leaf pass or the fp32 partial R of
// the Householder pass, whichever is larger (the two passes run one after the other).
static size_t tsqr_slot_bytes(int RT) {
    return RT == 16 ? gram_slot_bytes<16>() : (RT == 32 ? gram_slot_bytes<32>() : gram_slot_bytes<64>());
}

static TsqrLayout tsqr_layout(int32_t n, const TsqrPlan& p, const I8Plan& q) {
    Carver c(nullptr);
    TsqrLayout L;
#define LF_TAKE(field, T, cnt)                          \
    do {                                                \
        c.take<T>(cnt);                                 \
        L.field = c.off - (size_t)(cnt) * sizeof(T);    \
    } while (0)
    LF_TAKE(mods, lf_module, n);
    LF_TAKE(work, TsqrWork, p.work.size());
    LF_TAKE(nwork, int32_t, 1);
    LF_TAKE(info, TsqrInfo, p.info.size());
    LF_TAKE(n_dev, int32_t, 1);
    LF_TAKE(counters, int32_t, (size_t)6 * n);   // Gram counters, Householder counters, flags (2n each)
    LF_TAKE(partial, char, (size_t)p.slots * tsqr_slot_bytes(p.RT));
    LF_TAKE(i8work, TsqrWork, q.work.size());
    LF_TAKE(i8info, TsqrInfo, q.info.size());
    LF_TAKE(fb, int32_t, q.fb.size());
    LF_TAKE(amaps, CUtensorMap, (size_t)n);
    LF_TAKE(i8gram, char, (size_t)q.slots * i8_slot_bytes(p.RT));
#undef LF_TAKE
    L.total = c.off + 256;
    return L;
}

template <typename T, int RT>
static cudaError_t launch_tsqr(const TsqrArgs<T>& a, int n_items, cudaStream_t st) {
    auto k = tsqr_kernel<T, RT>;
    constexpr int W = tsqr_warps<T>();
    // the kernel strides over the device-side item count: a bounded grid (16 CTAs per
    // SM for fp32, 8 for fp64) covers any number of items
    const int grid = std::min((n_items + W - 1) / W, 148 * (sizeof(T) == 4 ? 16 : 8));
    if (grid > 0) LF_LAUNCH(sizeof(T) == 8 ? "tsqr_fp64_refine" : "tsqr_householder", k, grid, 32 * W, 0, st, a);
    return cudaGetLastError();
}

template <int RT>
static cudaError_t launch_gram_i8(const GramI8Args& a, const GramI8RootArgs& ra, cudaStream_t st) {
    if (a.n_work > 0) {
        int dev = 0, sms = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(gram_i8_kernel<RT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gram_i8_smem());
        if (e != cudaSuccess) return e;
        // one persistent CTA per SM (all of its tensor memory), static round-robin over the items
        const int grid = std::min(a.n_work, std::max(sms, 1));
        LF_LAUNCH("tsqr_gram_i8", gram_i8_kernel<RT>, grid, kI8Threads, gram_i8_smem(), st, a);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    constexpr size_t rsm = gram_i8_root_smem<RT>();
    cudaError_t e = cudaFuncSetAttribute(gram_i8_root_kernel<RT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsm);
    if (e != cudaSuccess) return e;
    if (ra.n_mf > 0)
        LF_LAUNCH("tsqr_gram_i8_root", gram_i8_root_kernel<RT>, (unsigned)cdiv(ra.n_mf, kI8RootWarps),
                  32 * kI8RootWarps, rsm, st, ra);
    return cudaGetLastError();
}

static cudaError_t launch_gram_i8_rt(int RT, const GramI8Args& a, const GramI8RootArgs& ra, cudaStream_t st) {
    if (RT == 16) return launch_gram_i8<16>(a, ra, st);
    if (RT == 32) return launch_gram_i8<32>(a, ra, st);
    return launch_gram_i8<64>(a, ra, st);
}

template <int RT>
static cudaError_t launch_gram(const GramArgs& a, int n_items, cudaStream_t st) {
    if (n_items > 0) LF_LAUNCH("tsqr_gram_leaf", gram_kernel<RT>, n_items, 32, 0, st, a);
    return cudaGetLastError();
}

static cudaError_t launch_gram_rt(int RT, const GramArgs& a, int n_items, cudaStream_t st) {
    if (RT == 16) return launch_gram<16>(a, n_items, st);
    if (RT == 32) return launch_gram<32>(a, n_items, st);
    return launch_gram<64>(a, n_items, st);
}

template <typename T>
static cudaError_t launch_tsqr_rt(int RT, const TsqrArgs<T>& a, int grid, cudaStream_t st) {
    if (RT == 16) return launch_tsqr<T, 16>(a, grid, st);
    if (RT == 32) return launch_tsqr<T, 32>(a, grid, st);
    return launch_tsqr<T, 64>(a, grid, st);
}

template <typename TIN, typename T, int RT>
static cudaError_t launch_svd(const SvdArgs<TIN, T>& a, int n_items, cudaStream_t st) {
    constexpr int W = svd_warps<T>();
    constexpr size_t smem = W * sizeof(SvdSmem<T, RT>);
    auto k = svd_kernel<TIN, T, RT>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const int grid = (n_items + W - 1) / W;
    if (grid > 0) LF_LAUNCH(sizeof(T) == 8 ? "svd_fp64_refine" : "svd_jacobi", k, grid, 32 * W, smem, st, a);
    return cudaGetLastError();
}

template <typename TIN, typename T>
static cudaError_t launch_svd_rt(int RT, const SvdArgs<TIN, T>& a, int n_items, cudaStream_t st) {
    if (RT == 16) return launch_svd<TIN, T, 16>(a, n_items, st);
    if (RT == 32) return launch_svd<TIN, T, 32>(a, n_items, st);
    return launch_svd<TIN, T, 64>(a, n_items, st);
}

// Routing block size: enough threads for one pass over the batch and the adapters
// (fewer warps make its block-wide barriers cheaper), at least 128, at most 1024.
static int route_threads(int T, int n_adapters) {
    const int need = std::max(T, n_adapters);
    return need >= kRouteThreads ? kRouteThreads : std::max(128, (need + 31) / 32 * 32);
}

// ------------------------------------------------------------ groups (S scope)
static void build_groups(const lf_module* mods, int32_t n, std::vector<int32_t>& ptr, std::vector<int32_t>& gm) {
    std::map<int32_t, std::vector<int32_t>> by;
    for (int32_t i = 0; i < n; ++i) by[mods[i].group].push_back(i);
    ptr.assign(1, 0);
    gm.clear();
    for (auto& kv : by) {
        for (int32_t i : kv.second) gm.push_back(i);
        ptr.push_back((int32_t)gm.size());
    }
}

// ----------------------------------------------------------- export planning
constexpr int kRefineChunk = 512;
constexpr int kExportItem = 2048;

struct ExportPlan {
    std::vector<int32_t> gptr, gmods;
    int32_t max_cand = 0;   // largest candidate count (sum of r - floor) over the groups
    std::vector<ExportWork> ework;
    int rs = 0, RT = 16;
    int32_t refine_cap = 0;
    int32_t refine_max_work = 0;
    int32_t refine_slots = 0;
};

static void plan_export(const lf_module* mods, int32_t n, ExportPlan& p) {
    p.rs = rank_stride(mods, n);
    p.RT = rt_bucket(p.rs);
    build_groups(mods, n, p.gptr, p.gmods);
    const int32_t ngroups = (int32_t)p.gptr.size() - 1;
    p.max_cand = 0;
    for (int32_t g = 0; g < ngroups; ++g) {
        int64_t c = 0;
        for (int32_t q = p.gptr[g]; q < p.gptr[g + 1]; ++q) c += mods[p.gmods[q]].r;
        p.max_cand = (int32_t)std::max<int64_t>(p.max_cand, std::min<int64_t>(c, kSelMaxCand));
    }
    p.ework.clear();
    int maxd = 1;
    for (int32_t i = 0; i < n; ++i) {
        for (int s = 0; s < mods[i].d_out; s += kExportItem)
            p.ework.push_back(ExportWork{i, 0, s, std::min(kExportItem, mods[i].d_out - s)});
        for (int s = 0; s < mods[i].d_in; s += kExportItem)
            p.ework.push_back(ExportWork{i, 1, s, std::min(kExportItem, mods[i].d_in - s)});
        maxd = std::max(maxd, std::max(mods[i].d_out, mods[i].d_in));
    }
    p.refine_cap = std::min<int32_t>(n, 8 * ngroups + 64);
    const int per = (int)cdiv(maxd, kRefineChunk);
    p.refine_max_work = p.refine_cap * 2 * per;
    p.refine_slots = p.refine_cap * 2 * (per > 1 ? tree_slots(per) : 0);
}

struct ExportLayout {
    size_t mods, gptr, gmods, ework, energy, sigref, flist, fcount, rwork, rnwork, rinfo, rcnt, rpart, rRB, rRA,
        rsig, CA, CB, total;
};

static ExportLayout export_layout(int32_t n, const ExportPlan& p) {
    Carver c(nullptr);
    ExportLayout L;
#define LF_TAKE(field, T, cnt)                          \
    do {                                                \
        c.take<T>(cnt);                                 \
        L.field = c.off - (size_t)(cnt) * sizeof(T);    \
    } while (0)
    const size_t rs2 = (size_t)p.rs * p.rs;
    LF_TAKE(mods, lf_module, n);
    LF_TAKE(gptr, int32_t, p.gptr.size());
    LF_TAKE(gmods, int32_t, p.gmods.size());
    LF_TAKE(ework, ExportWork, p.ework.size());
    LF_TAKE(energy, double, (size_t)n * p.rs);
    LF_TAKE(sigref, double, (size_t)n * p.rs);
    LF_TAKE(flist, int32_t, (size_t)n);
    LF_TAKE(fcount, int32_t, 2);
    LF_TAKE(rwork, TsqrWork, (size_t)p.refine_max_work);
    LF_TAKE(rnwork, int32_t, 1);
    LF_TAKE(rinfo, TsqrInfo, (size_t)2 * p.refine_cap);
    LF_TAKE(rcnt, int32_t, (size_t)p.refine_slots);
    LF_TAKE(rpart, double, (size_t)p.refine_slots * (p.RT * (p.RT + 1) / 2));
    LF_TAKE(rRB, double, (size_t)p.refine_cap * rs2);
    LF_TAKE(rRA, double, (size_t)p.refine_cap * rs2);
    LF_TAKE(rsig, double, (size_t)p.refine_cap * p.rs);
    LF_TAKE(CA, float, (size_t)n * rs2);
    LF_TAKE(CB, float, (size_t)n * rs2);
#undef LF_TAKE
    L.total = c.off + 256;
    return L;
}

// Caps the refinement list at `cap` and stores the capped count at count[1].
__global__ void cap_flags_kernel(int32_t* count, int cap) {
    if (threadIdx.x == 0 && blockIdx.x == 0) {
        int c = count[0];
        if (c > cap) {
            latch_error(LF_ERR_WORKSPACE);
            c = cap;
        }
        count[0] = c;
        count[1] = c;
    }
}

// ------------------------------------------------------------ apply workspace
struct ApplyWs {
    int32_t* tag;
    int32_t* counts;
    Seg* segs;
    int32_t* perm;
    GemvItem* items;
    float* t_buf;
    TcItem* tc_items;
    float* t_part;
    int32_t* runs;
    int32_t* tok_list;
};

// Carves (or, with base == nullptr, sizes) the side-path workspace for T tokens,
// n adapters and ns slices.
static size_t carve_apply(void* base, int64_t T, int64_t n, int ns, ApplyWs* w) {
    Carver c(base);
    const int64_t mseg = std::min<int64_t>(T, n);
    const int64_t T1 = std::max<int64_t>(T, 1);
    // routing tables first: their offsets depend on (T, n) only, so a routing pass on
    // this workspace serves calls with any number of slices
    w->tag = c.take<int32_t>(4);
    w->counts = c.take<int32_t>(8);
    w->segs = c.take<Seg>((size_t)std::max<int64_t>(mseg, 1));
    w->perm = c.take<int32_t>((size_t)T1);
    w->items = c.take<GemvItem>((size_t)(T / kGemvTok + mseg + 1));
    w->tc_items = c.take<TcItem>((size_t)(T / kTcM + mseg + 1));
    w->runs = c.take<int32_t>((size_t)2 * T1);   // run scratch of the routing pass
    w->tok_list = c.take<int32_t>((size_t)T1);   // tokens outside the tensor-core segments
    w->t_buf = c.take<float>((size_t)T1 * kMaxRank * ns);
    w->t_part = c.take<float>((size_t)kTcMaxSplit * T1 * kMaxRank * ns);
    return c.off + 256;
}

// Tensor maps for the tensor-core kernels' TMA stages: box of 64 elements (128 bytes)
// x 128 rows, 128-byte swizzle, out-of-range reads as zeros (and are not written by
// stores).  cuTensorMapEncodeTiled is looked up once through the runtime's driver
// entry point.  encode_rows_map returns false (the kernels then gather rows with
// cp.async) when the lookup or the encoding fails or the shape is below one box.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
static EncodeTiledFn encode_tiled_fn() {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Tensor map of a row-major bf16 matrix of `rows` rows of `cols` elements (row stride
// `cols`), box 64 x 128, for the tensor-core kernels' TMA stages (x for the shrink,
// y for the expand).
static bool encode_rows_map(CUtensorMap* map, const void* base, int32_t rows, int64_t cols) {
    if (rows < kTcM || cols < kTcKB || (cols & 7) || !aligned16(base)) return false;
    const EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kTcKB, (cuuint32_t)kTcM};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of a module's A (r x d_in fp32, row-major) read as A^T stages: dims
// {d_in, r}, box {32, r} (32 rows of A^T: one 128-byte run per column), 128-byte
// swizzle, rows past d_in read as zeros.  False when the encoder is unavailable or
// rejects the shape (the fp64 leaf then takes the matrix).
static bool encode_a_map(CUtensorMap* map, const float* A, int32_t r, int32_t d_in) {
    if (!aligned16(A) || (d_in & 3) || r < 1 || r > 64) return false;
    const EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)r};
    const cuuint64_t strides[1] = {(cuuint64_t)d_in * 4};
    const cuuint32_t box[2] = {32u, (cuuint32_t)r};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(A), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bounded grid of the grid-stride GEMV kernels: enough CTAs to fill the GPU (8 per
// SM of 148), never more than the largest possible number of work units.
static unsigned gemv_grid(int64_t max_units) {
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>(max_units, 8 * 148));
}

// Grid column chunks of width W over the slices (expand launches).
static void set_chunks(ApplyArgs& a, int W) {
    int c = 0;
    for (int q = 0; q < a.n_slices; ++q) {
        a.sl[q].chunk0 = c;
        c += (int)cdiv(a.sl[q].d_out, W);
    }
    a.n_chunks = c;
}

// Shared-factor slice for Sigma-sandwich serving (every adapter uses rank k_shared and
// the pools at offset 0).
struct SharedSlice {
    int32_t k = 0;
    const float* sigma = nullptr;
    int32_t mode = 0;
};

// Decode regime (token-parallel kernel, no routing pass): few tokens per resident adapter,
// T <= kGemvTok * n_adapters.  Other batches are routed: tensor-core tiles for segments of
// kTcMin or more tokens, the token-parallel kernel over the routing's list for the rest.
// Measured on the mixed batch of the large fleet (4096 tokens: 64 requests of 48 tokens and
// 1024 decode tokens over 1024 resident adapters), routing it anyway was 1.9x slower: its
// adapters of 64+ tokens gather scattered rows into tensor-core tiles.
static bool decode_regime(int64_t T, int64_t n_adapters) { return T <= (int64_t)kGemvTok * n_adapters; }

// Host checks of one apply's x, y and slices (shared: factors shared by all adapters,
// no per-adapter tables).
static lf_status check_apply(int32_t d_in, const void* x, const void* y, int64_t y_ld, const lf_slice* sl, int32_t ns,
                             bool shared) {
    if (d_in < 1 || !x || !y || !sl) return LF_ERR_INVALID_ARG;
    if ((d_in & 7) || (y_ld & 7)) return LF_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(y)) return LF_ERR_ALIGNMENT;
    for (int q = 0; q < ns; ++q) {
        const lf_slice& t = sl[q];
        if (t.d_out < 1 || t.pool_elems_A < 0 || t.pool_elems_Bt < 0 || t.y_offset < 0 || t.y_offset + t.d_out > y_ld ||
            t.max_rank < 0 || t.max_rank > kMaxRank)
            return LF_ERR_INVALID_ARG;
        if (!shared && (!t.ranks || !t.off_A || !t.off_Bt)) return LF_ERR_INVALID_ARG;
        if (!t.A_pool || !t.Bt_pool) return LF_ERR_INVALID_ARG;
        if ((t.d_out & 7) || (t.y_offset & 7)) return LF_ERR_ALIGNMENT;
        if (!aligned16(t.A_pool) || !aligned16(t.Bt_pool)) return LF_ERR_ALIGNMENT;
    }
    return LF_OK;
}

static lf_status apply_impl(int32_t T, int32_t d_in, const void* x, void* y, int64_t y_ld, const int32_t* ids,
                            int32_t n_adapters, const lf_slice* sl, int32_t ns, float scale, const float* scales,
                            int32_t* seg_out, void* ws, size_t ws_bytes, cudaStream_t s,
                            const SharedSlice* shared = nullptr, bool routed = false) {
    if (T < 0 || d_in < 1 || n_adapters < 1 || n_adapters > 16384 || ns < 1 || ns > kMaxSlices || !sl)
        return LF_ERR_INVALID_ARG;
    if (T == 0) return LF_OK;
    if (!ids || !ws) return LF_ERR_INVALID_ARG;
    const lf_status cs = check_apply(d_in, x, y, y_ld, sl, ns, shared != nullptr);
    if (cs != LF_OK) return cs;
    ApplyWs w;
    if (ws_bytes < carve_apply(nullptr, T, n_adapters, ns, &w)) return LF_ERR_WORKSPACE;
    carve_apply(reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256)), T, n_adapters,
                ns, &w);
    ApplyArgs A{};
    A.T = T;
    A.d_in = d_in;
    A.n_adapters = n_adapters;
    A.n_slices = ns;
    A.y_ld = y_ld;
    A.ldt = kMaxRank * ns;
    A.x = reinterpret_cast<const __nv_bfloat16*>(x);
    A.y = reinterpret_cast<__nv_bfloat16*>(y);
    A.ids = ids;
    A.scale = scale;
    A.scales = scales;
    if (shared) {
        A.sigma_mode = shared->mode;
        A.sigma = shared->sigma;
    }
    for (int q = 0; q < ns; ++q) {
        SliceTab& t = A.sl[q];
        t.d_out = sl[q].d_out;
        t.t_col = kMaxRank * q;
        t.k_shared = shared ? shared->k : 0;
        t.max_rank = shared ? 0 : sl[q].max_rank;
        t.y_off = sl[q].y_offset;
        t.ranks = sl[q].ranks;
        t.off_A = sl[q].off_A;
        t.off_Bt = sl[q].off_Bt;
        t.A_pool = reinterpret_cast<const __nv_bfloat16*>(sl[q].A_pool);
        t.Bt_pool = reinterpret_cast<const __nv_bfloat16*>(sl[q].Bt_pool);
        t.pool_A = sl[q].pool_elems_A;
        t.pool_Bt = sl[q].pool_elems_Bt;
    }
    A.counts = w.counts;
    A.segs = w.segs;
    A.perm = w.perm;
    A.items = w.items;
    A.tc_items = w.tc_items;
    A.t_buf = w.t_buf;
    A.t_part = w.t_part;
    A.tok_list = nullptr;

    RouteOut o{};
    o.counts = w.counts;
    o.segs = w.segs;
    o.perm = w.perm;
    o.items = w.items;
    o.tc_items = w.tc_items;
    o.run_start = w.runs;
    o.run_pos = w.runs + T;
    o.seg_out = seg_out;
    o.tag = w.tag;
    o.tok_list = w.tok_list;
    const bool token_parallel = decode_regime(T, n_adapters);
    o.tc_enable = token_parallel ? 0 : 1;
    const size_t rsmem = 2 * (size_t)n_adapters * sizeof(int32_t);
    LF_CUDA_TRY(cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem));
    if (token_parallel) {
        // few tokens per adapter: token-parallel shrink + expand, no sort; the routing
        // pass runs only when the caller asks for the segment table
        if (seg_out) {
            LF_LAUNCH("route", route_kernel, 1, route_threads(T, n_adapters), rsmem, s, ids, T, n_adapters, o);
            LF_CUDA_TRY(cudaGetLastError());
        }
        set_chunks(A, kBgmvCols);
        LF_LAUNCH("bgmv", bgmv_kernel<false>, dim3((unsigned)T, (unsigned)A.n_chunks), kBgmvThreads, 0, s, A);
        return launch_status();
    }
    if (routed)   // tables from an earlier routing pass on this workspace
        LF_LAUNCH("route_check", route_check_kernel, 1, 32, 0, s, w.tag, w.counts, T, n_adapters, 1);
    else
        LF_LAUNCH("route", route_kernel, 1, route_threads(T, n_adapters), rsmem, s, ids, T, n_adapters, o);
    LF_CUDA_TRY(cudaGetLastError());
    // segments under kTcMin tokens: the token-parallel kernel over the routing's token
    // list (adapter by adapter); the grid strides over the device-side count
    A.tok_list = w.tok_list;
    set_chunks(A, kBgmvCols);
    LF_LAUNCH("bgmv", bgmv_kernel<true>, dim3(gemv_grid(T), (unsigned)A.n_chunks), kBgmvThreads, 0, s, A);
    LF_CUDA_TRY(cudaGetLastError());
    // segments with >= kTcMin tokens: one tcgen05 shrink over all slices, then expand
    // tensor-core items: a segment of c >= kTcMin tokens gives ceil(c / kTcM) of them, so
    // there are at most T / kTcM + (segments of kTcMin or more tokens) + 1
    const int64_t mseg = std::min<int64_t>(T, n_adapters);
    const unsigned max_tc = (unsigned)(T / kTcM + std::min<int64_t>(mseg, T / kTcMin) + 1);
    const unsigned nsplit = (unsigned)cdiv(d_in, tc_split_len(d_in));
    set_chunks(A, kTcCols);
    alignas(64) CUtensorMap xmap, ymap;
    std::memset(&xmap, 0, sizeof(xmap));
    std::memset(&ymap, 0, sizeof(ymap));
    const int x_tma = encode_rows_map(&xmap, x, T, d_in) ? 1 : 0;
    const int y_tma = encode_rows_map(&ymap, y, T, y_ld) ? 1 : 0;
    if (ns == 1) {
        constexpr size_t sm = shrink_tc_smem<kMaxRank>();
        LF_CUDA_TRY(cudaFuncSetAttribute(shrink_tc_kernel<kMaxRank>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
        LF_LAUNCH("shrink_tc", shrink_tc_kernel<kMaxRank>, dim3(max_tc, nsplit), kTcThreads, sm, s, A, xmap, x_tma);
    } else {
        constexpr size_t sm = shrink_tc_smem<kMaxSlices * kMaxRank>();
        LF_CUDA_TRY(cudaFuncSetAttribute(shrink_tc_kernel<kMaxSlices * kMaxRank>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
        LF_LAUNCH("shrink_tc", shrink_tc_kernel<kMaxSlices * kMaxRank>, dim3(max_tc, nsplit), kTcThreads, sm, s, A,
                  xmap, x_tma);
    }
    LF_CUDA_TRY(cudaGetLastError());
    // two expand variants over the same grid, each taking its own (item, slice) pairs:
    // ranks up to 16 (three CTAs per SM) and the others (two), both in 64-column steps;
    // when every slice bounds its ranks by 16 the second has nothing to take and is left out
    bool small_only = !shared;
    for (int q = 0; q < ns; ++q) small_only = small_only && sl[q].max_rank >= 1 && sl[q].max_rank <= 16;
    {
        constexpr size_t sm16 = expand_tc_smem<16, 64>(), sm64 = expand_tc_smem<kMaxRank, 64>();
        LF_CUDA_TRY(cudaFuncSetAttribute(expand_tc_kernel<16, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm16));
        LF_CUDA_TRY(cudaFuncSetAttribute(expand_tc_kernel<kMaxRank, 64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm64));
        LF_LAUNCH("expand_tc", (expand_tc_kernel<16, 64>), dim3(max_tc, (unsigned)A.n_chunks), kTcExpThreads, sm16, s,
                  A, ymap, y_tma);
        LF_CUDA_TRY(cudaGetLastError());
        if (!small_only)
            LF_LAUNCH("expand_tc", (expand_tc_kernel<kMaxRank, 64>), dim3(max_tc, (unsigned)A.n_chunks), kTcExpThreads,
                      sm64, s, A, ymap, y_tma);
    }
    return launch_status();
}

// ------------------------------------------------- library-owned apply scratch
// Routing scratch for lf_lora_shrink_expand_noalloc, laid out exactly as the
// Carver lays out a caller workspace for (LF_NOALLOC_MAX_TOKENS, LF_NOALLOC_MAX_ADAPTERS).
constexpr size_t al256(size_t x) { return (x + 255) / 256 * 256; }
constexpr size_t kNoallocScratchBytes =
    al256(4 * sizeof(int32_t)) + al256((size_t)LF_NOALLOC_MAX_ADAPTERS * sizeof(Seg)) +
    al256((size_t)LF_NOALLOC_MAX_TOKENS * sizeof(int32_t)) +
    al256(((size_t)LF_NOALLOC_MAX_TOKENS / kGemvTok + LF_NOALLOC_MAX_ADAPTERS + 1) * sizeof(GemvItem)) +
    al256((size_t)LF_NOALLOC_MAX_TOKENS * kMaxRank * sizeof(float));
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

// In host code g_noalloc_scratch is only a host-side stand-in for the device array;
// its device address is looked up once per device (with that device current) and
// cached here.
constexpr int kMaxDevices = 64;
static std::mutex g_noalloc_mu;
static void* g_noalloc_addr[kMaxDevices] = {};

static lf_status noalloc_scratch(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return LF_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return LF_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_addr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return LF_ERR_CUDA;
        g_noalloc_addr[dev] = p;
    }
    *out = g_noalloc_addr[dev];
    return LF_OK;
}

// ------------------------------------------------------- bounded-wait check
// One thread waits on an mbarrier that nothing arrives at (no copy or MMA is in
// flight), so the wait runs out after `polls` polls and latches LF_ERR_TIMEOUT: the
// same exit every pipeline wait of the library takes when a producer never arrives.
__global__ void wait_selftest_kernel(int polls) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_barrier_init();
    mbar_wait_bounded(&bar, 0, polls);
}

// ------------------------------------------------------------ JD-Full plan
struct JdPlan {
    std::vector<JdMember> members;
    std::vector<JdProbDev> probs;
    std::vector<lf_module> basis_user, basis_ws;
    std::vector<TsqrWork> pwork;
    std::vector<TsqrInfo> pinfo;
    int32_t pslots = 0;
    std::vector<JdTile> tiles;
    std::vector<int32_t> tile0, ntiles;   // per mf = 2 * problem + factor
    TsqrPlan orth;
    int RX = 16, RY = 16;
    int64_t ws_U = 0, ws_Vt = 0;   // floats of the workspace copies of the state
};

static lf_status check_jd(const lf_module* mods, int32_t n_mods, const int32_t* members, int32_t n_members,
                          const lf_jd_problem* probs, int32_t n_probs) {
    lf_status st = check_mods(mods, n_mods);
    if (st != LF_OK) return st;
    if (n_members < 0 || n_probs < 0 || (n_members > 0 && !members) || (n_probs > 0 && !probs))
        return LF_ERR_INVALID_ARG;
    for (int32_t p = 0; p < n_probs; ++p) {
        const lf_jd_problem& q = probs[p];
        if (q.count < 1 || q.first < 0 || (int64_t)q.first + q.count > n_members) return LF_ERR_INVALID_ARG;
        if (q.d_out < 1 || q.d_in < 1 || q.rank < 1 || q.rank > kMaxRank || q.rank > q.d_out || q.rank > q.d_in)
            return LF_ERR_SHAPE;
        if (q.U_off < 0 || q.Vt_off < 0 || q.sigma_off < 0) return LF_ERR_INVALID_ARG;
        if ((q.U_off & 3) || (q.Vt_off & 3)) return LF_ERR_ALIGNMENT;
        for (int32_t j = 0; j < q.count; ++j) {
            const int32_t m = members[q.first + j];
            if (m < 0 || m >= n_mods) return LF_ERR_INVALID_ARG;
            if (mods[m].d_out != q.d_out || mods[m].d_in != q.d_in) return LF_ERR_SHAPE;
        }
    }
    return LF_OK;
}

static void plan_jd(const lf_module* mods, const int32_t* members, const lf_jd_problem* probs, int32_t n_probs,
                    JdPlan& P) {
    int rx = 1, ry = 1;
    for (int32_t p = 0; p < n_probs; ++p) {
        const lf_jd_problem& q = probs[p];
        P.probs.push_back(JdProbDev{(int32_t)P.members.size(), q.count, q.sigma_off});
        for (int32_t j = 0; j < q.count; ++j) {
            const int32_t m = members[q.first + j];
            P.members.push_back(JdMember{m, p, j, 0});
            rx = std::max(rx, (int)mods[m].r);
        }
        ry = std::max(ry, (int)q.rank);
        P.basis_user.push_back(lf_module{q.d_out, q.d_in, q.rank, 0, q.U_off, q.Vt_off});
        P.basis_ws.push_back(lf_module{q.d_out, q.d_in, q.rank, 0, P.ws_U, P.ws_Vt});
        P.ws_U += align_up((int64_t)q.d_out * q.rank, 4);
        P.ws_Vt += align_up((int64_t)q.rank * q.d_in, 4);
        for (int f = 0; f < 2; ++f) {
            const int rows = f == 0 ? q.d_out : q.d_in;
            P.tile0.push_back((int32_t)P.tiles.size());
            P.ntiles.push_back((int32_t)cdiv(rows, kJdTR));
            for (int r0 = 0; r0 < rows; r0 += kJdTR) P.tiles.push_back(JdTile{p, f, r0, std::min(kJdTR, rows - r0)});
        }
    }
    P.RX = rt_bucket(rx);
    P.RY = rt_bucket(ry);
    const int32_t ng = (int32_t)P.members.size();
    P.pinfo.resize((size_t)2 * ng);
    for (int32_t g = 0; g < ng; ++g) {
        const lf_module& md = mods[P.members[g].mod];
        for (int f = 0; f < 2; ++f) {
            const int rows = f == 0 ? md.d_out : md.d_in;
            const int nch = (int)cdiv(rows, kJdChunk);
            P.pinfo[2 * g + f] = TsqrInfo{nch, nch > 1 ? P.pslots : -1};
            for (int c = 0; c < nch; ++c)
                P.pwork.push_back(TsqrWork{2 * g + f, c * kJdChunk, std::min(kJdChunk, rows - c * kJdChunk),
                                           nch > 1 ? P.pslots + c : -1});
            if (nch > 1) P.pslots += nch;
        }
    }
    std::stable_sort(P.pwork.begin(), P.pwork.end(),
                     [](const TsqrWork& a, const TsqrWork& b) { return a.nrows > b.nrows; });
    plan_tsqr(P.basis_ws.data(), n_probs, P.orth);
}

struct JdLayout {
    size_t mods, members, probs, basis_user, basis_ws, pwork, pinfo, tiles, tile0, ntiles, owork, onwork, oinfo;
    size_t pcounters, ocounters, ppartial, opartial, tgram, gsum, QP, WZ, wsU, wsVt, RB, RA, R64, Rinv, total;
};

static JdLayout jd_layout(int32_t n_mods, int32_t n_probs, const JdPlan& P) {
    Carver c(nullptr);
    JdLayout L;
    const size_t ng = P.members.size();
    const size_t blk = (size_t)P.RX * P.RY;
    const size_t rs2 = (size_t)P.orth.rs * P.orth.rs;
#define LF_TAKE(field, T, cnt)                          \
    do {                                                \
        c.take<T>(cnt);                                 \
        L.field = c.off - (size_t)(cnt) * sizeof(T);    \
    } while (0)
    LF_TAKE(mods, lf_module, n_mods);
    LF_TAKE(members, JdMember, ng);
    LF_TAKE(probs, JdProbDev, n_probs);
    LF_TAKE(basis_user, lf_module, n_probs);
    LF_TAKE(basis_ws, lf_module, n_probs);
    LF_TAKE(pwork, TsqrWork, P.pwork.size());
    LF_TAKE(pinfo, TsqrInfo, P.pinfo.size());
    LF_TAKE(tiles, JdTile, P.tiles.size());
    LF_TAKE(tile0, int32_t, P.tile0.size());
    LF_TAKE(ntiles, int32_t, P.ntiles.size());
    LF_TAKE(owork, TsqrWork, P.orth.work.size());
    LF_TAKE(onwork, int32_t, 1);
    LF_TAKE(oinfo, TsqrInfo, P.orth.info.size());
    LF_TAKE(pcounters, int32_t, 2 * ng);
    // orthogonalize: flags of pass 1, Gram counters of pass 2, Householder counters of
    // both passes, flags of pass 2 (2 per problem each), zeroed every step
    LF_TAKE(ocounters, int32_t, (size_t)10 * n_probs);
    LF_TAKE(ppartial, double, (size_t)P.pslots * blk);
    LF_TAKE(opartial, char, (size_t)P.orth.slots * tsqr_slot_bytes(P.orth.RT));
    LF_TAKE(tgram, double, P.tiles.size() * (size_t)(P.RY * (P.RY + 1) / 2));
    LF_TAKE(gsum, double, (size_t)2 * n_probs * (P.RY * (P.RY + 1) / 2));
    LF_TAKE(QP, double, 2 * ng * blk);
    LF_TAKE(WZ, float, 2 * ng * blk);
    LF_TAKE(wsU, float, (size_t)P.ws_U);
    LF_TAKE(wsVt, float, (size_t)P.ws_Vt);
    LF_TAKE(RB, float, (size_t)n_probs * rs2);
    LF_TAKE(RA, float, (size_t)n_probs * rs2);
    LF_TAKE(R64, double, (size_t)2 * n_probs * rs2);   // pass 2, two factors per problem
    LF_TAKE(Rinv, double, (size_t)2 * n_probs * rs2);
#undef LF_TAKE
    L.total = c.off + 256;
    return L;
}

template <int RX, int RY>
static cudaError_t launch_jd_rxry(int which, const void* args, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    if (which == 0) {
        LF_LAUNCH("jd_project", (jd_project_kernel<RX, RY>), grid, 32 * jd_project_warps<RY>(), 0, st,
                  *static_cast<const JdProjArgs*>(args));
    } else if (which == 1) {
        auto k = jd_core_kernel<RX, RY>;
        constexpr size_t smem = jd_core_smem<RX, RY>();
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        LF_LAUNCH("jd_core", k, grid, 256, smem, st, *static_cast<const JdCoreArgs*>(args));
    } else {
        auto k = jd_update_kernel<RX, RY>;
        constexpr size_t smem = jd_update_smem<RX, RY>();
        cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        LF_LAUNCH("jd_update", k, grid, 128, smem, st, *static_cast<const JdUpdArgs*>(args));
    }
    return cudaGetLastError();
}

template <int RX>
static cudaError_t launch_jd_rx(int RY, int which, const void* args, int grid, cudaStream_t st) {
    if (RY == 16) return launch_jd_rxry<RX, 16>(which, args, grid, st);
    if (RY == 32) return launch_jd_rxry<RX, 32>(which, args, grid, st);
    return launch_jd_rxry<RX, 64>(which, args, grid, st);
}

static cudaError_t launch_jd(int RX, int RY, int which, const void* args, int grid, cudaStream_t st) {
    if (RX == 16) return launch_jd_rx<16>(RY, which, args, grid, st);
    if (RX == 32) return launch_jd_rx<32>(RY, which, args, grid, st);
    return launch_jd_rx<64>(RY, which, args, grid, st);
}

template <int RT>
static cudaError_t launch_jd_qform_rt(const JdQArgs& a, int grid, cudaStream_t st) {
    auto k = jd_qform_kernel<RT>;
    constexpr size_t smem = jd_qform_smem<RT>();
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LF_LAUNCH("jd_qform", k, grid, kJdTR, smem, st, a);
    return cudaGetLastError();
}

static cudaError_t launch_jd_qform(int RT, const JdQArgs& a, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    if (RT == 16) return launch_jd_qform_rt<16>(a, grid, st);
    if (RT == 32) return launch_jd_qform_rt<32>(a, grid, st);
    return launch_jd_qform_rt<64>(a, grid, st);
}

static cudaError_t launch_jd_gram_sum(int RT, const JdGramSumArgs& a, int n_mf, cudaStream_t st) {
    if (n_mf <= 0) return cudaSuccess;
    const dim3 grid(n_mf, (unsigned)cdiv(RT * (RT + 1) / 2, 128));
    if (RT == 16) LF_LAUNCH("jd_gram_sum", jd_gram_sum_kernel<16>, grid, 128, 0, st, a);
    else if (RT == 32) LF_LAUNCH("jd_gram_sum", jd_gram_sum_kernel<32>, grid, 128, 0, st, a);
    else LF_LAUNCH("jd_gram_sum", jd_gram_sum_kernel<64>, grid, 128, 0, st, a);
    return cudaGetLastError();
}

static cudaError_t launch_jd_rinv(int RT, const JdRinvArgs& a, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    if (RT == 16) LF_LAUNCH("jd_rinv", jd_rinv_kernel<16>, grid, 128, 0, st, a);
    else if (RT == 32) LF_LAUNCH("jd_rinv", jd_rinv_kernel<32>, grid, 128, 0, st, a);
    else LF_LAUNCH("jd_rinv", jd_rinv_kernel<64>, grid, 128, 0, st, a);
    return cudaGetLastError();
}

static cudaError_t launch_jd_chol(int RT, const JdCholArgs& a, int grid, cudaStream_t st) {
    if (grid <= 0) return cudaSuccess;
    if (RT == 16) LF_LAUNCH("jd_chol", jd_chol_kernel<16>, grid, 256, 0, st, a);
    else if (RT == 32) LF_LAUNCH("jd_chol", jd_chol_kernel<32>, grid, 256, 0, st, a);
    else LF_LAUNCH("jd_chol", jd_chol_kernel<64>, grid, 256, 0, st, a);
    return cudaGetLastError();
}

// ------------------------------------------------------- pool-wide subspace
static size_t pool_layout(int32_t R, int32_t d, size_t* off /* 10 entries or nullptr */) {
    Carver c(nullptr);
    size_t o[10];
    c.take<int64_t>((size_t)R); o[0] = c.off - (size_t)R * 8;          // row_off
    c.take<int32_t>((size_t)R); o[1] = c.off - (size_t)R * 4;          // row_step
    c.take<float>((size_t)R * d); o[2] = c.off - (size_t)R * d * 4;    // Sv
    c.take<double>((size_t)R * R); o[3] = c.off - (size_t)R * R * 8;   // X
    c.take<double>((size_t)R * R); o[4] = c.off - (size_t)R * R * 8;   // V
    c.take<double>((size_t)R); o[5] = c.off - (size_t)R * 8;           // lam
    c.take<int32_t>((size_t)R); o[6] = c.off - (size_t)R * 4;          // order
    c.take<uint32_t>(8); o[7] = c.off - 32;                            // barrier words
    c.take<double>((size_t)R); o[8] = c.off - (size_t)R * 8;           // resid parts
    o[9] = 0;
    if (off) std::memcpy(off, o, sizeof(o));
    return c.off + 256;
}

static lf_status check_pool(int32_t side, int32_t n_lora, const int32_t* ranks, const int64_t* offs, int32_t d,
                            int32_t* R_out) {
    if ((side != 0 && side != 1) || n_lora < 1 || !ranks || !offs || d < 1) return LF_ERR_INVALID_ARG;
    int64_t R = 0;
    for (int32_t i = 0; i < n_lora; ++i) {
        if (ranks[i] < 1 || offs[i] < 0) return LF_ERR_INVALID_ARG;
        R += ranks[i];
    }
    if (R > kPoolMaxRank || R > d) return LF_ERR_SHAPE;
    *R_out = (int32_t)R;
    return LF_OK;
}
}  // namespace lf

using namespace lf;

extern "C" {

int32_t lf_rank_stride(const lf_module* mods, int32_t n) { return mods && n > 0 ? rank_stride(mods, n) : 0; }

size_t lf_tsqr_workspace_size(const lf_module* mods, int32_t n) {
    if (check_mods(mods, n) != LF_OK) return 0;
    TsqrPlan p;
    plan_tsqr(mods, n, p);
    I8Plan q;
    plan_i8(mods, n, q);
    return tsqr_layout(n, p, q).total;
}

lf_status lf_tsqr_batched(const lf_module* mods, int32_t n, const float* B_base, const float* A_base, float* R_B,
                          float* R_A, double* sigma, double* U, double* V, void* ws, size_t ws_bytes,
                          lf_stream_t stream) {
    lf_status st = check_mods(mods, n);
    if (st != LF_OK) return st;
    if (n == 0) return LF_OK;
    if (!B_base || !A_base || !R_B || !R_A || !sigma || !ws) return LF_ERR_INVALID_ARG;
    if (!aligned16(B_base) || !aligned16(A_base)) return LF_ERR_ALIGNMENT;
    TsqrPlan p;
    plan_tsqr(mods, n, p);
    I8Plan q;
    plan_i8(mods, n, q);
    const TsqrLayout L = tsqr_layout(n, p, q);
    if (ws_bytes < L.total) return LF_ERR_WORKSPACE;
    char* base = reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    Staging h;
    const int32_t nwork = (int32_t)p.work.size();
    h.put(mods, n);
    h.put(p.work.data(), p.work.size());
    h.put(&nwork, 1);
    h.put(p.info.data(), p.info.size());
    h.put(&n, 1);
    LF_CUDA_TRY(cudaMemcpyAsync(base, h.buf.data(), h.off, cudaMemcpyHostToDevice, s));
    LF_CUDA_TRY(cudaMemsetAsync(base + L.counters, 0, (size_t)6 * n * sizeof(int32_t), s));
    // tensor maps of the A factors the integer leaf reads (a matrix whose map the encoder
    // rejects goes to the fp64 leaf with its items skipped)
    std::vector<CUtensorMap> amaps((size_t)n);
    std::vector<char> keep((size_t)2 * n, 1);
    for (int32_t i = 0; i < n; ++i) {
        std::memset(&amaps[i], 0, sizeof(CUtensorMap));
        if (q.fb[2 * i + 1] == 0 && !encode_a_map(&amaps[i], A_base + mods[i].A_off, mods[i].r, mods[i].d_in)) {
            q.fb[2 * i + 1] = 1;
            keep[2 * i + 1] = 0;
        }
    }
    std::vector<TsqrWork> work8;   // the items kept, then unused room up to the planned count
    work8.reserve(q.work.size());
    for (const TsqrWork& w : q.work)
        if (keep[w.mf]) work8.push_back(w);
    const int32_t n_work8 = (int32_t)work8.size();
    work8.resize(q.work.size(), TsqrWork{0, 0, 0, 0});
    Staging h8;   // the integer-Gram tables sit after the partial slots
    h8.put(work8.data(), work8.size());
    h8.put(q.info.data(), q.info.size());
    h8.put(q.fb.data(), q.fb.size());
    h8.put(amaps.data(), amaps.size());
    LF_CUDA_TRY(cudaMemcpyAsync(base + L.i8work, h8.buf.data(), h8.off, cudaMemcpyHostToDevice, s));
    int32_t* gram_counters = reinterpret_cast<int32_t*>(base + L.counters);
    int32_t* hh_counters = gram_counters + 2 * n;
    int32_t* flags = gram_counters + 4 * n;
    int32_t* fb = reinterpret_cast<int32_t*>(base + L.fb);

    // integer Gram on the tensor cores for every addressable matrix, then its root (sum of
    // the item Grams, fp64 Cholesky); a matrix it leaves (unaddressable rows, a value past
    // its column scale, a non-finite value) is marked in fb for the fp64 Gram leaf below
    GramI8Args ia;
    ia.mods = reinterpret_cast<const lf_module*>(base + L.mods);
    ia.B_base = B_base;
    ia.amaps = reinterpret_cast<const CUtensorMap*>(base + L.amaps);
    ia.work = reinterpret_cast<const TsqrWork*>(base + L.i8work);
    ia.n_work = n_work8;
    ia.gram = reinterpret_cast<double*>(base + L.i8gram);
    ia.fb = fb;
    GramI8RootArgs ra;
    ra.mods = ia.mods;
    ra.info = reinterpret_cast<const TsqrInfo*>(base + L.i8info);
    ra.gram = ia.gram;
    ra.fb = fb;
    ra.flags = flags;
    ra.R_B = R_B;
    ra.R_A = R_A;
    ra.rs = p.rs;
    ra.n_mf = 2 * n;
    LF_CUDA_TRY(launch_gram_i8_rt(p.RT, ia, ra, s));

    GramArgs ga;
    ga.mods = reinterpret_cast<const lf_module*>(base + L.mods);
    ga.B_base = B_base;
    ga.A_base = A_base;
    ga.work = reinterpret_cast<const TsqrWork*>(base + L.work);
    ga.n_work = reinterpret_cast<const int32_t*>(base + L.nwork);
    ga.info = reinterpret_cast<const TsqrInfo*>(base + L.info);
    ga.counters = gram_counters;
    ga.partial = reinterpret_cast<double*>(base + L.partial);
    ga.slot_doubles = (int64_t)(tsqr_slot_bytes(p.RT) / sizeof(double));
    ga.flags = flags;
    ga.R_B = R_B;
    ga.R_A = R_A;
    ga.rs = p.rs;
    ga.only = fb;
    ga.R64 = nullptr;
    LF_CUDA_TRY(launch_gram_rt(p.RT, ga, nwork, s));

    // structured-Householder TSQR for the matrices whose Gram Cholesky was rejected
    TsqrArgs<float> ta;
    ta.mods = reinterpret_cast<const lf_module*>(base + L.mods);
    ta.mod_ids = nullptr;
    ta.B_base = B_base;
    ta.A_base = A_base;
    ta.work = reinterpret_cast<const TsqrWork*>(base + L.work);
    ta.n_work = reinterpret_cast<const int32_t*>(base + L.nwork);
    ta.info = reinterpret_cast<const TsqrInfo*>(base + L.info);
    ta.counters = hh_counters;
    ta.partial = reinterpret_cast<float*>(base + L.partial);
    ta.R_B = R_B;
    ta.R_A = R_A;
    ta.rs = p.rs;
    ta.only = flags;
    ta.tree = 0;
    LF_CUDA_TRY(launch_tsqr_rt<float>(p.RT, ta, nwork, s));

    SvdArgs<float, float> sa;
    sa.mods = ta.mods;
    sa.mod_ids = nullptr;
    sa.n = reinterpret_cast<const int32_t*>(base + L.n_dev);
    sa.R_B = R_B;
    sa.R_A = R_A;
    sa.sigma = sigma;
    sa.U = U;
    sa.V = V;
    sa.rs = p.rs;
    sa.max_sweeps = 20;
    LF_CUDA_TRY(launch_svd_rt(p.RT, sa, n, s));
    return LF_OK;
}

size_t lf_select_workspace_size(const lf_module* mods, int32_t n) {
    if (check_mods(mods, n) != LF_OK) return 0;
    ExportPlan p;
    plan_export(mods, n, p);
    Carver c(nullptr);
    c.take<lf_module>(n);
    c.take<int32_t>(p.gptr.size());
    c.take<int32_t>(p.gmods.size());
    c.take<double>((size_t)n * p.rs);
    return c.off + 256;
}

// One selection CTA per group, with the group's candidate list in dynamic shared memory
// when it fits (kSelMaxCand entries at most; larger groups count from global memory).
static cudaError_t launch_select(SelArgs a, int ng, int32_t max_cand, cudaStream_t s) {
    a.cand_cap = std::min(max_cand, kSelMaxCand);
    const size_t smem = (size_t)a.cand_cap * sizeof(double);
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LF_LAUNCH("select", select_kernel, ng, kSelThreads, smem, s, a);
    return cudaGetLastError();
}

lf_status lf_select_ranks(const lf_module* mods, int32_t n, lf_policy pol, const double* sigma, int32_t* ranks,
                          int64_t* off_A, int64_t* off_Bt, void* ws, size_t ws_bytes, lf_stream_t stream) {
    lf_status st = check_mods(mods, n);
    if (st != LF_OK) return st;
    st = check_policy(mods, n, pol);
    if (st != LF_OK) return st;
    if (n == 0) return LF_OK;
    if (!sigma || !ranks || !off_A || !off_Bt || !ws) return LF_ERR_INVALID_ARG;
    if (ws_bytes < lf_select_workspace_size(mods, n)) return LF_ERR_WORKSPACE;
    ExportPlan p;
    plan_export(mods, n, p);
    char* base = reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    Staging h;
    const size_t om = h.put(mods, n);
    const size_t og = h.put(p.gptr.data(), p.gptr.size());
    const size_t ogm = h.put(p.gmods.data(), p.gmods.size());
    h.off = (size_t)align_up((int64_t)h.off, 256);
    const size_t oe = h.off;
    LF_CUDA_TRY(cudaMemcpyAsync(base, h.buf.data(), h.buf.size(), cudaMemcpyHostToDevice, s));
    SelArgs a;
    a.mods = reinterpret_cast<const lf_module*>(base + om);
    a.grp_ptr = reinterpret_cast<const int32_t*>(base + og);
    a.grp_mods = reinterpret_cast<const int32_t*>(base + ogm);
    a.sigma = sigma;
    a.energy = reinterpret_cast<double*>(base + oe);
    a.rs = p.rs;
    a.pol = pol;
    a.ranks = ranks;
    a.band = 0.0;
    a.flag_list = nullptr;
    a.flag_count = nullptr;
    const int ng = (int)p.gptr.size() - 1;
    LF_CUDA_TRY(launch_select(a, ng, p.max_cand, s));
    LF_LAUNCH("offsets", offsets_kernel, 1, 1024, 0, s, a.mods, n, ranks, off_A, off_Bt, INT64_MAX, INT64_MAX);
    return launch_status();
}

size_t lf_export_workspace_size(const lf_module* mods, int32_t n) {
    if (check_mods(mods, n) != LF_OK) return 0;
    ExportPlan p;
    plan_export(mods, n, p);
    return export_layout(n, p).total;
}

void lf_export_pool_bound(const lf_module* mods, int32_t n, lf_policy pol, int64_t* cap_A, int64_t* cap_Bt) {
    if (!cap_A || !cap_Bt) return;
    *cap_A = *cap_Bt = 0;
    if (check_mods(mods, n) != LF_OK || check_policy(mods, n, pol) != LF_OK) return;
    if (pol.kind == 0 || pol.kind == 3) {   // kind 3 may keep every direction: bound by r
        for (int32_t i = 0; i < n; ++i) {
            const int r = mods[i].r;
            const int k = pol.kind == 3 ? r
                                        : std::min(r, std::max(pol.floor, (pol.ratio_num * r + pol.ratio_den / 2) / pol.ratio_den));
            *cap_A += (int64_t)k * mods[i].d_in;
            *cap_Bt += (int64_t)k * mods[i].d_out;
        }
        return;
    }
    // S: floors everywhere, plus the group's extra slots on its widest modules
    std::map<int32_t, std::vector<int32_t>> by;
    for (int32_t i = 0; i < n; ++i) by[mods[i].group].push_back(i);
    for (auto& kv : by) {
        int64_t rsum = 0;
        for (int32_t i : kv.second) rsum += mods[i].r;
        const int64_t K = (int64_t)pol.ratio_num * rsum / pol.ratio_den;
        int64_t extra = K - (int64_t)pol.floor * (int64_t)kv.second.size();
        std::vector<std::pair<int, int>> slotsA, slotsB;  // (d, free slots)
        for (int32_t i : kv.second) {
            *cap_A += (int64_t)pol.floor * mods[i].d_in;
            *cap_Bt += (int64_t)pol.floor * mods[i].d_out;
            slotsA.push_back({mods[i].d_in, mods[i].r - pol.floor});
            slotsB.push_back({mods[i].d_out, mods[i].r - pol.floor});
        }
        auto fill = [&](std::vector<std::pair<int, int>>& v, int64_t* cap) {
            std::sort(v.begin(), v.end(), [](auto& x, auto& y) { return x.first > y.first; });
            int64_t left = extra;
            for (auto& s : v) {
                if (left <= 0) break;
                const int64_t t = std::min<int64_t>(left, s.second);
                *cap += t * s.first;
                left -= t;
            }
        };
        if (extra > 0) {
            fill(slotsA, cap_A);
            fill(slotsB, cap_Bt);
        }
    }
}

lf_status lf_truncate_export(const lf_module* mods, int32_t n, lf_policy pol, const float* B_base,
                             const float* A_base, const float* R_B, const float* R_A, const double* sigma,
                             const double* U, const double* V, int32_t* ranks, int64_t* off_A, int64_t* off_Bt,
                             float* A_pool, float* Bt_pool, void* A_pool_bf16, void* Bt_pool_bf16,
                             int64_t pool_cap_A, int64_t pool_cap_Bt, void* ws, size_t ws_bytes,
                             lf_stream_t stream) {
    lf_status st = check_mods(mods, n);
    if (st != LF_OK) return st;
    st = check_policy(mods, n, pol);
    if (st != LF_OK) return st;
    if (n == 0) return LF_OK;
    if (!B_base || !A_base || !R_B || !R_A || !sigma || !U || !V || !ranks || !off_A || !off_Bt || !A_pool ||
        !Bt_pool || !ws || pool_cap_A < 0 || pool_cap_Bt < 0)
        return LF_ERR_INVALID_ARG;
    if (!aligned16(B_base) || !aligned16(A_base)) return LF_ERR_ALIGNMENT;
    ExportPlan p;
    plan_export(mods, n, p);
    const ExportLayout L = export_layout(n, p);
    if (ws_bytes < L.total) return LF_ERR_WORKSPACE;
    char* base = reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);

    Staging h;
    h.put(mods, n);
    h.put(p.gptr.data(), p.gptr.size());
    h.put(p.gmods.data(), p.gmods.size());
    h.put(p.ework.data(), p.ework.size());
    LF_CUDA_TRY(cudaMemcpyAsync(base, h.buf.data(), h.off, cudaMemcpyHostToDevice, s));
    const lf_module* dmods = reinterpret_cast<const lf_module*>(base + L.mods);
    const int ng = (int)p.gptr.size() - 1;

    SelArgs a;
    a.mods = dmods;
    a.grp_ptr = reinterpret_cast<const int32_t*>(base + L.gptr);
    a.grp_mods = reinterpret_cast<const int32_t*>(base + L.gmods);
    a.sigma = sigma;
    a.energy = reinterpret_cast<double*>(base + L.energy);
    a.rs = p.rs;
    a.pol = pol;
    a.ranks = ranks;
    a.band = 1e-4;
    a.flag_list = nullptr;
    a.flag_count = nullptr;

    if (pol.kind >= 1) {   // spectral policies: refine the modules near the boundary
        int32_t* flist = reinterpret_cast<int32_t*>(base + L.flist);
        int32_t* fcount = reinterpret_cast<int32_t*>(base + L.fcount);
        LF_CUDA_TRY(cudaMemsetAsync(fcount, 0, 2 * sizeof(int32_t), s));
        a.flag_list = flist;
        a.flag_count = fcount;
        LF_CUDA_TRY(launch_select(a, ng, p.max_cand, s));
        LF_LAUNCH("refine_plan", cap_flags_kernel, 1, 32, 0, s, fcount, p.refine_cap);
        LF_CUDA_TRY(cudaGetLastError());
        TsqrWork* rwork = reinterpret_cast<TsqrWork*>(base + L.rwork);
        int32_t* rnwork = reinterpret_cast<int32_t*>(base + L.rnwork);
        TsqrInfo* rinfo = reinterpret_cast<TsqrInfo*>(base + L.rinfo);
        LF_LAUNCH("refine_plan", refine_plan_kernel, 1, 32, 0, s, dmods, flist, fcount, rwork, rnwork, rinfo, kRefineChunk);
        LF_CUDA_TRY(cudaGetLastError());
        if (p.refine_slots > 0)
            LF_CUDA_TRY(cudaMemsetAsync(base + L.rcnt, 0, (size_t)p.refine_slots * sizeof(int32_t), s));
        TsqrArgs<double> ta;
        ta.mods = dmods;
        ta.mod_ids = flist;
        ta.B_base = B_base;
        ta.A_base = A_base;
        ta.work = rwork;
        ta.n_work = rnwork;
        ta.info = rinfo;
        ta.counters = reinterpret_cast<int32_t*>(base + L.rcnt);
        ta.partial = reinterpret_cast<double*>(base + L.rpart);
        ta.R_B = reinterpret_cast<double*>(base + L.rRB);
        ta.R_A = reinterpret_cast<double*>(base + L.rRA);
        ta.rs = p.rs;
        ta.only = nullptr;
        ta.tree = 1;
        LF_CUDA_TRY(launch_tsqr_rt<double>(p.RT, ta, p.refine_max_work, s));
        SvdArgs<double, double> sa;
        sa.mods = dmods;
        sa.mod_ids = flist;
        sa.n = fcount + 1;
        sa.R_B = ta.R_B;
        sa.R_A = ta.R_A;
        sa.sigma = reinterpret_cast<double*>(base + L.rsig);
        sa.U = nullptr;
        sa.V = nullptr;
        sa.rs = p.rs;
        sa.max_sweeps = 20;
        LF_CUDA_TRY(launch_svd_rt(p.RT, sa, p.refine_cap, s));
        double* sigref = reinterpret_cast<double*>(base + L.sigref);
        LF_CUDA_TRY(cudaMemcpyAsync(sigref, sigma, (size_t)n * p.rs * sizeof(double), cudaMemcpyDeviceToDevice, s));
        LF_LAUNCH("refine_plan", scatter_sigma_kernel, p.refine_cap, 64, 0, s, flist, fcount + 1, sa.sigma, sigref, p.rs);
        LF_CUDA_TRY(cudaGetLastError());
        a.sigma = sigref;
        a.flag_list = nullptr;
        a.flag_count = nullptr;
    }
    LF_CUDA_TRY(launch_select(a, ng, p.max_cand, s));
    LF_LAUNCH("offsets", offsets_kernel, 1, 1024, 0, s, dmods, n, ranks, off_A, off_Bt, pool_cap_A, pool_cap_Bt);
    LF_CUDA_TRY(cudaGetLastError());
    float* CA = reinterpret_cast<float*>(base + L.CA);
    float* CB = reinterpret_cast<float*>(base + L.CB);
    LF_LAUNCH("export_coef", export_coef_kernel, n, 128, 0, s, dmods, ranks, R_B, R_A, sigma, U, V, p.rs, CA, CB);
    LF_CUDA_TRY(cudaGetLastError());
    ExportArgs ea;
    ea.mods = dmods;
    ea.work = reinterpret_cast<const ExportWork*>(base + L.ework);
    ea.B_base = B_base;
    ea.A_base = A_base;
    ea.ranks = ranks;
    ea.off_A = off_A;
    ea.off_Bt = off_Bt;
    ea.C_A = CA;
    ea.C_Bt = CB;
    ea.rs = p.rs;
    ea.A_pool = A_pool;
    ea.Bt_pool = Bt_pool;
    ea.A_pool16 = reinterpret_cast<__nv_bfloat16*>(A_pool_bf16);
    ea.Bt_pool16 = reinterpret_cast<__nv_bfloat16*>(Bt_pool_bf16);
    ea.cap_A = pool_cap_A;
    ea.cap_Bt = pool_cap_Bt;
    LF_CUDA_TRY(cudaFuncSetAttribute(export_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kExportSmem));
    LF_LAUNCH("export_stream", export_kernel, (int)p.ework.size(), kExpThreads, kExportSmem, s, ea);
    return launch_status();
}

size_t lf_apply_slices_workspace_size(int32_t T, int32_t n_adapters, int32_t n_slices) {
    if (T < 0 || n_adapters < 1 || n_slices < 1 || n_slices > kMaxSlices) return 0;
    ApplyWs w;
    return carve_apply(nullptr, T, n_adapters, n_slices, &w);
}

size_t lf_apply_workspace_size(int32_t T, int32_t n_adapters) { return lf_apply_slices_workspace_size(T, n_adapters, 1); }

lf_status lf_lora_sigma_sandwich(int32_t T, int32_t d_in, int32_t d_out, const void* x, void* y, const int32_t* ids,
                                 int32_t n_adapters, int32_t rank, const void* Vt, const void* Ut, const float* sigma,
                                 int32_t sigma_diag, float scale, void* ws, size_t ws_bytes, lf_stream_t stream) {
    if (rank < 1 || rank > kMaxRank || d_out < 1 || (sigma_diag != 0 && sigma_diag != 1)) return LF_ERR_INVALID_ARG;
    if (T > 0 && (!Vt || !Ut || !sigma)) return LF_ERR_INVALID_ARG;
    lf_slice one{};
    one.d_out = d_out;
    one.y_offset = 0;
    one.A_pool = Vt;
    one.Bt_pool = Ut;
    one.pool_elems_A = (int64_t)rank * d_in;
    one.pool_elems_Bt = (int64_t)rank * d_out;
    SharedSlice sh;
    sh.k = rank;
    sh.sigma = sigma;
    sh.mode = sigma_diag ? 1 : 2;
    return apply_impl(T, d_in, x, y, d_out, ids, n_adapters, &one, 1, scale, nullptr, nullptr, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), &sh);
}

lf_status lf_lora_shrink_expand(int32_t T, int32_t d_in, int32_t d_out, const void* x, void* y, const int32_t* ids,
                                int32_t n_adapters, const int32_t* ranks, const int64_t* off_A,
                                const int64_t* off_Bt, const void* A_pool, const void* Bt_pool,
                                int64_t pool_elems_A, int64_t pool_elems_Bt, float scale, int32_t* seg_out,
                                void* ws, size_t ws_bytes, lf_stream_t stream) {
    if (d_out < 1) return LF_ERR_INVALID_ARG;
    if (T > 0 && (!ranks || !off_A || !off_Bt || !A_pool || !Bt_pool)) return LF_ERR_INVALID_ARG;
    lf_slice one{};
    one.d_out = d_out;
    one.y_offset = 0;
    one.ranks = ranks;
    one.off_A = off_A;
    one.off_Bt = off_Bt;
    one.A_pool = A_pool;
    one.Bt_pool = Bt_pool;
    one.pool_elems_A = pool_elems_A;
    one.pool_elems_Bt = pool_elems_Bt;
    return apply_impl(T, d_in, x, y, d_out, ids, n_adapters, &one, 1, scale, nullptr, seg_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream));
}

lf_status lf_lora_shrink_expand_slices(int32_t T, int32_t d_in, const void* x, void* y, int64_t y_ld,
                                       const int32_t* ids, int32_t n_adapters, const lf_slice* slices,
                                       int32_t n_slices, float scale, const float* adapter_scale, int32_t* seg_out,
                                       void* ws, size_t ws_bytes, lf_stream_t stream) {
    return apply_impl(T, d_in, x, y, y_ld, ids, n_adapters, slices, n_slices, scale, adapter_scale, seg_out, ws,
                      ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

static_assert(kMaxProj == LF_MAX_PROJECTIONS, "projection table size");

lf_status lf_lora_shrink_expand_projections(int32_t T, const int32_t* ids, int32_t n_adapters,
                                            const lf_projection* projs, int32_t n_proj, float scale,
                                            const float* adapter_scale, void* ws, size_t ws_bytes,
                                            lf_stream_t stream) {
    if (T < 0 || n_adapters < 1 || n_adapters > 16384 || n_proj < 1 || n_proj > kMaxProj || !projs)
        return LF_ERR_INVALID_ARG;
    if (T == 0) return LF_OK;
    if (!ids) return LF_ERR_INVALID_ARG;
    for (int p = 0; p < n_proj; ++p) {
        if (projs[p].reserved != 0) return LF_ERR_INVALID_ARG;
        const lf_status st = check_apply(projs[p].d_in, projs[p].x, projs[p].y, projs[p].y_ld, &projs[p].slice, 1, false);
        if (st != LF_OK) return st;
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (!decode_regime(T, n_adapters)) {
        // routed path, projection by projection: the first call routes the batch into
        // ws, the others reuse its tables
        for (int p = 0; p < n_proj; ++p) {
            const lf_projection& q = projs[p];
            const lf_status st = apply_impl(T, q.d_in, q.x, q.y, q.y_ld, ids, n_adapters, &q.slice, 1, scale,
                                            adapter_scale, nullptr, ws, ws_bytes, s, nullptr, p > 0);
            if (st != LF_OK) return st;
        }
        return LF_OK;
    }
    ProjArgs A{};
    A.T = T;
    A.n_adapters = n_adapters;
    A.n_proj = n_proj;
    A.ids = ids;
    A.scale = scale;
    A.scales = adapter_scale;
    // the projections with the most work per token first along grid.y, so the long
    // CTAs start in the first waves (the table order is free: each CTA finds its
    // projection from the chunk ranges)
    int order[kMaxProj];
    for (int p = 0; p < n_proj; ++p) order[p] = p;
    std::stable_sort(order, order + n_proj, [&](int u, int v) {
        return (int64_t)projs[u].d_in + projs[u].slice.d_out > (int64_t)projs[v].d_in + projs[v].slice.d_out;
    });
    int chunks = 0;
    for (int i = 0; i < n_proj; ++i) {
        const lf_projection& q = projs[order[i]];
        ProjTab& t = A.p[i];
        t.x = reinterpret_cast<const __nv_bfloat16*>(q.x);
        t.y = reinterpret_cast<__nv_bfloat16*>(q.y);
        t.y_ld = q.y_ld;
        t.y_off = q.slice.y_offset;
        t.d_in = q.d_in;
        t.d_out = q.slice.d_out;
        t.chunk0 = chunks;
        t.max_rank = q.slice.max_rank;
        t.ranks = q.slice.ranks;
        t.off_A = q.slice.off_A;
        t.off_Bt = q.slice.off_Bt;
        t.A_pool = reinterpret_cast<const __nv_bfloat16*>(q.slice.A_pool);
        t.Bt_pool = reinterpret_cast<const __nv_bfloat16*>(q.slice.Bt_pool);
        t.pool_A = q.slice.pool_elems_A;
        t.pool_Bt = q.slice.pool_elems_Bt;
        chunks += (int)cdiv(q.slice.d_out, kBgmvCols);
    }
    A.n_chunks = chunks;
    LF_LAUNCH("bgmv", bgmv_proj_kernel, dim3((unsigned)T, (unsigned)chunks), kBgmvThreads, 0, s, A);
    return launch_status();
}

lf_status lf_route_tokens(int32_t T, const int32_t* ids, int32_t n_adapters, void* ws, size_t ws_bytes,
                          lf_stream_t stream) {
    if (T < 0 || n_adapters < 1 || n_adapters > 16384) return LF_ERR_INVALID_ARG;
    if (T == 0) return LF_OK;
    if (!ids || !ws) return LF_ERR_INVALID_ARG;
    ApplyWs w;
    if (ws_bytes < carve_apply(nullptr, T, n_adapters, 1, &w)) return LF_ERR_WORKSPACE;
    carve_apply(reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256)), T, n_adapters, 1,
                &w);
    RouteOut o{};
    o.counts = w.counts;
    o.segs = w.segs;
    o.perm = w.perm;
    o.items = w.items;
    o.tc_items = w.tc_items;
    o.run_start = w.runs;
    o.run_pos = w.runs + T;
    o.seg_out = nullptr;
    o.tag = w.tag;
    o.tok_list = w.tok_list;
    o.tc_enable = decode_regime(T, n_adapters) ? 0 : 1;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t rsmem = 2 * (size_t)n_adapters * sizeof(int32_t);
    LF_CUDA_TRY(cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem));
    LF_LAUNCH("route", route_kernel, 1, route_threads(T, n_adapters), rsmem, s, ids, T, n_adapters, o);
    return launch_status();
}

lf_status lf_lora_shrink_expand_slices_routed(int32_t T, int32_t d_in, const void* x, void* y, int64_t y_ld,
                                              const int32_t* ids, int32_t n_adapters, const lf_slice* slices,
                                              int32_t n_slices, float scale, const float* adapter_scale, void* ws,
                                              size_t ws_bytes, lf_stream_t stream) {
    return apply_impl(T, d_in, x, y, y_ld, ids, n_adapters, slices, n_slices, scale, adapter_scale, nullptr, ws,
                      ws_bytes, reinterpret_cast<cudaStream_t>(stream), nullptr, true);
}

lf_status lf_lora_shrink_expand_noalloc(int32_t T, int32_t d_in, int32_t d_out, const void* x, void* y,
                                        const int32_t* ids, int32_t n_adapters, const int32_t* ranks,
                                        const int64_t* off_A, const int64_t* off_Bt, const void* A_pool,
                                        const void* Bt_pool, int64_t pool_elems_A, int64_t pool_elems_Bt,
                                        float scale, int32_t* seg_out, lf_stream_t stream) {
    if (T < 0 || d_in < 1 || d_out < 1 || n_adapters < 1 || pool_elems_A < 0 || pool_elems_Bt < 0)
        return LF_ERR_INVALID_ARG;
    if (T > LF_NOALLOC_MAX_TOKENS || n_adapters > LF_NOALLOC_MAX_ADAPTERS) return LF_ERR_WORKSPACE;
    if (T == 0) return LF_OK;
    if (!x || !y || !ids || !ranks || !off_A || !off_Bt || !A_pool || !Bt_pool) return LF_ERR_INVALID_ARG;
    if ((d_in & 7) || (d_out & 7)) return LF_ERR_ALIGNMENT;
    if (!aligned16(x) || !aligned16(y) || !aligned16(A_pool) || !aligned16(Bt_pool)) return LF_ERR_ALIGNMENT;
    void* scratch = nullptr;
    lf_status st = noalloc_scratch(&scratch);
    if (st != LF_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // same carve as a caller workspace sized for the maxima (fits kNoallocScratchBytes)
    Carver c(scratch);
    RouteOut o{};
    o.counts = c.take<int32_t>(4);
    o.segs = c.take<Seg>((size_t)LF_NOALLOC_MAX_ADAPTERS);
    o.perm = c.take<int32_t>((size_t)LF_NOALLOC_MAX_TOKENS);
    o.items = c.take<GemvItem>((size_t)LF_NOALLOC_MAX_TOKENS / kGemvTok + LF_NOALLOC_MAX_ADAPTERS + 1);
    float* t_buf = c.take<float>((size_t)LF_NOALLOC_MAX_TOKENS * kMaxRank);
    o.seg_out = seg_out;
    o.tc_items = nullptr;
    o.tc_enable = 0;   // this entry point keeps every segment on the GEMV kernels
    if (c.off > kNoallocScratchBytes) return LF_ERR_WORKSPACE;
    const int64_t mseg = std::min<int64_t>(T, n_adapters);
    const size_t rsmem = 2 * (size_t)n_adapters * sizeof(int32_t);
    LF_CUDA_TRY(cudaFuncSetAttribute(route_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)rsmem));
    LF_LAUNCH("route", route_kernel, 1, route_threads(T, n_adapters), rsmem, s, ids, T, n_adapters, o);
    LF_CUDA_TRY(cudaGetLastError());
    ApplyArgs A{};
    A.T = T;
    A.d_in = d_in;
    A.n_adapters = n_adapters;
    A.n_slices = 1;
    A.y_ld = d_out;
    A.ldt = kMaxRank;
    A.x = reinterpret_cast<const __nv_bfloat16*>(x);
    A.y = reinterpret_cast<__nv_bfloat16*>(y);
    A.ids = ids;
    A.scale = scale;
    A.scales = nullptr;
    SliceTab& t = A.sl[0];
    t.d_out = d_out;
    t.t_col = 0;
    t.y_off = 0;
    t.ranks = ranks;
    t.off_A = off_A;
    t.off_Bt = off_Bt;
    t.A_pool = reinterpret_cast<const __nv_bfloat16*>(A_pool);
    t.Bt_pool = reinterpret_cast<const __nv_bfloat16*>(Bt_pool);
    t.pool_A = pool_elems_A;
    t.pool_Bt = pool_elems_Bt;
    A.counts = o.counts;
    A.segs = o.segs;
    A.perm = o.perm;
    A.items = o.items;
    A.t_buf = t_buf;
    set_chunks(A, kGemvCols);
    const unsigned max_items = (unsigned)(T / kGemvTok + mseg + 1);
    const dim3 grid2(max_items, (unsigned)A.n_chunks);
    if ((int64_t)T <= (int64_t)kGemvTok * n_adapters) {
        // decode regime (few tokens per adapter): shrink and expand in one launch
        LF_LAUNCH("fused_gemv", fused_gemv_kernel, grid2, kGemvThreads, 0, s, A);
    } else {
        LF_LAUNCH("shrink_gemv", shrink_kernel, gemv_grid(max_items), kGemvThreads, 0, s, A);
        LF_CUDA_TRY(cudaGetLastError());
        LF_LAUNCH("expand_gemv", expand_kernel, gemv_grid((int64_t)max_items * A.n_chunks), kGemvThreads, 0, s, A);
    }
    return launch_status();
}

size_t lf_jd_workspace_size(const lf_module* mods, int32_t n_mods, const int32_t* members, int32_t n_members,
                            const lf_jd_problem* probs, int32_t n_probs) {
    if (check_jd(mods, n_mods, members, n_members, probs, n_probs) != LF_OK) return 0;
    JdPlan P;
    plan_jd(mods, members, probs, n_probs, P);
    return jd_layout(n_mods, n_probs, P).total;
}

lf_status lf_jd_full(const lf_module* mods, int32_t n_mods, const int32_t* members, int32_t n_members,
                     const lf_jd_problem* probs, int32_t n_probs, const float* B_base, const float* A_base,
                     const double* weights, int32_t iters, float* U_base, float* Vt_base, float* sigma, void* ws,
                     size_t ws_bytes, lf_stream_t stream) {
    lf_status st = check_jd(mods, n_mods, members, n_members, probs, n_probs);
    if (st != LF_OK) return st;
    if (iters < 0) return LF_ERR_INVALID_ARG;
    if (n_probs == 0) return LF_OK;
    if (!B_base || !A_base || !U_base || !Vt_base || !ws) return LF_ERR_INVALID_ARG;
    if (!aligned16(B_base) || !aligned16(A_base) || !aligned16(U_base) || !aligned16(Vt_base))
        return LF_ERR_ALIGNMENT;
    JdPlan P;
    plan_jd(mods, members, probs, n_probs, P);
    const JdLayout L = jd_layout(n_mods, n_probs, P);
    if (ws_bytes < L.total) return LF_ERR_WORKSPACE;
    char* base = reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int32_t ng = (int32_t)P.members.size();

    Staging h;
    const int32_t onwork = (int32_t)P.orth.work.size();
    h.put(mods, n_mods);
    h.put(P.members.data(), P.members.size());
    h.put(P.probs.data(), P.probs.size());
    h.put(P.basis_user.data(), P.basis_user.size());
    h.put(P.basis_ws.data(), P.basis_ws.size());
    h.put(P.pwork.data(), P.pwork.size());
    h.put(P.pinfo.data(), P.pinfo.size());
    h.put(P.tiles.data(), P.tiles.size());
    h.put(P.tile0.data(), P.tile0.size());
    h.put(P.ntiles.data(), P.ntiles.size());
    h.put(P.orth.work.data(), P.orth.work.size());
    h.put(&onwork, 1);
    h.put(P.orth.info.data(), P.orth.info.size());
    LF_CUDA_TRY(cudaMemcpyAsync(base, h.buf.data(), h.off, cudaMemcpyHostToDevice, s));
    LF_CUDA_TRY(cudaMemsetAsync(base + L.pcounters, 0, (size_t)2 * ng * sizeof(int32_t), s));

    auto at = [&](size_t off) { return base + off; };
    const lf_module* d_mods = reinterpret_cast<const lf_module*>(at(L.mods));
    const JdMember* d_members = reinterpret_cast<const JdMember*>(at(L.members));
    const JdProbDev* d_probs = reinterpret_cast<const JdProbDev*>(at(L.probs));
    const lf_module* d_bu = reinterpret_cast<const lf_module*>(at(L.basis_user));
    const lf_module* d_bw = reinterpret_cast<const lf_module*>(at(L.basis_ws));
    float* wsU = reinterpret_cast<float*>(at(L.wsU));
    float* wsVt = reinterpret_cast<float*>(at(L.wsVt));
    float* RB = reinterpret_cast<float*>(at(L.RB));
    float* RA = reinterpret_cast<float*>(at(L.RA));
    const int npw = (int)P.pwork.size(), ntile = (int)P.tiles.size();

    JdProjArgs pa;
    pa.mods = d_mods;
    pa.members = d_members;
    pa.basis = d_bu;
    pa.B_base = B_base;
    pa.A_base = A_base;
    pa.U_base = U_base;
    pa.Vt_base = Vt_base;
    pa.work = reinterpret_cast<const TsqrWork*>(at(L.pwork));
    pa.info = reinterpret_cast<const TsqrInfo*>(at(L.pinfo));
    pa.counters = reinterpret_cast<int32_t*>(at(L.pcounters));
    pa.partial = reinterpret_cast<double*>(at(L.ppartial));
    pa.QP = reinterpret_cast<double*>(at(L.QP));

    JdCoreArgs ca;
    ca.members = d_members;
    ca.mods = d_mods;
    ca.basis = d_bu;
    ca.probs = d_probs;
    ca.QP = pa.QP;
    ca.weights = weights;
    ca.WZ = reinterpret_cast<float*>(at(L.WZ));
    ca.sigma = nullptr;
    ca.write_wz = 1;

    JdUpdArgs ua;
    ua.mods = d_mods;
    ua.members = d_members;
    ua.probs = d_probs;
    ua.basis_ws = d_bw;
    ua.B_base = B_base;
    ua.A_base = A_base;
    ua.WZ = ca.WZ;
    ua.tiles = reinterpret_cast<const JdTile*>(at(L.tiles));
    ua.U_ws = wsU;
    ua.Vt_ws = wsVt;
    ua.gram = reinterpret_cast<double*>(at(L.tgram));

    // orthogonalize (the state in the workspace -> the caller's U, V^T).  Pass 1: tile
    // Grams (update epilogue) -> jd_chol -> Householder TSQR for rejected matrices ->
    // Q = X R^-1, written to the caller's state, or back into the workspace for the
    // rejected ones, which pass 2 (Gram leaf + Cholesky on Q_1, Householder if
    // rejected again, Q = Q_1 R_2^-1) finishes.  Pass-2 kernels skip every other matrix.
    int32_t* oc = reinterpret_cast<int32_t*>(at(L.ocounters));
    int32_t* flags1 = oc;
    int32_t* gram2_cnt = oc + 2 * n_probs;
    int32_t* hh1_cnt = oc + 4 * n_probs;
    int32_t* hh2_cnt = oc + 6 * n_probs;
    int32_t* flags2 = oc + 8 * n_probs;
    double* R64_2 = reinterpret_cast<double*>(at(L.R64));   // pass 2's fp64 R (pass 1 inverts in jd_chol)
    const TsqrWork* owork = reinterpret_cast<const TsqrWork*>(at(L.owork));
    const int32_t* onw = reinterpret_cast<const int32_t*>(at(L.onwork));
    const TsqrInfo* oinfo = reinterpret_cast<const TsqrInfo*>(at(L.oinfo));

    JdGramSumArgs gsa;
    gsa.tile0 = reinterpret_cast<const int32_t*>(at(L.tile0));
    gsa.ntiles = reinterpret_cast<const int32_t*>(at(L.ntiles));
    gsa.gram = ua.gram;
    gsa.G = reinterpret_cast<double*>(at(L.gsum));
    double* Rinv = reinterpret_cast<double*>(at(L.Rinv));
    JdCholArgs cha;
    cha.basis = d_bw;
    cha.G = gsa.G;
    cha.Rinv = Rinv;
    cha.flags = flags1;
    cha.rs = P.orth.rs;
    JdRinvArgs ra1;   // pass 1: only the matrices the Cholesky rejected (Householder R)
    ra1.basis = d_bw;
    ra1.only = flags1;
    ra1.use32 = flags1;
    ra1.R64 = nullptr;   // pass 1 inverts only Householder R (use32 set for every matrix it takes)
    ra1.R_B = RB;
    ra1.R_A = RA;
    ra1.Rinv = Rinv;
    ra1.rs = P.orth.rs;
    JdRinvArgs ra2 = ra1;
    ra2.only = flags1;
    ra2.use32 = flags2;
    ra2.R64 = R64_2;

    auto householder = [&](const int32_t* only, int32_t* counters) -> cudaError_t {
        TsqrArgs<float> ta;
        ta.mods = d_bw;
        ta.mod_ids = nullptr;
        ta.B_base = wsU;
        ta.A_base = wsVt;
        ta.work = owork;
        ta.n_work = onw;
        ta.info = oinfo;
        ta.counters = counters;
        ta.partial = reinterpret_cast<float*>(at(L.opartial));
        ta.R_B = RB;
        ta.R_A = RA;
        ta.rs = P.orth.rs;
        ta.only = only;
        ta.tree = 0;
        return launch_tsqr_rt<float>(P.orth.RT, ta, onwork, s);
    };

    GramArgs ga;
    ga.mods = d_bw;
    ga.B_base = wsU;
    ga.A_base = wsVt;
    ga.work = owork;
    ga.n_work = onw;
    ga.info = oinfo;
    ga.counters = gram2_cnt;
    ga.partial = reinterpret_cast<double*>(at(L.opartial));
    ga.slot_doubles = (int64_t)(tsqr_slot_bytes(P.orth.RT) / sizeof(double));
    ga.flags = flags2;
    ga.R_B = RB;
    ga.R_A = RA;
    ga.rs = P.orth.rs;
    ga.only = flags1;
    ga.R64 = R64_2;

    JdQArgs q1;
    q1.src = d_bw;
    q1.src_U = wsU;
    q1.src_Vt = wsVt;
    q1.dst = d_bu;
    q1.dst_U = U_base;
    q1.dst_Vt = Vt_base;
    q1.alt = d_bw;
    q1.alt_U = wsU;
    q1.alt_Vt = wsVt;
    q1.route = flags1;
    q1.only = nullptr;
    q1.Rinv = Rinv;
    q1.rs = P.orth.rs;
    q1.tiles = ua.tiles;
    JdQArgs q2 = q1;
    q2.route = nullptr;
    q2.only = flags1;

    for (int32_t it = 0; it < iters; ++it) {
        LF_CUDA_TRY(cudaMemsetAsync(oc, 0, (size_t)10 * n_probs * sizeof(int32_t), s));
        LF_CUDA_TRY(launch_jd(P.RX, P.RY, 0, &pa, npw, s));
        LF_CUDA_TRY(launch_jd(P.RX, P.RY, 1, &ca, ng, s));
        LF_CUDA_TRY(launch_jd(P.RX, P.RY, 2, &ua, ntile, s));
        LF_CUDA_TRY(launch_jd_gram_sum(P.RY, gsa, 2 * n_probs, s));
        LF_CUDA_TRY(launch_jd_chol(P.RY, cha, 2 * n_probs, s));
        LF_CUDA_TRY(householder(flags1, hh1_cnt));
        LF_CUDA_TRY(launch_jd_rinv(P.RY, ra1, 2 * n_probs, s));
        LF_CUDA_TRY(launch_jd_qform(P.RY, q1, ntile, s));
        LF_CUDA_TRY(launch_gram_rt(P.orth.RT, ga, onwork, s));
        LF_CUDA_TRY(householder(flags2, hh2_cnt));
        LF_CUDA_TRY(launch_jd_rinv(P.RY, ra2, 2 * n_probs, s));
        LF_CUDA_TRY(launch_jd_qform(P.RY, q2, ntile, s));
    }
    if (sigma) {
        LF_CUDA_TRY(launch_jd(P.RX, P.RY, 0, &pa, npw, s));
        ca.sigma = sigma;
        ca.write_wz = 0;
        LF_CUDA_TRY(launch_jd(P.RX, P.RY, 1, &ca, ng, s));
    }
    return LF_OK;
}

size_t lf_pool_workspace_size(int32_t side, int32_t n_lora, const int32_t* ranks, const int64_t* offs, int32_t d) {
    int32_t R = 0;
    if (check_pool(side, n_lora, ranks, offs, d, &R) != LF_OK) return 0;
    return pool_layout(R, d, nullptr);
}

lf_status lf_pool_subspace(int32_t side, int32_t n_lora, const int32_t* ranks, const int64_t* offs, int32_t d,
                           const float* base, int32_t num, int32_t den, int32_t* k, double* sigma, float* basis,
                           float* coef, double* resid, void* ws, size_t ws_bytes, lf_stream_t stream) {
    int32_t R = 0;
    lf_status st = check_pool(side, n_lora, ranks, offs, d, &R);
    if (st != LF_OK) return st;
    if (num < 0 || den <= 0 || num > den) return LF_ERR_INVALID_ARG;
    if (!base || !k || !sigma || !basis || !coef || !resid || !ws) return LF_ERR_INVALID_ARG;
    size_t off[10];
    if (ws_bytes < pool_layout(R, d, off)) return LF_ERR_WORKSPACE;
    char* w = reinterpret_cast<char*>(align_up((int64_t)reinterpret_cast<uintptr_t>(ws), 256));
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // where each stack vector starts and its step: a row of A_i (r_i x d row-major, step 1)
    // or a column of B_i (d x r_i row-major, step r_i)
    std::vector<int64_t> row_off((size_t)R);
    std::vector<int32_t> row_step((size_t)R);
    for (int32_t i = 0, a = 0; i < n_lora; ++i)
        for (int32_t c = 0; c < ranks[i]; ++c, ++a) {
            row_off[a] = side == 0 ? offs[i] + (int64_t)c * d : offs[i] + c;
            row_step[a] = side == 0 ? 1 : ranks[i];
        }
    Staging h;
    h.put(row_off.data(), row_off.size());
    h.put(row_step.data(), row_step.size());
    LF_CUDA_TRY(cudaMemcpyAsync(w, h.buf.data(), h.off, cudaMemcpyHostToDevice, s));
    LF_CUDA_TRY(cudaMemsetAsync(w + off[7], 0, 32, s));
    PoolArgs a;
    a.R = R;
    a.d = d;
    a.num = num;
    a.den = den;
    a.base = base;
    a.row_off = reinterpret_cast<const int64_t*>(w + off[0]);
    a.row_step = reinterpret_cast<const int32_t*>(w + off[1]);
    a.Sv = reinterpret_cast<float*>(w + off[2]);
    a.X = reinterpret_cast<double*>(w + off[3]);
    a.V = reinterpret_cast<double*>(w + off[4]);
    a.lam = reinterpret_cast<double*>(w + off[5]);
    a.order = reinterpret_cast<int32_t*>(w + off[6]);
    a.bar = reinterpret_cast<uint32_t*>(w + off[7]);
    a.k_out = k;
    a.sigma = sigma;
    a.basis = basis;
    a.coef = coef;
    a.resid_part = reinterpret_cast<double*>(w + off[8]);
    a.resid = resid;
    const unsigned tiles = (unsigned)cdiv(R, kPoolTile);
    const unsigned xblocks = (unsigned)std::min<int64_t>(cdiv(d, kPoolThreads), 64);
    LF_LAUNCH("pool_gather", pool_gather_kernel, dim3(xblocks, (unsigned)R), kPoolThreads, 0, s, a);
    LF_LAUNCH("pool_gram", pool_gram_kernel, dim3(tiles, tiles), kPoolThreads, 0, s, a);
    // cooperative launch: every CTA resident (one per SM at most), so the grid barrier completes
    int dev = 0, sms = 0, per_sm = 0;
    LF_CUDA_TRY(cudaGetDevice(&dev));
    LF_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    LF_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pool_jacobi_kernel, kPoolThreads, 0));
    const int pairs = (R + 1) / 2;
    const int grid = std::max(1, std::min({sms * std::max(per_sm, 1), sms, (int)cdiv(pairs, kPoolThreads / 32)}));
    {
        PhaseScope ps_("pool_jacobi", s);
        void* args[] = {&a};
        LF_CUDA_TRY(cudaLaunchCooperativeKernel((const void*)pool_jacobi_kernel, dim3(grid), dim3(kPoolThreads), args,
                                                0, s));
    }
    LF_LAUNCH("pool_order", pool_order_kernel, 1, kPoolMaxRank, 0, s, a);
    LF_LAUNCH("pool_basis", pool_basis_kernel, dim3((unsigned)cdiv(d, kPoolThreads), tiles), kPoolThreads, 0, s, a);
    LF_LAUNCH("pool_coef", pool_coef_kernel, dim3(tiles, tiles), kPoolThreads, 0, s, a);
    LF_LAUNCH("pool_resid", pool_resid_kernel, 1, kPoolMaxRank, 0, s, a);
    return launch_status();
}

void lf_profile_enable(int on) { g_prof.on = on != 0; }

void lf_profile_reset(void) {
    for (auto& r : g_prof.pending) {
        g_prof.free_events.push_back(r.a);
        g_prof.free_events.push_back(r.b);
    }
    g_prof.pending.clear();
    std::fill(g_prof.ms.begin(), g_prof.ms.end(), 0.0);
    std::fill(g_prof.count.begin(), g_prof.count.end(), 0);
}

int32_t lf_profile_read(lf_phase_time* out, int32_t max_phases) {
    for (auto& r : g_prof.pending) {
        float t = 0.f;
        if (cudaEventSynchronize(r.b) == cudaSuccess && cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) {
            g_prof.ms[r.phase] += t;
            g_prof.count[r.phase] += 1;
        }
        g_prof.free_events.push_back(r.a);
        g_prof.free_events.push_back(r.b);
    }
    g_prof.pending.clear();
    const int32_t np = (int32_t)g_prof.names.size();
    for (int32_t i = 0; i < np && out && i < max_phases; ++i) {
        std::memset(out[i].name, 0, sizeof(out[i].name));
        std::strncpy(out[i].name, g_prof.names[i].c_str(), sizeof(out[i].name) - 1);
        out[i].total_ms = g_prof.ms[i];
        out[i].launches = g_prof.count[i];
    }
    return np;
}

int64_t lf_launch_count(void) { return g_prof.launches; }

const char* lf_status_string(lf_status s) {
    switch (s) {
        case LF_OK: return "ok";
        case LF_ERR_INVALID_ARG: return "invalid argument";
        case LF_ERR_SHAPE: return "bad shape (rank out of range or larger than a dimension)";
        case LF_ERR_BAD_INDEX: return "adapter id out of range";
        case LF_ERR_WORKSPACE: return "workspace or output pool too small";
        case LF_ERR_NUMERIC: return "non-finite value";
        case LF_ERR_TIMEOUT: return "bounded wait ran out";
        case LF_ERR_CUDA: return "CUDA runtime error";
        case LF_ERR_ALIGNMENT: return "misaligned pointer, offset or leading dimension";
    }
    return "unknown status";
}

lf_status lf_check_bounded_wait(int32_t polls, lf_stream_t stream) {
    if (polls < 0 || polls > (1 << 20)) return LF_ERR_INVALID_ARG;
    LF_LAUNCH("wait_selftest", wait_selftest_kernel, 1, 32, 0, reinterpret_cast<cudaStream_t>(stream), polls);
    return launch_status();
}

lf_status lf_get_device_status(lf_stream_t stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return LF_ERR_CUDA;
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error, sizeof(int)) != cudaSuccess) return LF_ERR_CUDA;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_error, &zero, sizeof(int)) != cudaSuccess) return LF_ERR_CUDA;
    return (lf_status)v;
}

}  // extern "C"
