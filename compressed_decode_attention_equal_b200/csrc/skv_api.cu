// C ABI of libskv (declared in include/skv.h): argument checks, the projection
// generator, workspace plans, TMA descriptors and kernel launches. No entry
// point allocates device memory; only skv_workspace_error synchronises.
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "skv_common.cuh"
#include "skv_internal.h"

using namespace skv;

namespace {

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// ---------------------------------------------------------------------------
// projection P (16 x 2d): SplitMix64 words -> Box-Muller (cosine branch) / 4
// ---------------------------------------------------------------------------
struct SplitMix64 {
    uint64_t state;
    uint64_t next() {
        state += 0x9e3779b97f4a7c15ULL;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
        z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
        return z ^ (z >> 31);
    }
};

void make_projection(uint64_t seed, int d, float *P) {
    const int cols = 2 * d;
    const double two_pi = 6.283185307179586476925286766559;
    const double scale = 1.0 / std::sqrt(static_cast<double>(kProjDim));
    SplitMix64 g{seed};
    for (int idx = 0; idx < kProjDim * cols; ++idx) {
        const uint64_t w1 = g.next();
        const uint64_t w2 = g.next();
        const double u1 = static_cast<double>((w1 >> 11) + 1) * 0x1p-53;   // (0, 1]
        const double u2 = static_cast<double>(w2 >> 11) * 0x1p-53;         // [0, 1)
        const double gauss = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
        P[idx] = static_cast<float>(gauss * scale);
    }
}

// bf16 bits of an fp32 value, rounded to nearest even (the inputs here are finite)
uint16_t bf16_rne_bits(float x) {
    uint32_t u;
    std::memcpy(&u, &x, 4);
    return static_cast<uint16_t>((u + 0x7fffu + ((u >> 16) & 1u)) >> 16);
}

// P16 = bf16(P) as the tensor-core projection's shared-memory image (see ProjFrag).
void make_projection_fragments(const float *P, int d, ProjFrag &out) {
    std::memset(&out, 0, sizeof out);
    const int cols = 2 * d, nchunk = cols / 32;
    uint16_t *img = reinterpret_cast<uint16_t *>(out.w);
    for (int c = 0; c < nchunk; ++c)
        for (int n = 0; n < kProjDim; ++n)
            for (int g = 0; g < 4; ++g)
                for (int e = 0; e < 8; ++e) {
                    const int k = 32 * c + 8 * g + e;   // feature
                    img[c * 512 + n * 32 + ((g ^ ((n >> 1) & 3)) * 8) + e] =
                        bf16_rne_bits(P[static_cast<size_t>(n) * cols + k]);
                }
}

// Small cache of the projection in both device forms -- transposed fp32 for the fixed recipe, the
// bf16 image for the tensor cores -- keyed by (seed, d), so that a call draws P only the first time.
struct ProjCache {
    std::mutex mu;
    struct Entry {
        uint64_t seed;
        int d;
        ProjT pt;
        ProjFrag frag;
    };
    std::vector<Entry> entries;
    void get(uint64_t seed, int d, ProjT *pt, ProjFrag *frag) {
        std::lock_guard<std::mutex> lock(mu);
        for (auto &e : entries)
            if (e.seed == seed && e.d == d) {
                if (pt) *pt = e.pt;
                if (frag) *frag = e.frag;
                return;
            }
        std::vector<float> P(static_cast<size_t>(kProjDim) * 2 * d);
        make_projection(seed, d, P.data());
        Entry e;
        e.seed = seed;
        e.d = d;
        std::memset(&e.pt, 0, sizeof e.pt);
        for (int i = 0; i < kProjDim; ++i)
            for (int j = 0; j < 2 * d; ++j) e.pt.pt[j * kProjDim + i] = P[static_cast<size_t>(i) * 2 * d + j];
        make_projection_fragments(P.data(), d, e.frag);
        if (entries.size() >= 16) entries.erase(entries.begin());
        entries.push_back(e);
        if (pt) *pt = e.pt;
        if (frag) *frag = e.frag;
    }
};
ProjCache g_proj;

// ---------------------------------------------------------------------------
// driver entry point for TMA descriptors (resolved once through the runtime)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Rows x d matrix of raw keys or values; boxes of 256 rows x 64 bytes, 64-byte swizzle.
bool make_row_map(CUtensorMap *map, const void *base, int dtype, int d, int64_t rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int elem = dtype == SKV_BF16 ? 2 : 4;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * elem};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(64 / elem), 256u};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype == SKV_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                          const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// ---------------------------------------------------------------------------
// coarsening plan
// ---------------------------------------------------------------------------
struct CoarsenPlan {
    int max_tiles = 0, max_emax = 0, Nmax = 0, max_blk = 0;
    int64_t rows = 0, mid = 0, bnd = 0, ent = 0;
    CoarsenLayout lay{};
};

skv_status plan_coarsen(int B, int Hkv, int d, const int32_t *T_host, const int32_t *N_host, int n_sink,
                        int n_recent, SeqTable *table, CoarsenPlan *plan) {
    if (B < 1 || B > SKV_MAX_SEQS || Hkv < 1 || !T_host || !N_host || n_sink < 0 || n_recent < 0)
        return SKV_ERR_INVALID_ARG;
    if (static_cast<int64_t>(B) * Hkv > 65535) return SKV_ERR_UNSUPPORTED;
    if (d != 64 && d != 128) return SKV_ERR_UNSUPPORTED;
    CoarsenPlan p;
    for (int b = 0; b < B; ++b) {
        const int T = T_host[b], N = N_host[b];
        if (T < 0 || T > SKV_MAX_TOKENS || N < 1 || N > (1 << 20)) return SKV_ERR_INVALID_ARG;
        SeqRow r{};
        r.T = T;
        r.N = N;
        r.s_eff = n_sink < T ? n_sink : T;
        r.w_eff = n_recent < T - r.s_eff ? n_recent : T - r.s_eff;
        r.M = T - r.s_eff - r.w_eff;
        r.tiles = (r.M + kTileOut - 1) / kTileOut;
        r.emax = r.s_eff + (r.M > 0 ? N : 0) + r.w_eff;
        r.row_off = p.rows;
        r.mid_off = p.mid;
        if (p.bnd > INT32_MAX - static_cast<int64_t>(Hkv) * (N + 1) ||
            p.ent > INT32_MAX - static_cast<int64_t>(Hkv) * r.emax)
            return SKV_ERR_UNSUPPORTED;
        r.bnd_off = static_cast<int32_t>(p.bnd);
        r.ent_off = static_cast<int32_t>(p.ent);
        p.rows += static_cast<int64_t>(Hkv) * T;
        p.mid += static_cast<int64_t>(Hkv) * r.M;
        p.bnd += static_cast<int64_t>(Hkv) * (N + 1);
        p.ent += static_cast<int64_t>(Hkv) * r.emax;
        if (r.tiles > p.max_tiles) p.max_tiles = r.tiles;
        const int nblk = (T + kMeanBlock - 1) / kMeanBlock;
        if (nblk > p.max_blk) p.max_blk = nblk;
        if (r.emax > p.max_emax) p.max_emax = r.emax;
        if (N > p.Nmax) p.Nmax = N;
        if (table) table->rows[b] = r;
    }
    if (p.rows > INT32_MAX) return SKV_ERR_UNSUPPORTED;   // TMA row coordinates are int32
    const int64_t units = static_cast<int64_t>(B) * Hkv;
    size_t off = kWsHeader;
    p.lay.seq = off;
    off += align256(sizeof(SeqRow) * B);
    p.lay.tile_total = off;
    off += align256(static_cast<size_t>(units) * p.max_tiles * 8);
    p.lay.unit_total = off;
    off += align256(static_cast<size_t>(units) * 8);
    p.lay.local_scan = off;
    off += align256(static_cast<size_t>(p.mid) * 8);
    p.lay.bounds = off;
    off += align256(static_cast<size_t>(p.bnd) * 4);
    p.lay.ents = off;
    off += align256(static_cast<size_t>(p.ent) * 8);
    p.lay.key_blk = off;   // the centring option's block sums and unit means
    off += align256(static_cast<size_t>(units) * p.max_blk * d * 4);
    p.lay.key_mu = off;
    off += align256(static_cast<size_t>(units) * d * 4);
    p.lay.total = off;
    *plan = p;
    return SKV_OK;
}

}  // namespace

namespace skv {

// ---------------------------------------------------------------------------
// decode plan (shared by skv_decode_attn_ex and skv_decode_attn_noalloc)
// ---------------------------------------------------------------------------
skv_status plan_decode(int dtype, int B, int R, int Hq, int Hkv, int d, int max_pages, DecodePlan *plan) {
    if (B < 1 || R < 1 || Hq < 1 || Hkv < 1 || max_pages < 1) return SKV_ERR_INVALID_ARG;
    if (Hq % Hkv != 0 || (d != 64 && d != 128) || (dtype != SKV_BF16 && dtype != SKV_F32))
        return SKV_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(max_pages) * kPageNodes > INT32_MAX / 2) return SKV_ERR_UNSUPPORTED;
    DecodePlan p{};
    const int64_t rows = static_cast<int64_t>(R) * (Hq / Hkv);
    if (rows > (1 << 20)) return SKV_ERR_UNSUPPORTED;
    p.rows = static_cast<int>(rows);
    p.row_passes = (p.rows + kRowsPerPass - 1) / kRowsPerPass;
    p.pass_rows = p.rows > kRowsPerPass ? kRowsPerPass : ((p.rows + 7) / 8) * 8;
    const int64_t nv = static_cast<int64_t>(B) * Hkv * p.row_passes;
    if (nv > kMaxVUnits) return SKV_ERR_UNSUPPORTED;
    // the page prefix is an int32 sum over all units
    if (static_cast<int64_t>(B) * Hkv * max_pages * p.row_passes > INT32_MAX / 2) return SKV_ERR_UNSUPPORTED;
    p.n_vunits = static_cast<int>(nv);
    p.lay = decode_layout(dtype, d, p, kMaxDecodeCtas);
    *plan = p;
    return SKV_OK;
}

DecodeLayout decode_layout(int dtype, int d, const DecodePlan &p, int ncta) {
    const auto al = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    DecodeLayout lay{};
    size_t off = kWsHeader;
    lay.counters = off;
    off += al(static_cast<size_t>(p.n_vunits) * 4);
    lay.part_v = off;
    if (dtype == SKV_BF16) off += al(static_cast<size_t>(ncta) * 2 * p.pass_rows * d * 4);
    lay.part_l = off;
    if (dtype == SKV_BF16) off += al(static_cast<size_t>(ncta) * 2 * p.pass_rows * 4);
    lay.total = off;
    return lay;
}

skv_status decode_args(const void *q, int dtype, int B, int R, int Hq, int Hkv, int d, const skv_node_pool *pool,
                       const int32_t *page_table, int max_pages, const int32_t *lens, void *out, float *lse,
                       int closure, DecodePlan *plan, DecodeArgs *args) {
    skv_status st = plan_decode(dtype, B, R, Hq, Hkv, d, max_pages, plan);
    if (st != SKV_OK) return st;
    if (!q || !out || !lse || !pool || !page_table || !lens) return SKV_ERR_INVALID_ARG;
    if (!pool->pages || pool->num_pages < 0) return SKV_ERR_INVALID_ARG;
    const auto al = [](const void *ptr, uintptr_t m) { return (reinterpret_cast<uintptr_t>(ptr) & (m - 1)) == 0; };
    if (!al(pool->pages, 16) || !al(q, 16) || !al(out, 16) || !al(lse, 4)) return SKV_ERR_INVALID_ARG;
    DecodeArgs a{};
    a.q = q;
    a.pages = static_cast<const uint8_t *>(pool->pages);
    a.num_pages = pool->num_pages;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.lens = lens;
    a.out = out;
    a.lse = lse;
    a.B = B;
    a.R = R;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.G = Hq / Hkv;
    a.d = d;
    a.dtype = dtype;
    a.rows = plan->rows;
    a.row_passes = plan->row_passes;
    a.pass_rows = plan->pass_rows;
    a.n_vunits = plan->n_vunits;
    a.closure = closure;
    *args = a;
    return SKV_OK;
}

}  // namespace skv

namespace skv {

// One thread arms an mbarrier for one arrival that nothing makes (no copy targets it), polls it at
// most `polls` times with the same try_wait the pipelines use, and raises FLAG_TIMEOUT when the
// polls run out -- the path every bounded wait of the library's kernels takes when it gives up.
__global__ void k_wait_selftest(uint32_t *flags, uint32_t polls) {
    __shared__ uint64_t bar;
    if (threadIdx.x != 0) return;
    mbar_init(&bar, 1);
    fence_mbar_init();
    bool done = false;
    for (uint32_t i = 0; i < polls && !done; ++i) done = mbar_try_wait(&bar, 0);
    if (!done) raise_flag(flags, FLAG_TIMEOUT);
    mbar_inval(&bar);
}

}  // namespace skv

// ===========================================================================
extern "C" {

const char *skv_status_string(int status) {
    switch (status) {
        case SKV_OK: return "SKV_OK";
        case SKV_ERR_INVALID_ARG: return "SKV_ERR_INVALID_ARG: invalid argument";
        case SKV_ERR_UNSUPPORTED: return "SKV_ERR_UNSUPPORTED: configuration not supported";
        case SKV_ERR_CUDA: return "SKV_ERR_CUDA: CUDA runtime error";
        case SKV_ERR_OVERFLOW: return "SKV_ERR_OVERFLOW: variation step above 2^20 (or not finite)";
        case SKV_ERR_TIMEOUT: return "SKV_ERR_TIMEOUT: a bounded device wait gave up (work abandoned)";
        case SKV_ERR_WORKSPACE: return "SKV_ERR_WORKSPACE: workspace too small or misaligned";
        case SKV_ERR_DEVICE: return "SKV_ERR_DEVICE: device detected a bad page id, lens entry or stuck wait";
        default: return "unknown skv status";
    }
}

int skv_abi_version(void) { return 203; }

size_t skv_page_bytes(skv_dtype dtype, int d) { return skv_page_bytes_ex(dtype, d, SKV_CLOSURE_SCALAR); }

size_t skv_page_bytes_ex(skv_dtype dtype, int d, skv_closure closure) {
    if ((dtype != SKV_BF16 && dtype != SKV_F32) || (d != 64 && d != 128)) return 0;
    if (closure != SKV_CLOSURE_SCALAR && closure != SKV_CLOSURE_DIAGONAL) return 0;
    const size_t elem = dtype == SKV_BF16 ? 2 : 4;
    const size_t vec = static_cast<size_t>(kPageNodes) * d * elem;
    return (closure == SKV_CLOSURE_DIAGONAL ? 3 : 2) * vec + kPageNodes * 8;
}

skv_status skv_projection_matrix(uint64_t proj_seed, int d, float *P_host) {
    if (!P_host || (d != 64 && d != 128)) return SKV_ERR_INVALID_ARG;
    make_projection(proj_seed, d, P_host);
    return SKV_OK;
}

size_t skv_coarsen_workspace_bytes(int B, int Hkv, int d, const int32_t *T_host, const int32_t *N_host, int n_sink,
                                   int n_recent) {
    CoarsenPlan p;
    if (plan_coarsen(B, Hkv, d, T_host, N_host, n_sink, n_recent, nullptr, &p) != SKV_OK) return 0;
    return p.lay.total;
}

// The coarsening pipeline; with `streaming` set, it also builds the streaming state (same stream).
static skv_status coarsen_impl(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                               const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                               uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                               int32_t *lens, int32_t *boundaries, int64_t *cumvar, void *workspace, size_t ws_bytes,
                               int representative, int closure, int center, int projection, StreamArgs *streaming,
                               void *stream);

skv_status skv_coarsen_ex(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                          const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host, uint64_t proj_seed,
                          const skv_node_pool *pool, const int32_t *page_table, int max_pages, int32_t *lens,
                          int32_t *boundaries, int64_t *cumvar, void *workspace, size_t ws_bytes,
                          const skv_coarsen_options *options, void *stream) {
    int representative = SKV_REP_MEAN, closure = SKV_CLOSURE_SCALAR, center = 0, projection = SKV_PROJECTION_FIXED_FP32;
    if (options) {
        if (options->representative != SKV_REP_MEAN && options->representative != SKV_REP_VARIATION_WEIGHTED)
            return SKV_ERR_INVALID_ARG;
        if (options->closure != SKV_CLOSURE_SCALAR && options->closure != SKV_CLOSURE_DIAGONAL)
            return SKV_ERR_INVALID_ARG;
        if (options->center_keys != 0 && options->center_keys != 1) return SKV_ERR_INVALID_ARG;
        if (options->projection != SKV_PROJECTION_FIXED_FP32 && options->projection != SKV_PROJECTION_TENSOR_BF16)
            return SKV_ERR_INVALID_ARG;
        for (int i = 0; i < 4; ++i)
            if (options->reserved[i] != 0) return SKV_ERR_INVALID_ARG;
        representative = options->representative;
        closure = options->closure;
        center = options->center_keys;
        projection = options->projection;
        if (projection == SKV_PROJECTION_TENSOR_BF16 && dtype != SKV_BF16) return SKV_ERR_UNSUPPORTED;
    }
    return coarsen_impl(k, v, dtype, B, Hkv, d, T_host, n_sink, n_recent, N_host, proj_seed, pool, page_table,
                        max_pages, lens, boundaries, cumvar, workspace, ws_bytes, representative, closure, center,
                        projection, nullptr, stream);
}

static skv_status coarsen_impl(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                               const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                               uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                               int32_t *lens, int32_t *boundaries, int64_t *cumvar, void *workspace, size_t ws_bytes,
                               int representative, int closure, int center, int projection, StreamArgs *streaming,
                               void *stream) {
    if (dtype != SKV_BF16 && dtype != SKV_F32) return SKV_ERR_UNSUPPORTED;
    static SeqTable table;   // host staging; guarded by the mutex below
    static std::mutex table_mu;
    std::lock_guard<std::mutex> lock(table_mu);
    CoarsenPlan plan;
    skv_status st = plan_coarsen(B, Hkv, d, T_host, N_host, n_sink, n_recent, &table, &plan);
    if (st != SKV_OK) return st;
    if (!pool || !page_table || !lens || max_pages < 1) return SKV_ERR_INVALID_ARG;
    if (!pool->pages || pool->num_pages < 0 || !aligned(pool->pages, 16)) return SKV_ERR_INVALID_ARG;
    if (plan.rows > 0 && (!k || !v || !aligned(k, 16) || !aligned(v, 16))) return SKV_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < plan.lay.total) return SKV_ERR_WORKSPACE;
    for (int b = 0; b < B; ++b)
        if (table.rows[b].emax > static_cast<int64_t>(max_pages) * kPageNodes) return SKV_ERR_INVALID_ARG;

    ProjT proj;
    static ProjFrag frag;   // host staging (guarded by table_mu)
    if (projection == SKV_PROJECTION_TENSOR_BF16) {
        std::memset(&proj, 0, sizeof proj);
        g_proj.get(proj_seed, d, nullptr, &frag);
    } else {
        g_proj.get(proj_seed, d, &proj, nullptr);
        std::memset(&frag, 0, sizeof frag);
    }
    CUtensorMap map_k, map_v;
    std::memset(&map_k, 0, sizeof map_k);
    std::memset(&map_v, 0, sizeof map_v);
    if (plan.max_tiles > 0) {
        if (!make_row_map(&map_k, k, dtype, d, plan.rows) || !make_row_map(&map_v, v, dtype, d, plan.rows))
            return SKV_ERR_CUDA;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    CoarsenArgs a{};
    a.k = k;
    a.v = v;
    a.B = B;
    a.Hkv = Hkv;
    a.d = d;
    a.dtype = dtype;
    a.max_tiles = plan.max_tiles;
    a.max_emax = plan.max_emax;
    a.Nmax = plan.Nmax;
    a.seq = reinterpret_cast<const SeqRow *>(ws + plan.lay.seq);
    a.tile_total = reinterpret_cast<int64_t *>(ws + plan.lay.tile_total);
    a.unit_total = reinterpret_cast<int64_t *>(ws + plan.lay.unit_total);
    a.local_scan = reinterpret_cast<int64_t *>(ws + plan.lay.local_scan);
    a.bounds = reinterpret_cast<int32_t *>(ws + plan.lay.bounds);
    a.ents = reinterpret_cast<int2 *>(ws + plan.lay.ents);
    a.flags = reinterpret_cast<uint32_t *>(ws);
    a.pages = static_cast<uint8_t *>(pool->pages);
    a.num_pages = pool->num_pages;
    a.page_table = page_table;
    a.max_pages = max_pages;
    a.lens = lens;
    a.user_bounds = boundaries;
    a.cumvar = cumvar;
    a.representative = representative;
    a.closure = closure;
    a.center = center;
    a.projection = projection;
    a.max_blk = plan.max_blk;
    a.key_blk = reinterpret_cast<float *>(ws + plan.lay.key_blk);
    a.key_mu = reinterpret_cast<float *>(ws + plan.lay.key_mu);
    cudaError_t e = launch_coarsen(a, table, proj, frag, map_k, map_v, static_cast<cudaStream_t>(stream));
    if (e == cudaSuccess && streaming) {
        streaming->flags = a.flags;
        streaming->pages = a.pages;
        streaming->num_pages = a.num_pages;
        streaming->page_table = page_table;
        streaming->max_pages = max_pages;
        streaming->lens = lens;
        e = launch_stream_init(a, *streaming, proj, static_cast<cudaStream_t>(stream));
    }
    return e == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// streaming coarsening
// ---------------------------------------------------------------------------
static bool stream_geometry(int B, int Hkv, int d, const int32_t *N_host, int n_sink, int n_recent, StreamArgs *s) {
    if (B < 1 || Hkv < 1 || B > SKV_MAX_SEQS || !N_host || n_sink < 0 || n_recent < 1 || (d != 64 && d != 128))
        return false;
    int Nmax = 0;
    for (int b = 0; b < B; ++b) {
        if (N_host[b] < 1 || N_host[b] > (1 << 20)) return false;
        Nmax = N_host[b] > Nmax ? N_host[b] : Nmax;
    }
    const int64_t ecap = static_cast<int64_t>(n_sink) + Nmax + 1 + n_recent;
    if (ecap > 8192) return false;   // the append kernel stages the node order in shared memory
    stream_layout(d, static_cast<int>(ecap), n_recent, s);
    return true;
}

size_t skv_stream_state_bytes(int B, int Hkv, int d, const int32_t *N_host, int n_sink, int n_recent) {
    StreamArgs s{};
    if (!stream_geometry(B, Hkv, d, N_host, n_sink, n_recent, &s)) return 0;
    return static_cast<size_t>(kStreamProjBytes + s.unit_bytes * B * Hkv);
}

skv_status skv_stream_init(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                           const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                           uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                           int32_t *lens, void *workspace, size_t ws_bytes, void *state, size_t state_bytes,
                           void *stream) {
    if (dtype != SKV_BF16 && dtype != SKV_F32) return SKV_ERR_UNSUPPORTED;
    StreamArgs s{};
    if (!T_host || !stream_geometry(B, Hkv, d, N_host, n_sink, n_recent, &s)) return SKV_ERR_INVALID_ARG;
    for (int b = 0; b < B; ++b)
        if (T_host[b] <= n_sink + n_recent) return SKV_ERR_UNSUPPORTED;   // streaming needs a middle
    if (!state || !aligned(state, 256) ||
        state_bytes < static_cast<size_t>(kStreamProjBytes + s.unit_bytes * B * Hkv))
        return SKV_ERR_WORKSPACE;
    if (static_cast<int64_t>(max_pages) * kPageNodes < s.Ecap) return SKV_ERR_INVALID_ARG;
    s.B = B;
    s.Hkv = Hkv;
    s.d = d;
    s.dtype = dtype;
    s.pt = static_cast<float *>(state);
    s.state = static_cast<uint8_t *>(state) + kStreamProjBytes;
    return coarsen_impl(k, v, dtype, B, Hkv, d, T_host, n_sink, n_recent, N_host, proj_seed, pool, page_table,
                        max_pages, lens, nullptr, nullptr, workspace, ws_bytes, SKV_REP_MEAN, SKV_CLOSURE_SCALAR, 0,
                        SKV_PROJECTION_FIXED_FP32, &s, stream);
}

skv_status skv_stream_append(const void *k_new, const void *v_new, skv_dtype dtype, int B, int Hkv, int d,
                             const int32_t *N_host, int n_sink, int n_recent, const skv_node_pool *pool,
                             const int32_t *page_table, int max_pages, int32_t *lens, void *state,
                             size_t state_bytes, void *workspace, size_t ws_bytes, void *stream) {
    if (dtype != SKV_BF16 && dtype != SKV_F32) return SKV_ERR_UNSUPPORTED;
    StreamArgs s{};
    if (!stream_geometry(B, Hkv, d, N_host, n_sink, n_recent, &s)) return SKV_ERR_INVALID_ARG;
    if (!k_new || !v_new || !pool || !pool->pages || pool->num_pages < 0 || !page_table || !lens)
        return SKV_ERR_INVALID_ARG;
    if (!aligned(pool->pages, 16) || static_cast<int64_t>(max_pages) * kPageNodes < s.Ecap) return SKV_ERR_INVALID_ARG;
    if (!state || !aligned(state, 256) ||
        state_bytes < static_cast<size_t>(kStreamProjBytes + s.unit_bytes * B * Hkv))
        return SKV_ERR_WORKSPACE;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return SKV_ERR_WORKSPACE;
    s.k_new = k_new;
    s.v_new = v_new;
    s.B = B;
    s.Hkv = Hkv;
    s.d = d;
    s.dtype = dtype;
    s.pages = static_cast<uint8_t *>(pool->pages);
    s.num_pages = pool->num_pages;
    s.page_table = page_table;
    s.max_pages = max_pages;
    s.lens = lens;
    s.pt = static_cast<float *>(state);
    s.state = static_cast<uint8_t *>(state) + kStreamProjBytes;
    s.flags = static_cast<uint32_t *>(workspace);
    return launch_stream_append(s, static_cast<cudaStream_t>(stream)) == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}

skv_status skv_coarsen(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d, const int32_t *T_host,
                       int n_sink, int n_recent, const int32_t *N_host, uint64_t proj_seed,
                       const skv_node_pool *pool, const int32_t *page_table, int max_pages, int32_t *lens,
                       int32_t *boundaries, int64_t *cumvar, void *workspace, size_t ws_bytes, void *stream) {
    return skv_coarsen_ex(k, v, dtype, B, Hkv, d, T_host, n_sink, n_recent, N_host, proj_seed, pool, page_table,
                          max_pages, lens, boundaries, cumvar, workspace, ws_bytes, nullptr, stream);
}

size_t skv_decode_workspace_bytes(int B, int R, int Hq, int Hkv, int d, int max_pages) {
    DecodePlan p;
    if (plan_decode(SKV_BF16, B, R, Hq, Hkv, d, max_pages, &p) != SKV_OK) return 0;
    return p.lay.total;
}

skv_status skv_decode_attn_ex(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                              const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                              const int32_t *lens, void *out, float *lse, void *workspace, size_t ws_bytes,
                              const skv_decode_options *options, void *stream) {
    int closure = SKV_CLOSURE_SCALAR;
    if (options) {
        if (options->closure != SKV_CLOSURE_SCALAR && options->closure != SKV_CLOSURE_DIAGONAL)
            return SKV_ERR_INVALID_ARG;
        for (int i = 0; i < 7; ++i)
            if (options->reserved[i] != 0) return SKV_ERR_INVALID_ARG;
        closure = options->closure;
    }
    DecodePlan plan;
    DecodeArgs a;
    skv_status st = decode_args(q, dtype, B, R, Hq, Hkv, d, pool, page_table, max_pages, lens, out, lse, closure,
                                &plan, &a);
    if (st != SKV_OK) return st;
    if (!workspace || !aligned(workspace, 256) || ws_bytes < plan.lay.total) return SKV_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    a.part_v = reinterpret_cast<float *>(ws + plan.lay.part_v);
    a.part_l = reinterpret_cast<float *>(ws + plan.lay.part_l);
    a.counters = reinterpret_cast<int32_t *>(ws + plan.lay.counters);
    a.flags = reinterpret_cast<uint32_t *>(ws);
    const cudaError_t e = launch_decode(a, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}

skv_status skv_decode_attn(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                           const skv_node_pool *pool, const int32_t *page_table, int max_pages, const int32_t *lens,
                           void *out, float *lse, void *workspace, size_t ws_bytes, void *stream) {
    return skv_decode_attn_ex(q, dtype, B, R, Hq, Hkv, d, pool, page_table, max_pages, lens, out, lse, workspace,
                              ws_bytes, nullptr, stream);
}

skv_status skv_wait_selftest(void *workspace, size_t ws_bytes, uint32_t polls, void *stream) {
    if (!workspace || !aligned(workspace, 256) || ws_bytes < kWsHeader) return SKV_ERR_WORKSPACE;
    if (polls > kWaitLimit) return SKV_ERR_INVALID_ARG;
    k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<uint32_t *>(workspace), polls);
    return cudaGetLastError() == cudaSuccess ? SKV_OK : SKV_ERR_CUDA;
}

skv_status skv_workspace_error(const void *workspace, void *stream, uint32_t *flags_host) {
    if (!workspace) return SKV_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // read and clear on the caller's stream, after everything already enqueued there
    uint32_t f = 0;
    if (cudaMemcpyAsync(&f, workspace, sizeof f, cudaMemcpyDeviceToHost, s) != cudaSuccess) return SKV_ERR_CUDA;
    if (cudaMemsetAsync(const_cast<void *>(workspace), 0, sizeof f, s) != cudaSuccess) return SKV_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return SKV_ERR_CUDA;
    if (flags_host) *flags_host = f;
    if (f & FLAG_OVERFLOW) return SKV_ERR_OVERFLOW;
    if (f & FLAG_TIMEOUT) return SKV_ERR_TIMEOUT;
    if (f) return SKV_ERR_DEVICE;
    return SKV_OK;
}

}  // extern "C"
