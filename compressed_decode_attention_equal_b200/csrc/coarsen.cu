// Equal-variation coarsening of a KV cache into macro-nodes.
//
// "Equal-Variation KV Cache" (synthcore idea 664), Mathematical statement and
// Implementation notes: the middle span of each (sequence, KV head) unit is cut
// at the first tokens whose cumulative variation of z_t = P [k_t; v_t] reaches
// j c_T / N. "SPICY-KV" demo page, Claims 2-3 and section 2: each segment keeps
// its mass m, mean key, mean value and per-dimension key variance, stored as
// alpha = ln m and beta = sigma^2 / (2 d).
//
// Pipeline (stream-ordered launches, all integer stages exact):
//   k_setup          copy the host-built per-sequence plan into the workspace
//   k_project_scan   TMA-staged tiles of 511 middle tokens (+1 halo): z via the
//                    fixed fp32 fma recipe, D_t = rne(d_t 2^20), tile-local
//                    inclusive int64 scan and tile totals
//   k_boundaries     c_T and each tile's start from the tile totals; every token
//                    writes the thresholds it crosses:
//                    b_j = t for N c_{t-1} < j c_T <= N c_t (128-bit products)
//   k_plan_entries   drop empty segments, lay out entries (sinks, segments,
//                    recents) and write lens
//   k_segment_reduce one warp per entry: two-pass mean / variance, node write
//                    into the paged pool (swizzled 16-byte chunks)
#include "skv_common.cuh"
#include "skv_internal.h"

namespace skv {

// ---------------------------------------------------------------------------
// k_setup: per-sequence plan -> workspace; clear the error flags
// ---------------------------------------------------------------------------
__global__ void k_setup(const __grid_constant__ SeqTable table, SeqRow *dst, int B, uint32_t *flags) {
    for (int b = threadIdx.x; b < B; b += blockDim.x) dst[b] = table.rows[b];
    if (threadIdx.x == 0) *flags = 0u;
}

// ---------------------------------------------------------------------------
// centring option ("SPICY-KV" Independent Claim 1(b), common-mode mean removal): the unit's
// mean key in one fixed fp32 order -- per dimension, blocks of kMeanBlock consecutive tokens
// summed in token order from 0, block sums added in block order from 0, total divided by T
// -- so that the centred keys fl32(k - mu) are the same bits wherever they are formed.
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ float to_f32(T x);
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <>
__device__ __forceinline__ float to_f32<float>(float x) { return x; }

// one thread per key dimension, one CTA per (block of kMeanBlock tokens, unit)
template <int D, typename T>
__global__ void __launch_bounds__(D) k_key_block_sums(const CoarsenArgs a) {
    const int u = blockIdx.y, blk = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    const int t0 = blk * kMeanBlock;
    if (t0 >= sr.T) return;
    const int n = min(kMeanBlock, sr.T - t0);
    const T *kp = static_cast<const T *>(a.k) + (sr.row_off + static_cast<int64_t>(h) * sr.T + t0) * D + threadIdx.x;
    float s = 0.0f;
#pragma unroll 16
    for (int t = 0; t < n; ++t) s = __fadd_rn(s, to_f32<T>(kp[static_cast<int64_t>(t) * D]));
    a.key_blk[(static_cast<int64_t>(u) * a.max_blk + blk) * D + threadIdx.x] = s;
}

template <int D>
__global__ void __launch_bounds__(D) k_key_mean(const CoarsenArgs a) {
    const int u = blockIdx.x;
    const SeqRow sr = a.seq[u / a.Hkv];
    const int nblk = (sr.T + kMeanBlock - 1) / kMeanBlock;
    const float *bs = a.key_blk + static_cast<int64_t>(u) * a.max_blk * D + threadIdx.x;
    float tot = 0.0f;
    // (unrolled so that the loads run ahead of the additions, which keep the fixed block order)
#pragma unroll 16
    for (int c = 0; c < nblk; ++c) tot = __fadd_rn(tot, bs[static_cast<int64_t>(c) * D]);
    a.key_mu[static_cast<int64_t>(u) * D + threadIdx.x] = sr.T > 0 ? __fdiv_rn(tot, static_cast<float>(sr.T)) : 0.0f;
}

// ---------------------------------------------------------------------------
// k_project_scan
// ---------------------------------------------------------------------------

constexpr int kK1Threads = 128;
constexpr int kK1Tok = kTileRows / kK1Threads;   // token rows per thread (4)
constexpr int kK1Stages = 2;
constexpr int kK1ColBytes = 64;                  // column chunk of every row per stage (64-byte swizzle)
constexpr int kK1BoxRows = 256;                  // TMA box height (two boxes per stage)
constexpr int kK1StageBytes = kTileRows * kK1ColBytes;
// floats per row of the z buffer: odd, so that 32 consecutive rows at one column hit 32 banks
constexpr int kZStride = 17;
// the steps of a tile's outputs, staged after the z buffer for the scan's thread mapping
constexpr int kZBytes = kTileRows * kZStride * 4;
static_assert(kTileRows % kK1BoxRows == 0 && kZBytes % 8 == 0 &&
                  kZBytes + kTileRows * 8 <= kK1Stages * kK1StageBytes, "tile");

template <int D>
constexpr size_t k1_smem_bytes() {
    // stages + P^T with one zero row of padding (the pipelined loop reads row j + 1) + barriers
    return 1024 /*alignment slack*/ + kK1Stages * kK1StageBytes + (2 * D + 1) * kProjDim * sizeof(float) + 64 + 64 +
           D * sizeof(float);
}

// x duplicated into both halves of an f32x2 operand, built with two different ALU operations (the
// pair then needs no register move): the bf16 in the low / high half of a 32-bit word as fp32.
__device__ __forceinline__ uint64_t dup_bf16lo(uint32_t w) {
    return f2pack(__uint_as_float(w << 16), __uint_as_float(__byte_perm(w, 0u, 0x1044)));
}
__device__ __forceinline__ uint64_t dup_bf16hi(uint32_t w) {
    return f2pack(__uint_as_float(w & 0xffff0000u), __uint_as_float(__byte_perm(w, 0u, 0x3244)));
}

template <typename T>
__device__ __forceinline__ uint64_t dup_elem(const uint4 &w, int e);

template <>
__device__ __forceinline__ uint64_t dup_elem<__nv_bfloat16>(const uint4 &w, int e) {
    const uint32_t x = (e >> 1) == 0 ? w.x : (e >> 1) == 1 ? w.y : (e >> 1) == 2 ? w.z : w.w;
    return (e & 1) ? dup_bf16hi(x) : dup_bf16lo(x);
}

template <>
__device__ __forceinline__ uint64_t dup_elem<float>(const uint4 &w, int e) {
    const uint32_t x = e == 0 ? w.x : e == 1 ? w.y : e == 2 ? w.z : w.w;
    return f2pack(__uint_as_float(x), __uint_as_float(x));
}

// 16-byte sub-chunk cc (0..3) of row r in a stage written by TMA with the 64-byte swizzle
// (sub-chunk index XOR bits [1:2] of the row: bank-conflict free for 8 consecutive rows)
__device__ __forceinline__ int k1_sub(int r, int cc) { return r * 4 + (cc ^ ((r >> 1) & 3)); }

// Quantised steps and the tile-local inclusive scan of one projection tile (z of its 512 rows in
// shared memory, row 0 the halo): D_t = rne(||z_t - z_{t-1}|| 2^20) by the fixed recipe for the
// tile's middle tokens, their running sums into local_scan, the tile total into tile_total.
__device__ __forceinline__ void scan_tile(const CoarsenArgs &a, const SeqRow &sr, int u, int h, int tile,
                                          const float *zb, long long *warp_sum) {
    const int tid = threadIdx.x;
    // steps of outputs l = tid + 1 + 128 q (rows l - 1 and l of the tile; row 0 is the halo):
    // consecutive threads read consecutive z rows (conflict-free at the odd row stride)
    long long *Ds = reinterpret_cast<long long *>(const_cast<float *>(zb) + kTileRows * kZStride);
#pragma unroll
    for (int q = 0; q < kK1Tok; ++q) {
        const int l = tid + 1 + kK1Threads * q;
        const int t = tile * kTileOut + l - 1;
        long long D_ = 0;
        if (l <= kTileOut && t < sr.M && t > 0) {
            D_ = quantised_step(zb + (l - 1) * kZStride, zb + l * kZStride);
            if (D_ < 0) {
                raise_flag(a.flags, FLAG_OVERFLOW);
                D_ = 0;
            }
        }
        if (l <= kTileOut) Ds[l] = D_;
    }
    __syncthreads();
    // the scan takes outputs l = 4 tid + 1 .. 4 tid + 4
    long long Dv[kK1Tok];
#pragma unroll
    for (int q = 0; q < kK1Tok; ++q) {
        const int l = kK1Tok * tid + 1 + q;
        Dv[q] = l <= kTileOut ? Ds[l] : 0;
    }
    // block inclusive scan of the per-thread sums
    const int lane = tid & 31, warp = tid >> 5;
    long long own = 0;
#pragma unroll
    for (int q = 0; q < kK1Tok; ++q) own += Dv[q];
    long long v = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, v, off);
        if (lane >= off) v += n;
    }
    if (lane == 31) warp_sum[warp] = v;
    __syncthreads();
    long long wp = 0;
    for (int w = 0; w < warp; ++w) wp += warp_sum[w];
    const long long incl = wp + v;
    long long run = incl - own;
    int64_t *ls = a.local_scan + sr.mid_off + static_cast<int64_t>(h) * sr.M;
#pragma unroll
    for (int q = 0; q < kK1Tok; ++q) {
        run += Dv[q];
        const int l = kK1Tok * tid + 1 + q;
        const int t = tile * kTileOut + l - 1;
        if (l <= kTileOut && t < sr.M) ls[t] = run;
    }
    if (tid == kK1Threads - 1) a.tile_total[static_cast<int64_t>(u) * a.max_tiles + tile] = incl;
}

// CENTER: the key features enter as fl32(k - mu) (the centring option)
template <int D, typename T, bool CENTER>
__global__ void __launch_bounds__(kK1Threads, 2)
    k_project_scan(const CoarsenArgs a, const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ ProjT proj) {
    constexpr int ELEM = sizeof(T);
    constexpr int KCHUNK = D * ELEM / kK1ColBytes;   // column chunks of one key row
    constexpr int NCHUNK = 2 * KCHUNK;               // key chunks, then value chunks
    constexpr int JPC = kK1ColBytes / ELEM;          // feature index j per chunk
    constexpr int EPS = 16 / ELEM;                   // elements per 16-byte sub-chunk

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t *stages = smem;
    float *pt = reinterpret_cast<float *>(smem + kK1Stages * kK1StageBytes);
    uint64_t *bar = reinterpret_cast<uint64_t *>(pt + (2 * D + 1) * kProjDim);
    long long *warp_sum = reinterpret_cast<long long *>(bar + 8);
    float *mus = reinterpret_cast<float *>(warp_sum + 8);   // the unit's mean key (CENTER)

    const int u = blockIdx.y;
    const int tile = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    if (tile >= sr.tiles) return;
    const int tid = threadIdx.x;

    const int y0 = static_cast<int>(sr.row_off + static_cast<int64_t>(h) * sr.T + sr.s_eff) + tile * kTileOut - 1;
    auto issue = [&](int c, int s) {
        mbar_arrive_expect_tx(&bar[s], kK1StageBytes);
        const CUtensorMap *map = c < KCHUNK ? &map_k : &map_v;
#pragma unroll
        for (int hb = 0; hb < kTileRows / kK1BoxRows; ++hb)
            tma_load_2d(stages + s * kK1StageBytes + hb * kK1BoxRows * kK1ColBytes, map, (c % KCHUNK) * JPC,
                        y0 + hb * kK1BoxRows, &bar[s]);
    };
    if (tid == 0) {
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        for (int s = 0; s < kK1Stages; ++s) mbar_init(&bar[s], 1);
        fence_mbar_init();
        for (int c = 0; c < NCHUNK && c < kK1Stages; ++c) issue(c, c);
    }
    for (int i = tid; i < (2 * D + 1) * kProjDim; i += kK1Threads) pt[i] = i < 2 * D * kProjDim ? proj.pt[i] : 0.0f;
    if constexpr (CENTER)
        for (int i = tid; i < D; i += kK1Threads) mus[i] = a.key_mu[static_cast<int64_t>(u) * D + i];
    __syncthreads();

    // rows tid + 128 t (t < 4) of the tile; each feature's P^T row is read once per 4 tokens
    uint64_t acc[kK1Tok][kProjDim / 2];
#pragma unroll
    for (int t = 0; t < kK1Tok; ++t)
#pragma unroll
        for (int i = 0; i < kProjDim / 2; ++i) acc[t][i] = 0ull;
    const float4 *ptv = reinterpret_cast<const float4 *>(pt);   // P^T row j = ptv[4 j .. 4 j + 3]
    // software pipeline: the P^T row of feature j + 1 and the next 16-byte sub-chunk of the rows
    // are read while feature j is accumulated (plain shared loads: never hoisted above the wait)
    float4 pc[4];
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) pc[q4] = ptv[q4];

    for (int c = 0; c < NCHUNK; ++c) {
        const int s = c % kK1Stages;
        const bool got = mbar_wait(&bar[s], (c / kK1Stages) & 1);
        const uint4 *st = reinterpret_cast<const uint4 *>(stages + s * kK1StageBytes);
        uint4 x[kK1Tok];
#pragma unroll
        for (int t = 0; t < kK1Tok; ++t) x[t] = st[k1_sub(tid + t * kK1Threads, 0)];
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
            const int ccn = cc < 3 ? cc + 1 : 3;
            uint4 xn[kK1Tok];
#pragma unroll
            for (int t = 0; t < kK1Tok; ++t) xn[t] = st[k1_sub(tid + t * kK1Threads, ccn)];
#pragma unroll
            for (int e = 0; e < EPS; ++e) {
                const int j = c * JPC + cc * EPS + e;
                float4 pn[4];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) pn[q4] = ptv[4 * (j + 1) + q4];
                float mu_j = 0.0f;
                if constexpr (CENTER) mu_j = mus[c < KCHUNK ? j : 0];   // value chunks: unused
#pragma unroll
                for (int t = 0; t < kK1Tok; ++t) {
                    uint64_t xx;
                    if constexpr (CENTER) {
                        float lo, hi;
                        f2unpack(dup_elem<T>(x[t], e), lo, hi);
                        const float xc = c < KCHUNK ? __fsub_rn(lo, mu_j) : lo;
                        xx = f2pack(xc, xc);
                    } else {
                        xx = dup_elem<T>(x[t], e);
                    }
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        acc[t][2 * q4] = ffma2(f2pack(pc[q4].x, pc[q4].y), xx, acc[t][2 * q4]);
                        acc[t][2 * q4 + 1] = ffma2(f2pack(pc[q4].z, pc[q4].w), xx, acc[t][2 * q4 + 1]);
                    }
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) pc[q4] = pn[q4];
            }
#pragma unroll
            for (int t = 0; t < kK1Tok; ++t) x[t] = xn[t];
        }
        // every thread's wait verdict: if any wait gave up, the CTA issues no further copy, thread 0
        // waits (bounded) for the copies already in flight into its shared memory (chunks c and
        // c + 1), and the tile writes nothing
        if (!__syncthreads_and(got)) {
            if (tid == 0) {
                for (int c2 = c; c2 < NCHUNK && c2 <= c + 1; ++c2)
                    (void)mbar_wait(&bar[c2 % kK1Stages], (c2 / kK1Stages) & 1);
                raise_flag(a.flags, FLAG_TIMEOUT);
            }
            return;
        }
        if (tid == 0 && c + kK1Stages < NCHUNK) issue(c + kK1Stages, s);
    }

    // z of the rows -> shared (the stages are free: every chunk has been consumed and synced)
    float *zb = reinterpret_cast<float *>(stages);
#pragma unroll
    for (int t = 0; t < kK1Tok; ++t) {
        const int r = tid + t * kK1Threads;
#pragma unroll
        for (int i = 0; i < kProjDim / 2; ++i) f2unpack(acc[t][i], zb[r * kZStride + 2 * i], zb[r * kZStride + 2 * i + 1]);
    }
    __syncthreads();

    scan_tile(a, sr, u, h, tile, zb, warp_sum);
}

// ---------------------------------------------------------------------------
// k_project_tc (option SKV_PROJECTION_TENSOR_BF16): the same tiles and scan, with z = P16 x on the
// fifth-generation tensor cores: P16 = bf16(P), x the bf16 features, fp32 accumulation in tensor
// memory. The products are exact; only the accumulation order and rounding differ from the fixed
// recipe, so the quantised steps differ from it by a bounded amount and the boundaries follow the
// steps the tensor cores produced.
//
// One thread issues everything: the TMA copies of a tile's 64-byte feature chunks (512 rows each,
// the 64-byte swizzle) into a kTcStages ring, and per chunk 8 MMAs (tcgen05.mma kind::f16, M = 128
// tokens, N = 16 outputs, K = 16 features: 4 row blocks x 2 feature halves) that read the chunk and
// P16's image straight from shared memory and accumulate z of the 4 row blocks in 64 columns of
// tensor memory; tcgen05.commit releases a stage to the next copy when its MMAs are done. The four
// warps then read z back (tcgen05.ld, one token row per thread) for the steps and the scan.
// ---------------------------------------------------------------------------
constexpr int kTcStages = 3;
constexpr int kTcCols = 4 * kProjDim;   // tensor-memory columns: z of the tile's 4 row blocks of 128

// Shared-memory matrix descriptor of a K-major operand in the 64-byte swizzle (rows of 64 bytes,
// 16-byte granule g of row r at g ^ ((r >> 1) & 3)): start address, 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t tc_desc_sw64(uint32_t saddr) {
    return static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4) | (static_cast<uint64_t>(1u) << 16) |
           (static_cast<uint64_t>(512u >> 4) << 32) | (static_cast<uint64_t>(1u) << 46) |
           (static_cast<uint64_t>(4u) << 61);
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both K-major, N = 16, M = 128.
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((kProjDim >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, bool accumulate) {
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(
            d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate ? 1u : 0u));
}

// arrive on `bar` once every MMA this thread has issued so far has completed
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 16 consecutive fp32 columns of this thread's tensor-memory lane
__device__ __forceinline__ void tc_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
        "%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

template <int D>
constexpr size_t tc_smem_bytes() {
    // alignment slack + stage ring + P16 image + barriers, tensor-memory slot, scan scratch
    return 1024 + kTcStages * kK1StageBytes + sizeof(ProjFrag) + 128 + 64;
}

template <int D>
__global__ void __launch_bounds__(kK1Threads, 2)
    k_project_tc(const CoarsenArgs a, const __grid_constant__ CUtensorMap map_k,
                 const __grid_constant__ CUtensorMap map_v, const __grid_constant__ ProjFrag pf) {
    constexpr int KCHUNK = D * 2 / kK1ColBytes;   // bf16 column chunks of one key row
    constexpr int NCHUNK = 2 * KCHUNK;            // key chunks, then value chunks
    constexpr int PIMG = NCHUNK * kProjDim * kK1ColBytes;   // bytes of P16's image
    static_assert(kTileRows == 4 * 128 && kK1StageBytes == kTileRows * kK1ColBytes, "4 row blocks of 128");
    static_assert(PIMG <= static_cast<int>(sizeof(ProjFrag)) && kTcCols == 64, "image and columns");

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t *smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);   // the swizzle atoms need 512-byte alignment
    uint8_t *stages = smem;
    uint8_t *pimg = stages + kTcStages * kK1StageBytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(pimg + sizeof(ProjFrag));
    uint64_t *consumed = full + kTcStages;
    uint64_t *done = consumed + kTcStages;
    uint32_t *tslot = reinterpret_cast<uint32_t *>(done + 1);
    int *ok_flag = reinterpret_cast<int *>(tslot + 1);
    long long *warp_sum = reinterpret_cast<long long *>(full + 16);

    const int u = blockIdx.y;
    const int tile = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    if (tile >= sr.tiles) return;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    const int y0 = static_cast<int>(sr.row_off + static_cast<int64_t>(h) * sr.T + sr.s_eff) + tile * kTileOut - 1;
    int n_issued = 0;   // (thread 0) chunks whose copy has been issued
    auto issue = [&](int c, int s) {
        ++n_issued;
        mbar_arrive_expect_tx(&full[s], kK1StageBytes);
        const CUtensorMap *map = c < KCHUNK ? &map_k : &map_v;
#pragma unroll
        for (int hb = 0; hb < kTileRows / kK1BoxRows; ++hb)
            tma_load_2d(stages + s * kK1StageBytes + hb * kK1BoxRows * kK1ColBytes, map, (c % KCHUNK) * 32,
                        y0 + hb * kK1BoxRows, &full[s]);
    };
    if (tid == 0) {
        prefetch_tensormap(&map_k);
        prefetch_tensormap(&map_v);
        for (int s = 0; s < kTcStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&consumed[s], 1);
        }
        mbar_init(done, 1);
        *ok_flag = 1;
        fence_mbar_init();
        for (int c = 0; c < NCHUNK && c < kTcStages; ++c) issue(c, c);
    }
    // P16's image (already in the 64-byte swizzle, chunk after chunk) into shared memory, then made
    // visible to the tensor cores (async proxy)
    for (int i = tid; i < PIMG / 16; i += kK1Threads)
        reinterpret_cast<uint4 *>(pimg)[i] = reinterpret_cast<const uint4 *>(pf.w)[i];
    fence_proxy_async_smem();
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tslot)),
                     "r"(static_cast<uint32_t>(kTcCols)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before_sync();
    __syncthreads();   // barriers, the image and the tensor-memory address are ready
    tc_fence_after_sync();
    const uint32_t tmem = *tslot;

    if (tid == 0) {
        bool ok = true;
        int n_landed = 0;   // chunks whose copy this thread has seen land
        for (int c = 0; c < NCHUNK; ++c) {
            const int s = c % kTcStages;
            if (!mbar_wait(&full[s], (c / kTcStages) & 1)) {
                ok = false;
                break;
            }
            ++n_landed;
            tc_fence_after_sync();
            const uint32_t sa = smem_u32(stages + s * kK1StageBytes);
            const uint32_t sb = smem_u32(pimg + c * kProjDim * kK1ColBytes);
#pragma unroll
            for (int mb = 0; mb < 4; ++mb)
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    tc_mma(tmem + mb * kProjDim, tc_desc_sw64(sa + mb * 128 * kK1ColBytes + ks * 32),
                           tc_desc_sw64(sb + ks * 32), c > 0 || ks > 0);
            tc_commit(&consumed[s]);   // the stage is free once these MMAs have read it
            if (c + kTcStages < NCHUNK) {
                if (!mbar_wait(&consumed[s], (c / kTcStages) & 1)) {
                    ok = false;
                    break;
                }
                issue(c + kTcStages, s);
            }
        }
        tc_commit(done);   // every MMA issued, also after a failed wait
        if (!ok) {
            // a wait gave up: no further copy or MMA; the copies already in flight land first
            for (int c2 = n_landed; c2 < n_issued; ++c2)
                (void)mbar_wait(&full[c2 % kTcStages], (c2 / kTcStages) & 1);
            *ok_flag = 0;
            raise_flag(a.flags, FLAG_TIMEOUT);
        }
    }
    const bool mma_done = mbar_wait(done, 0);
    __syncthreads();   // thread 0's verdict
    tc_fence_after_sync();
    const bool good = mma_done && *ok_flag != 0;
    // z of the tile's rows (the stages are free: every MMA has completed) -> shared, row after row
    float *zb = reinterpret_cast<float *>(stages);
    if (good) {
#pragma unroll 1
        for (int mb = 0; mb < 4; ++mb) {
            float z[kProjDim];
            tc_ld16(tmem + ((static_cast<uint32_t>(warp) * 32u) << 16) + mb * kProjDim, z);
            const int r = mb * 128 + warp * 32 + lane;
#pragma unroll
            for (int i = 0; i < kProjDim; ++i) zb[r * kZStride + i] = z[i];
        }
    }
    tc_fence_before_sync();
    __syncthreads();
    if (warp == 0)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(static_cast<uint32_t>(kTcCols)));
    if (!good) {
        if (tid == 0 && !mma_done) raise_flag(a.flags, FLAG_TIMEOUT);
        return;
    }
    scan_tile(a, sr, u, h, tile, zb, warp_sum);
}

// ---------------------------------------------------------------------------
// k_boundaries: b_j = first t with N c_t >= j c_T  (j = 1 .. N-1)
// ---------------------------------------------------------------------------
// floor(N * C / CT) for CT > 0, exact: the double estimate (inv_ct = 1 / CT) is off by at most one
// and corrected with exact 128-bit products
__device__ __forceinline__ long long floor_ratio(long long N, long long C, long long CT, double inv_ct) {
    long long q = static_cast<long long>(static_cast<double>(N) * static_cast<double>(C) * inv_ct);
    if (q < 0) q = 0;
    while (prod_ge(static_cast<uint64_t>(N), static_cast<uint64_t>(C), static_cast<uint64_t>(q + 1),
                   static_cast<uint64_t>(CT)))
        ++q;
    while (q > 0 && !prod_ge(static_cast<uint64_t>(N), static_cast<uint64_t>(C), static_cast<uint64_t>(q),
                             static_cast<uint64_t>(CT)))
        --q;
    return q;
}

// floor(N c / c_T) from the double estimate x = fl(fl(c) * scale), scale = fl(N * fl(1 / c_T)): four
// roundings, so |x - N c / c_T| <= N 2^-51 (the ratio is at most N). When x lies farther than
// guard = N 2^-48 from every integer its floor is the exact one (x - floor(x) is exact: both are
// multiples of x's ulp); -1 otherwise (undecided: the exact floor_ratio decides). c = 0 (the unit's
// first token, and threads without a token) is exact at once.
__device__ __forceinline__ int floor_estimate(long long c, double scale, double guard) {
    if (c == 0) return 0;
    const double x = static_cast<double>(c) * scale;
    const double f = floor(x);
    return x - f > guard && x - f < 1.0 - guard ? static_cast<int>(f) : -1;
}

// One thread per middle token t: the thresholds j with floor(N c_{t-1} / c_T) < j <= floor(N c_t / c_T)
// are first hit at t. Each thread takes its own floor once; its predecessor's comes from the lane
// below, across warps through shared memory, and for a tile's first token from the tile's start.
// A CTA takes kBndTiles consecutive tiles of one unit: c at the start of its first tile and c_T are
// sums of the unit's tile totals (exact integers), so no separate prefix pass over the tiles runs
// before it. All its loads are issued before the first floor is taken and the floors stay in
// registers: those of the double estimate first, then the exact ones for the few estimates that lie
// too close to an integer.
constexpr int kBndTiles = 4;

__global__ void __launch_bounds__(kTileRows, 3) k_boundaries(const CoarsenArgs a) {
    constexpr int WARPS = kTileRows / 32;
    __shared__ long long red[2][WARPS];
    __shared__ long long tts[kBndTiles];     // the CTA's tile totals
    __shared__ int qlast[kBndTiles][WARPS];  // the floor of each warp's last token, per tile
    __shared__ int qstart[kBndTiles];        // the floor at each tile's start (its first token's predecessor)
    const int u = blockIdx.y, tile0 = blockIdx.x * kBndTiles;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    if (tile0 >= sr.tiles) {
        if (blockIdx.x == 0 && threadIdx.x == 0) a.unit_total[u] = 0;   // a unit without middle tokens
        return;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t rowb = static_cast<int64_t>(u) * a.max_tiles;
    const int64_t *ls = a.local_scan + sr.mid_off + static_cast<int64_t>(h) * sr.M;
    long long before = 0, total = 0;   // this thread's share of the tile totals before tile0 / of all
    for (int i = tid; i < sr.tiles; i += kTileRows) {
        const long long x = a.tile_total[rowb + i];
        total += x;
        if (i < tile0) before += x;
    }
    long long lsv[kBndTiles];   // the tile-local scan at this thread's token of each tile; -1: none
#pragma unroll
    for (int g = 0; g < kBndTiles; ++g) {
        const int tile = tile0 + g;
        const int t = tile * kTileOut + tid;
        lsv[g] = tile < sr.tiles && tid < kTileOut && t < sr.M ? ls[t] : -1;   // inactive threads sit at the end
    }
    if (tid < kBndTiles) tts[tid] = tile0 + tid < sr.tiles ? a.tile_total[rowb + tile0 + tid] : 0;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        before += __shfl_xor_sync(0xffffffffu, before, off);
        total += __shfl_xor_sync(0xffffffffu, total, off);
    }
    if (lane == 0) {
        red[0][warp] = before;
        red[1][warp] = total;
    }
    __syncthreads();
    before = total = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
        before += red[0][w];
        total += red[1][w];
    }
    const long long CT = total;   // c_T
    if (blockIdx.x == 0 && tid == 0) a.unit_total[u] = CT;
    const int N = sr.N;
    if (a.cumvar) {   // c_t of the tiles' middle tokens
        long long tp = before;
#pragma unroll
        for (int g = 0; g < kBndTiles; ++g) {
            const int t = (tile0 + g) * kTileOut + tid;
            if (lsv[g] >= 0) a.cumvar[sr.row_off + static_cast<int64_t>(h) * sr.T + t] = tp + lsv[g];
            tp += tts[g];
        }
    }
    int32_t *bnd = a.bounds + sr.bnd_off + static_cast<int64_t>(h) * (N + 1);
    if (CT == 0) {
        if (tile0 == 0 && tid == 0)
            for (int j = 1; j < N; ++j) bnd[j] = 0;
        return;
    }
    const double inv = 1.0 / static_cast<double>(CT);
    const double scale = static_cast<double>(N) * inv, guard = static_cast<double>(N) * 0x1p-48;
    int q[kBndTiles];
    uint32_t undecided = 0;
    {
        long long tp = before;
#pragma unroll
        for (int g = 0; g < kBndTiles; ++g) {
            q[g] = floor_estimate(lsv[g] >= 0 ? tp + lsv[g] : 0, scale, guard);
            if (q[g] < 0) undecided |= 1u << g;
            tp += tts[g];
        }
    }
    if (undecided) {   // the exact floors with 128-bit products (rare)
        long long tp = before;
#pragma unroll
        for (int g = 0; g < kBndTiles; ++g) {
            if (undecided & (1u << g)) q[g] = static_cast<int>(floor_ratio(N, lsv[g] >= 0 ? tp + lsv[g] : 0, CT, inv));
            tp += tts[g];
        }
    }
    if (lane == 31) {
#pragma unroll
        for (int g = 0; g < kBndTiles; ++g) qlast[g][warp] = q[g];
    }
    if (tid < kBndTiles) {   // thread g: the floor at tile g's start
        long long tp = before;
        for (int g = 0; g < tid; ++g) tp += tts[g];
        int f = floor_estimate(tp, scale, guard);
        if (f < 0) f = static_cast<int>(floor_ratio(N, tp, CT, inv));
        qstart[tid] = f;
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < kBndTiles; ++g) {
        if (tile0 + g >= sr.tiles) break;   // (the same for the whole CTA)
        const int t = (tile0 + g) * kTileOut + tid;
        int qprev = __shfl_up_sync(0xffffffffu, q[g], 1);
        if (lane == 0) qprev = warp > 0 ? qlast[g][warp - 1] : qstart[g];
        if (lsv[g] >= 0 && t != 0) {
            const int jhi = q[g] > N - 1 ? N - 1 : q[g];
            for (int j = qprev + 1; j <= jhi; ++j) bnd[j] = t;
        }
    }
}

// ---------------------------------------------------------------------------
// k_plan_entries: entries (start, mass) in the order sinks, nonempty segments, recents
// ---------------------------------------------------------------------------
constexpr int kPlanSeg = 8;   // segments per thread and round of k_plan_entries

__global__ void __launch_bounds__(512) k_plan_entries(const CoarsenArgs a) {
    __shared__ int wsum[16];
    const int u = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    const int N = sr.N, M = sr.M;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    int32_t *bnd = a.bounds + sr.bnd_off + static_cast<int64_t>(h) * (N + 1);
    if (M == 0) {
        for (int j = tid; j <= N; j += 512) bnd[j] = 0;
    } else if (tid == 0) {
        bnd[0] = 0;
        bnd[N] = M;
    }
    __syncthreads();
    int2 *ents = a.ents + sr.ent_off + static_cast<int64_t>(h) * sr.emax;
    for (int e = tid; e < sr.s_eff; e += 512) ents[e] = make_int2(e, 1);
    // each thread takes kPlanSeg consecutive segments of a round: all its boundaries are read at once
    int carry = 0;
    for (int base = 0; base < N; base += 512 * kPlanSeg) {
        const int j0 = base + tid * kPlanSeg;
        int bv[kPlanSeg + 1];
#pragma unroll
        for (int i = 0; i <= kPlanSeg; ++i) bv[i] = j0 + i <= N ? bnd[j0 + i] : 0;
        int cnt = 0;
#pragma unroll
        for (int i = 0; i < kPlanSeg; ++i) cnt += (j0 + i < N && bv[i + 1] > bv[i]) ? 1 : 0;
        int v = cnt;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int n = __shfl_up_sync(0xffffffffu, v, off);
            if (lane >= off) v += n;
        }
        if (lane == 31) wsum[warp] = v;
        __syncthreads();
        int wp = 0, all = 0;
#pragma unroll
        for (int w = 0; w < 16; ++w) {
            const int x = wsum[w];
            all += x;
            if (w < warp) wp += x;
        }
        int e = sr.s_eff + carry + wp + v - cnt;   // this thread's first entry
#pragma unroll
        for (int i = 0; i < kPlanSeg; ++i)
            if (j0 + i < N && bv[i + 1] > bv[i]) ents[e++] = make_int2(sr.s_eff + bv[i], bv[i + 1] - bv[i]);
        carry += all;
        __syncthreads();   // wsum is read before the next round writes it
    }
    for (int i = tid; i < sr.w_eff; i += 512) ents[sr.s_eff + carry + i] = make_int2(sr.s_eff + M + i, 1);
    if (tid == 0) a.lens[u] = sr.s_eff + carry + sr.w_eff;
    if (a.user_bounds)
        for (int j = tid; j <= N; j += 512) a.user_bounds[static_cast<int64_t>(u) * (a.Nmax + 1) + j] = bnd[j];
}

// ---------------------------------------------------------------------------
// k_segment_reduce: one warp per entry
// ---------------------------------------------------------------------------
template <typename T>
struct Vec16;   // 16 bytes of elements as fp32

template <>
struct Vec16<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void cvt(const uint4 &w, float (&x)[8]) {
        x[0] = bf16lo(w.x); x[1] = bf16hi(w.x); x[2] = bf16lo(w.y); x[3] = bf16hi(w.y);
        x[4] = bf16lo(w.z); x[5] = bf16hi(w.z); x[6] = bf16lo(w.w); x[7] = bf16hi(w.w);
    }
    __device__ static void load(const void *p, float (&x)[8]) { cvt(__ldg(reinterpret_cast<const uint4 *>(p)), x); }
    __device__ static void store(void *p, const float (&x)[8]) {
        uint4 w;
        w.x = pack_bf16x2(x[0], x[1]); w.y = pack_bf16x2(x[2], x[3]);
        w.z = pack_bf16x2(x[4], x[5]); w.w = pack_bf16x2(x[6], x[7]);
        *reinterpret_cast<uint4 *>(p) = w;
    }
};

template <>
struct Vec16<float> {
    static constexpr int N = 4;
    __device__ static void cvt(const uint4 &w, float (&x)[4]) {
        x[0] = __uint_as_float(w.x); x[1] = __uint_as_float(w.y);
        x[2] = __uint_as_float(w.z); x[3] = __uint_as_float(w.w);
    }
    __device__ static void load(const void *p, float (&x)[4]) { cvt(__ldg(reinterpret_cast<const uint4 *>(p)), x); }
    __device__ static void store(void *p, const float (&x)[4]) {
        *reinterpret_cast<float4 *>(p) = make_float4(x[0], x[1], x[2], x[3]);
    }
};

constexpr int kK3Warps = 8;
constexpr int kSegPrefetchRows = 256;   // rows of a segment prefetched into L2 at its start

// W: the variation-weighted representative is compiled in (a separate instantiation, so the
// plain-mean kernel keeps its register budget).
// CENTER: keys enter as fl32(k - mu), mu the unit's mean key (the centring option)
template <int D, typename T, bool W, bool CENTER>
__global__ void __launch_bounds__(kK3Warps * 32) k_segment_reduce(const CoarsenArgs a) {
    constexpr int ELEM = sizeof(T);
    constexpr int ROWB = D * ELEM;        // bytes of one key row
    constexpr int CH = ROWB / 16;         // 16-byte chunks per row = lanes per token
    constexpr int TPS = 32 / CH;          // tokens per warp step
    constexpr int EPL = 16 / ELEM;        // elements per lane
    static_assert(CH >= 8 && CH <= 32, "row must span 8..32 chunks");

    const int u = blockIdx.y;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int e = blockIdx.x * kK3Warps + warp;
    const int n_ent = a.lens[u];
    if (e >= n_ent) return;
    const SeqRow sr = a.seq[b];
    const int2 ent = a.ents[sr.ent_off + static_cast<int64_t>(h) * sr.emax + e];
    const int start = ent.x, m = ent.y;
    const int sub = lane / CH, ch = lane % CH;

    float muv[EPL];   // the unit's mean key on this lane's dimensions (zero without centring)
#pragma unroll
    for (int i = 0; i < EPL; ++i) muv[i] = CENTER ? a.key_mu[static_cast<int64_t>(u) * D + ch * EPL + i] : 0.0f;
    const int64_t row0 = sr.row_off + static_cast<int64_t>(h) * sr.T + start;
    const uint8_t *kp = static_cast<const uint8_t *>(a.k) + row0 * ROWB + ch * 16;
    const uint8_t *vp = static_cast<const uint8_t *>(a.v) + row0 * ROWB + ch * 16;
    // The segment's rows are contiguous: one bulk L2 prefetch per tensor (its first kSegPrefetchRows
    // rows) puts the first pass's DRAM reads in flight at once, so that the warp's loads below wait
    // on L2 rather than on a chain of DRAM round trips. Taken by the weighted kernel only, whose
    // register budget leaves fewer warps per SM to cover the latency (the plain mean measured
    // slower with it).
    if (W && lane == 0 && m > 8) {
        const uint8_t *k0 = static_cast<const uint8_t *>(a.k) + row0 * ROWB;
        const uint8_t *v0 = static_cast<const uint8_t *>(a.v) + row0 * ROWB;
        const uint32_t bytes = static_cast<uint32_t>(m < kSegPrefetchRows ? m : kSegPrefetchRows) * ROWB;
        if (((reinterpret_cast<uintptr_t>(k0) | reinterpret_cast<uintptr_t>(v0)) & 15u) == 0) {
            bulk_prefetch_l2(k0, bytes);
            bulk_prefetch_l2(v0, bytes);
        }
    }

    // A middle segment with the variation-weighted representative ("Equal-Variation KV Cache",
    // "Implementation notes") also accumulates sum_r d_r k_r, sum_r d_r v_r and sum_r d_r with
    // d_r = D_r 2^-20, D_r recovered from the tile-local scan of the projection kernel.
    const int t_mid = start - sr.s_eff;   // middle index of the first member
    const bool weighted = W && m > 1 && t_mid >= 0 && t_mid < sr.M;
    const int64_t *ls = a.local_scan + sr.mid_off + static_cast<int64_t>(h) * sr.M;

    // loads are issued kUnroll token steps at a time (2 x kUnroll 16-byte loads in flight per lane).
    // The plain kernel takes 10 (74 registers, 3 CTAs per SM; 4, 6, 8, 12 and 16 measured slower),
    // the centred one 8 (10 costs it a CTA per SM). The weighted kernel takes 2 (75 registers, 3
    // CTAs per SM: its L2 prefetch already has the segment's rows in flight; 4 steps took 93
    // registers and 2 CTAs per SM and measured slower).
    constexpr int kUnroll = W ? 2 : (CENTER ? 8 : 10);
    float sk[EPL], sv[EPL], wk[EPL], wv[EPL], x[EPL], wsum = 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) sk[i] = sv[i] = wk[i] = wv[i] = 0.0f;
    for (int t0 = sub; t0 < m; t0 += TPS * kUnroll) {
        uint4 kw[kUnroll], vw[kUnroll];
        long long lc[kUnroll], lp[kUnroll];
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            const int t = t0 + r * TPS;
            kw[r] = vw[r] = make_uint4(0u, 0u, 0u, 0u);   // zero bits: +0.0 in both dtypes
            lc[r] = lp[r] = 0;
            if (t < m) {
                kw[r] = __ldg(reinterpret_cast<const uint4 *>(kp + static_cast<int64_t>(t) * ROWB));
                vw[r] = __ldg(reinterpret_cast<const uint4 *>(vp + static_cast<int64_t>(t) * ROWB));
                if (W && weighted) {   // D of middle token tm: its tile-local inclusive scan minus the previous
                    const int tm = t_mid + t;
                    lc[r] = __ldg(reinterpret_cast<const long long *>(ls + tm));
                    if (tm % kTileOut != 0) lp[r] = __ldg(reinterpret_cast<const long long *>(ls + tm - 1));
                }
            }
        }
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            const float w = W && weighted ? __ll2float_rn(lc[r] - lp[r]) * 0x1p-20f : 0.0f;
            if (W) wsum += w;
            Vec16<T>::cvt(kw[r], x);
            if constexpr (CENTER) {
#pragma unroll
                for (int i = 0; i < EPL; ++i) x[i] = t0 + r * TPS < m ? __fsub_rn(x[i], muv[i]) : 0.0f;
            }
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                sk[i] += x[i];
                if (W) wk[i] = __fmaf_rn(w, x[i], wk[i]);
            }
            Vec16<T>::cvt(vw[r], x);
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                sv[i] += x[i];
                if (W) wv[i] = __fmaf_rn(w, x[i], wv[i]);
            }
        }
    }
#pragma unroll
    for (int off = CH; off < 32; off <<= 1) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
            sv[i] += __shfl_xor_sync(0xffffffffu, sv[i], off);
        }
        if (W && weighted) {
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                wk[i] += __shfl_xor_sync(0xffffffffu, wk[i], off);
                wv[i] += __shfl_xor_sync(0xffffffffu, wv[i], off);
            }
            wsum += __shfl_xor_sync(0xffffffffu, wsum, off);
        }
    }
    const float fm = static_cast<float>(m);
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        sk[i] = __fdiv_rn(sk[i], fm);   // mean key
        sv[i] = __fdiv_rn(sv[i], fm);   // mean value
    }
    // the stored key and value: the mean, or the weighted average when the segment has variation
    float rk[EPL], rv[EPL];
    const bool use_w = W && weighted && wsum > 0.0f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        rk[i] = use_w ? __fdiv_rn(wk[i], wsum) : sk[i];
        rv[i] = use_w ? __fdiv_rn(wv[i], wsum) : sv[i];
    }
    // second pass over the keys (just read: served from L1 / L2)
    float q2[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) q2[i] = 0.0f;
    for (int t0 = sub; t0 < m; t0 += TPS * kUnroll) {
        uint4 kw[kUnroll];
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            const int t = t0 + r * TPS;
            kw[r] = make_uint4(0u, 0u, 0u, 0u);
            if (t < m) kw[r] = __ldg(reinterpret_cast<const uint4 *>(kp + static_cast<int64_t>(t) * ROWB));
        }
#pragma unroll
        for (int r = 0; r < kUnroll; ++r) {
            if (t0 + r * TPS >= m) break;
            Vec16<T>::cvt(kw[r], x);
            if constexpr (CENTER) {
#pragma unroll
                for (int i = 0; i < EPL; ++i) x[i] = __fsub_rn(x[i], muv[i]);
            }
#pragma unroll
            for (int i = 0; i < EPL; ++i) {
                const float dv = x[i] - sk[i];
                q2[i] = __fmaf_rn(dv, dv, q2[i]);
            }
        }
    }
    float var_lane = 0.0f, vd[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        float qi = q2[i];
#pragma unroll
        for (int off = CH; off < 32; off <<= 1) qi += __shfl_xor_sync(0xffffffffu, qi, off);
        vd[i] = __fdiv_rn(qi, fm);   // population variance of dimension i
        var_lane += vd[i];
    }
#pragma unroll
    for (int off = 1; off < CH; off <<= 1) var_lane += __shfl_xor_sync(0xffffffffu, var_lane, off);
    const float sigma2 = var_lane / static_cast<float>(D);

    const int32_t page = a.page_table[static_cast<int64_t>(u) * a.max_pages + e / kPageNodes];
    const int slot = e % kPageNodes;
    if (page < 0 || page >= a.num_pages) {
        if (lane == 0) raise_flag(a.flags, FLAG_BAD_PAGE);
        return;
    }
    constexpr int VEC_BYTES = kPageNodes * ROWB;   // keys (then values, then variances) of one page
    const bool diag = a.closure == SKV_CLOSURE_DIAGONAL;
    uint8_t *pg = a.pages + static_cast<int64_t>(page) * ((diag ? 3 : 2) * VEC_BYTES + kPageNodes * 8);
    if (sub == 0) {
        const int off = slot * ROWB + swz(ch, slot) * 16;
        Vec16<T>::store(pg + off, rk);
        Vec16<T>::store(pg + VEC_BYTES + off, rv);
        if (diag) Vec16<T>::store(pg + 2 * VEC_BYTES + kPageNodes * 8 + off, vd);   // per-dimension variances
    }
    if (lane == 0) {
        const float alpha = m == 1 ? 0.0f : logf(fm);
        reinterpret_cast<float2 *>(pg + 2 * VEC_BYTES)[slot] = make_float2(alpha, sigma2 / (2.0f * D));
    }
}

// ---------------------------------------------------------------------------
// host launcher
// ---------------------------------------------------------------------------
template <int D>
static cudaError_t launch_project_tc(const CoarsenArgs &a, int n_units, const ProjFrag &frag,
                                    const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s) {
    constexpr size_t smem = tc_smem_bytes<D>();
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_dev != dev) {
        e = cudaFuncSetAttribute(k_project_tc<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    k_project_tc<D><<<dim3(a.max_tiles, n_units), kK1Threads, smem, s>>>(a, map_k, map_v, frag);
    return cudaSuccess;
}

// The projection of the batch's n units: quantised steps and tile scans.
template <int D, typename T, bool CENTER>
static cudaError_t launch_projection(const CoarsenArgs &a, int n, const ProjT &proj, const ProjFrag &frag,
                                     const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s) {
    if (a.projection == SKV_PROJECTION_TENSOR_BF16) {
        // the variation is translation invariant: the tensor-core projection reads the raw keys
        // even when they are centred (a common shift cancels in z_t - z_{t-1})
        if constexpr (sizeof(T) == 2) return launch_project_tc<D>(a, n, frag, map_k, map_v, s);
        return cudaErrorInvalidValue;   // bf16 inputs only (host-checked)
    }
    constexpr size_t smem = k1_smem_bytes<D>();
    static thread_local int configured_dev = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (configured_dev != dev) {
        e = cudaFuncSetAttribute(k_project_scan<D, T, CENTER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    k_project_scan<D, T, CENTER><<<dim3(a.max_tiles, n), kK1Threads, smem, s>>>(a, map_k, map_v, proj);
    return cudaSuccess;
}

// Everything after the projection for the batch's n units: prefix over tiles, boundaries, entries,
// segment statistics.
template <int D, typename T, bool CENTER>
static void launch_segments(const CoarsenArgs &a, int n, cudaStream_t s) {
    const int bnd_ctas = (a.max_tiles + kBndTiles - 1) / kBndTiles;   // (one per unit writes c_T = 0 without tiles)
    k_boundaries<<<dim3(bnd_ctas > 0 ? bnd_ctas : 1, n), kTileRows, 0, s>>>(a);
    k_plan_entries<<<n, 512, 0, s>>>(a);
    if (a.max_emax > 0) {
        const dim3 g3((a.max_emax + kK3Warps - 1) / kK3Warps, n);
        if (a.representative == SKV_REP_VARIATION_WEIGHTED)
            k_segment_reduce<D, T, true, CENTER><<<g3, kK3Warps * 32, 0, s>>>(a);
        else
            k_segment_reduce<D, T, false, CENTER><<<g3, kK3Warps * 32, 0, s>>>(a);
    }
}

template <int D, typename T, bool CENTER>
static cudaError_t launch_typed(const CoarsenArgs &a, const SeqTable &table, const ProjT &proj, const ProjFrag &frag,
                                const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s) {
    const int units = a.B * a.Hkv;
    k_setup<<<1, 512, 0, s>>>(table, const_cast<SeqRow *>(a.seq), a.B, a.flags);
    if (CENTER && a.max_blk > 0) {
        k_key_block_sums<D, T><<<dim3(a.max_blk, units), D, 0, s>>>(a);
        k_key_mean<D><<<units, D, 0, s>>>(a);
    }
    if (a.max_tiles > 0) {
        const cudaError_t e = launch_projection<D, T, CENTER>(a, units, proj, frag, map_k, map_v, s);
        if (e != cudaSuccess) return e;
    }
    launch_segments<D, T, CENTER>(a, units, s);
    return cudaGetLastError();
}

template <int D, typename T>
static cudaError_t launch_dt(const CoarsenArgs &a, const SeqTable &table, const ProjT &proj, const ProjFrag &frag,
                             const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s) {
    return a.center ? launch_typed<D, T, true>(a, table, proj, frag, map_k, map_v, s)
                    : launch_typed<D, T, false>(a, table, proj, frag, map_k, map_v, s);
}

cudaError_t launch_coarsen(const CoarsenArgs &a, const SeqTable &table, const ProjT &proj, const ProjFrag &frag,
                           const CUtensorMap &map_k, const CUtensorMap &map_v, cudaStream_t s) {
    if (a.dtype == SKV_BF16) {
        if (a.d == 128) return launch_dt<128, __nv_bfloat16>(a, table, proj, frag, map_k, map_v, s);
        return launch_dt<64, __nv_bfloat16>(a, table, proj, frag, map_k, map_v, s);
    }
    if (a.d == 128) return launch_dt<128, float>(a, table, proj, frag, map_k, map_v, s);
    return launch_dt<64, float>(a, table, proj, frag, map_k, map_v, s);
}

}  // namespace skv
