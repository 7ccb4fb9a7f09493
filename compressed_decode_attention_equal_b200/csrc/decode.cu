// Compressed decode attention over the paged macro-node cache.
//
// "SPICY-KV" demo page, section 2 ("FlashAttention-2/3 & PagedAttention
// Online-Softmax Kernel Fusion"): every node carries alpha = ln m and
// beta = sigma^2 / (2 d_k); inside the K-tile loop the logit is
//   s = q.k / sqrt(d_k) + alpha + |q|^2 beta
// with |q|^2 computed once per query row in registers, and the online softmax
// proceeds as for exact tokens. Claim 3: the beta term is the second-order
// cumulant closure of the partition Z.
//
// bf16 path (k_decode_split, one launch per call), split-K over pages:
//  * the flat page space of all (unit, row-pass) "virtual units" is cut into
//    ncta equal ranges (one per CTA, a stream-K style split), so every CTA
//    streams the same number of 16-node pages whatever the length mix; the
//    part of one virtual unit inside one CTA's range is a "piece";
//  * one producer warp copies each page (keys 4 KB, values 4 KB, alpha/beta
//    128 B at d = 128, contiguous) with one TMA bulk copy into an 8-stage
//    mbarrier ring, and each piece's query rows into a double-buffered slot;
//  * four consumer warps run the GQA group's query rows through tensor cores:
//    S^T = K Q^T with nodes as the M = 16 dimension and up to 8 query rows as
//    N = 8 (a GQA group of 7 rows wastes 1/8), softmax on the accumulator, P^T
//    transposed in registers (movmatrix) into the B operand of O^T = V^T P^T;
//  * a piece that covers a whole unit writes out / lse directly; pieces of a
//    unit split across CTAs write normalised partials (out, log2 partition);
//    after streaming, each CTA counts its split pieces in per-unit counters,
//    and the CTA that completes a unit merges its pieces (log-sum-exp) and
//    resets the counter;
//  * launched with programmatic stream serialisation: the next launch's CTAs
//    become resident while this grid drains; each grid reads its inputs only
//    after griddepcontrol.wait, so data from any preceding kernel is visible.
// fp32 path (k_decode_f32): a plain CUDA-core kernel (exact fp32 arithmetic),
// one CTA per unit, for fp32 caches.
#include <mutex>
#include <vector>

#include "skv_common.cuh"
#include "skv_internal.h"

namespace skv {

constexpr int kDecConsumers = 4;
// Ring depth (here and in SplitSmem): a multiple of the page-group count, so that the pages i and
// i + STAGES that share a stage always go to the same consumer warp, in order. A warp that
// could poll a stage for page i + STAGES while it still held page i would see the previous
// phase's parity as complete (mbarrier parity aliasing) and read stale data.
constexpr int kDecStages = 8;
constexpr float kLog2e = 1.4426950408889634f;
// Lazy maximum of the online softmax: a row's reference maximum moves only when a page's maximum
// exceeds it by more than this (log2 units). Until then the page's exponents are taken against the
// stale reference, so they are at most 2^8 -- exact in fp32 and of unchanged relative precision in
// bf16 -- and O, l and the reference stay consistent (the final normalisation and log-partition use
// them together). The rescale of O, 64 multiplies per page, then runs rarely instead of on most
// pages.
constexpr float kLazyMax = 8.0f;
constexpr float kLn2 = 0.6931471805599453f;

// DIAG: the page also carries per-dimension key variances (the diagonal closure) after alpha/beta
template <int D, bool DIAG = false>
struct PageGeom {
    static constexpr int ROWB = D * 2;                    // bytes of one bf16 node vector
    static constexpr int VEC_BYTES = kPageNodes * ROWB;   // K (or V, or variance) bytes of a page
    static constexpr int AB_BYTES = kPageNodes * 8;
    static constexpr int VAR_OFF = 2 * VEC_BYTES + AB_BYTES;
    static constexpr int STAGE = 2 * VEC_BYTES + AB_BYTES + (DIAG ? VEC_BYTES : 0);
};

template <int D, int NT, bool DIAG = false>
struct SplitSmem {
    static constexpr int QROWB = D * 2 + 16;              // padded query row: conflict-free ldmatrix
    static constexpr int QBUF = NT * 8 * QROWB;           // the query rows of one piece
    // Consumer warps. With the variances a page carries 1.5x the bytes and 3x the MMAs before PV:
    // one CTA per SM with 8 consumer warps and 8 stages takes a whole unit (measured 27.5 us
    // against 32.2 us for 4 warps, 4 stages and 3 CTAs per SM on the 7B 3.5% shape). Otherwise
    // 4 consumer warps and two CTAs per SM. (Two row tiles per warp sharing the K and V
    // fragments, which needs one CTA of 6 consumer warps per SM for its registers, measured 94 us
    // against 81 us on the ragged paged 2% workload.)
    static constexpr int CONS = DIAG ? 8 : kDecConsumers;
    static constexpr int CTAS_PER_SM = DIAG ? 1 : 2;
    static constexpr int THREADS = (CONS + 1) * 32;
    // 16 or more query rows per unit (scalar closure): query rows are the MMA's M dimension, 16
    // rows per warp, and the softmax's P feeds the PV product from the accumulators directly
    static constexpr bool MR = !DIAG && NT >= 2;
    static constexpr int WPP = MR ? NT / 2 : NT;          // consumer warps per page
    static constexpr int PG = CONS / WPP;                 // page groups (pages i, i + PG, ... per warp)
    // four row tiles with rows as M: the doubled page-group buffer leaves room for six stages
    static constexpr int STAGES = DIAG ? 8 : (MR && NT == 4 ? 6 : kDecStages);
    static_assert(STAGES % PG == 0, "a stage's successive pages must go to one consumer warp");
    static constexpr int STAGES_BYTES = STAGES * PageGeom<D, DIAG>::STAGE;
    static constexpr int MST = D + 4;                     // mbuf row stride: 16-byte rows
    static constexpr int MBUF_FLOATS = PG * NT * 8 * MST; // per page group and query row: O, m, l
    static constexpr int BARS = 2 * STAGES + 4;
    static constexpr int ROWS = NT * 8;                   // query rows of one piece
    static constexpr int WST = 9;                         // merge weights per row (<= 8) + log2 partition
    static constexpr int EPI_BYTES = ROWS * 8 + ROWS * WST * 4;
    static constexpr int SVALID_INTS = (STAGES + 3) & ~3;   // padded: mbuf (read as float4) stays 16-byte aligned
    static constexpr int MBUF_OFF = STAGES_BYTES + 2 * QBUF + BARS * 8 + SVALID_INTS * 4;
    static_assert(MBUF_OFF % 16 == 0 && (MBUF_FLOATS * 4) % 16 == 0, "16-byte aligned epilogue buffers");
    static constexpr size_t FIXED = 128 + STAGES_BYTES + 2 * QBUF + BARS * 8 + SVALID_INTS * 4 + MBUF_FLOATS * 4 +
                                    16 * 4 + ((EPI_BYTES + 15) / 16) * 16;
};

__device__ __forceinline__ int clamp_len(const DecodeArgs &a, int L) {
    const int cap = a.max_pages * kPageNodes;
    if (L > cap) {
        raise_flag(a.flags, FLAG_BAD_LENS);
        L = cap;
    }
    return L < 0 ? 0 : L;
}

__device__ __forceinline__ int clamp_entries(const DecodeArgs &a, int u) { return clamp_len(a, a.lens[u]); }

// largest v with prefix[v] <= f
__device__ __forceinline__ int find_vunit(const int *prefix, int nv, long long f) {
    int lo = 0, hi = nv;   // prefix[lo] <= f < prefix[hi] (prefix[nv] = total > f)
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= f) lo = mid;
        else hi = mid;
    }
    return lo;
}

// The same search by a whole warp (every lane gets the answer): each round tests 32 evenly spaced
// entries at once, so nv = 8192 takes three rounds of shared loads instead of thirteen dependent ones.
__device__ __forceinline__ int find_vunit_warp(const int *prefix, int nv, long long f, int lane) {
    int lo = 0, hi = nv;   // prefix[lo] <= f < prefix[hi]
    while (hi - lo > 32) {
        const int step = (hi - lo + 31) / 32;
        const int idx = lo + lane * step;
        const unsigned ok = __ballot_sync(0xffffffffu, idx < hi && prefix[idx] <= f);   // lane 0 always
        const int k = 31 - __clz(ok);
        lo += k * step;
        hi = min(lo + step, hi);
    }
    const unsigned ok = __ballot_sync(0xffffffffu, lo + lane < hi && prefix[lo + lane] <= f);
    return lo + 31 - __clz(ok);
}

// floor(x / n) for 0 <= x < 2^53 and n > 0, exact: x and n are exact doubles and the division is
// correctly rounded, so a quotient that is not an integer stays more than 1/n away from the next one
// (far above the rounding error), and an integer quotient is exact. Much cheaper than a 64-bit integer
// division.
__device__ __forceinline__ long long floor_div(long long x, long long n) {
    return static_cast<long long>(floor(static_cast<double>(x) / static_cast<double>(n)));
}

// Work of one piece besides its pages, in pages: the stream-K split balances pages plus this much
// per unit, since each piece costs its CTA a query-row load and an epilogue (the page-group merge
// and the output or partial stores) on top of its pages, so a split by pages alone left the CTAs
// holding many short units last (28 query rows per unit: 2, 4, 6 and 8 measured 62.3, 58.0, 56.8
// and 57.0 us on the ragged 2% workload).
constexpr int kPieceWork = 6;

// Every CTA rebuilds the page prefix over virtual units (flat index of each unit's first page) and
// keeps every unit's clamped entry count, both in shared memory (lens are tiny and L2-resident).
// Run by the consumer warps alone (named barrier 1), so the producer can start copies meanwhile.
// `spec`: before the dependency wait, with lens that may still change: L2-only loads (no stale line
// is left in L1) and no flag raised; the result is checked against a second read after the wait.
template <int NCONS>
__device__ __forceinline__ void build_prefix(const DecodeArgs &a, int *prefix, int *ents, int *scratch, bool spec) {
    const int nv = a.n_vunits;
    const int tid = threadIdx.x, nth = NCONS * 32;
    const int per = (nv + nth - 1) / nth;
    const int lo = min(tid * per, nv), hi = min(lo + per, nv);
    const int cap = a.max_pages * kPageNodes;
    int local = 0;
    for (int v = lo; v < hi; v += 4) {
        int raw[4];   // four loads in flight before any is used
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int32_t *p = a.lens + (v + j) / a.row_passes;
            raw[j] = v + j < hi ? (spec ? ld_global_cg_s32(p) : *p) : 0;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (v + j < hi) {
                const int L = spec ? min(max(raw[j], 0), cap) : clamp_len(a, raw[j]);
                const int pages = (L + kPageNodes - 1) / kPageNodes;
                ents[v + j] = L;
                prefix[v + j] = pages;   // page count for now; made exclusive below
                local += pages;
            }
    }
    const int lane = tid & 31, warp = tid >> 5;
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += n;
    }
    if (lane == 31) scratch[warp] = x;
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
    int wp = 0;
    for (int w = 0; w < warp; ++w) wp += scratch[w];
    int run = wp + x - local;
    for (int v = lo; v < hi; ++v) {
        const int pages = prefix[v];
        prefix[v] = run;
        run += pages;
    }
    if (tid == nth - 1) prefix[nv] = wp + x;
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
}

// After the dependency wait: read the lens again (flagging bad ones) and check every clamped count
// against the one the speculative prefix was built from. Consumer warps alone; the verdict is
// the same in every consumer thread.
template <int NCONS>
__device__ __forceinline__ bool lens_unchanged(const DecodeArgs &a, const int *ents) {
    const int nv = a.n_vunits;
    const int tid = threadIdx.x, nth = NCONS * 32;
    const int per = (nv + nth - 1) / nth;
    const int lo = min(tid * per, nv), hi = min(lo + per, nv);
    bool same = true;
    for (int v = lo; v < hi; v += 4) {
        int raw[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) raw[j] = v + j < hi ? a.lens[(v + j) / a.row_passes] : 0;
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (v + j < hi) same &= clamp_len(a, raw[j]) == ents[v + j];
    }
    return bar_and(1, NCONS * 32, same);
}

// The work prefix of the stream-K split (built only when the grid splits that way): a unit's work
// is its pages plus kPieceWork if it has any, wpre[v] = prefix[v] + kPieceWork * (nonempty units
// before v). Consumer warps alone, after build_prefix.
template <int NCONS>
__device__ __forceinline__ void build_work(const DecodeArgs &a, const int *prefix, int *wpre, int *scratch) {
    const int nv = a.n_vunits;
    const int tid = threadIdx.x, nth = NCONS * 32;
    const int per = (nv + nth - 1) / nth;
    const int lo = min(tid * per, nv), hi = min(lo + per, nv);
    int local = 0;
    for (int v = lo; v < hi; ++v) local += prefix[v + 1] > prefix[v] ? 1 : 0;
    const int lane = tid & 31, warp = tid >> 5;
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += n;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));   // scratch free (build_prefix read it)
    if (lane == 31) scratch[warp] = x;
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
    int wp = 0;
    for (int w = 0; w < warp; ++w) wp += scratch[w];
    int run = wp + x - local;
    for (int v = lo; v < hi; ++v) {
        wpre[v] = prefix[v] + kPieceWork * run;
        run += prefix[v + 1] > prefix[v] ? 1 : 0;
    }
    if (tid == nth - 1) wpre[nv] = prefix[nv] + kPieceWork * (wp + x);
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
}

// Flat page index at work position w: the pages of the units before w's unit, plus those of w's
// unit that lie before w (a unit's pages follow its kPieceWork in the work order). A whole warp.
// (Not inlined: inlined twice, the searches' registers pushed the streaming loop into spills.)
__device__ __noinline__ long long flat_of_work(const int *wpre, const int *prefix, int nv, long long w, int lane) {
    if (w >= wpre[nv]) return prefix[nv];
    const int v = find_vunit_warp(wpre, nv, w, lane);
    const long long pages = prefix[v + 1] - prefix[v];
    const long long into = w - (wpre[v + 1] - pages);
    return prefix[v] + (into < 0 ? 0 : (into > pages ? pages : into));
}

// The CTA whose (nonempty) range holds work position f.
__device__ __forceinline__ long long cta_of(long long f, long long ptot, int ncta) {
    return floor_div((f + 1) * ncta + ptot - 1, ptot) - 1;
}

// Pieces of the unit whose pages lie at work positions [ps, pe): their count, and the partial-slot
// code (cta * 2 + slot) of piece i. With ptot >= ncta every CTA range is nonempty: the pieces sit
// in CTAs c_first..c_last, the first in its tail slot (1), the others in their head slot (0). With
// ptot < ncta every nonempty range holds exactly one work position: piece i is position ps + i's
// CTA.
__device__ __forceinline__ int piece_count(long long ps, long long pe, long long ptot, int ncta) {
    if (ptot < ncta) return static_cast<int>(pe - ps);
    return static_cast<int>(cta_of(pe - 1, ptot, ncta) - cta_of(ps, ptot, ncta) + 1);
}

__device__ __forceinline__ int piece_code(int i, long long ps, long long ptot, int ncta, long long c_first) {
    const long long c = ptot < ncta ? cta_of(ps + i, ptot, ncta) : c_first + i;
    return static_cast<int>(c * 2 + (i == 0 ? 1 : 0));
}

// Log-sum-exp merge of the n pieces (partial-slot codes in shared memory) of virtual unit v,
// by the CTA that completed it: one warp per query row, lanes over dimensions. Up to kFastPieces
// pieces, every load of two rows is issued before any is used (one round trip to L2).
constexpr int kFastPieces = 6;

// What the merge of a split unit reads and writes
struct MergeArgs {
    const float *part_l, *part_v;
    void *out;
    float *lse;
    int row_passes, Hkv, pass_rows, rows, R, Hq, G;
};

template <int D>
__device__ __forceinline__ void merge_store(const MergeArgs &m, int b, int h, int row, int lane, const float *acc,
                                            float M, float Ls) {
    constexpr int DPL = D / 32;
    const long long oi = (static_cast<long long>(b) * m.R + row / m.G) * m.Hq + h * m.G + row % m.G;
    const float inv = Ls > 0.0f ? 1.0f / Ls : 0.0f;
    __nv_bfloat16 *dst = static_cast<__nv_bfloat16 *>(m.out) + oi * D + lane * DPL;
    if constexpr (DPL == 4) {
        uint2 w;
        w.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
        w.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
        *reinterpret_cast<uint2 *>(dst) = w;
    } else {
        *reinterpret_cast<uint32_t *>(dst) = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    }
    if (lane == 0) m.lse[oi] = Ls > 0.0f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
}

template <int D, int NCONS>
__device__ void merge_unit(const MergeArgs m, int v, const int *codes, int n, int warp, int lane) {
    constexpr int DPL = D / 32;   // dimensions per lane
    const int u = v / m.row_passes, rpass = v % m.row_passes;
    const int b = u / m.Hkv, h = u % m.Hkv;
    const int rows_here = min(m.pass_rows, m.rows - rpass * kRowsPerPass);
    if (n <= 2) {
        // the common split: two pieces. Rows in groups of four per warp (two with eight warps),
        // every load of a group issued before any is used: one round trip to L2 per group.
        constexpr int RPW = kRowsPerPass / NCONS, CH = NCONS >= 8 ? 2 : (RPW < 4 ? RPW : 4);
#pragma unroll 1
        for (int t0 = 0; t0 < RPW && warp + t0 * NCONS < rows_here; t0 += CH) {
            float lv[CH][2], xv[CH][2][DPL];
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                const int rr = warp + (t0 + t) * NCONS;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    lv[t][i] = -INFINITY;
#pragma unroll
                    for (int j = 0; j < DPL; ++j) xv[t][i][j] = 0.0f;
                    if (i < n && rr < rows_here) {
                        const long long pr = static_cast<long long>(codes[i]) * m.pass_rows + rr;
                        lv[t][i] = __ldcg(m.part_l + pr);
                        const float *src = m.part_v + pr * D + lane * DPL;
                        if constexpr (DPL == 4) {
                            const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
                            xv[t][i][0] = x.x; xv[t][i][1] = x.y; xv[t][i][2] = x.z; xv[t][i][3] = x.w;
                        } else {
                            const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
                            xv[t][i][0] = x.x; xv[t][i][1] = x.y;
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < CH; ++t) {
                const int rr = warp + (t0 + t) * NCONS;
                if (rr >= rows_here) continue;
                const float M = fmaxf(lv[t][0], lv[t][1]);
                const float Mb = M == -INFINITY ? 0.0f : M;
                const float w0 = ex2(lv[t][0] - Mb), w1 = ex2(lv[t][1] - Mb);   // -inf (absent piece): 0
                float acc[DPL];
#pragma unroll
                for (int j = 0; j < DPL; ++j) acc[j] = fmaf(w1, xv[t][1][j], w0 * xv[t][0][j]);
                merge_store<D>(m, b, h, rpass * kRowsPerPass + rr, lane, acc, M, w0 + w1);
            }
        }
        return;
    }
    if (n <= kFastPieces) {
        for (int r0 = warp; r0 < rows_here; r0 += 2 * NCONS) {
            float lv[2][kFastPieces], xv[2][kFastPieces][DPL];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int rr = r0 + t * NCONS;
#pragma unroll
                for (int i = 0; i < kFastPieces; ++i) {
                    lv[t][i] = -INFINITY;
#pragma unroll
                    for (int j = 0; j < DPL; ++j) xv[t][i][j] = 0.0f;
                    if (i < n && rr < rows_here) {
                        const long long pr = static_cast<long long>(codes[i]) * m.pass_rows + rr;
                        lv[t][i] = __ldcg(m.part_l + pr);
                        const float *src = m.part_v + pr * D + lane * DPL;
                        if constexpr (DPL == 4) {
                            const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
                            xv[t][i][0] = x.x; xv[t][i][1] = x.y; xv[t][i][2] = x.z; xv[t][i][3] = x.w;
                        } else {
                            const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
                            xv[t][i][0] = x.x; xv[t][i][1] = x.y;
                        }
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                const int rr = r0 + t * NCONS;
                if (rr >= rows_here) continue;
                float M = -INFINITY;
#pragma unroll
                for (int i = 0; i < kFastPieces; ++i) M = fmaxf(M, lv[t][i]);
                const float Mb = M == -INFINITY ? 0.0f : M;
                float acc[DPL], Ls = 0.0f;
#pragma unroll
                for (int j = 0; j < DPL; ++j) acc[j] = 0.0f;
#pragma unroll
                for (int i = 0; i < kFastPieces; ++i) {
                    const float w = ex2(lv[t][i] - Mb);   // -inf (absent piece) gives 0
                    Ls += w;
#pragma unroll
                    for (int j = 0; j < DPL; ++j) acc[j] = fmaf(w, xv[t][i][j], acc[j]);
                }
                merge_store<D>(m, b, h, rpass * kRowsPerPass + rr, lane, acc, M, Ls);
            }
        }
        return;
    }
    for (int rr = warp; rr < rows_here; rr += NCONS) {
        float M = -INFINITY;
        for (int base = 0; base < n; base += 32) {
            const int i = base + lane;
            M = fmaxf(M, i < n ? __ldcg(m.part_l + static_cast<long long>(codes[i]) * m.pass_rows + rr) : -INFINITY);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
        const float Mb = M == -INFINITY ? 0.0f : M;
        float acc[DPL], Ls = 0.0f;
#pragma unroll
        for (int j = 0; j < DPL; ++j) acc[j] = 0.0f;
        for (int base = 0; base < n; base += 32) {
            const int i = base + lane;
            const float wi =
                i < n ? ex2(__ldcg(m.part_l + static_cast<long long>(codes[i]) * m.pass_rows + rr) - Mb) : 0.0f;
            Ls += wi;
            const int cnt = min(32, n - base);
#pragma unroll 4
            for (int k = 0; k < cnt; ++k) {
                const float w = __shfl_sync(0xffffffffu, wi, k);
                const float *src =
                    m.part_v + (static_cast<long long>(codes[base + k]) * m.pass_rows + rr) * D + lane * DPL;
                if constexpr (DPL == 4) {
                    const float4 x = __ldcg(reinterpret_cast<const float4 *>(src));
                    acc[0] = fmaf(w, x.x, acc[0]);
                    acc[1] = fmaf(w, x.y, acc[1]);
                    acc[2] = fmaf(w, x.z, acc[2]);
                    acc[3] = fmaf(w, x.w, acc[3]);
                } else {
                    const float2 x = __ldcg(reinterpret_cast<const float2 *>(src));
                    acc[0] = fmaf(w, x.x, acc[0]);
                    acc[1] = fmaf(w, x.y, acc[1]);
                }
            }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, off);
        merge_store<D>(m, b, h, rpass * kRowsPerPass + rr, lane, acc, M, Ls);
    }
}

template <int D, int NT, bool DIAG>
__global__ void __launch_bounds__(SplitSmem<D, NT, DIAG>::THREADS, SplitSmem<D, NT, DIAG>::CTAS_PER_SM)
    k_decode_split(const DecodeArgs a) {
    using G = PageGeom<D, DIAG>;
    using L = SplitSmem<D, NT, DIAG>;
    constexpr int NCONS = L::CONS;           // consumer warps (the producer is warp NCONS)
    constexpr int NTHR = L::THREADS;
    constexpr bool MR = L::MR;               // query rows as the MMA's M dimension
    constexpr int PG = L::PG;                // page groups: warps sharing a row tile split the pages
    constexpr int NKS = D / 16;              // QK k-steps over dims == PV m-tiles over dims
    constexpr int NS = L::STAGES;            // ring depth
    static_assert(NS % PG == 0, "a stage's successive pages must go to one consumer warp");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);   // 128-byte aligned (measured faster)
    uint8_t *stages = smem;
    uint8_t *qbuf = stages + L::STAGES_BYTES;
    uint64_t *full = reinterpret_cast<uint64_t *>(qbuf + 2 * L::QBUF);
    uint64_t *empty = full + NS;
    uint64_t *qfull = empty + NS;
    uint64_t *qempty = qfull + 2;
    int *svalid = reinterpret_cast<int *>(qempty + 2);
    float *mbuf = reinterpret_cast<float *>(svalid + L::SVALID_INTS);
    int *misc = reinterpret_cast<int *>(mbuf + L::MBUF_FLOATS);
    // epilogue tables: output row index and merge weights per query row of the piece
    long long *orow = reinterpret_cast<long long *>(misc + 16);
    float *wrow = reinterpret_cast<float *>(orow + L::ROWS);
    int *prefix = reinterpret_cast<int *>(reinterpret_cast<uint8_t *>(misc + 16) + ((L::EPI_BYTES + 15) / 16) * 16);
    __shared__ int scan_scratch[NTHR / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nv = a.n_vunits;
    // aligned split: rank r > 0 of a cluster stores its piece into rank 0's receive buffer
    // (cluster - 1 blocks of pass_rows x (D + 1) floats behind the page prefix)
    int *ents = prefix + ((nv + 1 + 3) & ~3);   // entries of every virtual unit
    float *xbuf = reinterpret_cast<float *>(ents + ((nv + 3) & ~3));   // 16-byte aligned
    // The stream-K split's work prefix shares the receive buffer's storage. Only a busy CTA of an
    // aligned cluster launch has its receive buffer written by other CTAs; such a CTA always takes
    // the producer's guess (try_spec below), and with the guess the set-up, work prefix included,
    // runs only after the dependency wait and is final -- it builds the work prefix only if the
    // split is not aligned, when no CTA writes a receive buffer.
    int *wpre = reinterpret_cast<int *>(xbuf);
    cluster_arrive_relaxed();   // this CTA has started (waited on before any remote access)
    if (tid == 0) {   // independent of the inputs: overlaps the wait below
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], L::WPP);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], NCONS);
        }
        fence_mbar_init();
    }
    for (int i = tid; i < 2 * L::QBUF / 4; i += NTHR) reinterpret_cast<uint32_t *>(qbuf)[i] = 0u;
    fence_proxy_async_smem();   // the zeros land before the query-row copies
    // Speculation, set up before the inputs may be read. The aligned split below, if every unit
    // fills its page-table row (P0 = max_pages), gives this CTA the table columns [c0, c1) of
    // virtual unit vc. As soon as the inputs are readable the producer copies that unit's query
    // rows and the range's first pages while the consumers read the lens; if the lens confirm the
    // guess the ring just continues, otherwise the copies are drained, the barriers re-armed and
    // the general split runs (a wrong guess costs up to NS page reads).
    const int kcl = a.cluster;
    const int crank = blockIdx.x % kcl, vc = blockIdx.x / kcl;   // clusters are consecutive blocks
    // (a cluster of one CTA per unit counts as aligned when it keeps 3/4 of the grid busy: every CTA
    // then owns a whole unit and nothing is merged)
    const bool try_spec = (kcl > 1 || 4LL * nv >= 3LL * a.ncta) && vc < nv && a.max_pages >= kcl &&
                          static_cast<long long>(nv) * kcl <= a.ncta;
    const int c0 = try_spec ? a.max_pages * crank / kcl : 0;   // max_pages * 8 fits in an int
    const int c1 = try_spec ? a.max_pages * (crank + 1) / kcl : 0;
    const int n_first = min(NS, c1 - c0);
    __syncthreads();   // barriers initialised, qbuf zeroed
    // let the next launch in the stream become resident as our CTAs retire
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    // While the preceding grid may still run, warm L2 with the guessed range's first pages: the
    // page ids read here may be stale (the preceding grid may write the table), so they feed only
    // L2 prefetches -- a stale id costs a wasted read, never a wrong result -- and are read again
    // after the wait below (this read is L2-only, so it leaves no stale line in L1). Ids outside
    // the pool are not touched. (Issuing the first copies with these ids and checking them against
    // the second read made the consumers wait for that read: measured slower.)
    if (warp == NCONS && try_spec && lane < n_first) {
        const long long u = vc / a.row_passes;
        const int phys = ld_global_cg_s32(a.page_table + u * a.max_pages + c0 + lane);
        if (phys >= 0 && phys < a.num_pages)
            bulk_prefetch_l2(a.pages + static_cast<long long>(phys) * G::STAGE, G::STAGE);
    }
    // wait for every preceding grid to complete (its writes visible) before reading any input (the
    // consumer warps wait below, after their speculative set-up)
    if (warp >= NCONS) asm volatile("griddepcontrol.wait;" ::: "memory");
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q);
    int spec_page = -1;      // producer lane j: page id of column c0 + j
    uint32_t spec_bad = 0;   // producer: first pages whose id lies outside the pool
    if (warp == NCONS) {
        if (try_spec) {
            const int u = vc / a.row_passes, rpass = vc % a.row_passes;
            if (lane < c1 - c0)
                spec_page = ld_global_s32(a.page_table + static_cast<long long>(u) * a.max_pages + c0 + lane);
            const int b = u / a.Hkv, h = u % a.Hkv;
            const int p0 = rpass * kRowsPerPass, p1 = min(p0 + a.pass_rows, a.rows);
            if (lane == 0) mbar_arrive_expect_tx(&qfull[0], (p1 - p0) * D * 2);
            __syncwarp();
            for (int row = p0 + lane; row < p1; row += 32) {
                const __nv_bfloat16 *src =
                    q + ((static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G) * D;
                bulk_g2s(qbuf + (row - p0) * L::QROWB, src, D * 2, &qfull[0]);
            }
            // lane k copies page k of the range into stage k (all issued at once)
            bool bad = false;
            if (lane < n_first) {
                if (spec_page < 0 || spec_page >= a.num_pages) {   // flagged only if the guess holds
                    bad = true;
                    svalid[lane] = 0;
                    mbar_arrive(&full[lane]);
                } else {
                    svalid[lane] = 1;
                    mbar_arrive_expect_tx(&full[lane], G::STAGE);
                    // pages are read once per call: evict-first, so that they do not push the small
                    // inputs (tables, lengths, queries) out of L2
                    bulk_g2s_hint(stages + lane * G::STAGE, a.pages + static_cast<long long>(spec_page) * G::STAGE,
                                  G::STAGE, &full[lane], createpolicy_evict_first());
                }
            }
            spec_bad = __ballot_sync(0xffffffffu, bad);
        }
        cluster_wait();   // pairs with the arrival above (the producer touches no remote memory)
        asm volatile("bar.sync 2, %0;" ::"n"(NTHR));   // the consumers' verdict and prefix
    } else {
        // Without the producer's guess (the stream-K split is likely), the set-up -- page prefix,
        // work prefix and this CTA's range -- first runs before the dependency wait on lens that
        // may be stale (misc[11..13]: the range's first and end flat page and first virtual unit,
        // misc[14] = 1), and is kept if the lens read after the wait are the same; otherwise, and
        // with the guess, it runs after the wait (where the producer's copies, not the set-up, are
        // the critical path).
        bool have = false;
        bool waited = false;
        // (built for the many-row shapes only: the code slowed the 7-row decode measurably even
        // where it did not run)
        if constexpr (MR) {
            if (!try_spec) {
                waited = true;
                build_prefix<NCONS>(a, prefix, ents, scan_scratch, true);
                const int P0s = prefix[1] - prefix[0];
                bool unis = true;
                {
                    const int per = (nv + NCONS * 32 - 1) / (NCONS * 32);
                    for (int v = min(tid * per, nv); v < min(tid * per + per, nv); ++v)
                        unis &= (prefix[v + 1] - prefix[v] == P0s);
                }
                unis = bar_and(1, NCONS * 32, unis);
                const bool als = unis && (kcl > 1 || 4LL * nv >= 3LL * a.ncta) && P0s >= kcl &&
                                 static_cast<long long>(nv) * kcl <= a.ncta;
                if (!als) {
                    build_work<NCONS>(a, prefix, wpre, scan_scratch);
                    if (warp == 0) {
                        const long long ptot_ = wpre[nv];
                        const long long pa_ = flat_of_work(wpre, prefix, nv, floor_div(ptot_ * blockIdx.x, a.ncta), lane);
                        const long long pb_ =
                            flat_of_work(wpre, prefix, nv, floor_div(ptot_ * (blockIdx.x + 1), a.ncta), lane);
                        const int v0_ = pa_ < pb_ ? find_vunit_warp(prefix, nv, pa_, lane) : 0;
                        if (lane == 0) {
                            misc[11] = static_cast<int>(pa_);
                            misc[12] = static_cast<int>(pb_);
                            misc[13] = v0_;
                        }
                    }
                }
                asm volatile("griddepcontrol.wait;" ::: "memory");
                have = lens_unchanged<NCONS>(a, ents) && !als;
                if (have && tid == 0) {
                    misc[8] = 0;
                    misc[9] = 0;
                }
            }
        }
        if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");
        if (MR && tid == 0) misc[14] = have ? 1 : 0;
        if (!have) {
            build_prefix<NCONS>(a, prefix, ents, scan_scratch, false);
            const int P0 = prefix[1] - prefix[0];
            bool uni = true;
            {
                const int per = (nv + NCONS * 32 - 1) / (NCONS * 32);
                for (int v = min(tid * per, nv); v < min(tid * per + per, nv); ++v)
                    uni &= (prefix[v + 1] - prefix[v] == P0);
            }
            uni = bar_and(1, NCONS * 32, uni);
            const bool al = uni && (kcl > 1 || 4LL * nv >= 3LL * a.ncta) && P0 >= kcl &&
                            static_cast<long long>(nv) * kcl <= a.ncta;
            if (tid == 0) {
                misc[8] = al ? 1 : 0;
                misc[9] = (al && try_spec && P0 == a.max_pages) ? 1 : 0;
            }
            if (!al) build_work<NCONS>(a, prefix, wpre, scan_scratch);
        }
        cluster_wait();   // every CTA of the cluster has started
        asm volatile("bar.arrive 2, %0;" ::"n"(NTHR));
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));   // misc visible to every consumer
    }
    const bool aligned = misc[8] != 0;
    const bool spec_ok = misc[9] != 0;
    bool alive = true;
    if (try_spec && !spec_ok) {
        // wrong guess: wait for the speculative copies, then re-arm every barrier
        if (warp == NCONS) {
            bool ok = true;
            for (int k = 0; k < n_first; ++k) ok &= mbar_wait(&full[k], 0);
            ok &= mbar_wait(&qfull[0], 0);
            if (lane == 0) misc[10] = ok ? 1 : 0;
            if (!ok && lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
        }
        __syncthreads();
        alive = misc[10] != 0;
        if (tid == 0 && alive) {
            for (int s2 = 0; s2 < NS; ++s2) {
                mbar_inval(&full[s2]);
                mbar_inval(&empty[s2]);
                mbar_init(&full[s2], 1);
                mbar_init(&empty[s2], L::WPP);
            }
            for (int s2 = 0; s2 < 2; ++s2) {
                mbar_inval(&qfull[s2]);
                mbar_inval(&qempty[s2]);
                mbar_init(&qfull[s2], 1);
                mbar_init(&qempty[s2], NCONS);
            }
            fence_mbar_init();
        }
        __syncthreads();
    }
    const long long ptot = aligned ? 0 : wpre[nv];   // total work of the stream-K split
    const int P0 = prefix[1] - prefix[0];
    const bool have_range = MR && misc[14] != 0;
    long long pa, pb;   // this CTA's flat pages
    if (aligned) {
        pa = vc < nv ? prefix[vc] + P0 * crank / kcl : 0;
        pb = vc < nv ? prefix[vc] + P0 * (crank + 1) / kcl : 0;
    } else if (have_range) {
        pa = misc[11];
        pb = misc[12];
    } else {
        pa = flat_of_work(wpre, prefix, nv, floor_div(ptot * blockIdx.x, a.ncta), lane);
        pb = flat_of_work(wpre, prefix, nv, floor_div(ptot * (blockIdx.x + 1), a.ncta), lane);
    }
    __nv_bfloat16 *outp = static_cast<__nv_bfloat16 *>(a.out);
    if (warp < NCONS) {
        // units with no entries get out = 0, lse = -inf (spread over the CTAs)
        for (int v = blockIdx.x; v < nv; v += a.ncta) {
            if (prefix[v + 1] != prefix[v]) continue;
            const int u = v / a.row_passes, rpass = v % a.row_passes;
            const int b = u / a.Hkv, h = u % a.Hkv;
            for (int idx = tid; idx < a.pass_rows * D; idx += NCONS * 32) {
                const int rr = idx / D, dim = idx % D;
                const int row = rpass * kRowsPerPass + rr;
                if (row >= a.rows) continue;
                const long long oi = (static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G;
                outp[oi * D + dim] = __float2bfloat16_rn(0.0f);
                if (dim == 0) a.lse[oi] = -INFINITY;
            }
        }
    }
    if (pa >= pb) return;
    const int v0 = aligned ? vc : (have_range ? misc[13] : find_vunit_warp(prefix, nv, pa, lane));
    const int n_my = static_cast<int>(pb - pa);

    if (warp == NCONS) {
        // ----------------------------- producer -----------------------------
        // a confirmed guess has issued piece 0's query rows and pages [0, n_first) already
        int v = spec_ok ? vc : -1, pi = spec_ok ? 0 : -1;   // current (nonempty) piece
        const int i_first = spec_ok ? n_first : 0;
        if (spec_ok && spec_bad != 0 && lane == 0) raise_flag(a.flags, FLAG_BAD_PAGE);
        // the query rows of piece vq into slot `slot` of the double buffer
        auto copy_q = [&](int vq, int slot) {
            const int u = vq / a.row_passes, rpass = vq % a.row_passes;
            const int b = u / a.Hkv, h = u % a.Hkv;
            const int p0 = rpass * kRowsPerPass, p1 = min(p0 + a.pass_rows, a.rows);
            if (lane == 0) mbar_arrive_expect_tx(&qfull[slot], (p1 - p0) * D * 2);
            __syncwarp();
            for (int row = p0 + lane; row < p1; row += 32) {
                const __nv_bfloat16 *src =
                    q + ((static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G) * D;
                bulk_g2s(qbuf + slot * L::QBUF + (row - p0) * L::QROWB, src, D * 2, &qfull[slot]);
            }
        };
        if (!spec_ok && alive) {   // the first piece's query rows need no page id: copy them first
            v = v0;
            pi = 0;
            copy_q(v, 0);
        }
        for (int base = 0; base < n_my && alive; base += 32) {
            int my_page = -1;
            if (base == 0 && spec_ok) {
                my_page = spec_page;   // the same columns, read before the lens were known
            } else if (base + lane < n_my) {
                const long long f = pa + base + lane;
                const int vv = find_vunit(prefix, nv, f);
                my_page = a.page_table[static_cast<long long>(vv / a.row_passes) * a.max_pages + (f - prefix[vv])];
            }
            const int cnt = min(32, n_my - base);
            for (int k = base < i_first ? i_first - base : 0; k < cnt; ++k) {
                const int i = base + k;
                const long long f = pa + i;
                if (v < 0 || f >= prefix[v + 1]) {
                    // first page of the next piece: copy its query rows first
                    v = find_vunit(prefix, nv, f);
                    ++pi;
                    const int slot = pi & 1;
                    if (pi >= 2 && !mbar_wait(&qempty[slot], ((pi >> 1) - 1) & 1)) {
                        if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                        alive = false;
                        break;
                    }
                    copy_q(v, slot);
                }
                const int s = i % NS;
                const int phys = __shfl_sync(0xffffffffu, my_page, k);
                if (i >= NS && !mbar_wait(&empty[s], ((i / NS) - 1) & 1)) {
                    if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                    alive = false;
                    break;
                }
                if (lane == 0) {
                    if (phys < 0 || phys >= a.num_pages) {
                        raise_flag(a.flags, FLAG_BAD_PAGE);
                        svalid[s] = 0;
                        mbar_arrive(&full[s]);
                    } else {
                        svalid[s] = 1;
                        mbar_arrive_expect_tx(&full[s], G::STAGE);
                        // a page is one contiguous [keys | values | alpha,beta] block: one copy
                        bulk_g2s_hint(stages + s * G::STAGE, a.pages + static_cast<long long>(phys) * G::STAGE,
                                      G::STAGE, &full[s], createpolicy_evict_first());
                    }
                }
                __syncwarp();
            }
        }
        if (aligned && kcl > 1) cluster_sync();   // the producer joins the consumers' cluster barrier
        return;
    }

    // ------------------------------- consumers -------------------------------
    // warp's row-tile group and page group (one n8 row tile nt = wt per warp; with rows as M, the
    // 16 rows of tiles 2 wt and 2 wt + 1)
    const int wt = warp % L::WPP, pg = warp / L::WPP;
    const int nt = wt;
    const int g = lane >> 2, c = lane & 3;
    const int ctid = tid;   // 0 .. NCONS * 32 - 1
    const float c_scale = kLog2e * rsqrtf(static_cast<float>(D));
    constexpr int MST = L::MST, WST = L::WST;
    int i0 = 0, pi = 0;
    int split_v[2] = {0, 0}, split_ps[2] = {0, 0}, split_pe[2] = {0, 0}, n_split = 0;   // (thread 0)
    int early_prev = -1;   // (thread 0) the count returned for the range's first piece, if counted early
    for (int v = v0; v < nv && prefix[v] < pb; ++v) {
        const long long ps = prefix[v], pe = prefix[v + 1];   // the unit's flat pages
        const int lo = static_cast<int>(max(pa, ps) - ps), hi = static_cast<int>(min(pb, pe) - ps);
        const int npg = hi - lo;
        if (npg <= 0) continue;   // an empty unit: written in the prologue
        const int u = v / a.row_passes, rpass = v % a.row_passes;
        const int b = u / a.Hkv, h = u % a.Hkv;
        const int Lent = ents[v];
        const int rows_here = min(a.pass_rows, a.rows - rpass * kRowsPerPass);
        if (ctid < rows_here) {   // output row of each query row (read after the page loop)
            const int row = rpass * kRowsPerPass + ctid;
            orow[ctid] = (static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G;
        }

        if constexpr (MR) {
            // ---- query rows as the MMA's M dimension (16 or more rows per unit) ----
            // Warp (wt, pg) takes rows 16 wt .. 16 wt + 15 of the piece for every page of its page
            // group: S (16 rows x 16 nodes) = Q K^T as two n8 tiles of nodes, the softmax on the
            // accumulators (each row spread over a quad of lanes), and P -- whose accumulator
            // layout is already the A operand of the next product -- times V into O (16 rows x D).
            // The A fragments of Q (rows g / g + 8, dims 2c, 2c + 1 (+ 8) of each k-step) are read
            // from the piece's query slot at every k-step rather than held in 32 registers across
            // the page loop; the slot is released at the piece's end.
            float qn_g = 0.0f, qn_h = 0.0f;   // |q|^2 of rows g and g + 8 (h: the row 8 below)
            const int qslot = pi & 1;
            const uint32_t qb =
                smem_u32(qbuf + qslot * L::QBUF) + (wt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1)) * L::QROWB;
            {
                if (alive && !mbar_wait(&qfull[qslot], (pi >> 1) & 1)) {
                    if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                    alive = false;
                }
#pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    uint32_t qf[4];
                    ldsm_x4(qb + ((2 * ks + (lane >> 4)) << 4), qf[0], qf[1], qf[2], qf[3]);
#pragma unroll
                    for (int r2 = 0; r2 < 4; r2 += 2) {
                        const uint32_t wg = qf[r2], wh = qf[r2 + 1];
                        qn_g = fmaf(bf16lo(wg), bf16lo(wg), qn_g);
                        qn_g = fmaf(bf16hi(wg), bf16hi(wg), qn_g);
                        qn_h = fmaf(bf16lo(wh), bf16lo(wh), qn_h);
                        qn_h = fmaf(bf16hi(wh), bf16hi(wh), qn_h);
                    }
                }
#pragma unroll
                for (int off = 1; off < 4; off <<= 1) {
                    qn_g += __shfl_xor_sync(0xffffffffu, qn_g, off);
                    qn_h += __shfl_xor_sync(0xffffffffu, qn_h, off);
                }
            }
            float m_g = -INFINITY, m_h = -INFINITY, l_g = 0.0f, l_h = 0.0f;
            float o[2 * NKS][4];   // d-tile j: rows g / g + 8, dims 8 j + 2c, 8 j + 2c + 1
#pragma unroll
            for (int j = 0; j < 2 * NKS; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;

            for (int k = ((pg - i0 % PG) + PG) % PG; k < npg && alive; k += PG) {
                const int i = i0 + k;
                const int s = i % NS;
                if (!mbar_wait(&full[s], (i / NS) & 1)) {
                    if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                    alive = false;
                    break;
                }
                const bool valid = svalid[s] != 0;
                const int nvalid = min(kPageNodes, Lent - (lo + k) * kPageNodes);
                if (valid) {
                    const uint32_t kb = smem_u32(stages + s * G::STAGE);
                    const uint32_t vb = kb + G::VEC_BYTES;
                    const float4 *ab4 = reinterpret_cast<const float4 *>(stages + s * G::STAGE + 2 * G::VEC_BYTES);
                    const int mi = lane >> 3;
                    // S = Q K^T: the x4 load of K rows at a k-step holds nodes 0-7 (r0, r2) and 8-15
                    // (r1, r3) as the B fragments of the two node tiles; the next k-step's load is
                    // issued before this one's MMAs
                    float sacc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
                    // odd k-steps accumulate apart: two chains of four dependent MMAs per node tile
                    float sodd[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
                    {
                        const int node = (lane & 7) + 8 * (mi & 1);
                        uint32_t kn[4], qn[4];
                        ldsm_x4(kb + node * G::ROWB + (swz(mi >> 1, node) << 4), kn[0], kn[1], kn[2], kn[3]);
                        ldsm_x4(qb + ((lane >> 4) << 4), qn[0], qn[1], qn[2], qn[3]);
#pragma unroll
                        for (int ks = 0; ks < NKS; ++ks) {
                            const uint32_t k0 = kn[0], k1 = kn[1], k2 = kn[2], k3 = kn[3];
                            const uint32_t q0 = qn[0], q1 = qn[1], q2 = qn[2], q3 = qn[3];
                            if (ks + 1 < NKS) {
                                ldsm_x4(kb + node * G::ROWB + (swz(2 * (ks + 1) + (mi >> 1), node) << 4), kn[0], kn[1],
                                        kn[2], kn[3]);
                                ldsm_x4(qb + ((2 * (ks + 1) + (lane >> 4)) << 4), qn[0], qn[1], qn[2], qn[3]);
                            }
                            mma_bf16((ks & 1) ? sodd[0] : sacc[0], q0, q1, q2, q3, k0, k2);
                            mma_bf16((ks & 1) ? sodd[1] : sacc[1], q0, q1, q2, q3, k1, k3);
                        }
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int r = 0; r < 4; ++r) sacc[nt][r] += sodd[nt][r];
                    }
                    // logits of nodes 8 nt + 2c + e for rows g (accumulator e) and g + 8 (2 + e)
                    const float4 abA = ab4[c], abB = ab4[4 + c];   // nodes 2c, 2c+1 and 8+2c, 9+2c
                    const float al[2][2] = {{abA.x, abA.z}, {abB.x, abB.z}};
                    const float be[2][2] = {{abA.y, abA.w}, {abB.y, abB.w}};
                    float sg[2][2], sh[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const bool in = 8 * nt + 2 * c + e < nvalid;
                            sg[nt][e] = in ? fmaf(sacc[nt][e], c_scale, kLog2e * fmaf(qn_g, be[nt][e], al[nt][e])) : -INFINITY;
                            sh[nt][e] = in ? fmaf(sacc[nt][2 + e], c_scale, kLog2e * fmaf(qn_h, be[nt][e], al[nt][e]))
                                           : -INFINITY;
                        }
                    float mxg = fmaxf(fmaxf(sg[0][0], sg[0][1]), fmaxf(sg[1][0], sg[1][1]));
                    float mxh = fmaxf(fmaxf(sh[0][0], sh[0][1]), fmaxf(sh[1][0], sh[1][1]));
#pragma unroll
                    for (int off = 1; off < 4; off <<= 1) {
                        mxg = fmaxf(mxg, __shfl_xor_sync(0xffffffffu, mxg, off));
                        mxh = fmaxf(mxh, __shfl_xor_sync(0xffffffffu, mxh, off));
                    }
                    const bool ug = mxg > m_g + kLazyMax, uh = mxh > m_h + kLazyMax;   // move the reference?
                    const float ng = ug ? mxg : m_g, nh = uh ? mxh : m_h;
                    const float bg = ng == -INFINITY ? 0.0f : ng, bh = nh == -INFINITY ? 0.0f : nh;
                    const float cg = ug ? ex2(m_g - bg) : 1.0f, ch = uh ? ex2(m_h - bh) : 1.0f;
                    float pg_[2][2], ph_[2][2];
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            pg_[nt][e] = ex2(sg[nt][e] - bg);
                            ph_[nt][e] = ex2(sh[nt][e] - bh);
                        }
                    l_g = fmaf(l_g, cg, (pg_[0][0] + pg_[0][1]) + (pg_[1][0] + pg_[1][1]));
                    l_h = fmaf(l_h, ch, (ph_[0][0] + ph_[0][1]) + (ph_[1][0] + ph_[1][1]));
                    m_g = ng;
                    m_h = nh;
                    if (__any_sync(0xffffffffu, ug || uh)) {
#pragma unroll
                        for (int j = 0; j < 2 * NKS; ++j) {
                            o[j][0] *= cg;
                            o[j][1] *= cg;
                            o[j][2] *= ch;
                            o[j][3] *= ch;
                        }
                    }
                    // P (16 rows x 16 nodes) as the A operand: accumulator layout, packed to bf16
                    const uint32_t pa0 = pack_bf16x2(pg_[0][0], pg_[0][1]), pa1 = pack_bf16x2(ph_[0][0], ph_[0][1]);
                    const uint32_t pa2 = pack_bf16x2(pg_[1][0], pg_[1][1]), pa3 = pack_bf16x2(ph_[1][0], ph_[1][1]);
                    // O += P V: the transposed x4 load of V at a pair of d-tiles holds nodes 0-7 of both
                    // (r0, r1) and nodes 8-15 of both (r2, r3). Slots past the unit's last entry may
                    // hold anything (NaN included): their V elements are zeroed, since P = 0 does not
                    // cancel NaN (b0 holds nodes 2c, 2c + 1; b1 nodes 2c + 8, 2c + 9).
                    const uint32_t m_lo = nvalid == kPageNodes ? 0xffffffffu
                                          : (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
                    const uint32_t m_hi = nvalid == kPageNodes ? 0xffffffffu
                                          : (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
                    {
                        const int node = (lane & 7) + 8 * (mi >> 1);
                        uint32_t vn[4];
                        ldsm_x4_t(vb + node * G::ROWB + (swz(mi & 1, node) << 4), vn[0], vn[1], vn[2], vn[3]);
#pragma unroll
                        for (int mt = 0; mt < NKS; ++mt) {
                            const uint32_t v0 = vn[0] & m_lo, v1 = vn[1] & m_lo, v2 = vn[2] & m_hi, v3 = vn[3] & m_hi;
                            if (mt + 1 < NKS)
                                ldsm_x4_t(vb + node * G::ROWB + (swz(2 * (mt + 1) + (mi & 1), node) << 4), vn[0], vn[1],
                                          vn[2], vn[3]);
                            mma_bf16(o[2 * mt], pa0, pa1, pa2, pa3, v0, v2);
                            mma_bf16(o[2 * mt + 1], pa0, pa1, pa2, pa3, v1, v3);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);   // K and V read: release the stage
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&qempty[qslot]);   // the piece's query rows are no longer read
            i0 += npg;
            ++pi;

            // ---- piece epilogue: O, m, l of rows g and g + 8 into the page-group buffer (the
            // n8 row tiles 2 wt and 2 wt + 1 of the one-tile layout) ----
#pragma unroll
            for (int off = 1; off < 4; off <<= 1) {
                l_g += __shfl_xor_sync(0xffffffffu, l_g, off);
                l_h += __shfl_xor_sync(0xffffffffu, l_h, off);
            }
            float *mw0 = mbuf + ((pg * NT + 2 * wt) * 8 + g) * MST;
            float *mw1 = mbuf + ((pg * NT + 2 * wt + 1) * 8 + g) * MST;
#pragma unroll
            for (int j = 0; j < 2 * NKS; ++j) {
                *reinterpret_cast<float2 *>(mw0 + 8 * j + 2 * c) = make_float2(o[j][0], o[j][1]);
                *reinterpret_cast<float2 *>(mw1 + 8 * j + 2 * c) = make_float2(o[j][2], o[j][3]);
            }
            if (c == 0) {
                mw0[D] = m_g;
                mw0[D + 1] = l_g;
                mw1[D] = m_h;
                mw1[D + 1] = l_h;
            }
        } else {
            // Q^T fragments of rows nt*8 + g of this piece (ldmatrix from the producer's copy), |q|^2
            uint32_t qf[NKS][2];
            float qn = 0.0f;
            {
                const int slot = pi & 1;
                if (alive && !mbar_wait(&qfull[slot], (pi >> 1) & 1)) {
                    if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                    alive = false;
                }
                const uint32_t qb = smem_u32(qbuf + slot * L::QBUF) + (nt * 8 + (lane & 7)) * L::QROWB;
    #pragma unroll
                for (int k2 = 0; k2 < NKS / 2; ++k2)
                    ldsm_x4(qb + ((4 * k2 + (lane >> 3)) << 4), qf[2 * k2][0], qf[2 * k2][1], qf[2 * k2 + 1][0],
                            qf[2 * k2 + 1][1]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&qempty[slot]);
    #pragma unroll
                for (int ks = 0; ks < NKS; ++ks) {
                    const uint32_t w0 = qf[ks][0], w1 = qf[ks][1];
                    qn = fmaf(bf16lo(w0), bf16lo(w0), qn);
                    qn = fmaf(bf16hi(w0), bf16hi(w0), qn);
                    qn = fmaf(bf16lo(w1), bf16lo(w1), qn);
                    qn = fmaf(bf16hi(w1), bf16hi(w1), qn);
                }
            }
            // diagonal closure: q_i^2 as the B operand of Var (16 x D) (q^2)^T, split into bf16 hi + lo
            // (q^2 of a bf16 q has at most 16 significant bits: hi + lo holds it exactly)
            uint32_t q2h[DIAG ? NKS : 1][2], q2l[DIAG ? NKS : 1][2];
            if constexpr (DIAG) {
    #pragma unroll
                for (int ks = 0; ks < NKS; ++ks)
    #pragma unroll
                    for (int r2 = 0; r2 < 2; ++r2) {
                        const float lo2 = bf16lo(qf[ks][r2]), hi2 = bf16hi(qf[ks][r2]);
                        const float slo = lo2 * lo2, shi = hi2 * hi2;
                        const uint32_t h2 = pack_bf16x2(slo, shi);
                        q2h[ks][r2] = h2;
                        q2l[ks][r2] = pack_bf16x2(slo - bf16lo(h2), shi - bf16hi(h2));
                    }
            }
            qn += __shfl_xor_sync(0xffffffffu, qn, 1);
            qn += __shfl_xor_sync(0xffffffffu, qn, 2);
            const float qn_r0 = __shfl_sync(0xffffffffu, qn, (2 * c) * 4);
            const float qn_r1 = __shfl_sync(0xffffffffu, qn, (2 * c + 1) * 4);

            float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.0f, 0.0f};
            float o[NKS][4];
    #pragma unroll
            for (int mt = 0; mt < NKS; ++mt) o[mt][0] = o[mt][1] = o[mt][2] = o[mt][3] = 0.0f;

            // page i of the CTA's range goes to page group i % PG (global index, not piece-local)
            for (int k = ((pg - i0 % PG) + PG) % PG; k < npg && alive; k += PG) {
                const int i = i0 + k;
                const int s = i % NS;
                if (!mbar_wait(&full[s], (i / NS) & 1)) {
                    if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                    alive = false;
                    break;
                }
                const bool valid = svalid[s] != 0;
                const int nvalid = min(kPageNodes, Lent - (lo + k) * kPageNodes);
                // S^T accumulators: even and odd k-steps apart, so that no chain of dependent MMAs is
                // longer than NKS / 2
                float sacc[2][4] = {{0.0f, 0.0f, 0.0f, 0.0f}, {0.0f, 0.0f, 0.0f, 0.0f}};
                float cacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // diagonal closure: sum_i q_i^2 var_i
                uint32_t vf[NKS][4];
                float2 ab0 = make_float2(0.0f, 0.0f), ab1 = ab0;
                if (valid) {
                    const uint32_t kb = smem_u32(stages + s * G::STAGE);
                    const uint32_t vb = kb + G::VEC_BYTES;
                    const float2 *ab = reinterpret_cast<const float2 *>(stages + s * G::STAGE + 2 * G::VEC_BYTES);
                    // S^T (16 nodes x 8 rows) = K (16 x D) Q^T (D x 8): every K fragment first
                    // (independent shared loads), then the MMAs
                    {
                        const int mi = lane >> 3, node = (lane & 7) + 8 * (mi & 1);
                        uint32_t kf[NKS][4];
    #pragma unroll
                        for (int ks = 0; ks < NKS; ++ks)
                            ldsm_x4(kb + node * G::ROWB + (swz(2 * ks + (mi >> 1), node) << 4), kf[ks][0], kf[ks][1],
                                    kf[ks][2], kf[ks][3]);
    #pragma unroll
                        for (int ks = 0; ks < NKS; ++ks)
                            mma_bf16(sacc[ks & 1], kf[ks][0], kf[ks][1], kf[ks][2], kf[ks][3], qf[ks][0], qf[ks][1]);
                        if constexpr (DIAG) {   // C^T (16 nodes x 8 rows) = Var (16 x D) (q^2)^T
                            const uint32_t varb = kb + G::VAR_OFF;
    #pragma unroll
                            for (int ks = 0; ks < NKS; ++ks) {
                                const int chunk = 2 * ks + (mi >> 1);
                                uint32_t a0, a1, a2, a3;
                                ldsm_x4(varb + node * G::ROWB + (swz(chunk, node) << 4), a0, a1, a2, a3);
                                mma_bf16(cacc, a0, a1, a2, a3, q2h[ks][0], q2h[ks][1]);
                                mma_bf16(cacc, a0, a1, a2, a3, q2l[ks][0], q2l[ks][1]);
                            }
                        }
                    }
                    // V^T fragments (A operand of O^T = V^T P^T) into registers now, so the stage goes
                    // back to the producer before the softmax
                    {
                        const int mi = lane >> 3, node = (lane & 7) + 8 * (mi >> 1);
    #pragma unroll
                        for (int mt = 0; mt < NKS; ++mt)
                            ldsm_x4_t(vb + node * G::ROWB + (swz(2 * mt + (mi & 1), node) << 4), vf[mt][0], vf[mt][1],
                                      vf[mt][2], vf[mt][3]);
                    }
                    ab0 = ab[g];
                    ab1 = ab[g + 8];
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);   // the page is in registers: release the stage
                if (valid) {
                    float sl[4];
                    // closure: |q|^2 beta, or sum_i q_i^2 var_i / (2d) with the diagonal variances
                    constexpr float kInv2d = 0.5f / D;
                    const float cl0 = DIAG ? fmaf(cacc[0], kInv2d, ab0.x) : fmaf(qn_r0, ab0.y, ab0.x);
                    const float cl1 = DIAG ? fmaf(cacc[1], kInv2d, ab0.x) : fmaf(qn_r1, ab0.y, ab0.x);
                    const float cl2 = DIAG ? fmaf(cacc[2], kInv2d, ab1.x) : fmaf(qn_r0, ab1.y, ab1.x);
                    const float cl3 = DIAG ? fmaf(cacc[3], kInv2d, ab1.x) : fmaf(qn_r1, ab1.y, ab1.x);
                    sl[0] = g < nvalid ? fmaf(sacc[0][0] + sacc[1][0], c_scale, kLog2e * cl0) : -INFINITY;
                    sl[1] = g < nvalid ? fmaf(sacc[0][1] + sacc[1][1], c_scale, kLog2e * cl1) : -INFINITY;
                    sl[2] = g + 8 < nvalid ? fmaf(sacc[0][2] + sacc[1][2], c_scale, kLog2e * cl2) : -INFINITY;
                    sl[3] = g + 8 < nvalid ? fmaf(sacc[0][3] + sacc[1][3], c_scale, kLog2e * cl3) : -INFINITY;
                    float mx0 = fmaxf(sl[0], sl[2]), mx1 = fmaxf(sl[1], sl[3]);
    #pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                    }
                    const bool u0 = mx0 > m_run[0] + kLazyMax, u1 = mx1 > m_run[1] + kLazyMax;   // move the reference?
                    const float mn0 = u0 ? mx0 : m_run[0], mn1 = u1 ? mx1 : m_run[1];
                    const float base0 = mn0 == -INFINITY ? 0.0f : mn0;
                    const float base1 = mn1 == -INFINITY ? 0.0f : mn1;
                    const float corr0 = u0 ? ex2(m_run[0] - base0) : 1.0f, corr1 = u1 ? ex2(m_run[1] - base1) : 1.0f;
                    const float p0 = ex2(sl[0] - base0), p1 = ex2(sl[1] - base1);
                    const float p2 = ex2(sl[2] - base0), p3 = ex2(sl[3] - base1);
                    l_run[0] = fmaf(l_run[0], corr0, p0 + p2);
                    l_run[1] = fmaf(l_run[1], corr1, p1 + p3);
                    m_run[0] = mn0;
                    m_run[1] = mn1;
                    if (__any_sync(0xffffffffu, u0 || u1)) {
    #pragma unroll
                        for (int mt = 0; mt < NKS; ++mt) {
                            o[mt][0] *= corr0;
                            o[mt][1] *= corr1;
                            o[mt][2] *= corr0;
                            o[mt][3] *= corr1;
                        }
                    }
                    // P^T as the B operand (16 nodes x 8 rows): transpose the 8x8 halves in registers
                    const uint32_t bp0 = movmatrix_t(pack_bf16x2(p0, p1));
                    const uint32_t bp1 = movmatrix_t(pack_bf16x2(p2, p3));
                    // O^T (D x 8) += V^T (D x 16) P^T (16 x 8)
                    if (nvalid == kPageNodes) {
    #pragma unroll
                        for (int mt = 0; mt < NKS; ++mt) mma_bf16(o[mt], vf[mt][0], vf[mt][1], vf[mt][2], vf[mt][3], bp0, bp1);
                    } else {
                        // slots past the unit's last entry may hold anything (NaN included): zero their
                        // V^T elements, since P = 0 does not cancel NaN in the product. This thread's
                        // fragment holds nodes 2c, 2c+1 (a0..a3) and 2c+8, 2c+9 (a4..a7).
                        const uint32_t m_lo =
                            (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
                        const uint32_t m_hi =
                            (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
    #pragma unroll
                        for (int mt = 0; mt < NKS; ++mt)
                            mma_bf16(o[mt], vf[mt][0] & m_lo, vf[mt][1] & m_lo, vf[mt][2] & m_hi, vf[mt][3] & m_hi, bp0,
                                     bp1);
                    }
                }
            }
            i0 += npg;
            ++pi;

            // ---- piece epilogue: merge the page groups through shared memory ----
    #pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
                l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], off);
                l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], off);
            }
            float *mw = mbuf + warp * 8 * MST;
    #pragma unroll
            for (int mt = 0; mt < NKS; ++mt) {
                mw[(2 * c) * MST + 16 * mt + g] = o[mt][0];
                mw[(2 * c + 1) * MST + 16 * mt + g] = o[mt][1];
                mw[(2 * c) * MST + 16 * mt + g + 8] = o[mt][2];
                mw[(2 * c + 1) * MST + 16 * mt + g + 8] = o[mt][3];
            }
            if (g == 0) {
                mw[(2 * c) * MST + D] = m_run[0];
                mw[(2 * c) * MST + D + 1] = l_run[0];
                mw[(2 * c + 1) * MST + D] = m_run[1];
                mw[(2 * c + 1) * MST + D + 1] = l_run[1];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
        const bool complete = (ps >= pa) && (pe <= pb);
        const int slot = ps < pa ? 0 : 1;
        // per query row: normalised page-group weights, log2 partition and output row
        if (ctid < rows_here) {
            const int rr = ctid, ntr = rr >> 3, j = rr & 7;
            float M = -INFINITY;
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) M = fmaxf(M, mbuf[((q2 * NT + ntr) * 8 + j) * MST + D]);
            const float Mb = M == -INFINITY ? 0.0f : M;
            float wq[PG], Ls = 0.0f;
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) {
                const float *st = mbuf + ((q2 * NT + ntr) * 8 + j) * MST;
                wq[q2] = ex2(st[D] - Mb);
                Ls = fmaf(st[D + 1], wq[q2], Ls);
            }
            const float inv = Ls > 0.0f ? __fdividef(1.0f, Ls) : 0.0f;   // Ls <= entries of a unit
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) wrow[rr * WST + q2] = wq[q2] * inv;
            wrow[rr * WST + 8] = Ls > 0.0f ? M + __log2f(Ls) : -INFINITY;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
        for (int it = ctid; it < rows_here * (D / 4); it += NCONS * 32) {
            const int rr = it / (D / 4), d4 = (it % (D / 4)) * 4;
            const int ntr = rr >> 3, j = rr & 7;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) {
                const float w = wrow[rr * WST + q2];
                const float4 x = *reinterpret_cast<const float4 *>(mbuf + ((q2 * NT + ntr) * 8 + j) * MST + d4);
                acc.x = fmaf(w, x.x, acc.x);
                acc.y = fmaf(w, x.y, acc.y);
                acc.z = fmaf(w, x.z, acc.z);
                acc.w = fmaf(w, x.w, acc.w);
            }
            const float lse2 = wrow[rr * WST + 8];
            if (complete) {
                const long long oi = orow[rr];
                *reinterpret_cast<uint2 *>(outp + oi * D + d4) =
                    make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                if (d4 == 0) a.lse[oi] = lse2 * kLn2;
            } else if (aligned) {
                // the CTA's only piece: rank 0 keeps it in its drained stage ring, the other ranks
                // store it into rank 0's receive buffer (no remote round trips)
                if (crank == 0) {
                    float *xl = reinterpret_cast<float *>(stages);
                    *reinterpret_cast<float4 *>(xl + rr * D + d4) = acc;
                    if (d4 == 0) xl[a.pass_rows * D + rr] = lse2;
                } else {
                    const uint32_t xr = dsmem_addr(smem_u32(xbuf + (crank - 1) * a.pass_rows * (D + 1)), 0);
                    st_dsmem_v4(xr + (rr * D + d4) * 4, acc);
                    if (d4 == 0) st_dsmem(xr + (a.pass_rows * D + rr) * 4, lse2);
                }
            } else {
                const long long pr = (static_cast<long long>(blockIdx.x) * 2 + slot) * a.pass_rows + rr;
                *reinterpret_cast<float4 *>(a.part_v + pr * D + d4) = acc;
                if (d4 == 0) a.part_l[pr] = lse2;
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));   // mbuf free; every partial of the piece stored
        if (!complete && !aligned && ctid == 0 && n_split < 2) {
            split_v[n_split] = v;
            // the unit's pages in work positions (the split's coordinates)
            split_ps[n_split] = wpre[v + 1] - static_cast<int>(pe - ps);
            split_pe[n_split] = wpre[v + 1];
            if (n_split == 0 && pe < pb) {
                // the range's first piece, with more of the range after it: its unit's other pieces
                // end the previous CTAs' ranges, so count it now and let one of them merge the unit
                // at its end (the count's result is read only at the end of this range)
                __threadfence();
                early_prev = atomicAdd(a.counters + v, 1);
            }
            ++n_split;
        }
    }

    if (aligned && kcl > 1) {
        // ---- cluster merge: rank 0 combines every rank's (out, log2 partition) of the unit ----
        cluster_sync();   // release / acquire: the other ranks' stores into xbuf are visible
        if (crank != 0) return;
        // orow[] still holds this unit's output rows (written by the piece epilogue)
        constexpr int WST = L::WST;
        const int rows_here = min(a.pass_rows, a.rows - (vc % a.row_passes) * kRowsPerPass);
        const float *own = reinterpret_cast<const float *>(stages);
        const int blk = a.pass_rows * (D + 1);
        if (ctid < rows_here) {
            const int rr = ctid;
            float M = -INFINITY;
            for (int r = 0; r < kcl; ++r) M = fmaxf(M, (r == 0 ? own : xbuf + (r - 1) * blk)[a.pass_rows * D + rr]);
            const float Mb = M == -INFINITY ? 0.0f : M;
            float Ls = 0.0f;
            for (int r = 0; r < kcl; ++r) {
                const float w = ex2((r == 0 ? own : xbuf + (r - 1) * blk)[a.pass_rows * D + rr] - Mb);
                wrow[rr * WST + r] = w;
                Ls += w;
            }
            const float inv = Ls > 0.0f ? __fdividef(1.0f, Ls) : 0.0f;   // 1 <= Ls <= kcl
            for (int r = 0; r < kcl; ++r) wrow[rr * WST + r] *= inv;
            wrow[rr * WST + 8] = Ls > 0.0f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
        for (int it = ctid; it < rows_here * (D / 4); it += NCONS * 32) {
            const int rr = it / (D / 4), d4 = (it % (D / 4)) * 4;
            float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            for (int r = 0; r < kcl; ++r) {
                const float w = wrow[rr * WST + r];
                const float4 x = *reinterpret_cast<const float4 *>((r == 0 ? own : xbuf + (r - 1) * blk) + rr * D + d4);
                acc.x = fmaf(w, x.x, acc.x);
                acc.y = fmaf(w, x.y, acc.y);
                acc.z = fmaf(w, x.z, acc.z);
                acc.w = fmaf(w, x.w, acc.w);
            }
            const long long oi = orow[rr];
            *reinterpret_cast<uint2 *>(outp + oi * D + d4) =
                make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
            if (d4 == 0) a.lse[oi] = wrow[rr * WST + 8];
        }
        return;
    }

    // ---- count this CTA's split pieces; merge the units it completes ----
    // (the barrier above ordered every thread's partial stores before thread 0's fence)
    int *pend = misc;   // pend[0] = count, then (v, ps, pe) per unit to merge
    if (ctid == 0) {
        int np = 0;
        if (n_split > 0) {
            __threadfence();
            // the counters not counted yet, both in flight at once: one round trip
            const int prev0 = early_prev >= 0 ? early_prev : atomicAdd(a.counters + split_v[0], 1);
            const int prev1 = n_split > 1 ? atomicAdd(a.counters + split_v[1], 1) : 0;
            for (int k = 0; k < n_split; ++k) {
                if ((k == 0 ? prev0 : prev1) == piece_count(split_ps[k], split_pe[k], ptot, a.ncta) - 1) {
                    pend[1 + 3 * np] = split_v[k];
                    pend[2 + 3 * np] = split_ps[k];
                    pend[3 + 3 * np] = split_pe[k];
                    ++np;
                }
            }
        }
        pend[0] = np;
    }
    asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
    const int np = pend[0];
    int *codes = reinterpret_cast<int *>(mbuf);
    for (int k = 0; k < np; ++k) {
        const int v = pend[1 + 3 * k];
        const long long ps = pend[2 + 3 * k], pe = pend[3 + 3 * k];
        const int n = piece_count(ps, pe, ptot, a.ncta);
        const long long c_first = cta_of(ps, ptot, a.ncta);
        for (int i = ctid; i < n; i += NCONS * 32) codes[i] = piece_code(i, ps, ptot, a.ncta, c_first);
        __threadfence();   // acquire: the other pieces' partials are visible after their counts
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
        merge_unit<D, NCONS>(MergeArgs{a.part_l, a.part_v, a.out, a.lse, a.row_passes, a.Hkv, a.pass_rows, a.rows, a.R,
                                       a.Hq, a.G},
                             v, codes, n, warp, lane);
        if (ctid == 0) a.counters[v] = 0;   // ready for the next call
        asm volatile("bar.sync 1, %0;" ::"n"(NCONS * 32));
    }
}

// fp32 caches: exact fp32 CUDA-core path, one CTA per unit, one warp per query row.
template <int D, bool DIAG>
__global__ void __launch_bounds__(128) k_decode_f32(const DecodeArgs a) {
    constexpr int PER = D / 32;
    const int u = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = clamp_entries(a, u);
    const float *q = static_cast<const float *>(a.q);
    constexpr int VEC_FLOATS = kPageNodes * D;   // fp32 keys (then values) of one page
    constexpr long long PAGE_FLOATS = (DIAG ? 3 : 2) * VEC_FLOATS + 2 * kPageNodes;
    const float *pool = reinterpret_cast<const float *>(a.pages);
    float *outp = static_cast<float *>(a.out);
    const float inv_sqrt_d = 1.0f / sqrtf(static_cast<float>(D));
    for (int row = warp; row < a.rows; row += 4) {
        const int r = row / a.G, gg = row % a.G;
        const long long oi = (static_cast<long long>(b) * a.R + r) * a.Hq + h * a.G + gg;
        float qv[PER], acc[PER];
        float qn = 0.0f;
#pragma unroll
        for (int i = 0; i < PER; ++i) {
            qv[i] = q[oi * D + lane + 32 * i];
            qn = fmaf(qv[i], qv[i], qn);
            acc[i] = 0.0f;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) qn += __shfl_xor_sync(0xffffffffu, qn, off);
        float m = -INFINITY, l = 0.0f;
        for (int e = 0; e < L; ++e) {
            const int page = a.page_table[static_cast<long long>(u) * a.max_pages + e / kPageNodes];
            if (page < 0 || page >= a.num_pages) {
                if (lane == 0) raise_flag(a.flags, FLAG_BAD_PAGE);
                continue;
            }
            const int slot = e % kPageNodes;
            const float *pk = pool + static_cast<long long>(page) * PAGE_FLOATS;
            const float *pv = pk + VEC_FLOATS;
            const long long nb = static_cast<long long>(slot) * D;
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int dim = lane + 32 * i;
                dot = fmaf(qv[i], pk[nb + swz(dim >> 2, slot) * 4 + (dim & 3)], dot);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            const float2 ab = reinterpret_cast<const float2 *>(pk + 2 * VEC_FLOATS)[slot];
            float closure = qn * ab.y;   // |q|^2 beta
            if constexpr (DIAG) {        // sum_i q_i^2 var_i / (2d)
                const float *pvar = pk + 2 * VEC_FLOATS + 2 * kPageNodes;
                float c = 0.0f;
#pragma unroll
                for (int i = 0; i < PER; ++i) {
                    const int dim = lane + 32 * i;
                    c = fmaf(qv[i] * qv[i], pvar[nb + swz(dim >> 2, slot) * 4 + (dim & 3)], c);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
                closure = c * (0.5f / D);
            }
            const float s = fmaf(dot, inv_sqrt_d, ab.x + closure);
            const float mn = fmaxf(m, s);
            const float corr = expf(m - mn);
            const float p = expf(s - mn);
            l = fmaf(l, corr, p);
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int dim = lane + 32 * i;
                acc[i] = fmaf(acc[i], corr, p * pv[nb + swz(dim >> 2, slot) * 4 + (dim & 3)]);
            }
            m = mn;
        }
#pragma unroll
        for (int i = 0; i < PER; ++i) outp[oi * D + lane + 32 * i] = l > 0.0f ? acc[i] / l : 0.0f;
        if (lane == 0) a.lse[oi] = l > 0.0f ? m + logf(l) : -INFINITY;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
template <int D, int NT, bool DIAG>
static size_t split_smem(int n_vunits, int cluster) {
    const size_t recv = static_cast<size_t>(cluster - 1) * (NT * 8) * (D + 1) * 4;   // aligned-split receive buffer
    const size_t work = static_cast<size_t>(n_vunits + 1) * 4;                       // or the work prefix
    return SplitSmem<D, NT, DIAG>::FIXED + static_cast<size_t>((n_vunits + 1 + 3) & ~3) * 4 +
           static_cast<size_t>((n_vunits + 3) & ~3) * 4 +   // entries per virtual unit
           (recv > work ? recv : work);
}

constexpr int kMaxCluster = 8;   // portable cluster size limit
// cluster > 1 needs n_vunits * cluster <= ncta <= kMaxDecodeCtas
template <int D, int NT, bool DIAG>
static size_t split_smem_max() {
    const size_t a = split_smem<D, NT, DIAG>(kMaxVUnits, 1);
    const size_t b = split_smem<D, NT, DIAG>(kMaxDecodeCtas / 2, kMaxCluster);
    return a > b ? a : b;
}

// Co-resident CTAs of the split kernel for one (device, shared-memory size, cluster size):
// SMs x resident CTAs without clusters, resident clusters x cluster size with them (a cluster
// must fit inside one GPC). Queried once and cached, so that later calls (and stream capture)
// issue no attribute queries.
template <int D, int NT, bool DIAG>
static cudaError_t split_grid(size_t smem, int cluster, int *ncta) {
    struct Entry {
        int dev;
        size_t smem;
        int cluster;
        int ncta;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &c : cache)
        if (c.dev == dev && c.smem == smem && c.cluster == cluster) {
            *ncta = c.ncta;
            return cudaSuccess;
        }
    static std::vector<std::pair<int, size_t>> limits;   // per device: the largest launchable request
    size_t limit = 0;
    for (const auto &l : limits)
        if (l.first == dev) limit = l.second;
    if (limit == 0) {
        // the largest request any call can make, within the device's opt-in maximum
        // (the opt-in maximum covers static and dynamic shared memory together)
        int optin = 0;
        if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
            return e;
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, k_decode_split<D, NT, DIAG>)) != cudaSuccess) return e;
        const size_t room = static_cast<size_t>(optin) - fa.sharedSizeBytes;
        limit = split_smem_max<D, NT, DIAG>();
        if (limit > room) limit = room;
        e = cudaFuncSetAttribute(k_decode_split<D, NT, DIAG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(limit));
        if (e != cudaSuccess) return e;
        limits.emplace_back(dev, limit);
    }
    int n = 0;
    if (smem > limit) {
        n = 0;   // does not fit this device: not launchable
    } else if (cluster == 1) {
        int sms = 0, occ = 0;
        if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_split<D, NT, DIAG>, (SplitSmem<D, NT, DIAG>::THREADS), smem)) !=
            cudaSuccess)
            return e;
        n = sms * (occ > 0 ? occ : 1);
    } else {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(cluster);
        cfg.blockDim = dim3((SplitSmem<D, NT, DIAG>::THREADS));
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = cluster;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int nc = 0;
        if (cudaOccupancyMaxActiveClusters(&nc, k_decode_split<D, NT, DIAG>, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();   // this cluster size is not available: not an error of the call
            nc = 0;
        }
        n = nc * cluster;
    }
    if (n > kMaxDecodeCtas) n = kMaxDecodeCtas - kMaxDecodeCtas % cluster;
    cache.push_back({dev, smem, cluster, n});
    *ncta = n;
    return cudaSuccess;
}

// Grid and cluster size of one call. The cluster size is the largest k <= 8 for which one
// cluster of k CTAs per virtual unit is co-resident and keeps at least 3/4 of the grid busy
// (an aligned split then streams at most 4/3 of the pages per CTA a stream-K split would, and
// saves its global merges). It is used only if the device finds every unit equally long;
// otherwise the same grid runs the stream-K split.
// Few pages (all units together, at max_pages pages each, give at most one page per CTA of the
// full grid): a stream-K split would leave most CTAs idle and merge each unit's one-page pieces
// through global partials. The grid then shrinks to exactly one cluster of k CTAs per virtual
// unit, k <= max_pages the largest co-resident size, so each CTA streams about max_pages / k
// pages and the pieces merge in distributed shared memory.
template <int D, int NT, bool DIAG>
static cudaError_t split_config(DecodeArgs *a, size_t *smem) {
    *smem = split_smem<D, NT, DIAG>(a->n_vunits, 1);
    cudaError_t e = split_grid<D, NT, DIAG>(*smem, 1, &a->ncta);
    if (e != cudaSuccess) return e;
    if (a->ncta < 1) return cudaErrorInvalidValue;
    a->cluster = 1;
    const long long nv = a->n_vunits;
    const bool few = nv * a->max_pages <= a->ncta;
    int kmax = a->ncta / a->n_vunits < kMaxCluster ? a->ncta / a->n_vunits : kMaxCluster;
    if (few && kmax > a->max_pages) kmax = a->max_pages;
    for (int k = kmax; k > 1; --k) {
        const size_t sk = split_smem<D, NT, DIAG>(a->n_vunits, k);
        int n = 0;
        if ((e = split_grid<D, NT, DIAG>(sk, k, &n)) != cudaSuccess) return e;
        if (nv * k <= n && (few || nv * k * 4 >= 3LL * n)) {
            a->cluster = k;
            a->ncta = few ? static_cast<int>(nv * k) : n;
            *smem = sk;
            break;
        }
    }
    return cudaSuccess;
}

template <int D, int NT, bool DIAG>
static cudaError_t launch_split(const DecodeArgs &a0, cudaStream_t s) {
    DecodeArgs a = a0;
    size_t smem = 0;
    cudaError_t e = split_config<D, NT, DIAG>(&a, &smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.ncta);
    cfg.blockDim = dim3((SplitSmem<D, NT, DIAG>::THREADS));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = a.cluster;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.cluster > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k_decode_split<D, NT, DIAG>, a);
}

template <bool DIAG>
static cudaError_t launch_decode_t(const DecodeArgs &a, cudaStream_t s) {
    if (a.dtype == SKV_F32) {
        if (a.d == 128) k_decode_f32<128, DIAG><<<a.B * a.Hkv, 128, 0, s>>>(a);
        else k_decode_f32<64, DIAG><<<a.B * a.Hkv, 128, 0, s>>>(a);
        return cudaGetLastError();
    }
    const int nt = a.pass_rows / 8 + (a.pass_rows % 8 ? 1 : 0);
    if (a.d == 128) {
        if (nt == 1) return launch_split<128, 1, DIAG>(a, s);
        if (nt == 2) return launch_split<128, 2, DIAG>(a, s);
        return launch_split<128, 4, DIAG>(a, s);
    }
    if (nt == 1) return launch_split<64, 1, DIAG>(a, s);
    if (nt == 2) return launch_split<64, 2, DIAG>(a, s);
    return launch_split<64, 4, DIAG>(a, s);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    return a.closure == SKV_CLOSURE_DIAGONAL ? launch_decode_t<true>(a, s) : launch_decode_t<false>(a, s);
}

}  // namespace skv

namespace skv {

template <int D, int NT, bool DIAG>
static cudaError_t split_ctas(const DecodeArgs &a0, int *ncta) {
    DecodeArgs a = a0;
    size_t smem = 0;
    const cudaError_t e = split_config<D, NT, DIAG>(&a, &smem);
    *ncta = a.ncta;
    return e;
}

// The grid k_decode_split would use for these arguments (bf16 caches), for callers that must size
// split-partial storage before launching. Queries (and caches) the same occupancy as the launcher.
template <bool DIAG>
static cudaError_t split_ctas_t(const DecodeArgs &a, int *ncta) {
    const int nt = a.pass_rows / 8 + (a.pass_rows % 8 ? 1 : 0);
    if (a.d == 128) {
        if (nt == 1) return split_ctas<128, 1, DIAG>(a, ncta);
        if (nt == 2) return split_ctas<128, 2, DIAG>(a, ncta);
        return split_ctas<128, 4, DIAG>(a, ncta);
    }
    if (nt == 1) return split_ctas<64, 1, DIAG>(a, ncta);
    if (nt == 2) return split_ctas<64, 2, DIAG>(a, ncta);
    return split_ctas<64, 4, DIAG>(a, ncta);
}

cudaError_t decode_split_ctas(const DecodeArgs &a, int *ncta) {
    return a.closure == SKV_CLOSURE_DIAGONAL ? split_ctas_t<true>(a, ncta) : split_ctas_t<false>(a, ncta);
}

}  // namespace skv
