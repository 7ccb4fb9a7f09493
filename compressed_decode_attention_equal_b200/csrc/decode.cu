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
//    streams the same number of 16-node pages whatever the length mix;
//  * one producer warp copies each page (K 4 KB, V 4 KB, alpha/beta 128 B at
//    d = 128) with three TMA bulk copies into an 8-stage mbarrier ring;
//  * four consumer warps run the GQA group's query rows through tensor cores:
//    S^T = K Q^T with nodes as the M = 16 dimension and up to 8 query rows as
//    N = 8 (a GQA group of 7 rows wastes 1/8), softmax on the accumulator, P^T
//    transposed in registers (movmatrix) into the B operand of O^T = V^T P^T;
//  * a piece that covers a whole unit writes out / lse directly; pieces of a
//    unit split across CTAs write (lse, out) partials, and the CTA that
//    finishes a unit last (an atomic per-unit counter, reset after use) merges
//    them with a log-sum-exp;
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
constexpr int kDecThreads = (kDecConsumers + 1) * 32;
constexpr int kDecStages = 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
struct PageGeom {
    static constexpr int ROWB = D * 2;                 // bytes of one bf16 node vector
    static constexpr int VEC_BYTES = kPageNodes * ROWB;   // K (or V) bytes of a page
    static constexpr int AB_BYTES = kPageNodes * 8;
    static constexpr int STAGE = 2 * VEC_BYTES + AB_BYTES;
};

template <int D>
constexpr size_t dec_smem_fixed() {
    return 16 /*align*/ + kDecStages * PageGeom<D>::STAGE + 2 * kDecStages * 8 + kDecStages * 4 +
           kDecConsumers * 8 * (D + 2) * 4;
}

__device__ __forceinline__ int clamp_entries(const DecodeArgs &a, int u) {
    int L = a.lens[u];
    const int cap = a.max_pages * kPageNodes;
    if (L > cap) {
        raise_flag(a.flags, FLAG_BAD_LENS);
        L = cap;
    }
    return L < 0 ? 0 : L;
}

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

// Every CTA rebuilds the page prefix over virtual units (lens are tiny and L2-resident).
__device__ __forceinline__ void build_prefix(const DecodeArgs &a, int *prefix, int *scratch) {
    const int nv = a.n_vunits;
    const int tid = threadIdx.x, nth = blockDim.x;
    const int per = (nv + nth - 1) / nth;
    const int lo = min(tid * per, nv), hi = min(lo + per, nv);
    int local = 0;
    for (int v = lo; v < hi; ++v) {
        const int pages = (clamp_entries(a, v / a.row_passes) + kPageNodes - 1) / kPageNodes;
        prefix[v] = pages;   // page count for now; made exclusive below
        local += pages;
    }
    // block exclusive scan of `local`
    const int lane = tid & 31, warp = tid >> 5;
    int x = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += n;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    int wp = 0;
    for (int w = 0; w < warp; ++w) wp += scratch[w];
    int run = wp + x - local;
    for (int v = lo; v < hi; ++v) {
        const int pages = prefix[v];
        prefix[v] = run;
        run += pages;
    }
    if (tid == nth - 1) prefix[nv] = wp + x;
    __syncthreads();
}

// First flat page of CTA c's range, and the CTA whose (nonempty) range holds page f.
__device__ __forceinline__ long long cta_begin(long long c, long long ptot, int ncta) { return ptot * c / ncta; }
__device__ __forceinline__ long long cta_of(long long f, long long ptot, int ncta) {
    return ((f + 1) * ncta + ptot - 1) / ptot - 1;
}

// Log-sum-exp merge of every piece of virtual unit v (run by the CTA that completed it).
template <int D>
__device__ void merge_unit(const DecodeArgs &a, int v, int b, int h, int rpass, long long ps, long long pe,
                           long long ptot, int tid, int nth) {
    const long long c_first = cta_of(ps, ptot, a.ncta), c_last = cta_of(pe - 1, ptot, a.ncta);
    const int rows_here = min(a.pass_rows, a.rows - rpass * kRowsPerPass);
    __nv_bfloat16 *outp = static_cast<__nv_bfloat16 *>(a.out);
    for (int idx = tid; idx < rows_here * D; idx += nth) {
        const int rr = idx / D, dim = idx % D;
        const int row = rpass * kRowsPerPass + rr;
        float M = -INFINITY;
        for (long long cc = c_first; cc <= c_last; ++cc) {
            const long long a_c = cta_begin(cc, ptot, a.ncta);
            if (a_c >= cta_begin(cc + 1, ptot, a.ncta)) continue;   // an empty range wrote no partial
            const int slot = ps < a_c ? 0 : 1;
            M = fmaxf(M, __ldcg(a.part + ((cc * 2 + slot) * a.pass_rows + rr) * (D + 1)));
        }
        const float Mb = M == -INFINITY ? 0.0f : M;
        float Ls = 0.0f, Os = 0.0f;
        for (long long cc = c_first; cc <= c_last; ++cc) {
            const long long a_c = cta_begin(cc, ptot, a.ncta);
            if (a_c >= cta_begin(cc + 1, ptot, a.ncta)) continue;
            const int slot = ps < a_c ? 0 : 1;
            const float *pp = a.part + ((cc * 2 + slot) * a.pass_rows + rr) * (D + 1);
            const float w = ex2(__ldcg(pp) - Mb);
            Ls += w;
            Os = fmaf(__ldcg(pp + 1 + dim), w, Os);
        }
        const long long oi = (static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G;
        outp[oi * D + dim] = __float2bfloat16_rn(Ls > 0.0f ? __fdividef(Os, Ls) : 0.0f);
        if (dim == 0) a.lse[oi] = Ls > 0.0f ? (M + __log2f(Ls)) * kLn2 : -INFINITY;
    }
}

template <int D, int NT>
__global__ void __launch_bounds__(kDecThreads, 2) k_decode_split(const DecodeArgs a) {
    using G = PageGeom<D>;
    constexpr int PG = kDecConsumers / NT;   // page groups: warps sharing a row tile split the pages
    constexpr int NKS = D / 16;              // QK k-steps over dims == PV m-tiles over dims

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((16 - (smem_u32(smem_raw) & 15)) & 15);
    uint8_t *stages = smem;
    uint64_t *full = reinterpret_cast<uint64_t *>(stages + kDecStages * G::STAGE);
    uint64_t *empty = full + kDecStages;
    int *svalid = reinterpret_cast<int *>(empty + kDecStages);
    float *mbuf = reinterpret_cast<float *>(svalid + kDecStages);
    int *prefix = reinterpret_cast<int *>(mbuf + kDecConsumers * 8 * (D + 2));
    __shared__ int scan_scratch[kDecThreads / 32];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nv = a.n_vunits;
    // let the next launch in the stream become resident as our CTAs retire; then wait for every
    // preceding grid to complete (its writes visible) before reading any input
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    build_prefix(a, prefix, scan_scratch);
    const long long ptot = prefix[nv];
    const long long ra = ptot * blockIdx.x / a.ncta;
    const long long rb = ptot * (blockIdx.x + 1) / a.ncta;
    // units with no entries get out = 0, lse = -inf (spread over the CTAs)
    for (int v = blockIdx.x; v < nv; v += a.ncta) {
        if (prefix[v + 1] != prefix[v]) continue;
        const int u = v / a.row_passes, rpass = v % a.row_passes;
        const int b = u / a.Hkv, h = u % a.Hkv;
        for (int idx = tid; idx < a.pass_rows * D; idx += kDecThreads) {
            const int rr = idx / D, dim = idx % D;
            const int row = rpass * kRowsPerPass + rr;
            if (row >= a.rows) continue;
            const long long oi = (static_cast<long long>(b) * a.R + row / a.G) * a.Hq + h * a.G + row % a.G;
            static_cast<__nv_bfloat16 *>(a.out)[oi * D + dim] = __float2bfloat16_rn(0.0f);
            if (dim == 0) a.lse[oi] = -INFINITY;
        }
    }
    if (ra >= rb) return;
    const int v0 = find_vunit(prefix, nv, ra);
    const int n_my = static_cast<int>(rb - ra);

    if (tid == 0) {
        for (int s = 0; s < kDecStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NT);
        }
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kDecConsumers) {
        // ----------------------------- producer -----------------------------
        bool alive = true;
        for (int base = 0; base < n_my && alive; base += 32) {
            int my_page = -1;
            if (base + lane < n_my) {
                const long long f = ra + base + lane;
                const int v = find_vunit(prefix, nv, f);
                const int u = v / a.row_passes;
                my_page = a.page_table[static_cast<long long>(u) * a.max_pages + (f - prefix[v])];
            }
            const int cnt = min(32, n_my - base);
            for (int k = 0; k < cnt; ++k) {
                const int i = base + k;
                const int s = i % kDecStages;
                const int phys = __shfl_sync(0xffffffffu, my_page, k);
                if (i >= kDecStages && !mbar_wait(&empty[s], ((i / kDecStages) - 1) & 1)) {
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
                        uint8_t *dst = stages + s * G::STAGE;
                        mbar_arrive_expect_tx(&full[s], G::STAGE);
                        bulk_g2s(dst, a.pool_k + static_cast<long long>(phys) * G::VEC_BYTES, G::VEC_BYTES, &full[s]);
                        bulk_g2s(dst + G::VEC_BYTES, a.pool_v + static_cast<long long>(phys) * G::VEC_BYTES,
                                 G::VEC_BYTES, &full[s]);
                        bulk_g2s(dst + 2 * G::VEC_BYTES, a.pool_ab + static_cast<long long>(phys) * kPageNodes,
                                 G::AB_BYTES, &full[s]);
                    }
                }
                __syncwarp();
            }
        }
        return;
    }

    // ------------------------------- consumers -------------------------------
    const int nt = warp % NT, pg = warp / NT;
    const int g = lane >> 2, c = lane & 3;
    const float c_scale = kLog2e * rsqrtf(static_cast<float>(D));
    const __nv_bfloat16 *q = static_cast<const __nv_bfloat16 *>(a.q);
    __nv_bfloat16 *outp = static_cast<__nv_bfloat16 *>(a.out);
    int i0 = 0;
    bool alive = true;
    for (int v = v0; v < nv && prefix[v] < rb; ++v) {
        const long long ps = prefix[v], pe = prefix[v + 1];
        const int lo = static_cast<int>(max(ra, ps) - ps), hi = static_cast<int>(min(rb, pe) - ps);
        const int npg = hi - lo;
        const int u = v / a.row_passes, rpass = v % a.row_passes;
        const int b = u / a.Hkv, h = u % a.Hkv;
        const int L = clamp_entries(a, u);

        // Q^T fragments of rows rpass*32 + nt*8 + g, and |q|^2 of rows 2c, 2c+1
        const int my_row = rpass * kRowsPerPass + nt * 8 + g;
        const bool row_ok = (nt * 8 + g) < a.pass_rows && my_row < a.rows;
        uint32_t qf[NKS][2];
        float qn = 0.0f;
        {
            const __nv_bfloat16 *qr = q;
            if (row_ok) {
                const int r = my_row / a.G, gg = my_row % a.G;
                qr = q + ((static_cast<long long>(b) * a.R + r) * a.Hq + h * a.G + gg) * D;
            }
#pragma unroll
            for (int ks = 0; ks < NKS; ++ks) {
                uint32_t w0 = 0, w1 = 0;
                if (row_ok) {
                    w0 = *reinterpret_cast<const uint32_t *>(qr + 16 * ks + 2 * c);
                    w1 = *reinterpret_cast<const uint32_t *>(qr + 16 * ks + 8 + 2 * c);
                }
                qf[ks][0] = w0;
                qf[ks][1] = w1;
                qn = fmaf(bf16lo(w0), bf16lo(w0), qn);
                qn = fmaf(bf16hi(w0), bf16hi(w0), qn);
                qn = fmaf(bf16lo(w1), bf16lo(w1), qn);
                qn = fmaf(bf16hi(w1), bf16hi(w1), qn);
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

        for (int k = pg; k < npg && alive; k += PG) {
            const int i = i0 + k;
            const int s = i % kDecStages;
            if (!mbar_wait(&full[s], (i / kDecStages) & 1)) {
                if (lane == 0) raise_flag(a.flags, FLAG_TIMEOUT);
                alive = false;
                break;
            }
            if (svalid[s]) {
                const int nvalid = min(kPageNodes, L - (lo + k) * kPageNodes);
                const uint32_t kb = smem_u32(stages + s * G::STAGE);
                const uint32_t vb = kb + G::VEC_BYTES;
                const float2 *ab = reinterpret_cast<const float2 *>(stages + s * G::STAGE + 2 * G::VEC_BYTES);
                // S^T (16 nodes x 8 rows) = K (16 x D) Q^T (D x 8)
                float sacc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
                {
                    const int mi = lane >> 3, node = (lane & 7) + 8 * (mi & 1);
#pragma unroll
                    for (int ks = 0; ks < NKS; ++ks) {
                        const int chunk = 2 * ks + (mi >> 1);
                        uint32_t a0, a1, a2, a3;
                        ldsm_x4(kb + node * G::ROWB + (swz(chunk, node) << 4), a0, a1, a2, a3);
                        mma_bf16(sacc, a0, a1, a2, a3, qf[ks][0], qf[ks][1]);
                    }
                }
                const float2 ab0 = ab[g], ab1 = ab[g + 8];
                float sl[4];
                sl[0] = g < nvalid ? fmaf(sacc[0], c_scale, kLog2e * fmaf(qn_r0, ab0.y, ab0.x)) : -INFINITY;
                sl[1] = g < nvalid ? fmaf(sacc[1], c_scale, kLog2e * fmaf(qn_r1, ab0.y, ab0.x)) : -INFINITY;
                sl[2] = g + 8 < nvalid ? fmaf(sacc[2], c_scale, kLog2e * fmaf(qn_r0, ab1.y, ab1.x)) : -INFINITY;
                sl[3] = g + 8 < nvalid ? fmaf(sacc[3], c_scale, kLog2e * fmaf(qn_r1, ab1.y, ab1.x)) : -INFINITY;
                float mx0 = fmaxf(sl[0], sl[2]), mx1 = fmaxf(sl[1], sl[3]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
                    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
                }
                const float mn0 = fmaxf(m_run[0], mx0), mn1 = fmaxf(m_run[1], mx1);
                const float base0 = mn0 == -INFINITY ? 0.0f : mn0;
                const float base1 = mn1 == -INFINITY ? 0.0f : mn1;
                const float corr0 = ex2(m_run[0] - base0), corr1 = ex2(m_run[1] - base1);
                const float p0 = ex2(sl[0] - base0), p1 = ex2(sl[1] - base1);
                const float p2 = ex2(sl[2] - base0), p3 = ex2(sl[3] - base1);
                l_run[0] = fmaf(l_run[0], corr0, p0 + p2);
                l_run[1] = fmaf(l_run[1], corr1, p1 + p3);
                m_run[0] = mn0;
                m_run[1] = mn1;
                if (!__all_sync(0xffffffffu, corr0 == 1.0f && corr1 == 1.0f)) {
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
                {
                    const int mi = lane >> 3, node = (lane & 7) + 8 * (mi >> 1);
                    if (nvalid == kPageNodes) {
#pragma unroll
                        for (int mt = 0; mt < NKS; ++mt) {
                            const int chunk = 2 * mt + (mi & 1);
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4_t(vb + node * G::ROWB + (swz(chunk, node) << 4), a0, a1, a2, a3);
                            mma_bf16(o[mt], a0, a1, a2, a3, bp0, bp1);
                        }
                    } else {
                        // slots past the unit's last entry may hold anything (NaN included):
                        // zero their V^T elements, since P = 0 does not cancel NaN in the product.
                        // This thread's fragment holds nodes 2c, 2c+1 (a0..a3) and 2c+8, 2c+9 (a4..a7).
                        const uint32_t m_lo = (2 * c < nvalid ? 0x0000ffffu : 0u) | (2 * c + 1 < nvalid ? 0xffff0000u : 0u);
                        const uint32_t m_hi =
                            (2 * c + 8 < nvalid ? 0x0000ffffu : 0u) | (2 * c + 9 < nvalid ? 0xffff0000u : 0u);
#pragma unroll
                        for (int mt = 0; mt < NKS; ++mt) {
                            const int chunk = 2 * mt + (mi & 1);
                            uint32_t a0, a1, a2, a3;
                            ldsm_x4_t(vb + node * G::ROWB + (swz(chunk, node) << 4), a0, a1, a2, a3);
                            mma_bf16(o[mt], a0 & m_lo, a1 & m_lo, a2 & m_hi, a3 & m_hi, bp0, bp1);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        i0 += npg;

        // ---- piece epilogue: merge the page groups through shared memory ----
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 4);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 4);
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 8);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 8);
        l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], 16);
        l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], 16);
        float *mw = mbuf + warp * 8 * (D + 2);
#pragma unroll
        for (int mt = 0; mt < NKS; ++mt) {
            mw[(2 * c) * (D + 2) + 16 * mt + g] = o[mt][0];
            mw[(2 * c + 1) * (D + 2) + 16 * mt + g] = o[mt][1];
            mw[(2 * c) * (D + 2) + 16 * mt + g + 8] = o[mt][2];
            mw[(2 * c + 1) * (D + 2) + 16 * mt + g + 8] = o[mt][3];
        }
        if (g == 0) {
            mw[(2 * c) * (D + 2) + D] = m_run[0];
            mw[(2 * c) * (D + 2) + D + 1] = l_run[0];
            mw[(2 * c + 1) * (D + 2) + D] = m_run[1];
            mw[(2 * c + 1) * (D + 2) + D + 1] = l_run[1];
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumers * 32));
        const bool complete = (ps >= ra) && (pe <= rb);
        const int slot = ps < ra ? 0 : 1;
        const int ctid = tid;   // 0 .. 127
        for (int idx = ctid; idx < NT * 8 * D; idx += kDecConsumers * 32) {
            const int rr = idx / D, dim = idx % D;
            const int ntr = rr >> 3, j = rr & 7;
            const int row = rpass * kRowsPerPass + rr;
            if (rr >= a.pass_rows || row >= a.rows) continue;
            float M = -INFINITY;
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) M = fmaxf(M, mbuf[((q2 * NT + ntr) * 8 + j) * (D + 2) + D]);
            float Ls = 0.0f, Os = 0.0f;
            const float Mb = M == -INFINITY ? 0.0f : M;
#pragma unroll
            for (int q2 = 0; q2 < PG; ++q2) {
                const float *st = mbuf + ((q2 * NT + ntr) * 8 + j) * (D + 2);
                const float w = ex2(st[D] - Mb);
                Ls = fmaf(st[D + 1], w, Ls);
                Os = fmaf(st[dim], w, Os);
            }
            const float val = Ls > 0.0f ? __fdividef(Os, Ls) : 0.0f;
            const float lse2 = Ls > 0.0f ? M + __log2f(Ls) : -INFINITY;
            if (complete) {
                const int r = row / a.G, gg = row % a.G;
                const long long oi = (static_cast<long long>(b) * a.R + r) * a.Hq + h * a.G + gg;
                outp[oi * D + dim] = __float2bfloat16_rn(val);
                if (dim == 0) a.lse[oi] = lse2 * kLn2;
            } else {
                float *pp = a.part + ((static_cast<long long>(blockIdx.x) * 2 + slot) * a.pass_rows + rr) * (D + 1);
                pp[1 + dim] = val;
                if (dim == 0) pp[0] = lse2;
            }
        }
        if (!complete) {
            // publish this piece; the CTA that completes the unit merges all of its pieces
            __threadfence();
            asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumers * 32));
            int *last = reinterpret_cast<int *>(mbuf);   // mbuf is free again after the barrier
            if (ctid == 0) {
                const long long c_first = cta_of(ps, ptot, a.ncta), c_last = cta_of(pe - 1, ptot, a.ncta);
                int pieces = 0;
                for (long long cc = c_first; cc <= c_last; ++cc) pieces += cta_begin(cc, ptot, a.ncta) <
                                                                            cta_begin(cc + 1, ptot, a.ncta);
                const int prev = atomicAdd(a.counters + v, 1);
                *last = (prev == pieces - 1) ? 1 : 0;
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumers * 32));
            if (*last) {
                __threadfence();
                merge_unit<D>(a, v, b, h, rpass, ps, pe, ptot, ctid, kDecConsumers * 32);
                if (ctid == 0) a.counters[v] = 0;   // ready for the next call
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(kDecConsumers * 32));
    }
}

// fp32 caches: exact fp32 CUDA-core path, one CTA per unit, one warp per query row.
template <int D>
__global__ void __launch_bounds__(128) k_decode_f32(const DecodeArgs a) {
    constexpr int PER = D / 32;
    const int u = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int L = clamp_entries(a, u);
    const float *q = static_cast<const float *>(a.q);
    const float *pk = reinterpret_cast<const float *>(a.pool_k);
    const float *pv = reinterpret_cast<const float *>(a.pool_v);
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
            const long long nb = (static_cast<long long>(page) * kPageNodes + slot) * D;
            float dot = 0.0f;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int dim = lane + 32 * i;
                dot = fmaf(qv[i], pk[nb + swz(dim >> 2, slot) * 4 + (dim & 3)], dot);
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
            const float2 ab = a.pool_ab[static_cast<long long>(page) * kPageNodes + slot];
            const float s = fmaf(dot, inv_sqrt_d, fmaf(qn, ab.y, ab.x));
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
template <int D, int NT>
static size_t split_smem(int n_vunits) {
    return dec_smem_fixed<D>() + static_cast<size_t>(n_vunits + 1) * 4;
}

// Grid size of the split kernel for one (device, shared-memory size): SMs x resident CTAs.
// Queried once and cached, so that later calls (and stream capture) issue no attribute queries.
template <int D, int NT>
static cudaError_t split_grid(size_t smem, int *ncta) {
    struct Entry {
        int dev;
        size_t smem;
        int ncta;
    };
    static std::mutex mu;
    static std::vector<Entry> cache;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    for (const Entry &c : cache)
        if (c.dev == dev && c.smem == smem) {
            *ncta = c.ncta;
            return cudaSuccess;
        }
    bool configured = false;
    for (const Entry &c : cache) configured |= (c.dev == dev);
    if (!configured) {
        // the largest request any call can make (the page prefix of kMaxVUnits virtual units)
        e = cudaFuncSetAttribute(k_decode_split<D, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(split_smem<D, NT>(kMaxVUnits)));
        if (e != cudaSuccess) return e;
    }
    int sms = 0, occ = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, k_decode_split<D, NT>, kDecThreads, smem)) !=
        cudaSuccess)
        return e;
    int n = sms * (occ > 0 ? occ : 1);
    if (n > kMaxDecodeCtas) n = kMaxDecodeCtas;
    cache.push_back({dev, smem, n});
    *ncta = n;
    return cudaSuccess;
}

template <int D, int NT>
static cudaError_t launch_split(const DecodeArgs &a0, cudaStream_t s) {
    DecodeArgs a = a0;
    const size_t smem = split_smem<D, NT>(a.n_vunits);
    cudaError_t e = split_grid<D, NT>(smem, &a.ncta);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(a.ncta);
    cfg.blockDim = dim3(kDecThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_decode_split<D, NT>, a);
}

cudaError_t launch_decode(const DecodeArgs &a, cudaStream_t s) {
    if (a.dtype == SKV_F32) {
        if (a.d == 128) k_decode_f32<128><<<a.B * a.Hkv, 128, 0, s>>>(a);
        else k_decode_f32<64><<<a.B * a.Hkv, 128, 0, s>>>(a);
        return cudaGetLastError();
    }
    const int nt = a.pass_rows / 8 + (a.pass_rows % 8 ? 1 : 0);
    if (a.d == 128) {
        if (nt == 1) return launch_split<128, 1>(a, s);
        if (nt == 2) return launch_split<128, 2>(a, s);
        return launch_split<128, 4>(a, s);
    }
    if (nt == 1) return launch_split<64, 1>(a, s);
    if (nt == 2) return launch_split<64, 2>(a, s);
    return launch_split<64, 4>(a, s);
}

}  // namespace skv
