// Streaming equal-variation coarsening: one token per (sequence, KV head) unit per call.
//
// "Equal-Variation KV Cache", "Implementation notes": in streaming inference a segment that
// exceeds its variation budget is split at the first threshold crossing and adjacent
// low-variation segments are merged; node merges follow the law of total variance ("SPICY-KV",
// dependent Claim 10). The policy (include/skv.h, skv_stream_append):
//  * the oldest recent token y enters the middle; its step D_y is the offline fixed fp32 recipe
//    against the previous middle token's feature; c_T += D_y;
//  * first hitting on the open (last) node's budget: N (V_open + D_y) >= c_T starts a new node at
//    y, else y joins the open node;
//  * while more than N middle nodes exist, the adjacent pair with the smallest V_j + V_{j+1}
//    (leftmost on ties) merges; means and summed squared deviations combine pairwise in fp64.
//
// k_stream_init builds the per-unit state after the offline coarsening of the prompt (same
// workspace: entry list and tile-local variation scans); k_stream_append runs one CTA per unit.
// Entries of a unit live in pool slots [0, lens) in no particular order: a merge frees a slot,
// which the unit's last entry then fills (decode attention does not depend on entry order).
#include <climits>

#include "skv_common.cuh"
#include "skv_internal.h"

namespace skv {

constexpr int kStreamThreads = 128;
constexpr int kStreamMaxNodes = 8192;   // node-order capacity the append kernel stages in shared memory

template <typename T>
struct Elem;
template <>
struct Elem<__nv_bfloat16> {
    static constexpr int SIZE = 2;
    __device__ static float get(const uint8_t *p) { return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(p)); }
    __device__ static void put(uint8_t *p, float x) { *reinterpret_cast<__nv_bfloat16 *>(p) = __float2bfloat16_rn(x); }
};
template <>
struct Elem<float> {
    static constexpr int SIZE = 4;
    __device__ static float get(const uint8_t *p) { return *reinterpret_cast<const float *>(p); }
    __device__ static void put(uint8_t *p, float x) { *reinterpret_cast<float *>(p) = x; }
};

// byte offset of element (slot, dim) inside a page's key (or value) block
template <int D, typename T>
__device__ __forceinline__ int vec_off(int slot, int dim) {
    constexpr int EPC = 16 / Elem<T>::SIZE;   // elements per 16-byte chunk
    return slot * D * Elem<T>::SIZE + swz(dim / EPC, slot) * 16 + (dim % EPC) * Elem<T>::SIZE;
}

template <int D, typename T>
struct UnitState {
    StreamHdr *hdr;
    int *order, *recent, *owner, *m, *start;
    long long *V;
    double *M2, *mk, *mv;
    __device__ UnitState(const StreamArgs &s, int u) {
        uint8_t *base = s.state + static_cast<int64_t>(u) * s.unit_bytes;
        hdr = reinterpret_cast<StreamHdr *>(base);
        order = reinterpret_cast<int *>(base + s.off_order);
        recent = reinterpret_cast<int *>(base + s.off_recent);
        owner = reinterpret_cast<int *>(base + s.off_owner);
        m = reinterpret_cast<int *>(base + s.off_m);
        start = reinterpret_cast<int *>(base + s.off_start);
        V = reinterpret_cast<long long *>(base + s.off_V);
        M2 = reinterpret_cast<double *>(base + s.off_M2);
        mk = reinterpret_cast<double *>(base + s.off_mk);
        mv = reinterpret_cast<double *>(base + s.off_mv);
    }
};

// page of entry e of unit u, or nullptr (flag raised) if the page id is outside the pool
template <int D, typename T>
__device__ __forceinline__ uint8_t *entry_page(const StreamArgs &s, int u, int e) {
    const int32_t page = s.page_table[static_cast<int64_t>(u) * s.max_pages + e / kPageNodes];
    if (page < 0 || page >= s.num_pages) {
        raise_flag(s.flags, FLAG_BAD_PAGE);
        return nullptr;
    }
    constexpr int VEC = kPageNodes * D * Elem<T>::SIZE;
    return s.pages + static_cast<int64_t>(page) * (2 * VEC + kPageNodes * 8);
}

// block-wide sum of a double (all threads return it)
__device__ double block_sum(double x, double *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    double t = 0.0;
    for (int w = 0; w < kStreamThreads / 32; ++w) t += red[w];
    return t;
}

__device__ long long block_sum_ll(long long x, long long *red) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    long long t = 0;
    for (int w = 0; w < kStreamThreads / 32; ++w) t += red[w];
    return t;
}

// write node e's mean key, mean value, alpha, beta into its pool slot (pg: its page if known)
template <int D, typename T>
__device__ void write_node(const StreamArgs &s, const UnitState<D, T> &st, int u, int e, uint8_t *pg = nullptr) {
    if (!pg) pg = entry_page<D, T>(s, u, e);
    if (!pg) return;
    constexpr int VEC = kPageNodes * D * Elem<T>::SIZE;
    const int slot = e % kPageNodes;
    for (int dim = threadIdx.x; dim < D; dim += kStreamThreads) {
        Elem<T>::put(pg + vec_off<D, T>(slot, dim), static_cast<float>(st.mk[static_cast<int64_t>(e) * D + dim]));
        Elem<T>::put(pg + VEC + vec_off<D, T>(slot, dim), static_cast<float>(st.mv[static_cast<int64_t>(e) * D + dim]));
    }
    if (threadIdx.x == 0) {
        const int m = st.m[e];
        const double sig2 = st.M2[e] / (static_cast<double>(m) * D);
        reinterpret_cast<float2 *>(pg + 2 * VEC)[slot] =
            make_float2(m == 1 ? 0.0f : logf(static_cast<float>(m)), static_cast<float>(sig2 / (2.0 * D)));
    }
}

// z = P [k; v] by the fixed recipe (z_i an fp32 fma chain over j ascending from 0); thread i < 16.
// pt: P^T (pt[j * 16 + i] = P[i][j]) in shared or parameter memory.
__device__ __forceinline__ float feature_i(const float *pt, const float *kx, const float *vx, int D, int i) {
    float z = 0.0f;
#pragma unroll 8
    for (int j = 0; j < D; ++j) z = __fmaf_rn(pt[j * kProjDim + i], kx[j], z);
#pragma unroll 8
    for (int j = 0; j < D; ++j) z = __fmaf_rn(pt[(D + j) * kProjDim + i], vx[j], z);
    return z;
}

// ---------------------------------------------------------------------------
// k_stream_init: per-unit state from the offline coarsening just run on the same workspace
// ---------------------------------------------------------------------------
template <int D, typename T>
__global__ void __launch_bounds__(kStreamThreads) k_stream_init(const CoarsenArgs a, const StreamArgs s,
                                                                const __grid_constant__ ProjT proj) {
    __shared__ double red_d[kStreamThreads / 32];
    __shared__ long long red_l[kStreamThreads / 32];
    __shared__ float xk[D], xv[D];
    const int u = blockIdx.x;
    const int b = u / a.Hkv, h = u % a.Hkv;
    const SeqRow sr = a.seq[b];
    UnitState<D, T> st(s, u);
    const int tid = threadIdx.x;
    const int n_ent = a.lens[u];
    const int n_mid = n_ent - sr.s_eff - sr.w_eff;
    if (n_ent > s.Ecap || n_mid < 1) {   // host-checked; never true for valid input
        if (tid == 0) raise_flag(a.flags, FLAG_BAD_LENS);
        return;
    }
    const int2 *ents = a.ents + sr.ent_off + static_cast<int64_t>(h) * sr.emax;
    const int64_t *ls = a.local_scan + sr.mid_off + static_cast<int64_t>(h) * sr.M;
    const T *kraw = static_cast<const T *>(a.k) + (sr.row_off + static_cast<int64_t>(h) * sr.T) * D;
    const T *vraw = static_cast<const T *>(a.v) + (sr.row_off + static_cast<int64_t>(h) * sr.T) * D;
    for (int e = tid; e < n_ent; e += kStreamThreads)
        st.owner[e] = e < sr.s_eff ? -1 : (e < sr.s_eff + n_mid ? 0 : -2 - (e - sr.s_eff - n_mid));
    for (int i = tid; i < n_mid; i += kStreamThreads) st.order[i] = sr.s_eff + i;
    for (int r = tid; r < sr.w_eff; r += kStreamThreads) st.recent[r] = sr.s_eff + n_mid + r;
    // fp64 statistics of every middle node (two passes over its members)
    for (int i = 0; i < n_mid; ++i) {
        const int e = sr.s_eff + i;
        const int2 en = ents[e];
        const int tok = en.x, m = en.y;
        double mk = 0.0, mv = 0.0;
        if (tid < D) {
            for (int r = 0; r < m; ++r) {
                mk += static_cast<double>(static_cast<float>(kraw[static_cast<int64_t>(tok + r) * D + tid]));
                mv += static_cast<double>(static_cast<float>(vraw[static_cast<int64_t>(tok + r) * D + tid]));
            }
            mk /= m;
            mv /= m;
        }
        double q = 0.0;
        if (tid < D)
            for (int r = 0; r < m; ++r) {
                const double dv = static_cast<double>(static_cast<float>(kraw[static_cast<int64_t>(tok + r) * D + tid])) - mk;
                q += dv * dv;
            }
        const double M2 = block_sum(q, red_d);
        long long vsum = 0;
        for (int r = tid; r < m; r += kStreamThreads) {
            const int t = tok - sr.s_eff + r;   // middle index
            vsum += ls[t] - (t % kTileOut != 0 ? ls[t - 1] : 0);
        }
        const long long V = block_sum_ll(vsum, red_l);
        if (tid < D) {
            st.mk[static_cast<int64_t>(e) * D + tid] = mk;
            st.mv[static_cast<int64_t>(e) * D + tid] = mv;
        }
        if (tid == 0) {
            st.m[e] = m;
            st.start[e] = tok;
            st.V[e] = V;
            st.M2[e] = M2;
        }
    }
    // the projection, kept for the appends (small kernel parameters keep their launches cheap)
    if (u == 0)
        for (int i = tid; i < 2 * D * kProjDim; i += kStreamThreads) s.pt[i] = proj.pt[i];
    // feature of the last middle token
    const int last = sr.s_eff + sr.M - 1;
    for (int dim = tid; dim < D; dim += kStreamThreads) {
        xk[dim] = static_cast<float>(kraw[static_cast<int64_t>(last) * D + dim]);
        xv[dim] = static_cast<float>(vraw[static_cast<int64_t>(last) * D + dim]);
    }
    __syncthreads();
    if (tid < kProjDim) st.hdr->z_last[tid] = feature_i(proj.pt, xk, xv, D, tid);
    if (tid == 0) {
        st.hdr->cT = a.unit_total[u];
        st.hdr->n_nodes = n_mid;
        st.hdr->T = sr.T;
        st.hdr->ring = 0;
        st.hdr->n_ent = n_ent;
        st.hdr->N = sr.N;
        st.hdr->S = sr.s_eff;
        st.hdr->W = sr.w_eff;
    }
}

// ---------------------------------------------------------------------------
// k_stream_append: one token per unit
// ---------------------------------------------------------------------------
// dynamic shared memory of the append kernel: P^T, the node order and the nodes' variations
template <int D>
__host__ __device__ constexpr size_t append_smem(int NM) {
    return static_cast<size_t>(2 * D * kProjDim) * 4 + static_cast<size_t>(NM) * 8 + static_cast<size_t>(NM) * 4;
}

template <int D, typename T>
__global__ void __launch_bounds__(kStreamThreads) k_stream_append(const StreamArgs s) {
    static_assert(D <= kStreamThreads, "one thread per dimension");
    extern __shared__ __align__(16) uint8_t dsm[];
    float *sP = reinterpret_cast<float *>(dsm);                               // [2D][16]
    long long *sV = reinterpret_cast<long long *>(dsm + 2 * D * kProjDim * 4);  // [NM] V in node order
    int *sOrder = reinterpret_cast<int *>(sV + s.NM);                          // [NM] node order
    __shared__ float ky[D], vy[D];
    __shared__ float zy[kProjDim];
    __shared__ double red_d[kStreamThreads / 32];
    __shared__ int sh_split, sh_merge_j, sh_pos, sh_ok, sh_yslot, sh_open, sh_mopen;
    __shared__ long long sh_D, sh_Vopen;
    __shared__ uint8_t *sh_opage;
    __shared__ unsigned long long sh_bmin;
    __shared__ float zl[kProjDim];
    const int u = blockIdx.x;
    const int tid = threadIdx.x;
    UnitState<D, T> st(s, u);
    StreamHdr &H = *st.hdr;
    constexpr int VEC = kPageNodes * D * Elem<T>::SIZE;
    // The loads are grouped into rounds of independent requests (every round is one L2 round trip):
    // header; ring slot, open node, last feature and projection; page id and the open node's
    // statistics; the leaving token.
    const int W = H.W, N = H.N;
    int n_nodes = H.n_nodes, n_ent = H.n_ent;
    const int ring = H.ring;
    {   // the projection: every load in flight at once
        constexpr int NV4 = 2 * D * kProjDim / 4 / kStreamThreads;
        float4 p4[NV4];
#pragma unroll
        for (int r = 0; r < NV4; ++r) p4[r] = reinterpret_cast<const float4 *>(s.pt)[r * kStreamThreads + tid];
#pragma unroll
        for (int r = 0; r < NV4; ++r) reinterpret_cast<float4 *>(sP)[r * kStreamThreads + tid] = p4[r];
    }
    if (tid == 0) sh_yslot = st.recent[ring];
    if (tid == 32) sh_open = n_nodes >= 1 ? st.order[n_nodes - 1] : -1;
    if (tid >= 64 && tid < 64 + kProjDim) zl[tid - 64] = H.z_last[tid - 64];
    __syncthreads();
    const int yslot = sh_yslot, open = sh_open;
    if (tid == 0) sh_ok = open >= 0 && entry_page<D, T>(s, u, yslot) != nullptr;
    if (tid == 32 && open >= 0) {
        sh_Vopen = st.V[open];
        sh_mopen = st.m[open];
        sh_opage = entry_page<D, T>(s, u, open);
    }
    // the open node's running means (used if y joins it)
    double mk_o = 0.0, mv_o = 0.0;
    if (tid < D && open >= 0) {
        mk_o = st.mk[static_cast<int64_t>(open) * D + tid];
        mv_o = st.mv[static_cast<int64_t>(open) * D + tid];
    }
    __syncthreads();
    if (!sh_ok) return;

    // 1. the oldest recent token y leaves the window: read it from its pool slot
    const uint8_t *ypg = entry_page<D, T>(s, u, yslot);
    for (int dim = tid; dim < D; dim += kStreamThreads) {
        ky[dim] = Elem<T>::get(ypg + vec_off<D, T>(yslot % kPageNodes, dim));
        vy[dim] = Elem<T>::get(ypg + VEC + vec_off<D, T>(yslot % kPageNodes, dim));
    }
    __syncthreads();
    // 2. its variation step, then first hitting on the open node's budget
    if (tid < kProjDim) zy[tid] = feature_i(sP, ky, vy, D, tid);
    __syncthreads();
    if (tid == 0) {
        long long Dy = quantised_step(zl, zy);
        if (Dy < 0) {
            raise_flag(s.flags, FLAG_OVERFLOW);
            Dy = 0;
        }
        const long long cT = H.cT + Dy;
        H.cT = cT;
        for (int i = 0; i < kProjDim; ++i) H.z_last[i] = zy[i];
        const long long Vo = sh_Vopen;
        sh_split = prod_ge(static_cast<unsigned long long>(N), static_cast<unsigned long long>(Vo + Dy), 1ull,
                           static_cast<unsigned long long>(cT))
                       ? 1
                       : 0;
        if (sh_split && n_ent >= s.Ecap) {   // no free slot: host-checked capacity, never true
            raise_flag(s.flags, FLAG_BAD_LENS);
            sh_split = 0;
        }
        sh_D = Dy;
    }
    __syncthreads();
    const long long Dy = sh_D;
    const int ypos = H.T - W;   // token index of y
    if (sh_split) {
        const int e = n_ent;
        for (int dim = tid; dim < D; dim += kStreamThreads) {
            st.mk[static_cast<int64_t>(e) * D + dim] = ky[dim];
            st.mv[static_cast<int64_t>(e) * D + dim] = vy[dim];
        }
        if (tid == 0) {
            st.m[e] = 1;
            st.V[e] = Dy;
            st.start[e] = ypos;
            st.M2[e] = 0.0;
            st.owner[e] = 0;
            st.order[n_nodes] = e;
        }
        ++n_nodes;
        ++n_ent;
    } else {   // y joins the open node (pairwise update with a one-member node)
        const int e = open;
        const int m = sh_mopen;
        const double inv = 1.0 / (m + 1);
        double q = 0.0;
        if (tid < D) {
            const double dk = static_cast<double>(ky[tid]) - mk_o;
            q = dk * dk;
            st.mk[static_cast<int64_t>(e) * D + tid] = mk_o + dk * inv;
            st.mv[static_cast<int64_t>(e) * D + tid] = mv_o + (static_cast<double>(vy[tid]) - mv_o) * inv;
        }
        const double dd = block_sum(q, red_d);
        if (tid == 0) {
            st.M2[e] += dd * m * inv;
            st.m[e] = m + 1;
            st.V[e] = sh_Vopen + Dy;
        }
    }
    __syncthreads();

    // 3. above N nodes: merge the adjacent pair with the smallest combined variation
    int merged = -1, moved = -1;
    if (n_nodes > N) {
        // the node order, then the nodes' variations, to shared memory (batches of loads in flight)
        for (int j0 = 0; j0 < n_nodes; j0 += 4 * kStreamThreads) {
            int o[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                o[r] = j < n_nodes ? st.order[j] : 0;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                if (j < n_nodes) sOrder[j] = o[r];
            }
        }
        __syncthreads();
        for (int j0 = 0; j0 < n_nodes; j0 += 4 * kStreamThreads) {
            long long vv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                vv[r] = j < n_nodes ? st.V[sOrder[j]] : 0;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                if (j < n_nodes) sV[j] = vv[r];
            }
        }
        __syncthreads();
        // the smallest V_j + V_{j+1} (all >= 0), then the smallest j attaining it
        long long best = LLONG_MAX;
        int bj = INT_MAX;
        for (int j = tid; j < n_nodes - 1; j += kStreamThreads) {
            const long long v2 = sV[j] + sV[j + 1];
            if (v2 < best) {   // j ascending per thread: keeps the leftmost of equal sums
                best = v2;
                bj = j;
            }
        }
        if (tid == 0) {
            sh_bmin = static_cast<unsigned long long>(LLONG_MAX);
            sh_merge_j = INT_MAX;
        }
        __syncthreads();
        atomicMin(&sh_bmin, static_cast<unsigned long long>(best));
        __syncthreads();
        if (static_cast<unsigned long long>(best) == sh_bmin) atomicMin(&sh_merge_j, bj);
        __syncthreads();
        const int j = sh_merge_j;
        const int ea = sOrder[j], eb = sOrder[j + 1];
        // pairwise update: a <- a + b
        const int ma = st.m[ea], mb = st.m[eb];
        const double wb = static_cast<double>(mb) / (ma + mb);
        double q = 0.0;
        for (int dim = tid; dim < D; dim += kStreamThreads) {
            double &ak = st.mk[static_cast<int64_t>(ea) * D + dim];
            double &av = st.mv[static_cast<int64_t>(ea) * D + dim];
            const double dk = st.mk[static_cast<int64_t>(eb) * D + dim] - ak;
            q += dk * dk;
            ak += dk * wb;
            av += (st.mv[static_cast<int64_t>(eb) * D + dim] - av) * wb;
        }
        const double dd = block_sum(q, red_d);
        if (tid == 0) {
            st.M2[ea] += st.M2[eb] + dd * static_cast<double>(ma) * mb / (ma + mb);
            st.m[ea] = ma + mb;
            st.V[ea] += st.V[eb];
        }
        // drop position j + 1 from the node order (from the shared copy)
        for (int t = j + 1 + tid; t < n_nodes - 1; t += kStreamThreads) st.order[t] = sOrder[t + 1];
        __syncthreads();
        --n_nodes;
        merged = ea;
        // the freed slot eb takes the unit's last entry
        const int last = n_ent - 1;
        if (eb != last) {
            const int kind = st.owner[last];
            if (kind <= -2) {   // a recent token: copy its pool entry
                const uint8_t *src = entry_page<D, T>(s, u, last);
                uint8_t *dst = entry_page<D, T>(s, u, eb);
                if (src && dst) {
                    for (int dim = tid; dim < D; dim += kStreamThreads) {
                        Elem<T>::put(dst + vec_off<D, T>(eb % kPageNodes, dim),
                                     Elem<T>::get(src + vec_off<D, T>(last % kPageNodes, dim)));
                        Elem<T>::put(dst + VEC + vec_off<D, T>(eb % kPageNodes, dim),
                                     Elem<T>::get(src + VEC + vec_off<D, T>(last % kPageNodes, dim)));
                    }
                    if (tid == 0)
                        reinterpret_cast<float2 *>(dst + 2 * VEC)[eb % kPageNodes] =
                            reinterpret_cast<const float2 *>(src + 2 * VEC)[last % kPageNodes];
                }
                if (tid == 0) {
                    st.recent[-2 - kind] = eb;
                    st.owner[eb] = kind;
                }
            } else {   // a middle node: move its state; its pool slot is rewritten below
                for (int dim = tid; dim < D; dim += kStreamThreads) {
                    st.mk[static_cast<int64_t>(eb) * D + dim] = st.mk[static_cast<int64_t>(last) * D + dim];
                    st.mv[static_cast<int64_t>(eb) * D + dim] = st.mv[static_cast<int64_t>(last) * D + dim];
                }
                if (tid == 0) {
                    st.m[eb] = st.m[last];
                    st.start[eb] = st.start[last];
                    st.V[eb] = st.V[last];
                    st.M2[eb] = st.M2[last];
                    st.owner[eb] = 0;
                    sh_pos = -1;
                }
                __syncthreads();
                // its position in the order before the shift (sOrder), then after it
                for (int p = tid; p < n_nodes + 1; p += kStreamThreads)
                    if (sOrder[p] == last) sh_pos = p > j + 1 ? p - 1 : p;
                __syncthreads();
                if (tid == 0 && sh_pos >= 0) st.order[sh_pos] = eb;
                if (merged == last) merged = eb;
                moved = eb;
            }
        }
        --n_ent;
        __syncthreads();
    }

    // 4. the new token takes y's (possibly moved) slot as an exact recent entry
    {
        const int ns = merged >= 0 ? st.recent[ring] : yslot;   // entries move only in a merge
        uint8_t *pg = ns == yslot ? const_cast<uint8_t *>(ypg) : entry_page<D, T>(s, u, ns);
        if (pg) {
            const T *kn = static_cast<const T *>(s.k_new) + static_cast<int64_t>(u) * D;
            const T *vn = static_cast<const T *>(s.v_new) + static_cast<int64_t>(u) * D;
            for (int dim = tid; dim < D; dim += kStreamThreads) {
                Elem<T>::put(pg + vec_off<D, T>(ns % kPageNodes, dim), static_cast<float>(kn[dim]));
                Elem<T>::put(pg + VEC + vec_off<D, T>(ns % kPageNodes, dim), static_cast<float>(vn[dim]));
            }
            if (tid == 0) reinterpret_cast<float2 *>(pg + 2 * VEC)[ns % kPageNodes] = make_float2(0.0f, 0.0f);
        }
    }
    // 5. changed middle nodes to the pool
    {
        const int last_node = merged >= 0 || sh_split ? st.order[n_nodes - 1] : open;
        write_node<D, T>(s, st, u, last_node, last_node == open ? sh_opage : nullptr);
    }
    if (merged >= 0) write_node<D, T>(s, st, u, merged);
    if (moved >= 0) write_node<D, T>(s, st, u, moved);
    __syncthreads();
    if (tid == 0) {
        H.n_nodes = n_nodes;
        H.n_ent = n_ent;
        H.ring = (ring + 1) % W;
        H.T = H.T + 1;
        s.lens[u] = n_ent;
    }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
static int64_t up256(int64_t x) { return (x + 255) & ~static_cast<int64_t>(255); }

void stream_layout(int d, int Ecap, int W, StreamArgs *s) {
    s->Ecap = Ecap;
    s->NM = Ecap;
    int64_t off = up256(sizeof(StreamHdr));
    s->off_order = off;
    off = up256(off + 4ll * Ecap);
    s->off_recent = off;
    off = up256(off + 4ll * (W > 0 ? W : 1));
    s->off_owner = off;
    off = up256(off + 4ll * Ecap);
    s->off_m = off;
    off = up256(off + 4ll * Ecap);
    s->off_start = off;
    off = up256(off + 4ll * Ecap);
    s->off_V = off;
    off = up256(off + 8ll * Ecap);
    s->off_M2 = off;
    off = up256(off + 8ll * Ecap);
    s->off_mk = off;
    off = up256(off + 8ll * Ecap * d);
    s->off_mv = off;
    off = up256(off + 8ll * Ecap * d);
    s->unit_bytes = off;
}

cudaError_t launch_stream_init(const CoarsenArgs &a, const StreamArgs &s, const ProjT &proj, cudaStream_t st) {
    const int units = a.B * a.Hkv;
    if (a.dtype == SKV_BF16) {
        if (a.d == 128) k_stream_init<128, __nv_bfloat16><<<units, kStreamThreads, 0, st>>>(a, s, proj);
        else k_stream_init<64, __nv_bfloat16><<<units, kStreamThreads, 0, st>>>(a, s, proj);
    } else {
        if (a.d == 128) k_stream_init<128, float><<<units, kStreamThreads, 0, st>>>(a, s, proj);
        else k_stream_init<64, float><<<units, kStreamThreads, 0, st>>>(a, s, proj);
    }
    return cudaGetLastError();
}

template <int D, typename T>
static cudaError_t append_typed(const StreamArgs &s, cudaStream_t st) {
    const size_t smem = append_smem<D>(s.NM);
    if (smem > 48 * 1024) {
        const cudaError_t e = cudaFuncSetAttribute(k_stream_append<D, T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   static_cast<int>(append_smem<D>(kStreamMaxNodes)));
        if (e != cudaSuccess) return e;
    }
    k_stream_append<D, T><<<s.B * s.Hkv, kStreamThreads, smem, st>>>(s);
    return cudaGetLastError();
}

cudaError_t launch_stream_append(const StreamArgs &s, cudaStream_t st) {
    if (s.NM > kStreamMaxNodes) return cudaErrorInvalidValue;
    if (s.dtype == SKV_BF16)
        return s.d == 128 ? append_typed<128, __nv_bfloat16>(s, st) : append_typed<64, __nv_bfloat16>(s, st);
    return s.d == 128 ? append_typed<128, float>(s, st) : append_typed<64, float>(s, st);
}

}  // namespace skv
