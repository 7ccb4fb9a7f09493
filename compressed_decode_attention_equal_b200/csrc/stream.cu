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
// The append is a chain of dependent memory round trips, so the state keeps beside each node
// list what lets the append issue every load it needs right after reading the unit's header:
// the nodes' variations in node order, the open node and its page, and the recent window's raw
// keys and values with their pages. One more round trip fetches the merged pair when a merge
// follows a split. A merge always follows a split (the node count is at most N before the
// append), so the entry it frees is refilled by the new node, the last entry.
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
    long long *V, *vord;
    int *rpage;
    float *ring;
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
        vord = reinterpret_cast<long long *>(base + s.off_vord);
        rpage = reinterpret_cast<int *>(base + s.off_rpage);
        ring = reinterpret_cast<float *>(base + s.off_ring);
    }
};

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
            st.vord[i] = V;
            st.M2[e] = M2;
        }
    }
    // the recent window: ring position r holds token T - W + r in pool slot s_eff + n_mid + r
    for (int r = 0; r < sr.w_eff; ++r) {
        const int tok = sr.T - sr.w_eff + r;
        for (int dim = tid; dim < D; dim += kStreamThreads) {
            st.ring[(static_cast<int64_t>(r) * 2) * D + dim] = static_cast<float>(kraw[static_cast<int64_t>(tok) * D + dim]);
            st.ring[(static_cast<int64_t>(r) * 2 + 1) * D + dim] = static_cast<float>(vraw[static_cast<int64_t>(tok) * D + dim]);
        }
        if (tid == 0) st.rpage[r] = s.page_table[static_cast<int64_t>(u) * s.max_pages + (sr.s_eff + n_mid + r) / kPageNodes];
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
        st.hdr->open = sr.s_eff + n_mid - 1;
        st.hdr->open_page = s.page_table[static_cast<int64_t>(u) * s.max_pages + (sr.s_eff + n_mid - 1) / kPageNodes];
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
    __shared__ float zy[kProjDim], zl[kProjDim];
    __shared__ double red_d[kStreamThreads / 32];
    __shared__ int sh_yslot, sh_ypage, sh_mopen, sh_newpage, sh_split, sh_merge_j, sh_pa, sh_pb, sh_ma, sh_mb;
    __shared__ long long sh_D, sh_Vo;
    __shared__ double sh_M2open, sh_M2a, sh_M2b;
    __shared__ unsigned long long sh_bmin;
    const int u = blockIdx.x;
    const int tid = threadIdx.x;
    UnitState<D, T> st(s, u);
    StreamHdr &H = *st.hdr;
    constexpr int VEC = kPageNodes * D * Elem<T>::SIZE;
    constexpr int PAGE = 2 * VEC + kPageNodes * 8;

    // round trip 0: the header
    const int W = H.W, N = H.N, n_nodes0 = H.n_nodes, n_ent0 = H.n_ent, ring = H.ring, Tcur = H.T;
    const int open = H.open, open_page = H.open_page;
    const long long cT0 = H.cT;

    // round trip 1: every other input the append may need, all loads in flight together -- the
    // projection, the last middle feature, the leaving token y (from the recent ring) and its pool
    // slot, the new token, the open node's statistics, the page of the slot a new node would take,
    // and, when the node count is at N (a split is then followed by a merge), the node order with
    // the nodes' variations
    {
        constexpr int NV4 = 2 * D * kProjDim / 4 / kStreamThreads;
        float4 p4[NV4];
#pragma unroll
        for (int r = 0; r < NV4; ++r) p4[r] = reinterpret_cast<const float4 *>(s.pt)[r * kStreamThreads + tid];
#pragma unroll
        for (int r = 0; r < NV4; ++r) reinterpret_cast<float4 *>(sP)[r * kStreamThreads + tid] = p4[r];
    }
    float kn = 0.0f, vn = 0.0f;   // the new token (dimension tid)
    double mk_o = 0.0, mv_o = 0.0;
    if (tid < D) {
        ky[tid] = st.ring[(static_cast<int64_t>(ring) * 2) * D + tid];
        vy[tid] = st.ring[(static_cast<int64_t>(ring) * 2 + 1) * D + tid];
        kn = static_cast<float>(static_cast<const T *>(s.k_new)[static_cast<int64_t>(u) * D + tid]);
        vn = static_cast<float>(static_cast<const T *>(s.v_new)[static_cast<int64_t>(u) * D + tid]);
        mk_o = st.mk[static_cast<int64_t>(open) * D + tid];
        mv_o = st.mv[static_cast<int64_t>(open) * D + tid];
    }
    if (tid >= 64 && tid < 64 + kProjDim) zl[tid - 64] = H.z_last[tid - 64];
    if (tid == 0) {
        sh_yslot = st.recent[ring];
        sh_ypage = st.rpage[ring];
        sh_Vo = st.vord[n_nodes0 - 1];
    }
    if (tid == 32) {
        sh_mopen = st.m[open];
        sh_M2open = st.M2[open];
        sh_newpage = n_ent0 < s.Ecap ? s.page_table[static_cast<int64_t>(u) * s.max_pages + n_ent0 / kPageNodes] : -1;
    }
    const bool may_merge = n_nodes0 >= N;
    if (may_merge) {
        for (int j0 = 0; j0 < n_nodes0; j0 += 4 * kStreamThreads) {
            int o[4];
            long long vv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                o[r] = j < n_nodes0 ? st.order[j] : 0;
                vv[r] = j < n_nodes0 ? st.vord[j] : 0;
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int j = j0 + r * kStreamThreads + tid;
                if (j < n_nodes0) {
                    sOrder[j] = o[r];
                    sV[j] = vv[r];
                }
            }
        }
    }
    __syncthreads();
    const int yslot = sh_yslot, ypage = sh_ypage, m_open = sh_mopen;
    if (ypage < 0 || ypage >= s.num_pages) {
        if (tid == 0) raise_flag(s.flags, FLAG_BAD_PAGE);
        return;
    }
    uint8_t *ypg = s.pages + static_cast<int64_t>(ypage) * PAGE;

    // the leaving token's step (the offline fixed fp32 recipe), then first hitting on the open
    // node's budget
    if (tid < kProjDim) zy[tid] = feature_i(sP, ky, vy, D, tid);
    __syncthreads();
    if (tid == 0) {
        long long Dy = quantised_step(zl, zy);
        if (Dy < 0) {
            raise_flag(s.flags, FLAG_OVERFLOW);
            Dy = 0;
        }
        const long long cT = cT0 + Dy;
        H.cT = cT;
        int split = prod_ge(static_cast<unsigned long long>(N), static_cast<unsigned long long>(sh_Vo + Dy), 1ull,
                            static_cast<unsigned long long>(cT))
                        ? 1
                        : 0;
        if (split && n_ent0 >= s.Ecap) {   // no free slot: host-checked capacity, never true
            raise_flag(s.flags, FLAG_BAD_LENS);
            split = 0;
        }
        sh_split = split;
        sh_D = Dy;
    }
    if (tid < kProjDim) H.z_last[tid] = zy[tid];
    __syncthreads();
    const long long Dy = sh_D;
    const bool split = sh_split != 0;
    const int ypos = Tcur - W;   // token index of y
    int n_nodes = n_nodes0, n_ent = n_ent0;
    int new_open = open, new_open_page = open_page;
    // the node whose pool entry is rewritten at the end, with its statistics (dimension tid)
    int wr_node = -1, wr_page = -1, wr_m = 0;
    double wr_M2 = 0.0, wr_k = 0.0, wr_v = 0.0;

    if (!split) {   // y joins the open node (pairwise update with a one-member node)
        const double inv = 1.0 / (m_open + 1);
        double q = 0.0;
        if (tid < D) {
            const double dk = static_cast<double>(ky[tid]) - mk_o;
            q = dk * dk;
            wr_k = mk_o + dk * inv;
            wr_v = mv_o + (static_cast<double>(vy[tid]) - mv_o) * inv;
            st.mk[static_cast<int64_t>(open) * D + tid] = wr_k;
            st.mv[static_cast<int64_t>(open) * D + tid] = wr_v;
        }
        const double dd = block_sum(q, red_d);
        wr_M2 = sh_M2open + dd * m_open * inv;
        wr_m = m_open + 1;
        if (tid == 0) {
            st.M2[open] = wr_M2;
            st.m[open] = wr_m;
            st.V[open] = sh_Vo + Dy;
            st.vord[n_nodes0 - 1] = sh_Vo + Dy;
        }
        wr_node = open;
        wr_page = open_page;
    } else {
        // y starts a new node in the next free entry
        const int e = n_ent0;
        if (tid < D) {
            st.mk[static_cast<int64_t>(e) * D + tid] = ky[tid];
            st.mv[static_cast<int64_t>(e) * D + tid] = vy[tid];
        }
        if (tid == 0) {
            st.m[e] = 1;
            st.V[e] = Dy;
            st.start[e] = ypos;
            st.M2[e] = 0.0;
            st.owner[e] = 0;
            st.order[n_nodes0] = e;
            st.vord[n_nodes0] = Dy;
            if (may_merge) {
                sOrder[n_nodes0] = e;
                sV[n_nodes0] = Dy;
            }
        }
        n_nodes = n_nodes0 + 1;
        n_ent = n_ent0 + 1;
        new_open = e;
        new_open_page = sh_newpage;
        wr_node = e;
        wr_page = sh_newpage;
        wr_m = 1;
        if (tid < D) {
            wr_k = ky[tid];
            wr_v = vy[tid];
        }
        __syncthreads();

        // above N nodes: merge the adjacent pair with the smallest combined variation. The new
        // node is the last entry and the last in node order, so it is never the left node of the
        // pair; the slot a merge frees is refilled by the new node (unless the new node is the one
        // merged away, which frees its own slot).
        if (n_nodes > N) {
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
            const bool b_new = eb == e;
            // round trip 2: the pair's statistics and the page ids of their slots
            double ak = 0.0, av = 0.0, bk = 0.0, bv = 0.0;
            if (tid < D) {
                ak = st.mk[static_cast<int64_t>(ea) * D + tid];
                av = st.mv[static_cast<int64_t>(ea) * D + tid];
                bk = b_new ? static_cast<double>(ky[tid]) : st.mk[static_cast<int64_t>(eb) * D + tid];
                bv = b_new ? static_cast<double>(vy[tid]) : st.mv[static_cast<int64_t>(eb) * D + tid];
            }
            if (tid == 0) {
                sh_ma = st.m[ea];
                sh_mb = b_new ? 1 : st.m[eb];
                sh_M2a = st.M2[ea];
                sh_M2b = b_new ? 0.0 : st.M2[eb];
                sh_pa = s.page_table[static_cast<int64_t>(u) * s.max_pages + ea / kPageNodes];
                sh_pb = s.page_table[static_cast<int64_t>(u) * s.max_pages + eb / kPageNodes];
            }
            __syncthreads();
            const int ma = sh_ma, mb = sh_mb;
            // pairwise update: a <- a + b (means and summed squared deviations)
            const double wb = static_cast<double>(mb) / (ma + mb);
            double q = 0.0, nk = 0.0, nv = 0.0;
            if (tid < D) {
                const double dk = bk - ak;
                q = dk * dk;
                nk = ak + dk * wb;
                nv = av + (bv - av) * wb;
                st.mk[static_cast<int64_t>(ea) * D + tid] = nk;
                st.mv[static_cast<int64_t>(ea) * D + tid] = nv;
            }
            const double dd = block_sum(q, red_d);
            const double M2ab = sh_M2a + sh_M2b + dd * static_cast<double>(ma) * mb / (ma + mb);
            const long long Vab = sV[j] + sV[j + 1];
            if (tid == 0) {
                st.M2[ea] = M2ab;
                st.m[ea] = ma + mb;
                st.V[ea] = Vab;
                st.vord[j] = Vab;
            }
            // drop position j + 1 from the node order (and its variation)
            for (int t = j + 1 + tid; t < n_nodes - 1; t += kStreamThreads) {
                st.order[t] = sOrder[t + 1];
                st.vord[t] = sV[t + 1];
            }
            __syncthreads();
            n_nodes -= 1;
            n_ent -= 1;
            if (b_new) {
                // the new node merged into its left neighbour, which becomes the open node; the
                // new node's slot (the last entry) is released
                new_open = ea;
                new_open_page = sh_pa;
                wr_node = -1;
            } else {
                // the new node moves into the freed slot eb, at order position n_nodes - 1
                if (tid < D) {
                    st.mk[static_cast<int64_t>(eb) * D + tid] = ky[tid];
                    st.mv[static_cast<int64_t>(eb) * D + tid] = vy[tid];
                }
                if (tid == 0) {
                    st.m[eb] = 1;
                    st.start[eb] = ypos;
                    st.V[eb] = Dy;
                    st.M2[eb] = 0.0;
                    st.owner[eb] = 0;
                    st.order[n_nodes - 1] = eb;
                }
                new_open = eb;
                new_open_page = sh_pb;
                wr_node = eb;
                wr_page = sh_pb;
            }
            // the merged node's pool entry
            if (sh_pa >= 0 && sh_pa < s.num_pages) {
                uint8_t *pg = s.pages + static_cast<int64_t>(sh_pa) * PAGE;
                const int slot = ea % kPageNodes;
                if (tid < D) {
                    Elem<T>::put(pg + vec_off<D, T>(slot, tid), static_cast<float>(nk));
                    Elem<T>::put(pg + VEC + vec_off<D, T>(slot, tid), static_cast<float>(nv));
                }
                if (tid == 0) {
                    const int m = ma + mb;
                    reinterpret_cast<float2 *>(pg + 2 * VEC)[slot] = make_float2(
                        logf(static_cast<float>(m)), static_cast<float>(M2ab / (static_cast<double>(m) * D) / (2.0 * D)));
                }
            } else if (tid == 0) {
                raise_flag(s.flags, FLAG_BAD_PAGE);
            }
        }
    }

    // the new token takes y's slot as an exact recent entry, and y's place in the ring
    if (tid < D) {
        Elem<T>::put(ypg + vec_off<D, T>(yslot % kPageNodes, tid), kn);
        Elem<T>::put(ypg + VEC + vec_off<D, T>(yslot % kPageNodes, tid), vn);
        st.ring[(static_cast<int64_t>(ring) * 2) * D + tid] = kn;
        st.ring[(static_cast<int64_t>(ring) * 2 + 1) * D + tid] = vn;
    }
    if (tid == 0) reinterpret_cast<float2 *>(ypg + 2 * VEC)[yslot % kPageNodes] = make_float2(0.0f, 0.0f);
    // the open node's (or the moved new node's) pool entry, from the statistics held here
    if (wr_node >= 0) {
        if (wr_page >= 0 && wr_page < s.num_pages) {
            uint8_t *pg = s.pages + static_cast<int64_t>(wr_page) * PAGE;
            const int slot = wr_node % kPageNodes;
            if (tid < D) {
                Elem<T>::put(pg + vec_off<D, T>(slot, tid), static_cast<float>(wr_k));
                Elem<T>::put(pg + VEC + vec_off<D, T>(slot, tid), static_cast<float>(wr_v));
            }
            if (tid == 0)
                reinterpret_cast<float2 *>(pg + 2 * VEC)[slot] = make_float2(
                    wr_m == 1 ? 0.0f : logf(static_cast<float>(wr_m)),
                    static_cast<float>(wr_M2 / (static_cast<double>(wr_m) * D) / (2.0 * D)));
        } else if (tid == 0) {
            raise_flag(s.flags, FLAG_BAD_PAGE);
        }
    }
    if (tid == 0) {
        H.n_nodes = n_nodes;
        H.n_ent = n_ent;
        H.open = new_open;
        H.open_page = new_open_page;
        H.ring = (ring + 1) % W;
        H.T = Tcur + 1;
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
    s->off_vord = off;
    off = up256(off + 8ll * Ecap);
    s->off_rpage = off;
    off = up256(off + 4ll * (W > 0 ? W : 1));
    s->off_ring = off;
    off = up256(off + 4ll * 2 * (W > 0 ? W : 1) * d);
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
