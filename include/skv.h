/*
 * skv.h -- C ABI of libskv: equal-variation KV-cache coarsening and compressed
 * (macro-node) single-query decode attention on one NVIDIA B200 (sm_100a).
 *
 * Two operations, from two web pages:
 *
 *  1. skv_coarsen: "Equal-Variation KV Cache" (synthcore idea 664),
 *     "Mathematical statement" and "Implementation notes". Per (sequence, KV
 *     head) unit the first n_sink tokens and the last n_recent tokens stay
 *     exact; the middle span is cut into N segments of equal cumulative
 *     variation of the projected trajectory z_t = P [k_t; v_t] (first token
 *     whose cumulative variation reaches j c_T / N starts segment j); each
 *     nonempty segment becomes one macro-node. Node statistics follow the
 *     "SPICY-KV" demo page, Independent Claims 2-3 and section 2: mass m =
 *     member count, mean key, mean value, per-dimension key variance sigma^2
 *     averaged over the d dimensions, alpha = ln m, beta = sigma^2 / (2 d).
 *
 *  2. skv_decode_attn: "SPICY-KV" demo page, section 2 ("FlashAttention-2/3 &
 *     PagedAttention Online-Softmax Kernel Fusion") and Claim 3. For each
 *     query row q and each entry j of its KV head's compressed cache,
 *     s_j = q.k_j / sqrt(d) + alpha_j + |q|^2 beta_j; out = softmax(s) V and
 *     lse = ln sum_j exp(s_j).
 *
 * Conventions shared by every entry point:
 *  - All tensor arguments are DEVICE pointers unless the name ends in _host.
 *    The caller owns every buffer (inputs, outputs, node pool, page table,
 *    workspace). No entry point allocates device memory or synchronises the
 *    stream, except skv_workspace_error, which synchronises to read a flag.
 *  - stream is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued on it in order; the call returns before it finishes.
 *  - Host-detectable errors return before anything is enqueued. Errors that
 *    only the device can see (a page id outside the pool, a lens entry above
 *    the page table's capacity, a variation overflow) set a flag in the
 *    workspace header that skv_workspace_error reports; the offending access
 *    is skipped, never performed out of bounds. Flags are sticky: they
 *    accumulate until skv_workspace_error reads and clears them (skv_coarsen
 *    also clears them when it starts).
 *  - A workspace must be zero-filled before its first use (cudaMemsetAsync or
 *    torch.zeros); every call leaves it ready for the next call. Calls that
 *    share a workspace must be ordered on one stream.
 *  - Supported: d in {64, 128}; dtype SKV_F32 or SKV_BF16 (keys, values,
 *    queries, node vectors and outputs share the dtype; alpha/beta and lse are
 *    fp32); at most SKV_MAX_SEQS sequences per call.
 *
 * Node pool layout (produced by skv_coarsen, consumed by skv_decode_attn):
 *  A page holds SKV_PAGE_NODES = 16 consecutive entries of ONE unit, stored
 *  as one contiguous block of skv_page_bytes(dtype, d) bytes:
 *    [0, V)        keys   [16][d] in the dtype         (V = 16 * d * elem)
 *    [V, 2V)       values [16][d] in the dtype
 *    [2V, 2V+128)  {alpha, beta} fp32 pairs [16]
 *  and, in a pool built for the diagonal closure (SKV_CLOSURE_DIAGONAL), also
 *    [2V+128, 3V+128)  per-dimension key variances [16][d] in the dtype
 *  (skv_page_bytes_ex gives the page size of either layout). Within the key,
 *  value and variance blocks the 16-byte chunk c of slot n's vector is
 *  stored at chunk position c ^ (n & 7) (a bank-conflict-free order for the
 *  tensor-core fragment loads; d * elem >= 128 bytes). One page is one copy.
 *  page_table : [B][Hkv][max_pages] int32 physical page ids; entry e of unit
 *               (b, h) lives in page page_table[b][h][e / 16], slot e % 16.
 *  lens       : [B][Hkv] int32 entries per unit, in the order sinks, nonempty
 *               middle segments (in token order), recents.
 *  The pool pointer must be 16-byte aligned.
 */
#ifndef SKV_H
#define SKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SKV_OK = 0,
    SKV_ERR_INVALID_ARG = -1, /* null pointer, bad size, misaligned buffer */
    SKV_ERR_UNSUPPORTED = -2, /* valid but outside the built configurations */
    SKV_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed */
    SKV_ERR_OVERFLOW = -4,    /* variation step above 2^20 or too many tokens */
    SKV_ERR_TIMEOUT = -5,     /* a bounded device wait gave up; that work was abandoned */
    SKV_ERR_WORKSPACE = -6,   /* workspace smaller than the *_workspace_bytes query */
    SKV_ERR_DEVICE = -7       /* device-detected bad page id or lens (see flags) */
} skv_status;

typedef enum { SKV_F32 = 0, SKV_BF16 = 1 } skv_dtype;

#define SKV_PAGE_NODES 16
#define SKV_PROJ_DIM 16
#define SKV_MAX_SEQS 512
#define SKV_MAX_TOKENS ((1 << 22) - 1) /* per sequence */

typedef struct {
    void *pages;       /* [num_pages][skv_page_bytes(dtype, d)] (device) */
    int64_t num_pages; /* capacity, in pages */
} skv_node_pool;

/* Human-readable name of a status code (static storage; never NULL). */
const char *skv_status_string(int status);

/* ABI version of this header (major * 100 + minor). */
int skv_abi_version(void);

/* Bytes of one node-pool page: 2 * 16 * d * elem + 128 (0 for an unsupported dtype or d). */
size_t skv_page_bytes(skv_dtype dtype, int d);

/*
 * The variance a node carries into the decode logit ("SPICY-KV" Independent
 * Claim 3: a scalar sigma_m^2 or a diagonal vector):
 *   SKV_CLOSURE_SCALAR (0): beta = sigma^2 / (2d), logit term |q|^2 beta.
 *   SKV_CLOSURE_DIAGONAL (1): the node also stores var_i, the members'
 *     population variance of key dimension i; logit term
 *     sum_i q_i^2 var_i / (2d) (the second cumulant of q.eps/sqrt(d) for
 *     independent per-dimension deviations; equal to the scalar term when
 *     every var_i equals sigma^2). The pages grow by 16 * d * elem bytes.
 * A pool is built for one closure: skv_coarsen_ex and skv_decode_attn_ex must
 * be given the closure its pages were sized for.
 */
typedef enum { SKV_CLOSURE_SCALAR = 0, SKV_CLOSURE_DIAGONAL = 1 } skv_closure;

/* Bytes of one page for a closure: skv_page_bytes, plus 16 * d * elem for
 * SKV_CLOSURE_DIAGONAL (0 for an unsupported dtype, d or closure). */
size_t skv_page_bytes_ex(skv_dtype dtype, int d, skv_closure closure);

/*
 * The projection the coarsener draws from proj_seed ("Equal-Variation KV
 * Cache", "Implementation notes": z_t = P [k_t; v_t] with P a fixed random
 * projection). P_host: [16][2d] fp32 row-major, written on the host; no GPU
 * work. Entry e consumes two SplitMix64 words a, b of the stream seeded by
 * proj_seed: u1 = ((a >> 11) + 1) 2^-53, u2 = (b >> 11) 2^-53, entry =
 * fp32(sqrt(-2 ln u1) cos(2 pi u2) / 4).
 * Errors: SKV_ERR_INVALID_ARG for P_host == NULL or d not in {64, 128}.
 */
skv_status skv_projection_matrix(uint64_t proj_seed, int d, float *P_host);

/*
 * Bytes of device workspace skv_coarsen needs for this batch (0 on invalid
 * arguments). T_host, N_host: [B] host arrays of sequence lengths and segment
 * counts.
 */
size_t skv_coarsen_workspace_bytes(int B, int Hkv, int d, const int32_t *T_host, const int32_t *N_host,
                                   int n_sink, int n_recent);

/*
 * Coarsen B sequences x Hkv KV heads into the node pool.
 *
 * k, v      : raw keys/values in dtype. Sequence b occupies the contiguous
 *             block [Hkv][T_b][d] starting at element offset
 *             (T_0 + ... + T_{b-1}) * Hkv * d (for equal T this is
 *             [B][Hkv][T][d]). Read only.
 * T_host    : [B] host, tokens per sequence, 0 <= T_b <= SKV_MAX_TOKENS.
 * n_sink, n_recent : exact tokens kept at the start / end (>= 0). When
 *             T_b < n_sink + n_recent the sinks take priority.
 * N_host    : [B] host, middle segments per sequence, 1 <= N_b <= 2^20.
 * proj_seed : seed of the projection P (see skv_projection_matrix).
 * pool, page_table, max_pages : output node pool and the caller's page
 *             assignment ([B][Hkv][max_pages] int32, device). Unit (b, h)
 *             needs ceil((S_eff + N_b + W_eff) / 16) pages (host-checked
 *             against max_pages; page ids device-checked against num_pages).
 * lens      : [B][Hkv] int32 device output, entries written per unit.
 * boundaries: optional ([B][Hkv][Nmax+1] int32 device, Nmax = max_b N_b):
 *             middle-local segment boundaries b_0 = 0 <= ... <= b_N = M_b.
 * cumvar    : optional int64 device array with the token layout of k (one
 *             value per token and head); position t < M_b of unit (b, h)
 *             receives the cumulative quantised variation c_t of middle
 *             token t. Other positions are left untouched.
 * workspace : device scratch of at least skv_coarsen_workspace_bytes bytes,
 *             256-byte aligned; its header holds the device error flags.
 *
 * The variation step d_t = ||z_t - z_{t-1}||_2 is quantised to
 * D_t = rne(d_t * 2^20) (int64) through one fixed fp32 recipe: each z_i is an
 * fp32 fma chain over j = 0..2d-1 ascending from 0; d_t = sqrtf of an fma
 * chain of squared differences over i = 0..15 ascending. The boundaries are
 * therefore exact integers: b_j = min{ t : N c_t >= j c_T } (128-bit
 * products). Node statistics are fp32 (two-pass variance), node vectors are
 * stored in dtype (round to nearest even).
 *
 * Errors: SKV_ERR_INVALID_ARG (null pointers, negative sizes, B > SKV_MAX_SEQS,
 * misalignment, workspace too small -> SKV_ERR_WORKSPACE), SKV_ERR_UNSUPPORTED
 * (d, dtype), SKV_ERR_CUDA (launch failure). A step above 2^20 sets the
 * device overflow flag (SKV_ERR_OVERFLOW from skv_workspace_error).
 */
skv_status skv_coarsen(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                       const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                       uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table,
                       int max_pages, int32_t *lens, int32_t *boundaries, int64_t *cumvar,
                       void *workspace, size_t ws_bytes, void *stream);

/*
 * Options of skv_coarsen_ex.
 *
 * representative: the key and value a middle segment stores.
 *   SKV_REP_MEAN (0): the plain member mean ("SPICY-KV" demo page, Claim 2),
 *     what skv_coarsen stores.
 *   SKV_REP_VARIATION_WEIGHTED (1): the variation-weighted average of
 *     "Equal-Variation KV Cache", "Implementation notes":
 *     k_j = sum_{r in S_j} d_r k_r / sum_{r in S_j} d_r, and the same for v,
 *     with d_r the variation step into token r taken as the fixed-point step
 *     D_r * 2^-20 (so both the weights and which segments have none are exact;
 *     D_0 = 0 for the first middle token). A segment whose steps are all zero
 *     stores the plain mean. Exact tokens (sinks, recents) are unchanged.
 *   In both cases sigma^2 (and beta) is the members' population key variance
 *   about their plain mean (Claim 3 defines it on the members), m and alpha are
 *   unchanged, and the boundaries do not depend on the option.
 * closure: the pool's skv_closure; SKV_CLOSURE_DIAGONAL also writes each
 *   node's per-dimension key variances (zero for exact tokens).
 * center_keys: 1 selects the common-mode mean removal of "SPICY-KV"
 *   Independent Claim 1(b) (keys mapped into a less anisotropic space
 *   before coarsening): every key of a unit enters the pipeline -- the
 *   projection, the segment statistics and the exact tokens alike -- as
 *   fl32(k_t - mu) with mu the unit's mean key over all T_b tokens. mu follows
 *   one fixed fp32 order (per dimension: blocks of 256 consecutive tokens
 *   summed in token order, block sums added in block order, total divided by
 *   T_b), so the centred keys, and hence the boundaries, are exact. The stored
 *   keys are centred: decode outputs are unchanged up to rounding and each
 *   lse moves by -q.mu/sqrt(d). Not available for streaming coarsening.
 * projection: how z_t = P [k_t; v_t] is computed for the variation steps.
 *   SKV_PROJECTION_FIXED_FP32 (0, default): the fixed fp32 fma recipe above;
 *     steps, boundaries and node counts are reproducible bit for bit by any
 *     IEEE fp32 implementation of the recipe.
 *   SKV_PROJECTION_TENSOR_BF16 (1, bf16 inputs only): z = P16 [k; v] on the
 *     tensor cores, P16 = P rounded to bf16 (nearest even), exact products
 *     accumulated in fp32 in the hardware's order; d_t and D_t then follow the
 *     same recipe from z. A different fixed random projection (P16) and a
 *     different summation order: each step D_t stays within the fp32
 *     accumulation bound of the exact P16 projection's step, and the
 *     boundaries are the exact first-hitting boundaries of those steps (given
 *     the steps, every later stage is exact), but the steps are not those of
 *     the fixed recipe, so boundaries may differ from the default's. The
 *     projection reads the raw keys even with center_keys (a common shift
 *     cancels in z_t - z_{t-1}). fp32 inputs: SKV_ERR_UNSUPPORTED.
 * reserved: must be zero.
 */
typedef enum { SKV_REP_MEAN = 0, SKV_REP_VARIATION_WEIGHTED = 1 } skv_representative;

typedef enum { SKV_PROJECTION_FIXED_FP32 = 0, SKV_PROJECTION_TENSOR_BF16 = 1 } skv_projection;

typedef struct {
    int32_t representative; /* skv_representative */
    int32_t closure;        /* skv_closure */
    int32_t center_keys;    /* 0 or 1: common-mode mean removal (see above) */
    int32_t projection;     /* skv_projection (see above) */
    int32_t reserved[4];
} skv_coarsen_options;

/*
 * skv_coarsen with options (NULL = defaults, identical to skv_coarsen). Same
 * arguments, layouts, ownership and errors as skv_coarsen; additionally
 * SKV_ERR_INVALID_ARG for an unknown representative, closure or projection,
 * center_keys not 0 or 1, or a nonzero reserved field; SKV_ERR_UNSUPPORTED for
 * the tensor-core projection on fp32 inputs.
 */
skv_status skv_coarsen_ex(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                          const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                          uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table,
                          int max_pages, int32_t *lens, int32_t *boundaries, int64_t *cumvar,
                          void *workspace, size_t ws_bytes, const skv_coarsen_options *options,
                          void *stream);

/*
 * Streaming coarsening ("Equal-Variation KV Cache", "Implementation notes":
 * in streaming inference a segment that exceeds its variation budget is
 * split at the first threshold crossing and adjacent low-variation segments
 * are merged; node merges follow the law of total variance, "SPICY-KV"
 * dependent Claim 10). The page leaves the policy open; this library fixes:
 *  - skv_stream_init coarsens the prompt exactly as skv_coarsen (plain mean,
 *    scalar closure) and records per-unit streaming state: each middle node's
 *    mass m, variation V (sum of its steps D), first token and fp64 mean key,
 *    mean value and summed squared key deviations M2, in token order; c_T;
 *    the last middle token's feature; the recent window's pool slots.
 *  - skv_stream_append appends one token per unit (k_new, v_new: [B][Hkv][d]
 *    in dtype, device). The oldest recent token y enters the middle: its step
 *    D_y (the offline fixed fp32 recipe against the previous middle token) is
 *    added to c_T; if N (V_open + D_y) >= c_T (exact 128-bit comparison; the
 *    open node is the last middle node) y starts a new node with V = D_y,
 *    otherwise it joins the open node. While more than N middle nodes exist
 *    the adjacent pair with the smallest V_j + V_{j+1} merges (leftmost on
 *    ties): masses and variations add, means and M2 combine by the pairwise
 *    update. The new token takes y's pool slot as an exact recent entry.
 *    Node outputs as offline: alpha = ln m (0 for m = 1),
 *    beta = M2 / (m d) / (2 d); lens is updated.
 * Entries of a streamed unit are kept in no particular order in its pool
 * slots [0, lens) (decode attention does not depend on their order): a merge
 * frees a slot, which the unit's last entry then fills.
 * Requirements: bf16 or fp32, d in {64, 128}, n_recent >= 1; every sequence
 * has T_b > n_sink + n_recent at init (a non-empty middle; else
 * SKV_ERR_UNSUPPORTED); each unit's page table row holds
 * n_sink + max_b N_b + 1 + n_recent <= 8192 entries (host-checked; larger
 * capacities return SKV_ERR_INVALID_ARG). skv_stream_append
 * takes the N_host, n_sink and n_recent given to skv_stream_init (they fix
 * the state layout).
 * state: device buffer of skv_stream_state_bytes bytes (caller-owned, written
 * by skv_stream_init -- including the projection P drawn from proj_seed,
 * which the appends reuse -- and read and updated by each skv_stream_append;
 * calls that share a state must be ordered on one stream).
 * workspace (append): any zero-filled device buffer of >= 256 bytes whose
 * header holds the device error flags (see skv_workspace_error), e.g. the
 * coarsen workspace.
 */
size_t skv_stream_state_bytes(int B, int Hkv, int d, const int32_t *N_host, int n_sink, int n_recent);

skv_status skv_stream_init(const void *k, const void *v, skv_dtype dtype, int B, int Hkv, int d,
                           const int32_t *T_host, int n_sink, int n_recent, const int32_t *N_host,
                           uint64_t proj_seed, const skv_node_pool *pool, const int32_t *page_table,
                           int max_pages, int32_t *lens, void *workspace, size_t ws_bytes, void *state,
                           size_t state_bytes, void *stream);

skv_status skv_stream_append(const void *k_new, const void *v_new, skv_dtype dtype, int B, int Hkv, int d,
                             const int32_t *N_host, int n_sink, int n_recent, const skv_node_pool *pool,
                             const int32_t *page_table, int max_pages, int32_t *lens, void *state,
                             size_t state_bytes, void *workspace, size_t ws_bytes, void *stream);

/* Bytes of device workspace skv_decode_attn needs (0 on invalid arguments). */
size_t skv_decode_workspace_bytes(int B, int R, int Hq, int Hkv, int d, int max_pages);

/*
 * Compressed decode attention.
 *
 * q     : [B][R][Hq][d] queries in dtype (R independent query rows per
 *         sequence, pre-RoPE basis). Query head hq reads KV head hq / (Hq/Hkv).
 * pool, page_table, max_pages, lens : the compressed cache (layout above).
 * out   : [B][R][Hq][d] in dtype, softmax(s) V.
 * lse   : [B][R][Hq] fp32, natural-log partition ln sum_j exp(s_j); a unit
 *         with zero entries gives out = 0 and lse = -inf.
 * workspace : device scratch of at least skv_decode_workspace_bytes bytes,
 *         256-byte aligned (split partials, per-unit completion counters that
 *         every call returns to zero, and the device error flags).
 *
 * One kernel launch per call (programmatic stream serialisation: it becomes
 * resident while the previous launch drains, and reads its inputs only after
 * every preceding grid in the stream has completed). Graph-capturable.
 *
 * Errors: SKV_ERR_INVALID_ARG, SKV_ERR_UNSUPPORTED (d, dtype, Hq % Hkv != 0),
 * SKV_ERR_WORKSPACE, SKV_ERR_CUDA. Device-detected bad page ids or lens above
 * max_pages * 16 set the device flag (SKV_ERR_DEVICE from
 * skv_workspace_error); those pages are skipped.
 */
skv_status skv_decode_attn(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                           const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                           const int32_t *lens, void *out, float *lse, void *workspace, size_t ws_bytes,
                           void *stream);

/*
 * Options of skv_decode_attn_ex. closure: the pool's skv_closure
 * (SKV_CLOSURE_DIAGONAL reads each node's per-dimension variances and uses
 * sum_i q_i^2 var_i / (2d) in place of |q|^2 beta). reserved: must be zero.
 */
typedef struct {
    int32_t closure; /* skv_closure */
    int32_t reserved[7];
} skv_decode_options;

/*
 * skv_decode_attn with options (NULL = defaults, identical to
 * skv_decode_attn). Same arguments, layouts, ownership, workspace and errors;
 * additionally SKV_ERR_INVALID_ARG for an unknown closure or a nonzero
 * reserved field.
 */
skv_status skv_decode_attn_ex(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                              const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                              const int32_t *lens, void *out, float *lse, void *workspace, size_t ws_bytes,
                              const skv_decode_options *options, void *stream);

/*
 * Decode attention without any caller-provided workspace. (The sources describe no such entry
 * point; it exists for callers of this library that cannot allocate device memory.)
 *
 * Some callers cannot allocate: a plugin that a host framework hands only its input and output
 * buffers, a runtime whose device allocator is fixed when it starts, or code on a latency-critical
 * path where cudaMalloc, which may synchronise the device, is not allowed. This entry point takes
 * the same arguments as skv_decode_attn minus the workspace, applies the same checks and launches
 * the same kernel with the same grid, so its out and lse are bit-identical to skv_decode_attn's
 * for the same inputs. Its scratch -- device flags, per-unit completion counters and split
 * partials -- lives in one array of SKV_NOALLOC_SCRATCH_BYTES that the library defines at file
 * scope. Every GPU that loads the library reserves that array once and keeps it until the
 * process exits.
 *  - No cudaMalloc, cudaFree or other allocating call is made.
 *  - The first call on each device looks up the array's device address (cudaGetSymbolAddress)
 *    with that device current and caches it; make that first call before any stream capture.
 *  - All calls on a device share the array and it keeps the last call's contents: each call
 *    clears the flags and counters on `stream` before its kernel runs, and calls whose kernels
 *    may overlap on the GPU (other streams, or other threads' streams) race on the array and
 *    must be serialised by the caller.
 *  - A request whose scratch would exceed SKV_NOALLOC_SCRATCH_BYTES (bf16: split partials of
 *    2 x grid x rows-per-pass x (d + 1) floats, plus 4 bytes per unit and row pass) returns
 *    SKV_ERR_WORKSPACE before anything is enqueued; use skv_decode_attn for such sizes.
 *  - Scalar-closure pools only (the pools skv_coarsen builds).
 *  - Device-detected errors (bad page id, lens above capacity) still skip the bad access, but
 *    their flags live in the library's array and are not reported; diagnose with skv_decode_attn.
 * Other errors: as skv_decode_attn.
 */
#define SKV_NOALLOC_SCRATCH_BYTES (4u << 20)
skv_status skv_decode_attn_noalloc(const void *q, skv_dtype dtype, int B, int R, int Hq, int Hkv, int d,
                                   const skv_node_pool *pool, const int32_t *page_table, int max_pages,
                                   const int32_t *lens, void *out, float *lse, void *stream);

/*
 * Check of the device error path that a stuck pipeline takes. Every wait of
 * the library's kernels on an mbarrier (a copy landing, a stage being freed)
 * polls at most 2^20 times; when the polls run out the kernel raises the
 * timeout flag, abandons the work it cannot finish (after waiting, again
 * bounded, for its copies in flight) and returns, so the context stays
 * usable. This call launches one thread that waits in the same way on a
 * barrier nothing ever arrives at, for `polls` polls (0 .. 2^20), no copy
 * outstanding, and raises the flag in `workspace` (any zero-filled buffer of
 * >= 256 bytes, 256-byte aligned, e.g. a decode workspace). Afterwards
 * skv_workspace_error returns SKV_ERR_TIMEOUT with flag bit 8. No counterpart
 * in the sources: it exists to test failure reporting without a GPU fault.
 * Errors: SKV_ERR_WORKSPACE (NULL, misaligned or too small), SKV_ERR_INVALID_ARG
 * (polls above 2^20), SKV_ERR_CUDA (launch failure).
 */
skv_status skv_wait_selftest(void *workspace, size_t ws_bytes, uint32_t polls, void *stream);

/*
 * Read and clear the device error flags raised on this workspace since they
 * were last cleared. The read and the clear are enqueued on `stream` (after
 * the work already there) and the call then synchronises that stream. Returns
 * SKV_OK, SKV_ERR_OVERFLOW (a variation step above 2^20), SKV_ERR_TIMEOUT (a
 * bounded wait gave up and its work was abandoned), or SKV_ERR_DEVICE (a bad
 * page id or lens entry was skipped); in that order of precedence when
 * several flags are set (SKV_ERR_CUDA if a copy or the synchronisation
 * fails). *flags_host (optional) receives the raw bits: 1 overflow, 2 bad page
 * id, 4 lens above capacity, 8 a bounded wait gave up.
 */
skv_status skv_workspace_error(const void *workspace, void *stream, uint32_t *flags_host);

#ifdef __cplusplus
}
#endif

#endif /* SKV_H */
