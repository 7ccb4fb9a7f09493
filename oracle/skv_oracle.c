/*
 * skv_oracle.c -- plain, slow CPU reference for equal-variation KV coarsening
 * and compressed (macro-node) decode attention.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the package's smoke check and the
 * benchmark's CPU-baseline leg load this file's library. The GPU library never
 * links, includes or calls it, and it includes nothing from the GPU library.
 *
 * Every floating-point result is computed in fp64 from the fp32 values of the
 * inputs (bf16 and fp32 inputs convert to fp32 exactly), with one exception:
 * the per-token variation d_t that decides the integer segmentation. Where a
 * floating-point value decides an integer, both sides must take the decision
 * in the same precision, so d_t follows one fixed fp32 recipe (below) using
 * only correctly rounded IEEE operations (fmaf, subtraction, sqrtf, scaling by
 * a power of two, llrintf). Build with -ffp-contract=off and without
 * -ffast-math. An fp64 d_t is produced beside it for information.
 *
 * Sources:
 *  [EV]  "Equal-Variation KV Cache" (synthcore idea 664): "Mathematical
 *        statement", "Key formulas", "Implementation notes".
 *  [SK]  "SPICY-KV" demo page: section 2 "FlashAttention-2/3 & PagedAttention
 *        Online-Softmax Kernel Fusion" and Independent Claims 1-3.
 *
 * Readings of the pages that this file fixes (the pages leave them open):
 *  R1  Exact tokens: the first S tokens (sinks) and the last W tokens (recent
 *      window) stay exact; when T < S + W the sinks take priority.
 *  R2  The feature is z_t = P [k_t ; v_t] (no hidden state), P is r x 2d with
 *      r = 16, entries N(0,1)/sqrt(r) from a SplitMix64 + Box-Muller stream.
 *  R3  Variation is measured on the middle span only; d_0 = 0.
 *  R4  d_t is quantised to int64 fixed point D_t = rne(d_t * 2^20) and the
 *      cumulative variation c_t is the exact integer prefix sum of D.
 *  R5  "first token whose cumulative variation crosses q_j = j c_T / N" is
 *      b_j = min{ t : N * c_t >= j * c_T }, compared in 128-bit integers; the
 *      boundary token starts the new segment; empty segments are dropped.
 *  R6  A node stores the plain member mean of keys and values, mass m, and
 *      the per-dimension population key variance averaged over dimensions.
 *  R6b Option (orc_coarsen_unit2, rep = 1): a middle segment stores instead
 *      the variation-weighted averages of [EV] "Implementation notes",
 *      k = sum_r d_r k_r / sum_r d_r (same for v), with d_r the fixed-point
 *      step D_r (the common 2^-20 scale cancels); a segment whose steps are
 *      all zero keeps the plain mean. sigma^2, m and alpha stay as in R6
 *      (the variance is about the plain mean of the members).
 *  R7  Decode logit s = q.k/sqrt(d) + ln m + |q|^2 sigma^2/(2d); lse is the
 *      natural-log partition; an empty entry list gives out = 0, lse = -inf.
 *  R7b Option (orc_decode_rows2 with var): the diagonal closure of [SK]
 *      Claim 3 ("diagonal vector sigma_m^2"): the second cumulant of
 *      q.eps/sqrt(d) for independent per-dimension deviations,
 *      s = q.k/sqrt(d) + ln m + sum_i q_i^2 var_i / (2d), var_i the members'
 *      population variance of key dimension i (orc_coarsen_unit2's var). With
 *      var_i = sigma^2 for every i it is the scalar form of R7.
 *  R8  Option (orc_key_mean_f32): common-mode mean removal of [SK]
 *      Independent Claim 1(b) (keys mapped into a less anisotropic space
 *      before coarsening): every key of a unit has the unit's mean key mu
 *      (over all T tokens) subtracted in fp32, and the coarsening then runs on
 *      the centred keys. Because the centred keys feed the fixed fp32
 *      variation recipe, mu itself follows one fixed fp32 order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_OK 0
#define ORC_ERR_ARG (-1)
#define ORC_ERR_OVERFLOW (-4)

#define ORC_PROJ_DIM 16
/* largest D_t accepted (d_t < 2^20); with M < 2^22 tokens c_T stays below 2^62 */
#define ORC_D_MAX 0x1p40f
#define ORC_M_MAX (1 << 22)

/* ------------------------------------------------------------------------ */
/* SplitMix64 (Steele, Lea & Flood, "Fast Splittable Pseudorandom Number     */
/* Generators", OOPSLA 2014): a Weyl sequence with step 0x9e3779b97f4a7c15   */
/* passed through the variant-13 64-bit finaliser of Stafford's mix.         */
/* ------------------------------------------------------------------------ */
static uint64_t orc_splitmix64(uint64_t *state)
{
    uint64_t z;
    *state += 0x9e3779b97f4a7c15ULL;
    z = *state;
    z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
    z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
    return z ^ (z >> 31);
}

void orc_splitmix64_stream(uint64_t seed, int n, uint64_t *out)
{
    uint64_t s = seed;
    for (int i = 0; i < n; ++i) out[i] = orc_splitmix64(&s);
}

/*
 * Projection matrix P (reading R2; [EV] "Implementation notes": "P is a fixed
 * random projection"). Row-major r x cols. Each entry draws two 64-bit words
 * a, b: u1 = ((a >> 11) + 1) 2^-53 in (0, 1], u2 = (b >> 11) 2^-53 in [0, 1),
 * g = sqrt(-2 ln u1) cos(2 pi u2) (Box-Muller, cosine branch), entry =
 * fp32(g / sqrt(r)).
 */
int orc_projection(uint64_t seed, int r, int cols, float *P)
{
    if (r <= 0 || cols <= 0 || !P) return ORC_ERR_ARG;
    const double two_pi = 6.283185307179586476925286766559;
    const double inv_sqrt_r = 1.0 / sqrt((double)r);
    uint64_t s = seed;
    for (long idx = 0; idx < (long)r * cols; ++idx) {
        uint64_t a = orc_splitmix64(&s);
        uint64_t b = orc_splitmix64(&s);
        double u1 = (double)((a >> 11) + 1) * 0x1p-53;
        double u2 = (double)(b >> 11) * 0x1p-53;
        double g = sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
        P[idx] = (float)(g * inv_sqrt_r);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Variation of the projected trajectory ([EV] "Implementation notes":       */
/* z_t = P[k_t; v_t], d_t = ||z_t - z_{t-1}||_2).                            */
/* ------------------------------------------------------------------------ */

/* z = P [k; v] under the fixed fp32 recipe: for each output row i, an fp32
 * accumulator starts at 0 and takes fmaf(P[i][j], x_j, acc) for j = 0..2d-1
 * in ascending order, x = [k; v]. */
void orc_feature_f32(const float *P, const float *k, const float *v, int d, float *z)
{
    const int cols = 2 * d;
    for (int i = 0; i < ORC_PROJ_DIM; ++i) {
        float acc = 0.0f;
        for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + j], k[j], acc);
        for (int j = 0; j < d; ++j) acc = fmaf(P[i * cols + d + j], v[j], acc);
        z[i] = acc;
    }
}

/* The same feature in fp64 (information only). */
static void orc_feature_f64(const float *P, const float *k, const float *v, int d, double *z)
{
    const int cols = 2 * d;
    for (int i = 0; i < ORC_PROJ_DIM; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += (double)P[i * cols + j] * (double)k[j];
        for (int j = 0; j < d; ++j) acc += (double)P[i * cols + d + j] * (double)v[j];
        z[i] = acc;
    }
}

/* D = rne(d * 2^20) with d = sqrtf(sum_i fmaf(delta_i, delta_i, .)), delta_i =
 * zc_i - zp_i in fp32, i ascending. Returns ORC_ERR_OVERFLOW when d * 2^20 is
 * not finite or exceeds 2^40. */
int orc_quantised_step(const float *zp, const float *zc, int64_t *D)
{
    float s = 0.0f;
    for (int i = 0; i < ORC_PROJ_DIM; ++i) {
        float di = zc[i] - zp[i];
        s = fmaf(di, di, s);
    }
    float dd = sqrtf(s);
    float scaled = dd * 1048576.0f; /* exact: power-of-two scaling */
    if (!(scaled <= ORC_D_MAX)) return ORC_ERR_OVERFLOW;
    *D = (int64_t)llrintf(scaled);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Equal-variation boundaries ([EV] "Mathematical statement": breakpoints    */
/* with V(t_j) = j Var / N, first-hitting convention; "Implementation        */
/* notes": thresholds q_j = j c_T / N, boundary = first token whose          */
/* cumulative variation crosses the next threshold).                         */
/* ------------------------------------------------------------------------ */

/* b[0] = 0, b[N] = M, and for j = 1..N-1 the first t with N c_t >= j c_T,
 * found by walking the tokens in order and advancing j each time the running
 * cumulative variation reaches the next threshold. */
int orc_segment(const int64_t *C, int M, int N, int32_t *b)
{
    if (M < 0 || N < 1 || !b) return ORC_ERR_ARG;
    b[0] = 0;
    b[N] = M;
    if (M == 0) {
        for (int j = 1; j < N; ++j) b[j] = 0;
        return ORC_OK;
    }
    const __int128 cT = (__int128)C[M - 1];
    int j = 1;
    for (int t = 0; t < M && j <= N - 1; ++t) {
        const __int128 lhs = (__int128)N * (__int128)C[t];
        while (j <= N - 1 && lhs >= (__int128)j * cT) {
            b[j] = t;
            ++j;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* One (sequence, KV head) unit: split, variation, segmentation, node stats. */
/* ------------------------------------------------------------------------ */

/* Number of entries the unit can produce: S_eff + N + W_eff (upper bound). */
int orc_split(int T, int S, int W, int *S_eff, int *W_eff, int *M)
{
    if (T < 0 || S < 0 || W < 0) return ORC_ERR_ARG;
    int s = S < T ? S : T;
    int w = W < T - s ? W : T - s;
    *S_eff = s;
    *W_eff = w;
    *M = T - s - w;
    return ORC_OK;
}

/* R8: the unit's mean key in a fixed fp32 order. Per dimension i, blocks of
 * ORC_MEAN_BLOCK consecutive tokens are summed in token order from 0 (each
 * addition an IEEE fp32 addition), the block sums are added in block order
 * from 0, and the total is divided by T (IEEE fp32 division); mu = 0 for
 * T = 0. The centred key is then fl32(k_ti - mu_i). */
#define ORC_MEAN_BLOCK 256
int orc_key_mean_f32(const float *k, int T, int d, float *mu)
{
    if (T < 0 || d < 1 || !mu || (T > 0 && !k)) return ORC_ERR_ARG;
    for (int i = 0; i < d; ++i) {
        float total = 0.0f;
        for (int b0 = 0; b0 < T; b0 += ORC_MEAN_BLOCK) {
            const int b1 = b0 + ORC_MEAN_BLOCK < T ? b0 + ORC_MEAN_BLOCK : T;
            float blk = 0.0f;
            for (int t = b0; t < b1; ++t) blk = blk + k[(long)t * d + i];
            total = total + blk;
        }
        mu[i] = T > 0 ? total / (float)T : 0.0f;
    }
    return ORC_OK;
}

/* Node statistics of tokens [start, start + m) ([SK] Claim 2: mass, mean key,
 * mean value; Claim 3: subgrid key variance; section 2: alpha = log m,
 * beta = sigma^2 / (2 d_k)). Two-pass population variance in fp64.
 * w (may be NULL): the members' variation steps D; when given and not all
 * zero, the stored key and value are the D-weighted averages ([EV]
 * "Implementation notes"), the variance still being about the plain mean. */
static void orc_node_stats(const float *k, const float *v, int d, int start, int m, const int64_t *w,
                           double *kt, double *vt, double *var_vec, double *sig2, double *alpha, double *beta)
{
    for (int i = 0; i < d; ++i) {
        double sk = 0.0, sv = 0.0;
        for (int t = start; t < start + m; ++t) {
            sk += (double)k[(long)t * d + i];
            sv += (double)v[(long)t * d + i];
        }
        kt[i] = sk / m;
        vt[i] = sv / m;
    }
    double var_sum = 0.0;
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int t = start; t < start + m; ++t) {
            double dev = (double)k[(long)t * d + i] - kt[i];
            acc += dev * dev;
        }
        var_sum += acc / m;
        if (var_vec) var_vec[i] = acc / m;
    }
    *sig2 = var_sum / d;
    *alpha = log((double)m);
    *beta = *sig2 / (2.0 * d);
    if (w) {
        double W = 0.0;
        for (int r = 0; r < m; ++r) W += (double)w[r];
        if (W > 0.0) {
            for (int i = 0; i < d; ++i) {
                double wk = 0.0, wv = 0.0;
                for (int r = 0; r < m; ++r) {
                    wk += (double)w[r] * (double)k[(long)(start + r) * d + i];
                    wv += (double)w[r] * (double)v[(long)(start + r) * d + i];
                }
                kt[i] = wk / W;
                vt[i] = wv / W;
            }
        }
    }
}

/*
 * Coarsen one unit. k, v: [T][d] fp32 values of the unit's tokens. P: 16 x 2d.
 * Outputs (caller-sized): D, C, d64: [max(M,1)]; b: [N+1]; ent_start,
 * ent_len: [S_eff+N+W_eff]; kt, vt: [(S_eff+N+W_eff) d]; sig2, alpha, beta:
 * [S_eff+N+W_eff]. *E receives the number of entries (sinks, nonempty
 * segments in order, recents). d64 (may be NULL) is the fp64 variation.
 */
/* The coarsening of one unit; D_in (may be NULL): quantised steps given by the caller for the
 * middle tokens (D_in[0] the first middle token's), in place of the fixed fp32 recipe -- the
 * integer stages (prefix sums, first-hitting boundaries) and the node statistics then follow
 * those steps (the stage-wise check of a projection computed another way). */
static int coarsen_core(const float *k, const float *v, int T, int d, int S, int W, int N,
                        const float *P, int rep, const int64_t *D_in, int64_t *D, int64_t *C, double *d64,
                        int32_t *b, int32_t *ent_start, int32_t *ent_len, double *kt, double *vt,
                        double *var_vec, double *sig2, double *alpha, double *beta, int32_t *E)
{
    int s_eff, w_eff, M;
    if (d <= 0 || N < 1 || (!P && !D_in) || !b || !E) return ORC_ERR_ARG;
    if (rep != 0 && (rep != 1 || !D)) return ORC_ERR_ARG;
    if (orc_split(T, S, W, &s_eff, &w_eff, &M) != ORC_OK) return ORC_ERR_ARG;
    if (M >= ORC_M_MAX) return ORC_ERR_OVERFLOW;
    if (D_in) {
        int64_t run = 0;
        for (int t = 0; t < M; ++t) {
            if (D_in[t] < 0 || D_in[t] > ((int64_t)1 << 40)) return ORC_ERR_ARG;
            run += D_in[t];
            if (D) D[t] = D_in[t];
            if (C) C[t] = run;
            if (d64) d64[t] = 0.0;
        }
        if (!C && M > 0) return ORC_ERR_ARG;   /* the given-steps path needs C for the boundaries */
        int rc = orc_segment(C, M, N, b);
        if (rc != ORC_OK) return rc;
        goto entries;
    }

    /* variation on the middle span [s_eff, s_eff + M) */
    float zp[ORC_PROJ_DIM], zc[ORC_PROJ_DIM];
    double zp64[ORC_PROJ_DIM], zc64[ORC_PROJ_DIM];
    int64_t run = 0;
    for (int t = 0; t < M; ++t) {
        const long tok = (long)(s_eff + t) * d;
        orc_feature_f32(P, k + tok, v + tok, d, zc);
        if (d64) orc_feature_f64(P, k + tok, v + tok, d, zc64);
        int64_t Dt = 0;
        double dt64 = 0.0;
        if (t > 0) {
            if (orc_quantised_step(zp, zc, &Dt) != ORC_OK) return ORC_ERR_OVERFLOW;
            if (d64) {
                double s2 = 0.0;
                for (int i = 0; i < ORC_PROJ_DIM; ++i) s2 += (zc64[i] - zp64[i]) * (zc64[i] - zp64[i]);
                dt64 = sqrt(s2);
            }
        }
        run += Dt;
        if (D) D[t] = Dt;
        if (C) C[t] = run;
        if (d64) d64[t] = dt64;
        memcpy(zp, zc, sizeof zp);
        memcpy(zp64, zc64, sizeof zp64);
    }

    /* boundaries need the prefix sums even when the caller did not ask for them */
    int64_t *Cw = C;
    if (!Cw && M > 0) {
        Cw = (int64_t *)malloc(sizeof(int64_t) * (size_t)M);
        if (!Cw) return ORC_ERR_ARG;
        run = 0;
        for (int t = 0; t < M; ++t) {
            const long tok = (long)(s_eff + t) * d;
            orc_feature_f32(P, k + tok, v + tok, d, zc);
            int64_t Dt = 0;
            if (t > 0 && orc_quantised_step(zp, zc, &Dt) != ORC_OK) { free(Cw); return ORC_ERR_OVERFLOW; }
            run += Dt;
            Cw[t] = run;
            memcpy(zp, zc, sizeof zp);
        }
    }
    int rc = orc_segment(Cw, M, N, b);
    if (Cw != C) free(Cw);
    if (rc != ORC_OK) return rc;

entries:;
    /* entries: sinks, nonempty middle segments in order, recents */
    int e = 0;
    for (int t = 0; t < s_eff; ++t, ++e) { ent_start[e] = t; ent_len[e] = 1; }
    for (int j = 0; j < N; ++j) {
        if (b[j + 1] > b[j]) { ent_start[e] = s_eff + b[j]; ent_len[e] = b[j + 1] - b[j]; ++e; }
    }
    for (int t = 0; t < w_eff; ++t, ++e) { ent_start[e] = s_eff + M + t; ent_len[e] = 1; }
    *E = e;
    for (int i = 0; i < e; ++i) {
        /* weights only for middle segments (exact tokens are their own representative) */
        const int mid = ent_start[i] - s_eff;
        const int64_t *w = (rep == 1 && mid >= 0 && mid < M) ? D + mid : NULL;
        orc_node_stats(k, v, d, ent_start[i], ent_len[i], w, kt + (long)i * d, vt + (long)i * d,
                       var_vec ? var_vec + (long)i * d : NULL, sig2 + i, alpha + i, beta + i);
    }
    return ORC_OK;
}

int orc_coarsen_unit2(const float *k, const float *v, int T, int d, int S, int W, int N,
                      const float *P, int rep, int64_t *D, int64_t *C, double *d64, int32_t *b,
                      int32_t *ent_start, int32_t *ent_len, double *kt, double *vt, double *var_vec,
                      double *sig2, double *alpha, double *beta, int32_t *E)
{
    return coarsen_core(k, v, T, d, S, W, N, P, rep, NULL, D, C, d64, b, ent_start, ent_len, kt, vt, var_vec,
                        sig2, alpha, beta, E);
}

/* orc_coarsen_unit2 from given quantised steps D_in[0..M) (see coarsen_core). */
int orc_coarsen_unit_steps(const float *k, const float *v, int T, int d, int S, int W, int N, int rep,
                           const int64_t *D_in, int64_t *D, int64_t *C, int32_t *b, int32_t *ent_start,
                           int32_t *ent_len, double *kt, double *vt, double *var_vec, double *sig2,
                           double *alpha, double *beta, int32_t *E)
{
    if (!D_in) return ORC_ERR_ARG;
    return coarsen_core(k, v, T, d, S, W, N, NULL, rep, D_in, D, C, NULL, b, ent_start, ent_len, kt, vt,
                        var_vec, sig2, alpha, beta, E);
}

/* orc_coarsen_unit2 with the plain-mean representative (R6). */
int orc_coarsen_unit(const float *k, const float *v, int T, int d, int S, int W, int N,
                     const float *P, int64_t *D, int64_t *C, double *d64, int32_t *b,
                     int32_t *ent_start, int32_t *ent_len, double *kt, double *vt,
                     double *sig2, double *alpha, double *beta, int32_t *E)
{
    return orc_coarsen_unit2(k, v, T, d, S, W, N, P, 0, D, C, d64, b, ent_start, ent_len, kt, vt, NULL, sig2,
                             alpha, beta, E);
}

/* ------------------------------------------------------------------------ */
/* Compressed decode attention ([SK] section 2: s = q.k/sqrt(d_k) + log m +  */
/* |q|^2 sigma^2/(2 d_k); the softmax over the entries is then the standard  */
/* one; Claim 3: the closure term).                                          */
/* ------------------------------------------------------------------------ */

/* rows query rows q [rows][d] against E entries (kt, vt [E][d]; alpha, beta
 * [E]). out [rows][d], lse [rows]. fp64 throughout, max-shifted. */
int orc_decode_rows2(const double *q, int rows, int d, const double *kt, const double *vt,
                     const double *alpha, const double *beta, const double *var, int E, double *out,
                     double *lse)
{
    if (rows < 0 || d <= 0 || E < 0) return ORC_ERR_ARG;
    double *s = (double *)malloc(sizeof(double) * (size_t)(E > 0 ? E : 1));
    if (!s) return ORC_ERR_ARG;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    for (int r = 0; r < rows; ++r) {
        const double *qr = q + (long)r * d;
        double *o = out + (long)r * d;
        for (int i = 0; i < d; ++i) o[i] = 0.0;
        if (E == 0) { lse[r] = -INFINITY; continue; }
        double qn2 = 0.0;
        for (int i = 0; i < d; ++i) qn2 += qr[i] * qr[i];
        double mx = -INFINITY;
        for (int j = 0; j < E; ++j) {
            double dot = 0.0;
            for (int i = 0; i < d; ++i) dot += qr[i] * kt[(long)j * d + i];
            double closure = qn2 * beta[j];
            if (var) {   /* R7b: sum_i q_i^2 var_i / (2d) */
                double c = 0.0;
                for (int i = 0; i < d; ++i) c += qr[i] * qr[i] * var[(long)j * d + i];
                closure = c / (2.0 * d);
            }
            s[j] = dot * inv_sqrt_d + alpha[j] + closure;
            if (s[j] > mx) mx = s[j];
        }
        double Z = 0.0;
        for (int j = 0; j < E; ++j) Z += exp(s[j] - mx);
        const double l = mx + log(Z);
        for (int j = 0; j < E; ++j) {
            const double p = exp(s[j] - l);
            for (int i = 0; i < d; ++i) o[i] += p * vt[(long)j * d + i];
        }
        lse[r] = l;
    }
    free(s);
    return ORC_OK;
}

/* orc_decode_rows2 with the scalar closure (R7). */
int orc_decode_rows(const double *q, int rows, int d, const double *kt, const double *vt,
                    const double *alpha, const double *beta, int E, double *out, double *lse)
{
    return orc_decode_rows2(q, rows, d, kt, vt, alpha, beta, NULL, E, out, lse);
}
