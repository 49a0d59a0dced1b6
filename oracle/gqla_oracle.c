/*
 * gqla_oracle.c -- plain fp64 CPU oracle for GQLA decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link
 * or call this file: only the tests, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant generator
 * with the CUDA library.
 *
 * What it computes, and where the definition comes from:
 *
 *  - GQLA keeps one latent row per cached token: c_t (r_kv = 512) followed by
 *    one RoPE key k^R_t (64) shared by all heads, 576 elements in all
 *    ("GQLA: Group-Query Latent Attention ..." on paperlayer.ai, sec. 3
 *    Methods, "Architecture"; sec. 5 Experiments, "Conversion setup").
 *  - The up-projections W_UK and W_UV are indexed by g groups, not by the h_q
 *    query heads (gist.science technical summary, sec. 2 "Architektur";
 *    paperlayer.ai sec. 6 Conclusion).  Head h belongs to group h / (h_q/g):
 *    h_q/g = 16 query heads share one group (pwwt.cn article, sec. 5, "128/8=16").
 *  - GQA path (the un-absorbed definition): K_nope = c_t W_UK_g and
 *    V = c_t W_UV_g are materialised per group, the key is [K_nope ; k^R_t],
 *    and decoding is standard grouped-query attention (paperlayer.ai sec. 2
 *    "Algebraically equivalent decoding paths", sec. 3 "Two equivalent
 *    decoding paths").  This is `gqla_oracle_decode`.
 *  - MQA-absorb path: W_UK is folded into the query and W_UV into the output,
 *    every head attends over the latent row itself (same sections).  It is
 *    algebraically equal to the GQA path; `gqla_oracle_decode_absorbed`
 *    writes it out separately so the two forms can be checked against each
 *    other.
 *  - s_q query tokens per step (multi-token prediction) see the cache
 *    causally (paperlayer.ai sec. 4 Roofline Analysis, "MQA-absorb path" and
 *    "GQA path").
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *  - softmax scale 1/sqrt(d_nope + d_R) = 1/sqrt(192), passed in as `scale`;
 *  - the cached row is [c (512) | k^R (64)], latent first;
 *  - the s_q new tokens are already the last s_q cache entries, so query s of
 *    a sequence of length L sees tokens t <= L - s_q + s (bottom-right causal);
 *  - an empty visible set gives out = 0 and lse = -inf;
 *  - lse is the natural log of sum_t exp(scale * q.k_t).
 *
 * Layouts (all row-major, fp64 unless noted):
 *   q            [batch][s_q][h][192]   (0..127 nope, 128..191 rope)
 *   cache        [num_pages][page_size][576]
 *   page_table   int32 [batch][max_pages]; token t of sequence b lives in
 *                page page_table[b][t / page_size], row t % page_size
 *   seqlens      int32 [batch]
 *   w_uk, w_uv   [g][512][128]
 *   out          [batch][s_q][h][128]
 *   lse          [batch][s_q][h]
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { LAT = 512, ROPE = 64, NOPE = 128, DV = 128, QK = NOPE + ROPE, ROW = LAT + ROPE };

static const double *token_row(const double *cache, const int32_t *page_table, int max_pages,
                               int page_size, int b, int64_t t)
{
    int64_t page = page_table[(int64_t)b * max_pages + t / page_size];
    return cache + (page * page_size + t % page_size) * (int64_t)ROW;
}

/* Softmax-weighted average of `vals` ([n][dv]) with weights exp(score - max). */
static void softmax_average(const double *score, const double *vals, int64_t n, int dv,
                            double *out, double *lse)
{
    if (n <= 0) {
        for (int d = 0; d < dv; ++d) out[d] = 0.0;
        *lse = -INFINITY;
        return;
    }
    double m = -INFINITY;
    for (int64_t t = 0; t < n; ++t) if (score[t] > m) m = score[t];
    double sum = 0.0;
    for (int d = 0; d < dv; ++d) out[d] = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        double p = exp(score[t] - m);
        sum += p;
        for (int d = 0; d < dv; ++d) out[d] += p * vals[t * dv + d];
    }
    for (int d = 0; d < dv; ++d) out[d] /= sum;
    *lse = m + log(sum);
}

static int num_units_all(int batch, int g) { return batch * g; }

/*
 * GQA-path definition: for each requested (b, group) unit, materialise
 * K = [c W_UK_g ; k^R] and V = c W_UV_g for every cached token of sequence b,
 * then run standard attention for the heads of that group.
 * `units` holds pairs (b, group); NULL means every pair.  Outputs of units
 * not listed are left untouched.  Returns 0, or -1 on bad arguments.
 */
int gqla_oracle_decode(int batch, int s_q, int num_heads, int num_groups, int page_size,
                       int max_pages, const double *q, const double *cache,
                       const int32_t *page_table, const int32_t *seqlens, const double *w_uk,
                       const double *w_uv, double scale, const int32_t *units, int num_units,
                       double *out, double *lse)
{
    if (batch <= 0 || s_q <= 0 || num_groups <= 0 || num_heads % num_groups) return -1;
    const int G = num_heads / num_groups;
    if (!units) num_units = num_units_all(batch, num_groups);
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int u = 0; u < num_units; ++u) {
        int b = units ? units[2 * u] : u / num_groups;
        int gi = units ? units[2 * u + 1] : u % num_groups;
        if (b < 0 || b >= batch || gi < 0 || gi >= num_groups) { bad = 1; continue; }
        int64_t L = seqlens[b];
        if (L < 0) { bad = 1; continue; }
        double *K = malloc(sizeof(double) * (size_t)(L ? L : 1) * QK);
        double *V = malloc(sizeof(double) * (size_t)(L ? L : 1) * DV);
        double *score = malloc(sizeof(double) * (size_t)(L ? L : 1));
        const double *wk = w_uk + (int64_t)gi * LAT * NOPE;
        const double *wv = w_uv + (int64_t)gi * LAT * DV;
        for (int64_t t = 0; t < L; ++t) {
            const double *c = token_row(cache, page_table, max_pages, page_size, b, t);
            double *k = K + t * QK, *v = V + t * DV;
            for (int d = 0; d < NOPE; ++d) k[d] = v[d] = 0.0;
            for (int r = 0; r < LAT; ++r)      /* each sum still runs over r = 0..511 in order */
                for (int d = 0; d < NOPE; ++d) {
                    k[d] += c[r] * wk[r * NOPE + d];
                    v[d] += c[r] * wv[r * DV + d];
                }
            for (int j = 0; j < ROPE; ++j) k[NOPE + j] = c[LAT + j];
        }
        for (int s = 0; s < s_q; ++s) {
            int64_t visible = L - s_q + s + 1;
            if (visible > L) visible = L;
            for (int hg = 0; hg < G; ++hg) {
                int h = gi * G + hg;
                const double *qv = q + (((int64_t)b * s_q + s) * num_heads + h) * QK;
                for (int64_t t = 0; t < visible; ++t) {
                    double acc = 0.0;
                    for (int d = 0; d < QK; ++d) acc += qv[d] * K[t * QK + d];
                    score[t] = scale * acc;
                }
                int64_t o = ((int64_t)b * s_q + s) * num_heads + h;
                softmax_average(score, V, visible, DV, out + o * DV, lse + o);
            }
        }
        free(K); free(V); free(score);
    }
    return bad ? -1 : 0;
}

/*
 * MQA-absorb form of the same attention, written independently:
 *   q~ = [W_UK_g q^C ; q^R]  (576),   s_t = scale * q~ . row_t,
 *   o~ = sum_t p_t c_t        (512),   out = W_UV_g^T o~  (128).
 * Used only to check that the two decoding paths agree.
 */
int gqla_oracle_decode_absorbed(int batch, int s_q, int num_heads, int num_groups, int page_size,
                                int max_pages, const double *q, const double *cache,
                                const int32_t *page_table, const int32_t *seqlens,
                                const double *w_uk, const double *w_uv, double scale,
                                double *out, double *lse)
{
    if (batch <= 0 || s_q <= 0 || num_groups <= 0 || num_heads % num_groups) return -1;
    const int G = num_heads / num_groups;
    const int rows = batch * s_q * num_heads;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int r = 0; r < rows; ++r) {
        int h = r % num_heads, s = (r / num_heads) % s_q, b = r / (num_heads * s_q);
        int gi = h / G;
        int64_t L = seqlens[b];
        if (L < 0) { bad = 1; continue; }
        const double *qv = q + (int64_t)r * QK;
        const double *wk = w_uk + (int64_t)gi * LAT * NOPE;
        const double *wv = w_uv + (int64_t)gi * LAT * DV;
        double qa[ROW];
        for (int k = 0; k < LAT; ++k) {
            double acc = 0.0;
            for (int d = 0; d < NOPE; ++d) acc += wk[k * NOPE + d] * qv[d];
            qa[k] = acc;
        }
        for (int j = 0; j < ROPE; ++j) qa[LAT + j] = qv[NOPE + j];
        int64_t visible = L - s_q + s + 1;
        if (visible > L) visible = L;
        double *score = malloc(sizeof(double) * (size_t)(visible > 0 ? visible : 1));
        double *lat = malloc(sizeof(double) * (size_t)(visible > 0 ? visible : 1) * LAT);
        for (int64_t t = 0; t < visible; ++t) {
            const double *c = token_row(cache, page_table, max_pages, page_size, b, t);
            double acc = 0.0;
            for (int k = 0; k < ROW; ++k) acc += qa[k] * c[k];
            score[t] = scale * acc;
            memcpy(lat + t * LAT, c, sizeof(double) * LAT);
        }
        double olat[LAT];
        softmax_average(score, lat, visible, LAT, olat, lse + r);
        for (int d = 0; d < DV; ++d) {
            double acc = 0.0;
            for (int k = 0; k < LAT; ++k) acc += olat[k] * wv[k * DV + d];
            out[(int64_t)r * DV + d] = visible > 0 ? acc : 0.0;
        }
        free(score); free(lat);
    }
    return bad ? -1 : 0;
}

/* Absorbed query q~ = [W_UK_{g(h)} q^C ; q^R] for every (b, s, h) row, fp64. */
int gqla_oracle_absorb_query(int rows, int num_heads, int num_groups, const double *q,
                             const double *w_uk, double *q_absorbed)
{
    if (num_groups <= 0 || num_heads % num_groups) return -1;
    const int G = num_heads / num_groups;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        const double *qv = q + (int64_t)r * QK;
        const double *wk = w_uk + (int64_t)((r % num_heads) / G) * LAT * NOPE;
        double *qa = q_absorbed + (int64_t)r * ROW;
        for (int k = 0; k < LAT; ++k) {
            double acc = 0.0;
            for (int d = 0; d < NOPE; ++d) acc += wk[k * NOPE + d] * qv[d];
            qa[k] = acc;
        }
        for (int j = 0; j < ROPE; ++j) qa[LAT + j] = qv[NOPE + j];
    }
    return 0;
}

/*
 * One-shot cache expansion for the GQA path, exact fp64:
 *   kv[g][n][0:128]   = c_n W_UK_g,   kv[g][n][128:256] = c_n W_UV_g,
 *   k_rope[n][0:64]   = k^R_n.
 * `latent` is [n_slots][576].
 */
void gqla_oracle_expand_f64(int64_t n_slots, int num_groups, const double *latent,
                            const double *w_uk, const double *w_uv, double *kv, double *k_rope)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_slots; ++n) {
        const double *c = latent + n * ROW;
        for (int gi = 0; gi < num_groups; ++gi) {
            const double *wk = w_uk + (int64_t)gi * LAT * NOPE;
            const double *wv = w_uv + (int64_t)gi * LAT * DV;
            double *dst = kv + ((int64_t)gi * n_slots + n) * (NOPE + DV);
            for (int d = 0; d < NOPE; ++d) {
                double k = 0.0, v = 0.0;
                for (int r = 0; r < LAT; ++r) {
                    k += c[r] * wk[r * NOPE + d];
                    v += c[r] * wv[r * DV + d];
                }
                dst[d] = k;
                dst[NOPE + d] = v;
            }
        }
        for (int j = 0; j < ROPE; ++j) k_rope[n * ROPE + j] = c[LAT + j];
    }
}

/* IEEE binary32 -> bfloat16, round to nearest, ties to even (NaN kept quiet). */
static uint16_t bf16_round_nearest_even(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7fffu + lsb;
    return (uint16_t)(u >> 16);
}

uint16_t gqla_oracle_bf16_rne(float f) { return bf16_round_nearest_even(f); }

/*
 * The same expansion with a fixed single-precision rounding order, so that a
 * GPU kernel can be checked bit for bit: every output starts from +0.0f and
 * takes one fused multiply-add per latent index r = 0, 1, ..., 511 in
 * ascending order, then is rounded once to bf16 (nearest, ties to even).
 * Inputs are the bf16 values widened to float.  k_rope is copied bit-exactly.
 */
void gqla_oracle_expand_f32seq(int64_t n_slots, int num_groups, const float *latent,
                               const float *w_uk, const float *w_uv, uint16_t *kv,
                               uint16_t *k_rope)
{
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_slots; ++n) {
        const float *c = latent + n * ROW;
        for (int gi = 0; gi < num_groups; ++gi) {
            const float *wk = w_uk + (int64_t)gi * LAT * NOPE;
            const float *wv = w_uv + (int64_t)gi * LAT * DV;
            uint16_t *dst = kv + ((int64_t)gi * n_slots + n) * (NOPE + DV);
            for (int d = 0; d < NOPE; ++d) {
                float k = 0.0f, v = 0.0f;
                for (int r = 0; r < LAT; ++r) {
                    k = fmaf(c[r], wk[r * NOPE + d], k);
                    v = fmaf(c[r], wv[r * DV + d], v);
                }
                dst[d] = bf16_round_nearest_even(k);
                dst[NOPE + d] = bf16_round_nearest_even(v);
            }
        }
        for (int j = 0; j < ROPE; ++j) k_rope[n * ROPE + j] = bf16_round_nearest_even(c[LAT + j]);
    }
}

int gqla_oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
