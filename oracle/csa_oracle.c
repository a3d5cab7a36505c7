/*
 * csa_oracle.c -- plain, slow fp64 CPU oracle of the DeepSeek-V4 CSA / HCA attention forward.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * load this library. It shares no code, header, table or helper with the CUDA library; the two
 * meet only in the seeded inputs the tests hand to both.
 *
 * Every step follows the method as stated on the source pages, in their order, in double
 * precision, with no blocking, fusion or reordering:
 *   Hugging Face Transformers docs, "DeepSeek-V4", section "Hybrid attention (§2.3)": compressor,
 *     lightning indexer + top-k (eqs. 13-17), shared K=V MQA, partial interleaved RoPE with the
 *     output rope slice rotated at -i (eq. 26), per-head sink (eq. 27), sliding-window branch;
 *   same page, "Attention mask layout": visibility w < (t+1)//m, -1 sentinels, window mask;
 *   insight.ai.kr digest of the HF blog: softmax-gated pooling with a learned position bias,
 *     ReLU multi-head indexer, FP8 KV with BF16 RoPE dims;
 *   llm-atlas "DeepSeek-V4-Flash", table "config.json full fields": rope_theta,
 *     compress_rope_theta, qk_rope_head_dim, sliding_window, index sizes.
 * Where the pages leave a step open the reading taken is the one the package definition fixes
 * (window [(w+1)m-L, (w+1)m), entry position w*m, theta_tok for raw tokens and theta_cmp for
 * entries with per-branch de-rotation, lambda default 1/sqrt(D), ties to the smaller index).
 *
 * bf16 and FP8 E4M3 inputs are decoded exactly from their public definitions.
 * Parallelism: OpenMP over independent query rows only; each row is computed the same way
 * whatever the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- scalar decoders ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32: widen by shifting into the high 16 bits. */
double orc_bf16_to_f64(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.
 * Exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there is no infinity, so
 * S.1111.110 = 448 is the largest finite value. */
double orc_e4m3_to_f64(uint8_t v)
{
    int sign = v >> 7, e = (v >> 3) & 0xF, mant = v & 0x7;
    double mag;
    if (e == 0xF && mant == 0x7)
        return NAN;
    if (e == 0)
        mag = ldexp((double)mant / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)mant / 8.0, e - 7);
    return sign ? -mag : mag;
}

/* The E4M3 code nearest to a binary32 value, as the OCP definition's saturating conversion
 * rounds it: round to nearest, ties to the code with an even mantissa (its lowest bit 0); finite
 * values beyond the largest magnitude (448) saturate to +-448; NaN gives the NaN code 0x7F. The sign
 * bit is kept, also on a result of zero. The nearest magnitude is found by comparing |x| with every
 * finite non-negative code in turn (codes 0x00..0x7E increase with their value). */
uint8_t orc_e4m3_from_f32(float x)
{
    if (isnan(x))
        return 0x7F;
    int sign = signbit(x) ? 1 : 0;
    double a = fabs((double)x);
    if (a >= 448.0)
        return (uint8_t)(0x7E | (sign << 7));
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7E; ++c) {
        double err = fabs(a - orc_e4m3_to_f64((uint8_t)c));
        if (err < best_err || (err == best_err && (c & 1) == 0)) {
            best = c;
            best_err = err;
        }
    }
    return (uint8_t)(best | (sign << 7));
}

void orc_e4m3_from_f32_array(const float *x, int64_t n, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_e4m3_from_f32(x[i]);
}

/* FP8 form of entry rows (the FP8 KV cache of the insight.ai.kr digest: most of each entry in FP8,
 * the rope channels kept in BF16; the per-entry scale reading): per row of `cols` binary32 values,
 * scale = amax / 448 rounded to binary32 (1 when the row is all zero), each code the E4M3 encoding
 * of x / scale rounded to binary32. Both roundings are single roundings of the exact quotient:
 * a quotient of two binary32 values never lies closer to a binary32 rounding boundary than the
 * binary64 rounding error, so rounding through binary64 first changes nothing. */
void orc_fp8_entry_rows(const float *x, int64_t rows, int cols, uint8_t *codes, float *scale)
{
    for (int64_t i = 0; i < rows; ++i) {
        const float *xr = x + i * (int64_t)cols;
        double amax = 0.0;
        for (int c = 0; c < cols; ++c)
            if (fabs((double)xr[c]) > amax) amax = fabs((double)xr[c]);
        float s = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;
        scale[i] = s;
        for (int c = 0; c < cols; ++c)
            codes[i * (int64_t)cols + c] = orc_e4m3_from_f32((float)((double)xr[c] / (double)s));
    }
}

void orc_bf16_array_to_f64(const uint16_t *x, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = orc_bf16_to_f64(x[i]);
}

/* ---- RoPE: interleaved pairs of the last r channels ------------------------------------------
 * pair p = channels (D-r+2p, D-r+2p+1), frequency theta^(-2p/r), angle pos * frequency. */
void orc_rope(double *x, int D, int r, double pos, double theta)
{
    for (int p = 0; p < r / 2; ++p) {
        double freq = pow(theta, -(2.0 * p) / (double)r);
        double ang = pos * freq;
        double c = cos(ang), s = sin(ang);
        double *a = x + (D - r) + 2 * p;
        double x0 = a[0], x1 = a[1];
        a[0] = x0 * c - x1 * s;
        a[1] = x0 * s + x1 * c;
    }
}

/* ---- 1. compressor ---------------------------------------------------------------------------
 * Entry w pools win(w) = [(w+1)m - L, (w+1)m) clipped to [0,S) with a per-channel softmax over
 * positions of gate[j,d] + bias[j - ((w+1)m - L)], then is rotated at w*m with theta_cmp.
 * kv_rot[j] = kv[j] rotated at j with theta_tok. T = floor(S/m) entries (complete windows only).
 * Either output may be NULL. Returns T, or -1 on bad arguments. */
int64_t orc_compress(const uint16_t *kv, const uint16_t *gate, const float *pos_bias,
                     int64_t S, int D, int m, int L, int r, double theta_cmp, double theta_tok,
                     double *C, double *kv_rot)
{
    if (S < 0 || D <= 0 || m <= 0 || L <= 0 || r < 0 || r > D || (r & 1))
        return -1;
    int64_t T = S / m;
    if (C) {
#pragma omp parallel for schedule(static)
        for (int64_t w = 0; w < T; ++w) {
            int64_t start = (w + 1) * (int64_t)m - L;
            int64_t end = (w + 1) * (int64_t)m; /* exclusive; <= S since w < T */
            int64_t lo = start < 0 ? 0 : start;
            double *out = C + w * (int64_t)D;
            for (int d = 0; d < D; ++d) {
                double mx = -INFINITY;
                for (int64_t j = lo; j < end; ++j) {
                    double a = orc_bf16_to_f64(gate[j * D + d]) + (double)pos_bias[j - start];
                    if (a > mx) mx = a;
                }
                double num = 0.0, den = 0.0;
                for (int64_t j = lo; j < end; ++j) {
                    double a = orc_bf16_to_f64(gate[j * D + d]) + (double)pos_bias[j - start];
                    double e = exp(a - mx);
                    den += e;
                    num += e * orc_bf16_to_f64(kv[j * D + d]);
                }
                out[d] = num / den;
            }
            orc_rope(out, D, r, (double)(w * (int64_t)m), theta_cmp);
        }
    }
    if (kv_rot) {
#pragma omp parallel for schedule(static)
        for (int64_t j = 0; j < S; ++j) {
            double *out = kv_rot + j * (int64_t)D;
            for (int d = 0; d < D; ++d)
                out[d] = orc_bf16_to_f64(kv[j * D + d]);
            orc_rope(out, D, r, (double)j, theta_tok);
        }
    }
    return T;
}

/* ---- 2. visibility ---------------------------------------------------------------------------
 * entry w is visible to query t iff w < floor((t+1)/m); never more than the T entries that exist. */
int64_t orc_visible(int64_t t, int m, int64_t T)
{
    int64_t v = (t + 1) / m;
    return v < T ? v : T;
}

/* ---- 4. lightning indexer --------------------------------------------------------------------
 * I[t,s] = sum_h w[t,h] * ReLU(q^I[t,h,:] . k^I[s,:]) for one query row and one key row. */
static double index_score(const uint16_t *qrow, const float *wrow, const uint16_t *krow, int HI, int dI)
{
    double total = 0.0;
    for (int h = 0; h < HI; ++h) {
        double dot = 0.0;
        for (int c = 0; c < dI; ++c)
            dot += orc_bf16_to_f64(qrow[h * dI + c]) * orc_bf16_to_f64(krow[c]);
        double relu = dot > 0.0 ? dot : 0.0;
        total += (double)wrow[h] * relu;
    }
    return total;
}

/* Prefill scores for the query rows listed in rows[]: out[i, s] = I[rows[i], s] for s < vis,
 * NaN for entries not yet visible. */
void orc_index_scores(const uint16_t *qI, const uint16_t *kI, const float *w,
                      int64_t S, int64_t T, int HI, int dI, int m,
                      const int64_t *rows, int64_t nrows, double *out)
{
    (void)S;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t t = rows[i];
        int64_t vis = orc_visible(t, m, T);
        for (int64_t s = 0; s < T; ++s)
            out[i * T + s] = s < vis ? index_score(qI + t * (int64_t)HI * dI, w + t * (int64_t)HI,
                                                   kI + s * (int64_t)dI, HI, dI)
                                     : NAN;
    }
}

/* Decode scores: one query per sequence b = rows[i], all T entries visible. */
void orc_decode_index_scores(const uint16_t *qI, const float *w, const uint16_t *kI,
                             int64_t B, int64_t T, int HI, int dI,
                             const int64_t *rows, int64_t nrows, double *out)
{
    (void)B;
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t b = rows[i];
#pragma omp parallel for schedule(static)
        for (int64_t s = 0; s < T; ++s)
            out[i * T + s] = index_score(qI + b * (int64_t)HI * dI, w + b * (int64_t)HI,
                                         kI + (b * T + s) * (int64_t)dI, HI, dI);
    }
}

/* ---- 4b. top-k ---------------------------------------------------------------------------------
 * Order candidates by score descending, ties by smaller entry index, keep min(k, vis); the kept
 * set is written in ascending index order and the remaining slots are -1. */
typedef struct { double score; int64_t index; } cand_t;

static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index > b->index) - (a->index < b->index);
}

static int idx_cmp(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

void orc_topk(const double *scores, const int64_t *vis, int64_t nrows, int64_t ld, int k, int32_t *idx)
{
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t v = vis[i];
        cand_t *c = (cand_t *)malloc(sizeof(cand_t) * (size_t)(v > 0 ? v : 1));
        for (int64_t s = 0; s < v; ++s) {
            c[s].score = scores[i * ld + s];
            c[s].index = s;
        }
        qsort(c, (size_t)v, sizeof(cand_t), cand_cmp);
        int64_t keep = v < k ? v : k;
        int32_t *out = idx + i * (int64_t)k;
        for (int64_t j = 0; j < keep; ++j)
            out[j] = (int32_t)c[j].index;
        qsort(out, (size_t)keep, sizeof(int32_t), idx_cmp);
        for (int64_t j = keep; j < k; ++j)
            out[j] = -1;
        free(c);
    }
}

/* ---- 5. core attention for one (query, head) -------------------------------------------------
 * qh: un-rotated query head [D]; wk: nw window rows (post-RoPE, theta_tok); ek: ne entry rows
 * (post-RoPE, theta_cmp); z: sink logit. One softmax over window + entries + sink, K = V, output
 * rope slice of each branch rotated back by -t with that branch's theta. */
static void attend_one(const double *qh, int D, int r, int64_t t,
                       const double *const *wk, int64_t nw, const double *const *ek, int64_t ne,
                       double z, double theta_tok, double theta_cmp, double scale,
                       double *work /* [5*D + nw + ne] */, double *out)
{
    double *q_tok = work, *q_cmp = work + D, *u_win = work + 2 * D, *u_ent = work + 3 * D;
    double *logit = work + 4 * D;
    memcpy(q_tok, qh, sizeof(double) * D);
    memcpy(q_cmp, qh, sizeof(double) * D);
    orc_rope(q_tok, D, r, (double)t, theta_tok);
    orc_rope(q_cmp, D, r, (double)t, theta_cmp);

    double mx = z;
    for (int64_t i = 0; i < nw; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q_tok[d] * wk[i][d];
        logit[i] = scale * dot;
        if (logit[i] > mx) mx = logit[i];
    }
    for (int64_t i = 0; i < ne; ++i) {
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += q_cmp[d] * ek[i][d];
        logit[nw + i] = scale * dot;
        if (logit[nw + i] > mx) mx = logit[nw + i];
    }
    double den = exp(z - mx);
    for (int64_t i = 0; i < nw + ne; ++i) den += exp(logit[i] - mx);

    for (int d = 0; d < D; ++d) u_win[d] = u_ent[d] = 0.0;
    for (int64_t i = 0; i < nw; ++i) {
        double p = exp(logit[i] - mx) / den;
        for (int d = 0; d < D; ++d) u_win[d] += p * wk[i][d];
    }
    for (int64_t i = 0; i < ne; ++i) {
        double p = exp(logit[nw + i] - mx) / den;
        for (int d = 0; d < D; ++d) u_ent[d] += p * ek[i][d];
    }
    orc_rope(u_win, D, r, -(double)t, theta_tok);
    orc_rope(u_ent, D, r, -(double)t, theta_cmp);
    for (int d = 0; d < D; ++d) out[d] = u_win[d] + u_ent[d];
}

/* Prefill attention (CSA when idx != NULL, HCA when idx == NULL) for the listed query rows.
 * q [S,H,D] bf16 un-rotated; C [T,D] and kv_rot [S,D] post-RoPE in double; idx [S,k] int32
 * with -1 sentinels; sinks [H]; out [nrows,H,D]. scale <= 0 selects 1/sqrt(D). */
void orc_attend(const uint16_t *q, const double *C, const double *kv_rot, const int32_t *idx,
                const float *sinks, int64_t S, int H, int D, int64_t T, int k, int W, int r,
                double theta_tok, double theta_cmp, int m, double scale,
                const int64_t *rows, int64_t nrows, double *out)
{
    (void)S;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
#pragma omp parallel
    {
        int64_t cap = (int64_t)W + (idx ? k : T) + 1;
        const double **wk = (const double **)malloc(sizeof(double *) * (size_t)cap);
        const double **ek = (const double **)malloc(sizeof(double *) * (size_t)cap);
        double *qh = (double *)malloc(sizeof(double) * (size_t)D);
        double *work = (double *)malloc(sizeof(double) * (size_t)(5 * D + 2 * cap));
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < nrows; ++i) {
            int64_t t = rows[i];
            int64_t nw = 0, ne = 0;
            for (int64_t j = t - W + 1; j <= t; ++j)
                if (j >= 0) wk[nw++] = kv_rot + j * (int64_t)D;
            if (idx) {
                for (int j = 0; j < k; ++j) {
                    int32_t s = idx[t * (int64_t)k + j];
                    if (s >= 0) ek[ne++] = C + (int64_t)s * D;
                }
            } else {
                int64_t vis = orc_visible(t, m, T);
                for (int64_t s = 0; s < vis; ++s) ek[ne++] = C + s * (int64_t)D;
            }
            for (int h = 0; h < H; ++h) {
                orc_bf16_array_to_f64(q + (t * H + h) * (int64_t)D, D, qh);
                attend_one(qh, D, r, t, wk, nw, ek, ne, (double)sinks[h], theta_tok, theta_cmp, scale,
                           work, out + (i * H + h) * (int64_t)D);
            }
        }
        free(wk); free(ek); free(qh); free(work);
    }
}

/* Decode attention for the listed sequences b = rows[i]: the single query of sequence b sits at
 * position P; window rows win[b, i] hold positions P-W+1+i (post-RoPE, theta_tok); entries are
 * post-RoPE (theta_cmp), either bf16 C [B,T,D] or, when C == NULL, FP8 codes c8 [B,T,D-r] times
 * scale [B,T] on channels [0,D-r) and bf16 rope [B,T,r] on [D-r,D). idx [B,k] (-1 = empty). */
void orc_decode_attend(const uint16_t *q, const uint16_t *C, const uint8_t *c8, const float *c8_scale,
                       const uint16_t *c_rope, const uint16_t *win, const int32_t *idx, const float *sinks,
                       int64_t B, int H, int D, int64_t T, int k, int W, int r, int64_t P,
                       double theta_tok, double theta_cmp, double scale,
                       const int64_t *rows, int64_t nrows, double *out)
{
    (void)B;
    if (scale <= 0.0) scale = 1.0 / sqrt((double)D);
    int64_t cap = (int64_t)W + k + 1;
    double *keys = (double *)malloc(sizeof(double) * (size_t)(cap * D));
    const double **wk = (const double **)malloc(sizeof(double *) * (size_t)cap);
    const double **ek = (const double **)malloc(sizeof(double *) * (size_t)cap);
    for (int64_t i = 0; i < nrows; ++i) {
        int64_t b = rows[i];
        int64_t nw = 0, ne = 0, used = 0;
        for (int j = 0; j < W; ++j) {
            int64_t pos = P - W + 1 + j;
            if (pos < 0) continue;
            double *row = keys + (used++) * (int64_t)D;
            orc_bf16_array_to_f64(win + (b * W + j) * (int64_t)D, D, row);
            wk[nw++] = row;
        }
        for (int j = 0; j < k; ++j) {
            int32_t s = idx[b * (int64_t)k + j];
            if (s < 0) continue;
            double *row = keys + (used++) * (int64_t)D;
            if (C) {
                orc_bf16_array_to_f64(C + (b * T + s) * (int64_t)D, D, row);
            } else {
                const uint8_t *codes = c8 + (b * T + s) * (int64_t)(D - r);
                double sc = (double)c8_scale[b * T + s];
                for (int d = 0; d < D - r; ++d) row[d] = orc_e4m3_to_f64(codes[d]) * sc;
                orc_bf16_array_to_f64(c_rope + (b * T + s) * (int64_t)r, r, row + (D - r));
            }
            ek[ne++] = row;
        }
#pragma omp parallel
        {
            double *qh = (double *)malloc(sizeof(double) * (size_t)D);
            double *work = (double *)malloc(sizeof(double) * (size_t)(5 * D + 2 * cap));
#pragma omp for schedule(static)
            for (int h = 0; h < H; ++h) {
                orc_bf16_array_to_f64(q + (b * H + h) * (int64_t)D, D, qh);
                attend_one(qh, D, r, P, wk, nw, ek, ne, (double)sinks[h], theta_tok, theta_cmp, scale,
                           work, out + (i * H + h) * (int64_t)D);
            }
            free(qh); free(work);
        }
    }
    free(keys); free(wk); free(ek);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
