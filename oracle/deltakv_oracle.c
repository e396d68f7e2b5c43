/*
 * deltakv_oracle.c -- plain, slow, fp64 CPU oracle for DeltaKV residual
 * KV-cache compression and for attention over the reconstructed cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is used by the test-suite, by the
 * smoke check and by the CPU-baseline leg of the benchmark.  The product path
 * (the CUDA library under decode_attention_strided_b200/csrc) never links,
 * loads or calls it, and the two share no code, header or table.
 *
 * Source of the method: "DeltaKV: Residual-Based KV Cache Compression via
 * Long-Range Similarity" (gist.science summary, section 3 "Metodologia",
 * subsections "Struttura della Compressione", "Processo di Compressione"
 * steps 1-4 and "Ricostruzione").  The summary gives no formulas; the
 * readings taken here for the steps it leaves open are:
 *   - references: token t is a reference iff t mod s == 0; reference slot j
 *     is token j*s (the "fixed stride" of "Struttura della Compressione");
 *   - candidates of a non-reference token t: the slots j with j*s < t
 *     (the "historical" tokens of step 1); there are ceil(t/s) of them;
 *   - similarity: squared L2 distance over the concatenation [K_t ; V_t] of
 *     one kv-head (step 1);
 *   - selection: the k_eff = min(k, ceil(t/s)) smallest distances, ties going
 *     to the lower slot index, stored in ascending (distance, slot) order,
 *     unused entries padded with -1;
 *   - KV_R is the plain mean of the chosen reference rows (step 2) and the
 *     residual is x_t - KV_R (step 3);
 *   - compressor (step 4): code = W2 act(W1 r + b1) + b2, act = exact GELU
 *     x * Phi(x) by default; the stored code is rounded to the cache's
 *     element type (round-to-nearest-even);
 *   - reconstruction ("Ricostruzione"): reference rows are stored as they
 *     are; other tokens become KV_R + W4 act(W3 code + b3) + b4, whose first
 *     d_h entries are K and last d_h entries are V;
 *   - attention of one query head over T reconstructed tokens:
 *     softmax(q . K_t / sqrt(d_h)) . V_t, no mask.
 *
 * Everything is computed in double precision from the exact input values.
 * Arrays are dense, row-major, double unless stated otherwise.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_ACT_GELU_ERF = 0, ORACLE_ACT_GELU_TANH = 1, ORACLE_ACT_NONE = 2 };
enum { ORACLE_ROUND_NONE = 0, ORACLE_ROUND_F32 = 1, ORACLE_ROUND_BF16 = 2, ORACLE_ROUND_Q4 = 3 };

/* ---------------------------------------------------------------- helpers */

/* The nonlinearity between the two linear layers.  Exact GELU is
 * z * Phi(z) = z/2 * (1 + erf(z/sqrt 2)); the tanh form is the usual
 * approximation, offered only when a caller asks for it by name. */
double deltakv_oracle_act(int act, double z)
{
    if (act == ORACLE_ACT_GELU_ERF)
        return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));
    if (act == ORACLE_ACT_GELU_TANH) {
        const double c = sqrt(2.0 / 3.14159265358979323846);
        return 0.5 * z * (1.0 + tanh(c * (z + 0.044715 * z * z * z)));
    }
    return z;
}

/* Round a double to the nearest value with `bits` significant bits
 * (ties to even), keeping the binary exponent range of IEEE float.
 * bits = 24 is IEEE single, bits = 8 is bfloat16.  Written from the
 * definition: scale the value so that its significand becomes an integer
 * with `bits` digits, round that integer with ties-to-even, scale back. */
static double round_sig_bits(double v, int bits)
{
    if (v == 0.0 || !isfinite(v))
        return v;
    int e;
    (void)frexp(v, &e);                 /* v = m * 2^e, 0.5 <= |m| < 1 */
    if (e < -125)                       /* below float's normal range: keep */
        e = -125;                       /* float's fixed subnormal spacing  */
    double scaled = ldexp(v, bits - e); /* |scaled| in [2^(bits-1), 2^bits) */
    double r = nearbyint(scaled);       /* default mode: ties to even        */
    return ldexp(r, e - bits);
}

double deltakv_oracle_round(int mode, double v)
{
    if (mode == ORACLE_ROUND_F32)
        return round_sig_bits(v, 24);
    if (mode == ORACLE_ROUND_BF16)
        return round_sig_bits(v, 8);
    return v;
}

/* 4-bit codes (the summary's section 5, "Efficienza di Memoria": the
 * memory saving is largest combined with 4-bit quantisation; which tensors
 * and which grid the summary does not say).  Reading taken: one code row
 * (the d_c values of one compressed token) is quantised symmetrically to
 * signed 4-bit integers with one scale per row,
 *     scale = bf16(max_i |c_i| / 7),   q_i = clamp(rne(c_i / scale), -7, 7),
 * and the stored (dequantised) code is q_i * scale.  A zero row has scale 0
 * and q = 0.  rne is round to nearest, ties to even; the scale is rounded to
 * bfloat16 first so that the value stored with the codes is the one they were
 * quantised against.  Writes q[0..d_c) and returns the scale. */
double deltakv_oracle_quantize_row4(int d_c, const double* c, int8_t* q)
{
    double amax = 0.0;
    for (int i = 0; i < d_c; ++i)
        if (fabs(c[i]) > amax) amax = fabs(c[i]);
    double scale = deltakv_oracle_round(ORACLE_ROUND_BF16, amax / 7.0);
    for (int i = 0; i < d_c; ++i) {
        double v = scale > 0.0 ? nearbyint(c[i] / scale) : 0.0;
        if (v > 7.0) v = 7.0;
        if (v < -7.0) v = -7.0;
        q[i] = (int8_t)v;
    }
    return scale;
}

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/* Squared L2 distance between token rows a and b of X = [K | V]. */
static double dist2(const double* K, const double* V, int d_h, int a, int b)
{
    double acc = 0.0;
    for (int e = 0; e < d_h; ++e) {
        double d = K[(size_t)a * d_h + e] - K[(size_t)b * d_h + e];
        acc += d * d;
    }
    for (int e = 0; e < d_h; ++e) {
        double d = V[(size_t)a * d_h + e] - V[(size_t)b * d_h + e];
        acc += d * d;
    }
    return acc;
}

/* ------------------------------------------------------ step 1: selection */

/* For a non-reference token t, choose the k_eff nearest strided references.
 * Writes idx[0..k-1] (slots, ascending (distance, slot), -1 padded) and the
 * k-th and (k+1)-th smallest distances (INFINITY where they do not exist).
 * The selection is done by k+1 plain linear scans: each scan takes the
 * smallest distance not yet taken, and a strict '<' over increasing slot
 * numbers makes the lower slot win a tie.  Returns k_eff. */
int deltakv_oracle_select(int t, int d_h, int s, int k,
                          const double* K, const double* V,
                          int32_t* idx, double* d_k, double* d_k1)
{
    int n_cand = ceil_div(t, s); /* slots j with j*s < t */
    double* d = (double*)malloc(sizeof(double) * (size_t)(n_cand > 0 ? n_cand : 1));
    char* taken = (char*)calloc((size_t)(n_cand > 0 ? n_cand : 1), 1);
    for (int j = 0; j < n_cand; ++j)
        d[j] = dist2(K, V, d_h, t, j * s);

    int k_eff = k < n_cand ? k : n_cand;
    double last = INFINITY, next = INFINITY;
    for (int r = 0; r <= k; ++r) {
        int best = -1;
        for (int j = 0; j < n_cand; ++j)
            if (!taken[j] && (best < 0 || d[j] < d[best]))
                best = j;
        if (r < k) {
            idx[r] = best; /* -1 when no candidate is left */
            if (best >= 0) {
                taken[best] = 1;
                last = d[best];
            }
        } else {
            next = best >= 0 ? d[best] : INFINITY;
        }
    }
    if (d_k) *d_k = k_eff > 0 ? last : INFINITY;
    if (d_k1) *d_k1 = next;
    free(d);
    free(taken);
    return k_eff;
}

/* ---------------------------------- steps 2-4: mean, residual, compressor */

/* x_t - mean of the chosen reference rows, written into r[0..2*d_h). */
static void residual(int t, int d_h, int s, int k, const double* K, const double* V,
                     const int32_t* idx, double* r)
{
    int D = 2 * d_h, k_eff = 0;
    for (int e = 0; e < D; ++e) r[e] = 0.0;
    for (int i = 0; i < k; ++i) {
        if (idx[i] < 0) continue;
        int u = idx[i] * s;
        for (int e = 0; e < d_h; ++e) {
            r[e] += K[(size_t)u * d_h + e];
            r[d_h + e] += V[(size_t)u * d_h + e];
        }
        ++k_eff;
    }
    for (int e = 0; e < D; ++e) r[e] /= (double)k_eff;
    for (int e = 0; e < d_h; ++e) {
        r[e] = K[(size_t)t * d_h + e] - r[e];
        r[d_h + e] = V[(size_t)t * d_h + e] - r[d_h + e];
    }
}

/* y = W2 act(W1 x + b1) + b2 with W1 [hid][n_in], W2 [n_out][hid]. */
void deltakv_oracle_mlp(int n_in, int hid, int n_out, int act,
                        const double* W1, const double* b1,
                        const double* W2, const double* b2,
                        const double* x, double* y)
{
    double* h = (double*)malloc(sizeof(double) * (size_t)hid);
    for (int i = 0; i < hid; ++i) {
        double acc = b1 ? b1[i] : 0.0;
        for (int e = 0; e < n_in; ++e) acc += W1[(size_t)i * n_in + e] * x[e];
        h[i] = deltakv_oracle_act(act, acc);
    }
    for (int o = 0; o < n_out; ++o) {
        double acc = b2 ? b2[o] : 0.0;
        for (int i = 0; i < hid; ++i) acc += W2[(size_t)o * hid + i] * h[i];
        y[o] = acc;
    }
    free(h);
}

/* Compress one non-reference or reference token t of a (sequence, kv-head):
 * idx row [k], code row [d_c], and the k-th / (k+1)-th smallest distances.
 * r and c are caller scratch of 2*d_h and d_c doubles. */
static void compress_token(int t, int d_h, int s, int k, int d_c, int hidden, int act,
                           int round_mode, const double* K, const double* V,
                           const double* W1, const double* b1,
                           const double* W2, const double* b2,
                           int32_t* it, double* ct, double* dk, double* dk1,
                           double* r, double* c)
{
    if (t % s == 0) { /* reference token: stored as it is */
        for (int i = 0; i < k; ++i) it[i] = -1;
        for (int o = 0; o < d_c; ++o) ct[o] = 0.0;
        if (dk) *dk = NAN;
        if (dk1) *dk1 = NAN;
        return;
    }
    double a, b;
    deltakv_oracle_select(t, d_h, s, k, K, V, it, &a, &b);
    if (dk) *dk = a;
    if (dk1) *dk1 = b;
    residual(t, d_h, s, k, K, V, it, r);
    deltakv_oracle_mlp(2 * d_h, hidden, d_c, act, W1, b1, W2, b2, r, c);
    if (round_mode == ORACLE_ROUND_Q4) {
        int8_t q[256];
        double scale = deltakv_oracle_quantize_row4(d_c, c, q);
        for (int o = 0; o < d_c; ++o) ct[o] = (double)q[o] * scale;
        return;
    }
    for (int o = 0; o < d_c; ++o) ct[o] = deltakv_oracle_round(round_mode, c[o]);
}

/* Compress the tokens listed in rows[0..n_rows) of one (sequence, kv-head)
 * whose K, V are [T][d_h].  Output row i belongs to token rows[i]:
 *   idx  [n_rows][k]   chosen slots (-1 for reference tokens and padding),
 *   code [n_rows][d_c] the stored code, rounded per round_mode (0 for refs;
 *                      with ORACLE_ROUND_Q4 the dequantised 4-bit code),
 *   d_k, d_k1 [n_rows] the k-th and (k+1)-th smallest distances (NAN for
 *   references).  Tokens are independent, so the loop may run on several
 *   threads (n_threads <= 0 keeps the library default). */
int deltakv_oracle_compress_rows(int T, int d_h, int s, int k, int d_c, int hidden,
                                 int act, int round_mode,
                                 const double* K, const double* V,
                                 const double* W1, const double* b1,
                                 const double* W2, const double* b2,
                                 int n_rows, const int32_t* rows,
                                 int32_t* idx, double* code, double* d_k, double* d_k1,
                                 int n_threads)
{
    if (T < 0 || d_h <= 0 || s <= 0 || k <= 0 || d_c <= 0 || hidden <= 0 || n_rows < 0)
        return -1;
    if (round_mode == ORACLE_ROUND_Q4 && d_c > 256)
        return -1;
    for (int i = 0; i < n_rows; ++i)
        if (rows[i] < 0 || rows[i] >= T) return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double* r = (double*)malloc(sizeof(double) * (size_t)(2 * d_h));
        double* c = (double*)malloc(sizeof(double) * (size_t)d_c);
#pragma omp for schedule(dynamic, 16)
        for (int i = 0; i < n_rows; ++i)
            compress_token(rows[i], d_h, s, k, d_c, hidden, act, round_mode, K, V, W1, b1, W2, b2,
                           idx + (size_t)i * k, code + (size_t)i * d_c,
                           d_k ? d_k + i : NULL, d_k1 ? d_k1 + i : NULL, r, c);
        free(r);
        free(c);
    }
    return 0;
}

/* Compress every token 0..T-1 (rows = 0, 1, ..., T-1). */
int deltakv_oracle_compress(int T, int d_h, int s, int k, int d_c, int hidden,
                            int act, int round_mode,
                            const double* K, const double* V,
                            const double* W1, const double* b1,
                            const double* W2, const double* b2,
                            int32_t* idx, double* code, double* d_k, double* d_k1,
                            int n_threads)
{
    if (T < 0) return -1;
    int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)(T > 0 ? T : 1));
    for (int t = 0; t < T; ++t) rows[t] = t;
    int rc = deltakv_oracle_compress_rows(T, d_h, s, k, d_c, hidden, act, round_mode, K, V,
                                          W1, b1, W2, b2, T, rows, idx, code, d_k, d_k1,
                                          n_threads);
    free(rows);
    return rc;
}

/* ------------------------------------------------------- reconstruction */

/* Rebuild token t ("Ricostruzione") into kh, vh [d_h] from what the cache
 * holds for it: a reference token (t mod s == 0) is its stored row of K, V;
 * any other token is KV_R + W4 act(W3 code + b3) + b4, where KV_R is the mean
 * of the reference rows of the slots it (k entries, -1 unused) lists and
 * code [d_c] is its stored code.  y and mean are caller scratch of 2*d_h. */
static void reconstruct_token(int t, int d_h, int s, int k, int d_c, int hidden, int act,
                              const double* K, const double* V,
                              const int32_t* it, const double* code,
                              const double* W3, const double* b3,
                              const double* W4, const double* b4,
                              double* kh, double* vh, double* y, double* mean)
{
    int D = 2 * d_h;
    if (t % s == 0) {
        for (int e = 0; e < d_h; ++e) {
            kh[e] = K[(size_t)t * d_h + e];
            vh[e] = V[(size_t)t * d_h + e];
        }
        return;
    }
    int k_eff = 0;
    for (int e = 0; e < D; ++e) mean[e] = 0.0;
    for (int i = 0; i < k; ++i) {
        if (it[i] < 0) continue;
        int u = it[i] * s;
        for (int e = 0; e < d_h; ++e) {
            mean[e] += K[(size_t)u * d_h + e];
            mean[d_h + e] += V[(size_t)u * d_h + e];
        }
        ++k_eff;
    }
    deltakv_oracle_mlp(d_c, hidden, D, act, W3, b3, W4, b4, code, y);
    for (int e = 0; e < d_h; ++e) {
        kh[e] = mean[e] / (double)k_eff + y[e];
        vh[e] = mean[d_h + e] / (double)k_eff + y[d_h + e];
    }
}

/* Rebuild K_hat, V_hat [T][d_h] from what the compressed cache holds: the
 * reference rows (read from K, V at tokens j*s only), the slots idx and the
 * codes.  x_hat = KV_R + W4 act(W3 code + b3) + b4 for non-reference tokens. */
int deltakv_oracle_reconstruct(int T, int d_h, int s, int k, int d_c, int hidden, int act,
                               const double* K, const double* V,
                               const int32_t* idx, const double* code,
                               const double* W3, const double* b3,
                               const double* W4, const double* b4,
                               double* K_hat, double* V_hat, int n_threads)
{
    int D = 2 * d_h;
    if (T < 0 || d_h <= 0 || s <= 0 || k <= 0 || d_c <= 0 || hidden <= 0)
        return -1;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double* y = (double*)malloc(sizeof(double) * (size_t)D);
        double* mean = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
        for (int t = 0; t < T; ++t)
            reconstruct_token(t, d_h, s, k, d_c, hidden, act, K, V, idx + (size_t)t * k,
                              code + (size_t)t * d_c, W3, b3, W4, b4,
                              K_hat + (size_t)t * d_h, V_hat + (size_t)t * d_h, y, mean);
        free(y);
        free(mean);
    }
    return 0;
}

/* Rebuild only the tokens rows[0..n_rows) of a (sequence, kv-head) whose raw
 * K, V are [T][d_h] (only their reference rows are read).  Row i of idx_rows
 * [n_rows][k] and code_rows [n_rows][d_c] holds what the cache stores for
 * token rows[i]; K_hat, V_hat [n_rows][d_h] receive the rebuilt rows.  Same
 * arithmetic as deltakv_oracle_reconstruct, token by token. */
int deltakv_oracle_reconstruct_rows(int T, int d_h, int s, int k, int d_c, int hidden, int act,
                                    const double* K, const double* V,
                                    int n_rows, const int32_t* rows,
                                    const int32_t* idx_rows, const double* code_rows,
                                    const double* W3, const double* b3,
                                    const double* W4, const double* b4,
                                    double* K_hat, double* V_hat, int n_threads)
{
    int D = 2 * d_h;
    if (T < 0 || d_h <= 0 || s <= 0 || k <= 0 || d_c <= 0 || hidden <= 0 || n_rows < 0)
        return -1;
    for (int i = 0; i < n_rows; ++i) {
        if (rows[i] < 0 || rows[i] >= T) return -1;
        for (int j = 0; j < k; ++j)
            if (idx_rows[(size_t)i * k + j] >= 0 && idx_rows[(size_t)i * k + j] * s >= rows[i]) return -1;
    }
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
#pragma omp parallel
    {
        double* y = (double*)malloc(sizeof(double) * (size_t)D);
        double* mean = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
        for (int i = 0; i < n_rows; ++i)
            reconstruct_token(rows[i], d_h, s, k, d_c, hidden, act, K, V, idx_rows + (size_t)i * k,
                              code_rows + (size_t)i * d_c, W3, b3, W4, b4,
                              K_hat + (size_t)i * d_h, V_hat + (size_t)i * d_h, y, mean);
        free(y);
        free(mean);
    }
    return 0;
}

/* ------------------------------------------------------------ attention */

/* out[g][:] = sum_t softmax_t(q_g . K_t / sqrt(d_h)) V_t for G query heads
 * that share one kv-head; K, V are [T][d_h]; the largest logit is subtracted
 * before exponentiation.  T must be >= 1. */
int deltakv_oracle_attention(int T, int d_h, int G, const double* q,
                             const double* K, const double* V, double* out)
{
    if (T < 1) return -1;
    double* lg = (double*)malloc(sizeof(double) * (size_t)T);
    double scale = 1.0 / sqrt((double)d_h);
    for (int g = 0; g < G; ++g) {
        const double* qg = q + (size_t)g * d_h;
        double m = -INFINITY;
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int e = 0; e < d_h; ++e) acc += qg[e] * K[(size_t)t * d_h + e];
            lg[t] = acc * scale;
            if (lg[t] > m) m = lg[t];
        }
        double l = 0.0;
        for (int t = 0; t < T; ++t) {
            lg[t] = exp(lg[t] - m);
            l += lg[t];
        }
        for (int e = 0; e < d_h; ++e) {
            double acc = 0.0;
            for (int t = 0; t < T; ++t) acc += lg[t] * V[(size_t)t * d_h + e];
            out[(size_t)g * d_h + e] = acc / l;
        }
    }
    free(lg);
    return 0;
}
