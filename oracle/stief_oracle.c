/*
 * stief_oracle.c -- plain fp64 CPU oracle for StiefAttention latent-KV decode.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the correctness reference that the
 * CUDA path is checked against.  Only tests/, __graft_entry__.smoke() and the
 * CPU-baseline / reference arm of bench.py load it.  The product library never
 * links, calls or falls back to it, and it shares no code, header or table with
 * the CUDA sources.
 *
 * What it computes, and where the pages define it ("Don't be so Stief! Learning
 * KV Cache low-rank approximation over the Stiefel manifold", StiefAttention
 * technical summary, section "Mecanismo Central"/"Kernmechanismus", item 5
 * "Inferencia"/"Inferenz"):
 *
 *   - keys and values are stored compressed, K_down = K . P_K and
 *     V_down = V . P_V, with P_K (d x r_K) and P_V (d x r_V) having orthonormal
 *     columns (item 2, "Stiefel manifold");
 *   - before attention the full dimensions are reconstructed on the fly,
 *     K~ = K_down . P_K^T and V~ = V_down . P_V^T;
 *   - attention itself is ordinary softmax attention over the reconstructed
 *     keys and values.
 *
 * Readings taken where the pages are silent:
 *   - one basis pair per KV head, stored [Hkv][d][r];
 *   - scores scaled by 1/sqrt(d) with d the full head dimension;
 *   - grouped-query attention with contiguous groups, query head h reads KV
 *     head h / (Hq/Hkv);
 *   - the stored latent is rounded once, round-to-nearest-even, to bfloat16;
 *   - a sequence of length 0 attends to nothing and yields a zero output.
 *
 * Everything is computed in IEEE double precision, in the order the definition
 * states: no blocking, no fusion, no reordering of a sum.  OpenMP only runs
 * independent (sequence, KV head) problems side by side; the arithmetic of each
 * problem is sequential and identical with any thread count.
 *
 * Parity pins (tests/test_oracle_pins.py): bf16 rounding against torch's
 * float32->bfloat16 conversion, r = d reduces to textbook softmax attention
 * (torch scaled_dot_product_attention in float64), invariance under the basis
 * change P -> P.O (the QR "change of coordinates" remark, item 3), closed forms
 * for one and two tokens, token-order invariance, and compression with
 * P = [I; 0] reproducing the first r coordinates exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------- */
/* bfloat16 rounding                                                           */
/* ------------------------------------------------------------------------- */

/*
 * Round a double to the nearest bfloat16 value, ties to even.
 *
 * bfloat16 has 8 significant bits (7 stored), the exponent range of binary32
 * (smallest normal 2^-126) and subnormals down to 2^-133.  The value is
 * rounded by scaling onto the integer grid of its binade and applying
 * nearbyint() in the default round-to-nearest-even mode.  Magnitudes that
 * round to 2^128 or beyond become infinity.  NaN stays NaN.
 */
double stief_oracle_round_bf16(double x)
{
    if (isnan(x) || isinf(x) || x == 0.0)
        return x;
    int e;
    frexp(fabs(x), &e);                     /* |x| = m * 2^e, m in [0.5, 1) */
    /* spacing of bf16 values in this binade: 2^(e-8) for normals,
       fixed 2^-133 in the subnormal range */
    int q_exp = e - 8;
    if (q_exp < -133)
        q_exp = -133;
    double q = ldexp(1.0, q_exp);
    double r = nearbyint(x / q) * q;
    if (fabs(r) >= ldexp(1.0, 128))
        r = copysign(INFINITY, x);
    return r;
}

/* Elementwise rounding of an array (n values). */
void stief_oracle_round_bf16_array(const double* x, double* y, long n)
{
    for (long i = 0; i < n; ++i)
        y[i] = stief_oracle_round_bf16(x[i]);
}

/* ------------------------------------------------------------------------- */
/* Compressed storage: K_down = K . P                                          */
/* ------------------------------------------------------------------------- */

/*
 * y[t][c] = sum_{i<d} x[t][i] * P[i][c]     for t < T, c < r
 * optionally rounded once to bf16 (round_bf16 != 0).
 * x is [T][d], P is [d][r], y is [T][r], all row-major doubles.
 */
void stief_oracle_project(const double* x, const double* P, double* y,
                          long T, int d, int r, int round_bf16)
{
    for (long t = 0; t < T; ++t) {
        for (int c = 0; c < r; ++c) {
            double acc = 0.0;
            for (int i = 0; i < d; ++i)
                acc += x[t * d + i] * P[(long)i * r + c];
            y[t * r + c] = round_bf16 ? stief_oracle_round_bf16(acc) : acc;
        }
    }
}

/*
 * Append T new rows per (sequence, KV head) to the latent cache.
 *
 *   k_new, v_new : [B][Hkv][T][d]
 *   P_K, P_V     : [Hkv][d][rK], [Hkv][d][rV]
 *   k_lat, v_lat : [B][Hkv][L_max][rK], [B][Hkv][L_max][rV]
 *   seq_lens     : [B], updated in place
 *
 * Sequence b writes rows [seq_lens[b], seq_lens[b] + T) of every KV head and
 * then advances seq_lens[b] by T.  If seq_lens[b] + T would exceed L_max (or
 * seq_lens[b] is negative) nothing of sequence b is written, its length is left
 * unchanged, and the return value counts it.  round_bf16 selects the stored
 * precision (1: bf16 RNE as stored by the product; 0: exact fp64).
 */
int stief_oracle_compress_append(const double* k_new, const double* v_new,
                                 const double* P_K, const double* P_V,
                                 double* k_lat, double* v_lat, int32_t* seq_lens,
                                 int B, int Hkv, int T, int d, int rK, int rV,
                                 int L_max, int round_bf16)
{
    int overflowed = 0;
    for (int b = 0; b < B; ++b) {
        long L = seq_lens[b];
        if (L < 0 || L + T > L_max) {
            ++overflowed;
            continue;
        }
        for (int h = 0; h < Hkv; ++h) {
            long src = ((long)b * Hkv + h) * T * d;
            long dst = ((long)b * Hkv + h) * L_max + L;
            stief_oracle_project(k_new + src, P_K + (long)h * d * rK,
                                 k_lat + dst * rK, T, d, rK, round_bf16);
            stief_oracle_project(v_new + src, P_V + (long)h * d * rV,
                                 v_lat + dst * rV, T, d, rV, round_bf16);
        }
        seq_lens[b] = (int32_t)(L + T);
    }
    return overflowed;
}

/* ------------------------------------------------------------------------- */
/* Decode attention over the reconstructed cache                               */
/* ------------------------------------------------------------------------- */

/* Reconstruct one full-dimension row: out[i] = sum_c lat[c] * P[i][c]. */
static void reconstruct_row(const double* lat, const double* P, int d, int r,
                            double* out)
{
    for (int i = 0; i < d; ++i) {
        double acc = 0.0;
        for (int c = 0; c < r; ++c)
            acc += lat[c] * P[(long)i * r + c];
        out[i] = acc;
    }
}

/*
 * One decode step for every (sequence, query head).
 *
 *   q            : [B][Hq][d]
 *   P_K, P_V     : [Hkv][d][rK], [Hkv][d][rV]
 *   k_lat, v_lat : [B][Hkv][L_max][rK], [B][Hkv][L_max][rV]
 *   seq_lens     : [B]; sequence b attends to its rows [0, seq_lens[b])
 *   out          : [B][Hq][d]
 *
 * For each (b, KV head g) and each of its query heads h (h / G == g, G = Hq/Hkv):
 *   K~_t = K_down[t] . P_K[g]^T,  V~_t = V_down[t] . P_V[g]^T      (t < L)
 *   s_t  = (q_h . K~_t) / sqrt(d)
 *   p    = softmax(s)   (maximum subtracted, then normalised)
 *   o_h  = sum_t p_t V~_t
 * L == 0 gives o_h = 0.  Returns 0, or -1 if a length is outside [0, L_max]
 * (that sequence's output is then left as zeros).
 */
int stief_oracle_decode(const double* q, const double* P_K, const double* P_V,
                        const double* k_lat, const double* v_lat,
                        const int32_t* seq_lens, double* out,
                        int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
                        int num_threads)
{
    const int G = Hq / Hkv;
    const double scale = 1.0 / sqrt((double)d);
    int bad = 0;
    memset(out, 0, sizeof(double) * (size_t)B * Hq * d);

#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (long unit = 0; unit < (long)B * Hkv; ++unit) {
        const int b = (int)(unit / Hkv);
        const int g = (int)(unit % Hkv);
        const long L = seq_lens[b];
        if (L < 0 || L > L_max) {
            bad |= 1;
            continue;
        }
        if (L == 0)
            continue;
        const double* PK = P_K + (long)g * d * rK;
        const double* PV = P_V + (long)g * d * rV;
        const double* Kd = k_lat + ((long)b * Hkv + g) * L_max * rK;
        const double* Vd = v_lat + ((long)b * Hkv + g) * L_max * rV;

        double* s = (double*)malloc(sizeof(double) * (size_t)G * L);
        double* row = (double*)malloc(sizeof(double) * (size_t)d);

        /* scores: s[j][t] = q_h . K~_t / sqrt(d) */
        for (long t = 0; t < L; ++t) {
            reconstruct_row(Kd + t * rK, PK, d, rK, row);
            for (int j = 0; j < G; ++j) {
                const double* qh = q + ((long)b * Hq + (long)g * G + j) * d;
                double acc = 0.0;
                for (int i = 0; i < d; ++i)
                    acc += qh[i] * row[i];
                s[(long)j * L + t] = acc * scale;
            }
        }
        /* softmax per query head: subtract the maximum, exponentiate, sum */
        double* denom = (double*)malloc(sizeof(double) * (size_t)G);
        for (int j = 0; j < G; ++j) {
            double* sj = s + (long)j * L;
            double mx = sj[0];
            for (long t = 1; t < L; ++t)
                if (sj[t] > mx)
                    mx = sj[t];
            double sum = 0.0;
            for (long t = 0; t < L; ++t) {
                sj[t] = exp(sj[t] - mx);
                sum += sj[t];
            }
            denom[j] = sum;
        }
        /* value mix: o_h = sum_t p_t V~_t */
        for (long t = 0; t < L; ++t) {
            reconstruct_row(Vd + t * rV, PV, d, rV, row);
            for (int j = 0; j < G; ++j) {
                double p = s[(long)j * L + t] / denom[j];
                double* oh = out + ((long)b * Hq + (long)g * G + j) * d;
                for (int i = 0; i < d; ++i)
                    oh[i] += p * row[i];
            }
        }
        free(denom);
        free(row);
        free(s);
    }
    return bad ? -1 : 0;
}

/*
 * Decode in the latent space, for models whose attention weights absorb the bases
 * (StiefAttention technical summary, "Mecanismo Central" item 5, last sentence:
 * the projection bases can be folded into the attention's linear weights).
 *
 *   q_lat        : [B][Hq][rK]   (the query already projected, q~ = q . P_K)
 *   k_lat, v_lat : [B][Hkv][L_max][rK], [B][Hkv][L_max][rV]
 *   seq_lens     : [B]
 *   out_lat      : [B][Hq][rV]   (o~; the model's folded output weight applies P_V^T)
 *
 * For each (b, KV head g) and each of its query heads h (h / G == g):
 *   s_t = (q~_h . K_down[t]) / sqrt(d)        t < L, d the full head dimension
 *   p   = softmax(s)   (maximum subtracted, then normalised)
 *   o~_h = sum_t p_t V_down[t]
 * L == 0 gives o~_h = 0.  Returns 0, or -1 if a length is outside [0, L_max].
 */
int stief_oracle_decode_latent(const double* q_lat, const double* k_lat, const double* v_lat,
                               const int32_t* seq_lens, double* out_lat,
                               int B, int Hq, int Hkv, int d, int rK, int rV, int L_max,
                               int num_threads)
{
    const int G = Hq / Hkv;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    int bad = 0;
    memset(out_lat, 0, sizeof(double) * (size_t)B * Hq * rV);

#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
#endif
    for (long unit = 0; unit < (long)B * Hkv; ++unit) {
        const int b = (int)(unit / Hkv);
        const int g = (int)(unit % Hkv);
        const long L = seq_lens[b];
        if (L < 0 || L > L_max) {
            bad |= 1;
            continue;
        }
        if (L == 0)
            continue;
        const double* Kd = k_lat + ((long)b * Hkv + g) * L_max * rK;
        const double* Vd = v_lat + ((long)b * Hkv + g) * L_max * rV;
        double* w_lat = (double*)malloc(sizeof(double) * (size_t)L);
        for (int j = 0; j < G; ++j) {
            const long head = (long)b * Hq + (long)g * G + j;  /* query head of group g */
            const double* qh = q_lat + head * rK;
            /* scores */
            for (long t = 0; t < L; ++t) {
                double acc = 0.0;
                for (int c = 0; c < rK; ++c)
                    acc += qh[c] * Kd[t * rK + c];
                w_lat[t] = acc * inv_sqrt_d;
            }
            /* softmax: subtract the maximum, exponentiate, sum */
            double mx = w_lat[0];
            for (long t = 1; t < L; ++t)
                if (w_lat[t] > mx)
                    mx = w_lat[t];
            double sum_lat = 0.0;
            for (long t = 0; t < L; ++t) {
                w_lat[t] = exp(w_lat[t] - mx);
                sum_lat += w_lat[t];
            }
            /* value mix in the latent space */
            double* oh = out_lat + head * rV;
            for (long t = 0; t < L; ++t) {
                const double p_lat = w_lat[t] / sum_lat;
                for (int c = 0; c < rV; ++c)
                    oh[c] += p_lat * Vd[t * rV + c];
            }
        }
        free(w_lat);
    }
    return bad ? -1 : 0;
}

/* Number of OpenMP threads a parallel region would use (1 without OpenMP). */
int stief_oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
