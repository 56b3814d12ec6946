/*
 * hsa_oracle.c -- plain, slow, fp64 CPU reference of Hierarchical Sparse
 * Attention (HSA).  TEST INFRASTRUCTURE ONLY: the tests, the smoke check and
 * the CPU-baseline leg of the benchmark use it; the library never does.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * What it computes follows the HSA summary page, "Every Token Counts 16m
 * Context": Core Technique (fixed-length non-overlapping chunks, one landmark
 * per chunk, top-k retrieval per query), Implementation (landmark =
 * projection of the mean-pooled chunk; scores = similarity(query, landmarks);
 * keep the k best; attend inside each kept chunk with standard attention; fuse
 * the chunk outputs weighted by their retrieval scores) and the gap router of
 * the value-of-information router page ("double the kept set where the k-th /
 * (k+1)-th gap is smallest").  Readings where the pages are silent:
 *   - the landmark is mean(keys of the chunk) times a d x d matrix W_L
 *     (row vector times W_L, W_L[e_in][e_out]), no refiner layer;
 *   - the similarity is the raw dot product; with grouped-query attention a
 *     kv head's G query heads share one selection whose score is the sum of
 *     the G per-head dot products;
 *   - candidates of a query at absolute position p are the complete chunks
 *     c < floor(p / S); none -> the output is 0;
 *   - ranking is by score descending, ties to the lower chunk index;
 *   - fusion weights are the softmax, over the kept set, of those same
 *     retrieval scores; in-chunk attention is softmax(q k^T / sqrt(d)) v;
 *   - router: if tau > 0, the row has more than k candidates and
 *     (s_k - s_{k+1}) < tau * |s_k|, keep min(2k, #candidates) chunks.
 * Everything is accumulated in double; inputs are read from their storage
 * dtype (fp32 or bf16) exactly.
 *
 * Parity pins: every function here is checked in tests/test_oracle_pins.py
 * against brute force, closed forms, invariants and library routines.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORC_F32 = 0, ORC_BF16 = 1, ORC_F64 = 2 };

static double load(const void *p, size_t i, int dt)
{
    if (dt == ORC_F64) return ((const double *)p)[i];
    if (dt == ORC_F32) return (double)((const float *)p)[i];
    uint32_t bits = (uint32_t)((const uint16_t *)p)[i] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 value (ties to even), in one step. */
static double round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e = ilogb(x);
    if (e < -126) e = -126;                 /* bf16 shares fp32's exponent range */
    double ulp = ldexp(1.0, e - 7);         /* 8 significant bits */
    double r = nearbyint(x / ulp) * ulp;    /* default rounding mode: ties to even */
    if (fabs(r) > 0x1.FEp127) r = copysign(INFINITY, x);
    return r;
}

/* y[i] = x[i] rounded to the storage dtype (fp32 or bf16), kept as double. */
void hsa_oracle_round(int dt, const double *x, long long n, double *y)
{
    for (long long i = 0; i < n; ++i)
        y[i] = (dt == ORC_BF16) ? round_bf16(x[i]) : (dt == ORC_F32 ? (double)(float)x[i] : x[i]);
}

/*
 * Landmarks of every complete chunk.
 *   K  [B][T][Hkv][d]  (dtype dt)      W [d][d] (dtype dt, row = input dim)
 *   L  [B][Hkv][C][d]  double, C = T / S, NOT rounded to the storage dtype.
 * L[b][j][c][f] = sum_e ( (1/S) sum_{u<S} K[b][cS+u][j][e] ) * W[e][f]
 */
void hsa_oracle_landmarks(int dt, int B, long long T, int Hkv, int d, int S,
                          const void *K, const void *W, double *L)
{
    long long C = T / S;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (long long c = 0; c < C; ++c) {
            double *mean = (double *)malloc(sizeof(double) * (size_t)d);
            for (int j = 0; j < Hkv; ++j) {
                for (int e = 0; e < d; ++e) mean[e] = 0.0;
                for (int u = 0; u < S; ++u) {
                    size_t row = (((size_t)b * (size_t)T + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                    for (int e = 0; e < d; ++e) mean[e] += load(K, row + e, dt);
                }
                for (int e = 0; e < d; ++e) mean[e] /= (double)S;
                double *out = L + (((size_t)b * Hkv + j) * (size_t)C + (size_t)c) * (size_t)d;
                for (int f = 0; f < d; ++f) {
                    double acc = 0.0;
                    for (int e = 0; e < d; ++e) acc += mean[e] * load(W, (size_t)e * d + f, dt);
                    out[f] = acc;
                }
            }
            free(mean);
        }
    }
}

typedef struct { double s; long long c; } cand_t;

/* score descending, then chunk index ascending */
static int cand_order(const void *a, const void *b)
{
    const cand_t *x = (const cand_t *)a, *y = (const cand_t *)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->c > y->c) - (x->c < y->c);
}

/*
 * Top-k chunk selection for n query rows.
 *   row_b[r], row_p[r]: batch index and absolute position of row r
 *   Qr [n][H][d] (dtype dt_q)          L [B][Hkv][C][d] double (storage values)
 * Outputs, per row and kv head j:
 *   idx   [n][Hkv][kmax]  kept chunks in rank order, -1 padding
 *   score [n][Hkv][kmax]  their group scores, -inf padding
 *   keff  [n][Hkv]        number kept
 *   allscores [n][Hkv][C] (optional) every group score, -inf for non-candidates
 */
void hsa_oracle_select(int dt_q, int H, int Hkv, int d, int S, long long C, int k,
                       double tau, int kmax, long long n, const int *row_b,
                       const long long *row_p, const void *Qr, const double *L,
                       int *idx, double *score, int *keff, double *allscores)
{
    int G = H / Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long r = 0; r < n; ++r) {
        long long ncand = row_p[r] / S;
        if (ncand > C) ncand = C;
        if (ncand < 0) ncand = 0;
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(ncand > 0 ? ncand : 1));
        for (int j = 0; j < Hkv; ++j) {
            const double *Lj = L + ((size_t)row_b[r] * Hkv + j) * (size_t)C * d;
            for (long long c = 0; c < ncand; ++c) {
                double s = 0.0;
                for (int h = j * G; h < (j + 1) * G; ++h) {
                    double dot = 0.0;
                    for (int e = 0; e < d; ++e)
                        dot += load(Qr, ((size_t)r * H + h) * d + e, dt_q) * Lj[(size_t)c * d + e];
                    s += dot;
                }
                cand[c].s = s;
                cand[c].c = c;
                if (allscores) allscores[((size_t)r * Hkv + j) * (size_t)C + c] = s;
            }
            if (allscores)
                for (long long c = ncand; c < C; ++c)
                    allscores[((size_t)r * Hkv + j) * (size_t)C + c] = -INFINITY;
            qsort(cand, (size_t)ncand, sizeof(cand_t), cand_order);
            long long ke = ncand < k ? ncand : k;
            if (tau > 0.0 && ncand > k) {
                double sk = cand[k - 1].s, sk1 = cand[k].s;
                if (sk - sk1 < tau * fabs(sk)) ke = ncand < 2 * k ? ncand : 2 * k;
            }
            size_t o = ((size_t)r * Hkv + j) * kmax;
            for (int i = 0; i < kmax; ++i) {
                idx[o + i] = i < ke ? (int)cand[i].c : -1;
                score[o + i] = i < ke ? cand[i].s : -INFINITY;
            }
            keff[(size_t)r * Hkv + j] = (int)ke;
        }
        free(cand);
    }
}

/*
 * Chunk attention and retrieval-weighted fusion for n query rows.
 *   Qr [n][H][d] (dt)       K, V [B][Tkv][Hkv][d] (dt)
 *   idx, score [n][Hkv][kmax], keff [n][Hkv]: a selection (from hsa_oracle_select)
 *   O [n][H][d] double
 * For kv head j and each head h of its group:
 *   w_i  = exp(score_i - max) / sum_i' exp(score_i' - max),   i < keff
 *   o_i  = sum_u softmax_u(q_h . K[c_i S + u] / sqrt(d)) V[c_i S + u]
 *   O[h] = sum_i w_i o_i   (0 when keff == 0)
 */
void hsa_oracle_attend(int dt, long long Tkv, int H, int Hkv, int d, int S, int kmax,
                       long long n, const int *row_b, const void *Qr, const void *K,
                       const void *V, const int *idx, const double *score,
                       const int *keff, double *O)
{
    int G = H / Hkv;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 4)
    for (long long r = 0; r < n; ++r) {
        double *w = (double *)malloc(sizeof(double) * (size_t)kmax);
        double *a = (double *)malloc(sizeof(double) * (size_t)S);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
        size_t b = (size_t)row_b[r];
        for (int j = 0; j < Hkv; ++j) {
            size_t so = ((size_t)r * Hkv + j) * kmax;
            int ke = keff[(size_t)r * Hkv + j];
            double m = -INFINITY, z = 0.0;
            for (int i = 0; i < ke; ++i) if (score[so + i] > m) m = score[so + i];
            for (int i = 0; i < ke; ++i) { w[i] = exp(score[so + i] - m); z += w[i]; }
            for (int i = 0; i < ke; ++i) w[i] /= z;
            for (int h = j * G; h < (j + 1) * G; ++h) {
                double *out = O + ((size_t)r * H + h) * d;
                for (int e = 0; e < d; ++e) out[e] = 0.0;
                for (int i = 0; i < ke; ++i) {
                    long long c = idx[so + i];
                    double amax = -INFINITY, l = 0.0;
                    for (int u = 0; u < S; ++u) {
                        size_t row = ((b * (size_t)Tkv + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                        double dot = 0.0;
                        for (int e = 0; e < d; ++e)
                            dot += load(Qr, ((size_t)r * H + h) * d + e, dt) * load(K, row + e, dt);
                        a[u] = dot * scale;
                        if (a[u] > amax) amax = a[u];
                    }
                    for (int e = 0; e < d; ++e) o[e] = 0.0;
                    for (int u = 0; u < S; ++u) {
                        double p = exp(a[u] - amax);
                        l += p;
                        size_t row = ((b * (size_t)Tkv + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                        for (int e = 0; e < d; ++e) o[e] += p * load(V, row + e, dt);
                    }
                    for (int e = 0; e < d; ++e) out[e] += w[i] * (o[e] / l);
                }
            }
        }
        free(w); free(a); free(o);
    }
}
