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
 * the value-of-information router page (abstract: rows whose top-k cut is
 * nearly tied, a small gap between the k-th and (k+1)-th scores, keep twice
 * as many chunks).  Readings where the pages are silent:
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

/*
 * Gradients of the method with the selection held fixed (the chunk choice is a
 * discrete decision: it has no gradient, and the kept chunks' scores still
 * carry one through the fusion weights).  The forward this differentiates,
 * for the rows given and kv head j, each head h of its group and kept slot i:
 *   s_i  = sum_{h in group} q_h . L[c_i]          (L = mean-pooled keys * W_L)
 *   w    = softmax_i(s)                           (i < keff)
 *   a_iu = softmax_u(q_h . K[c_i S + u] / sqrt(d)),  o_hi = sum_u a_iu V[c_i S + u]
 *   O_h  = sum_i w_i o_hi
 * Given dO [n][H][d] (double), the chain rule gives, in this order:
 *   e_hi  = dO_h . o_hi,   dw_i = sum_h e_hi,   ds_i = w_i (dw_i - sum_i' w_i' dw_i')
 *   dq_h += sum_i ds_i L[c_i],                  dL[c_i] += ds_i q_h
 *   with g = w_i dO_h:  dV_u += a_iu g,  dz_u = a_iu (g . V_u - g . o_hi),
 *                       dq_h += (1/sqrt d) sum_u dz_u K_u,  dK_u += (1/sqrt d) dz_u q_h
 * and, through the landmark of every complete chunk c (m_c = its key mean):
 *   dW_L += m_c^T dL[c],   dK_u += (dL[c] W_L^T) / S   for the S keys of chunk c.
 * Inputs: Qr [n][H][d] (dt), row_b [n], K, V [B][Tkv][Hkv][d] (dt), W [d][d]
 * (dt), L [B][Hkv][C][d] (double: the landmarks the scores are taken from),
 * idx, keff as from hsa_oracle_select.  Outputs, all double and OVERWRITTEN:
 * dQ [n][H][d], dK, dV [B][Tkv][Hkv][d], dW [d][d], dL [B][Hkv][C][d].
 * L enters the scores as given, so rounding it to a storage dtype is taken as
 * the identity in the chain rule (the rounding has no useful derivative).
 */
void hsa_oracle_backward(int dt, int B, long long Tkv, int H, int Hkv, int d, int S, int kmax,
                         long long n, const int *row_b, const void *Qr, const void *K,
                         const void *V, const void *W, const double *L, const int *idx,
                         const int *keff, const double *dO, double *dQ, double *dK,
                         double *dV, double *dW, double *dL)
{
    int G = H / Hkv;
    long long C = Tkv / S;
    double scale = 1.0 / sqrt((double)d);
    memset(dQ, 0, sizeof(double) * (size_t)n * H * d);
    memset(dK, 0, sizeof(double) * (size_t)B * Tkv * Hkv * d);
    memset(dV, 0, sizeof(double) * (size_t)B * Tkv * Hkv * d);
    memset(dW, 0, sizeof(double) * (size_t)d * d);
    memset(dL, 0, sizeof(double) * (size_t)B * Hkv * C * d);
    /* kv heads touch disjoint parts of dQ, dK, dV and dL: one thread per head */
#pragma omp parallel for schedule(static)
    for (int j = 0; j < Hkv; ++j) {
        double *w = (double *)malloc(sizeof(double) * (size_t)kmax);
        double *dw = (double *)malloc(sizeof(double) * (size_t)kmax);
        double *e = (double *)malloc(sizeof(double) * (size_t)kmax * G);
        double *a = (double *)malloc(sizeof(double) * (size_t)kmax * G * S);   /* a[(i*G+g)*S+u] */
        double *o = (double *)malloc(sizeof(double) * (size_t)kmax * G * d);   /* o[(i*G+g)*d+x] */
        for (long long r = 0; r < n; ++r) {
            size_t b = (size_t)row_b[r];
            size_t so = ((size_t)r * Hkv + j) * kmax;
            int ke = keff[(size_t)r * Hkv + j];
            if (ke <= 0) continue;
            const double *Lj = L + (b * Hkv + j) * (size_t)C * d;
            /* scores and fusion weights */
            double m = -INFINITY, z = 0.0;
            for (int i = 0; i < ke; ++i) {
                double s = 0.0;
                for (int g = 0; g < G; ++g)
                    for (int x = 0; x < d; ++x)
                        s += load(Qr, ((size_t)r * H + j * G + g) * d + x, dt) * Lj[(size_t)idx[so + i] * d + x];
                w[i] = s;
                if (s > m) m = s;
            }
            for (int i = 0; i < ke; ++i) { w[i] = exp(w[i] - m); z += w[i]; }
            for (int i = 0; i < ke; ++i) w[i] /= z;
            /* in-chunk attention of every (slot, head) and e = dO . o */
            for (int i = 0; i < ke; ++i) {
                size_t c = (size_t)idx[so + i];
                for (int g = 0; g < G; ++g) {
                    size_t qh = ((size_t)r * H + j * G + g) * d;
                    double *ai = a + ((size_t)i * G + g) * S, *oi = o + ((size_t)i * G + g) * d;
                    double amax = -INFINITY, l = 0.0;
                    for (int u = 0; u < S; ++u) {
                        size_t kr = ((b * (size_t)Tkv + c * S + u) * Hkv + j) * (size_t)d;
                        double dot = 0.0;
                        for (int x = 0; x < d; ++x) dot += load(Qr, qh + x, dt) * load(K, kr + x, dt);
                        ai[u] = dot * scale;
                        if (ai[u] > amax) amax = ai[u];
                    }
                    for (int u = 0; u < S; ++u) { ai[u] = exp(ai[u] - amax); l += ai[u]; }
                    for (int u = 0; u < S; ++u) ai[u] /= l;
                    for (int x = 0; x < d; ++x) oi[x] = 0.0;
                    for (int u = 0; u < S; ++u) {
                        size_t vr = ((b * (size_t)Tkv + c * S + u) * Hkv + j) * (size_t)d;
                        for (int x = 0; x < d; ++x) oi[x] += ai[u] * load(V, vr + x, dt);
                    }
                    double ev = 0.0;
                    for (int x = 0; x < d; ++x) ev += dO[qh + x] * oi[x];
                    e[(size_t)i * G + g] = ev;
                }
            }
            /* fusion softmax: dw, then ds */
            double wdw = 0.0;
            for (int i = 0; i < ke; ++i) {
                dw[i] = 0.0;
                for (int g = 0; g < G; ++g) dw[i] += e[(size_t)i * G + g];
                wdw += w[i] * dw[i];
            }
            for (int i = 0; i < ke; ++i) {
                double ds = w[i] * (dw[i] - wdw);
                size_t c = (size_t)idx[so + i];
                double *dLc = dL + ((b * Hkv + j) * (size_t)C + c) * d;
                for (int g = 0; g < G; ++g) {
                    size_t qh = ((size_t)r * H + j * G + g) * d;
                    for (int x = 0; x < d; ++x) {
                        dQ[qh + x] += ds * Lj[c * d + x];
                        dLc[x] += ds * load(Qr, qh + x, dt);
                    }
                }
            }
            /* in-chunk attention backward with the output gradient w_i dO_h */
            for (int i = 0; i < ke; ++i) {
                size_t c = (size_t)idx[so + i];
                for (int g = 0; g < G; ++g) {
                    size_t qh = ((size_t)r * H + j * G + g) * d;
                    const double *ai = a + ((size_t)i * G + g) * S, *oi = o + ((size_t)i * G + g) * d;
                    double go = 0.0;
                    for (int x = 0; x < d; ++x) go += w[i] * dO[qh + x] * oi[x];
                    for (int u = 0; u < S; ++u) {
                        size_t kr = ((b * (size_t)Tkv + c * S + u) * Hkv + j) * (size_t)d;
                        double gv = 0.0;
                        for (int x = 0; x < d; ++x) {
                            double gx = w[i] * dO[qh + x];
                            dV[kr + x] += ai[u] * gx;
                            gv += gx * load(V, kr + x, dt);
                        }
                        double dz = ai[u] * (gv - go) * scale;
                        for (int x = 0; x < d; ++x) {
                            dQ[qh + x] += dz * load(K, kr + x, dt);
                            dK[kr + x] += dz * load(Qr, qh + x, dt);
                        }
                    }
                }
            }
        }
        free(w); free(dw); free(e); free(a); free(o);
    }
    /* landmark backward: dW_L and the keys' share through the chunk mean */
    double *mean = (double *)malloc(sizeof(double) * (size_t)d);
    double *dm = (double *)malloc(sizeof(double) * (size_t)d);
    for (int b = 0; b < B; ++b)
        for (int j = 0; j < Hkv; ++j)
            for (long long c = 0; c < C; ++c) {
                const double *dLc = dL + (((size_t)b * Hkv + j) * (size_t)C + (size_t)c) * d;
                for (int x = 0; x < d; ++x) mean[x] = 0.0;
                for (int u = 0; u < S; ++u) {
                    size_t kr = (((size_t)b * Tkv + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                    for (int x = 0; x < d; ++x) mean[x] += load(K, kr + x, dt);
                }
                for (int x = 0; x < d; ++x) mean[x] /= (double)S;
                for (int x = 0; x < d; ++x) {
                    double acc = 0.0;
                    for (int f = 0; f < d; ++f) {
                        dW[(size_t)x * d + f] += mean[x] * dLc[f];
                        acc += dLc[f] * load(W, (size_t)x * d + f, dt);
                    }
                    dm[x] = acc / (double)S;
                }
                for (int u = 0; u < S; ++u) {
                    size_t kr = (((size_t)b * Tkv + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                    for (int x = 0; x < d; ++x) dK[kr + x] += dm[x];
                }
            }
    free(mean); free(dm);
}

/* ------------------------------------------------------------------------
 * Selection variants.
 *
 * Landmark refiner (HSA summary page, Implementation: a learned layer with
 * cross-attention refines the mean-pooled landmark).  Reading: one head of
 * cross-attention whose query is the pooled landmark and whose keys and
 * values are the chunk's own S keys, added back to the landmark:
 *   L0  = mean_u(K_u) W_L
 *   q   = L0 W_q,     kap_u = K_u W_k,     nu_u = K_u W_v
 *   a   = softmax_u(q . kap_u / sqrt(d))
 *   L   = L0 + sum_u a_u nu_u
 * W_L, W_q, W_k, W_v: d x d, row = input dim, dtype dt.  L: double, NOT
 * rounded to the storage dtype.
 */
void hsa_oracle_landmarks_refined(int dt, int B, long long T, int Hkv, int d, int S,
                                  const void *K, const void *WL, const void *Wq,
                                  const void *Wk, const void *Wv, double *L)
{
    long long C = T / S;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int b = 0; b < B; ++b) {
        for (long long c = 0; c < C; ++c) {
            double *mean = (double *)malloc(sizeof(double) * (size_t)d);
            double *l0 = (double *)malloc(sizeof(double) * (size_t)d);
            double *q = (double *)malloc(sizeof(double) * (size_t)d);
            double *kap = (double *)malloc(sizeof(double) * (size_t)d);
            double *nu = (double *)malloc(sizeof(double) * (size_t)d);
            double *logit = (double *)malloc(sizeof(double) * (size_t)S);
            double *acc = (double *)malloc(sizeof(double) * (size_t)d);
            for (int j = 0; j < Hkv; ++j) {
                size_t row0 = (((size_t)b * (size_t)T + (size_t)(c * S)) * Hkv + j) * (size_t)d;
                size_t rstride = (size_t)Hkv * d;
                for (int e = 0; e < d; ++e) mean[e] = 0.0;
                for (int u = 0; u < S; ++u)
                    for (int e = 0; e < d; ++e) mean[e] += load(K, row0 + u * rstride + e, dt);
                for (int e = 0; e < d; ++e) mean[e] = mean[e] / (double)S;
                for (int f = 0; f < d; ++f) {
                    double s = 0.0;
                    for (int e = 0; e < d; ++e) s += mean[e] * load(WL, (size_t)e * d + f, dt);
                    l0[f] = s;
                }
                for (int f = 0; f < d; ++f) {
                    double s = 0.0;
                    for (int e = 0; e < d; ++e) s += l0[e] * load(Wq, (size_t)e * d + f, dt);
                    q[f] = s;
                }
                /* logits of the landmark query against every key of the chunk */
                double mx = -INFINITY;
                for (int u = 0; u < S; ++u) {
                    for (int f = 0; f < d; ++f) {
                        double s = 0.0;
                        for (int e = 0; e < d; ++e)
                            s += load(K, row0 + u * rstride + e, dt) * load(Wk, (size_t)e * d + f, dt);
                        kap[f] = s;
                    }
                    double dot = 0.0;
                    for (int f = 0; f < d; ++f) dot += q[f] * kap[f];
                    logit[u] = dot * scale;
                    if (logit[u] > mx) mx = logit[u];
                }
                double z = 0.0;
                for (int u = 0; u < S; ++u) { logit[u] = exp(logit[u] - mx); z += logit[u]; }
                for (int f = 0; f < d; ++f) acc[f] = 0.0;
                for (int u = 0; u < S; ++u) {
                    double a = logit[u] / z;
                    for (int f = 0; f < d; ++f) {
                        double s = 0.0;
                        for (int e = 0; e < d; ++e)
                            s += load(K, row0 + u * rstride + e, dt) * load(Wv, (size_t)e * d + f, dt);
                        nu[f] = s;
                    }
                    for (int f = 0; f < d; ++f) acc[f] += a * nu[f];
                }
                double *out = L + (((size_t)b * Hkv + j) * (size_t)C + (size_t)c) * (size_t)d;
                for (int f = 0; f < d; ++f) out[f] = l0[f] + acc[f];
            }
            free(mean); free(l0); free(q); free(kap); free(nu); free(logit); free(acc);
        }
    }
}

/*
 * Quest-style chunk summaries (value-of-information router page, abstract:
 * the router stacks on block-scoring methods such as Quest).  Reading: Quest's
 * page summary with the chunk as the page -- per complete chunk and kv head,
 * the channel-wise maximum and minimum of its S keys:
 *   Lq[b][j][c][e] = max_u K[b][cS+u][j][e],   Lq[b][j][c][d + e] = min_u K[b][cS+u][j][e]
 * Lq [B][Hkv][C][2d] double (the values are stored values: no rounding).
 */
void hsa_oracle_quest_summaries(int dt, int B, long long T, int Hkv, int d, int S,
                                const void *K, double *Lq)
{
    long long C = T / S;
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (long long c = 0; c < C; ++c) {
            for (int j = 0; j < Hkv; ++j) {
                double *out = Lq + (((size_t)b * Hkv + j) * (size_t)C + (size_t)c) * (size_t)(2 * d);
                for (int e = 0; e < d; ++e) { out[e] = -INFINITY; out[d + e] = INFINITY; }
                for (int u = 0; u < S; ++u) {
                    size_t row = (((size_t)b * (size_t)T + (size_t)(c * S + u)) * Hkv + j) * (size_t)d;
                    for (int e = 0; e < d; ++e) {
                        double x = load(K, row + e, dt);
                        if (x > out[e]) out[e] = x;
                        if (x < out[d + e]) out[d + e] = x;
                    }
                }
            }
        }
    }
}

/*
 * Top-k selection with Quest's criticality score in place of the landmark dot
 * product.  For chunk c and a query row's kv head j:
 *   s_c = sum_{h in group j} sum_e max(q_h[e] * Lq_c[e], q_h[e] * Lq_c[d + e])
 * -- for each head the largest value any key of the chunk could give each
 * product q_h[e] k[e], summed: an upper bound of sum_h max_u q_h . K_u.  The
 * candidates, ranking, ties, keff and router are those of hsa_oracle_select.
 *   Lq [B][Hkv][C][2d] double; other arguments as hsa_oracle_select.
 */
void hsa_oracle_select_quest(int dt_q, int H, int Hkv, int d, int S, long long C, int k,
                             double tau, int kmax, long long n, const int *row_b,
                             const long long *row_p, const void *Qr, const double *Lq,
                             int *idx, double *score, int *keff, double *allscores)
{
    int G = H / Hkv;
#pragma omp parallel for schedule(dynamic, 4)
    for (long long r = 0; r < n; ++r) {
        long long ncand = row_p[r] / (long long)S;
        if (ncand > C) ncand = C;
        if (ncand < 0) ncand = 0;
        cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(ncand > 0 ? ncand : 1));
        for (int j = 0; j < Hkv; ++j) {
            const double *Lj = Lq + ((size_t)row_b[r] * Hkv + j) * (size_t)C * (size_t)(2 * d);
            for (long long c = 0; c < ncand; ++c) {
                const double *mx = Lj + (size_t)c * (2 * d), *mn = mx + d;
                double s = 0.0;
                for (int h = j * G; h < (j + 1) * G; ++h) {
                    double bound = 0.0;
                    for (int e = 0; e < d; ++e) {
                        double qe = load(Qr, ((size_t)r * H + h) * d + e, dt_q);
                        double hi = qe * mx[e], lo = qe * mn[e];
                        bound += hi > lo ? hi : lo;
                    }
                    s += bound;
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
                double gap = cand[k - 1].s - cand[k].s;
                if (gap < tau * fabs(cand[k - 1].s)) ke = ncand < 2 * k ? ncand : 2 * k;
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
