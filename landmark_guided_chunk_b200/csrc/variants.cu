// variants.cu -- the two selection variants.
//
// Landmark refiner (HSA summary page, Implementation: a learned layer with
// cross-attention refines the mean-pooled landmark).  One head of
// cross-attention whose query is the pooled landmark and whose keys and values
// are the chunk's own keys, added back:
//     L0 = mean_u(K_u) W_L
//     L  = L0 + softmax_u((L0 W_q) . (K_u W_k) / sqrt(d)) (K_u W_v)
// computed as q' = (L0 W_q) W_k^T, logits q' . K_u, z = sum_u a_u K_u and
// L = L0 + z W_v: four d x d products per (chunk, kv head) instead of 2S.
// One CTA per (chunk, kv head, sequence): the chunk's S keys are staged once
// in shared memory (fp32), everything else is d-vectors.  fp32 throughout,
// one rounding of L to the dtype.
//
// Quest block scoring (value-of-information router page, abstract: the router
// stacks on block scorers such as Quest).  Each chunk is summarised by the
// channel-wise max Mx and min Mn of its keys, and a query row's score is
//     s_c = sum_{h in group} sum_e max(q_h[e] Mx_c[e], q_h[e] Mn_c[e])
//         = P . Mx_c + N . Mn_c,   P = sum_h max(q_h, 0),  N = sum_h min(q_h, 0)
// (Mx >= Mn, so the larger product is the max's for q >= 0 and the min's
// otherwise).  That is a width-2d contraction of [P | N] with [Mx | Mn], so
// the selection kernels run unchanged on a transformed problem: d' = 2d,
// landmarks = the summaries, and per (token, kv head) a query group of G'
// rows whose sum is [P | N].  In bf16 G' = 2: row 0 = [hi(P) | hi(N)], row 1
// = [lo(P) | lo(N)], hi = P rounded to bf16 and lo = the remainder rounded,
// so the pair carries P to ~2^-18 relative; in fp32 G' = 1.
#include "common.cuh"

namespace hsa {
namespace {

constexpr int RT = 256;   // threads of a refiner CTA

// y[f] = sum_e x[e] W[e][f] (W row-major d x d in global memory; x, y, part in
// shared memory).  Thread t sums column f = t % d over its share of e; the
// RT / d shares are added through `part`.
template <typename T>
__device__ __forceinline__ void gemv_rows(const float *x, const T *__restrict__ W, float *y, float *part, int d) {
    const int nh = RT / d;
    const int f = threadIdx.x % d, h = threadIdx.x / d;
    if (h < nh) {
        float s = 0.f;
        for (int e = h; e < d; e += nh) s = fmaf(x[e], to_f32(__ldg(W + (size_t)e * d + f)), s);
        part[h * d + f] = s;
    }
    __syncthreads();
    if ((int)threadIdx.x < d) {
        float s = 0.f;
        for (int g = 0; g < nh; ++g) s += part[g * d + threadIdx.x];
        y[threadIdx.x] = s;
    }
    __syncthreads();
}

// y[e] = sum_f W[e][f] x[f]: one warp per row e, lanes over f.
template <typename T>
__device__ __forceinline__ void gemv_cols(const float *x, const T *__restrict__ W, float *y, int d) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int e = warp; e < d; e += RT / 32) {
        float s = 0.f;
        for (int f = lane; f < d; f += 32) s = fmaf(to_f32(__ldg(W + (size_t)e * d + f)), x[f], s);
        s = warp_sum(s);
        if (lane == 0) y[e] = s;
    }
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(RT) refine_kernel(const T *__restrict__ K, const T *__restrict__ WL,
                                                    const T *__restrict__ Wq, const T *__restrict__ Wk,
                                                    const T *__restrict__ Wv, T *__restrict__ L, int Tcap, int Hkv,
                                                    int d, int S, int Lc, float scale) {
    extern __shared__ __align__(16) float rs[];
    const int c = blockIdx.x / Hkv, j = blockIdx.x % Hkv, b = blockIdx.y;
    float *ks = rs;                 // [S][d] the chunk's keys
    float *xv = ks + (size_t)S * d; // d: the mean, later z
    float *l0 = xv + d;             // d: pooled landmark
    float *qv = l0 + d;             // d: L0 W_q
    float *qp = qv + d;             // d: q' = q W_k^T
    float *yv = qp + d;             // d: z W_v
    float *lg = yv + d;             // S: logits, then probabilities
    float *part = lg + S;           // (RT / d) x d partial sums
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const size_t rstride = (size_t)Hkv * d;
    const T *src = K + ((size_t)b * Tcap + (size_t)c * S) * rstride + (size_t)j * d;
    for (int i = threadIdx.x; i < S * d; i += RT) {
        const int u = i / d, e = i - u * d;
        ks[i] = to_f32(__ldg(src + (size_t)u * rstride + e));
    }
    __syncthreads();
    {   // mean over the S keys
        const int nh = RT / d;
        const int e = threadIdx.x % d, h = threadIdx.x / d;
        if (h < nh) {
            float s = 0.f;
            for (int u = h; u < S; u += nh) s += ks[u * d + e];
            part[h * d + e] = s;
        }
        __syncthreads();
        if ((int)threadIdx.x < d) {
            float s = 0.f;
            for (int g = 0; g < nh; ++g) s += part[g * d + threadIdx.x];
            xv[threadIdx.x] = s / (float)S;
        }
        __syncthreads();
    }
    gemv_rows(xv, WL, l0, part, d);   // L0 = mean W_L
    gemv_rows(l0, Wq, qv, part, d);   // q = L0 W_q
    gemv_cols(qv, Wk, qp, d);         // q' = q W_k^T, so q . (K_u W_k) = q' . K_u
    for (int u = warp; u < S; u += RT / 32) {
        float s = 0.f;
        for (int e = lane; e < d; e += 32) s = fmaf(qp[e], ks[u * d + e], s);
        s = warp_sum(s);
        if (lane == 0) lg[u] = s * scale;
    }
    __syncthreads();
    if (warp == 0) {   // softmax over the S logits
        float m = -INFINITY;
        for (int u = lane; u < S; u += 32) m = fmaxf(m, lg[u]);
        m = warp_max(m);
        float z = 0.f;
        for (int u = lane; u < S; u += 32) {
            const float p = expf(lg[u] - m);
            lg[u] = p;
            z += p;
        }
        z = warp_sum(z);
        __syncwarp();
        const float inv = 1.f / z;
        for (int u = lane; u < S; u += 32) lg[u] *= inv;
    }
    __syncthreads();
    {   // z = sum_u a_u K_u
        const int nh = RT / d;
        const int e = threadIdx.x % d, h = threadIdx.x / d;
        if (h < nh) {
            float s = 0.f;
            for (int u = h; u < S; u += nh) s = fmaf(lg[u], ks[u * d + e], s);
            part[h * d + e] = s;
        }
        __syncthreads();
        if ((int)threadIdx.x < d) {
            float s = 0.f;
            for (int g = 0; g < nh; ++g) s += part[g * d + threadIdx.x];
            xv[threadIdx.x] = s;
        }
        __syncthreads();
    }
    gemv_rows(xv, Wv, yv, part, d);   // z W_v
    if ((int)threadIdx.x < d)
        L[(((size_t)b * Hkv + j) * Lc + c) * d + threadIdx.x] = from_f32<T>(l0[threadIdx.x] + yv[threadIdx.x]);
}

// Quest summaries: one CTA per (chunk, sequence); thread = one 16-byte column of
// the chunk's token rows (all kv heads), running max and min over the S rows.
template <typename T>
__global__ void __launch_bounds__(256) quest_summary_kernel(const T *__restrict__ K, T *__restrict__ Lq, int Tcap,
                                                            int Hkv, int d, int S, int Lc, int c0) {
    constexpr int NV = 16 / (int)sizeof(T);
    const int c = c0 + blockIdx.x, b = blockIdx.y;
    const int n = Hkv * d, nv = n / NV;
    const uint4 *src = reinterpret_cast<const uint4 *>(K + ((size_t)b * Tcap + (size_t)c * S) * n);
    for (int v = threadIdx.x; v < nv; v += blockDim.x) {
        float mx[NV], mn[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            mx[i] = -INFINITY;
            mn[i] = INFINITY;
        }
        for (int u0 = 0; u0 < S; u0 += 8) {
            uint4 x[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) x[k] = __ldg(src + (size_t)(u0 + k) * nv + v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const T *e = reinterpret_cast<const T *>(&x[k]);
#pragma unroll
                for (int i = 0; i < NV; ++i) {
                    const float f = to_f32(e[i]);
                    mx[i] = fmaxf(mx[i], f);
                    mn[i] = fminf(mn[i], f);
                }
            }
        }
        const int ch = v * NV, j = ch / d, e0 = ch - j * d;
        T *dst = Lq + (((size_t)b * Hkv + j) * Lc + c) * (size_t)(2 * d);
#pragma unroll
        for (int i = 0; i < NV; ++i) {
            dst[e0 + i] = from_f32<T>(mx[i]);       // exact: a stored value
            dst[d + e0 + i] = from_f32<T>(mn[i]);
        }
    }
}

// The transformed query of Quest scoring: per (token, kv head), P and N summed
// over the group's heads in fp32, in head order.
template <typename T>
__global__ void __launch_bounds__(256) quest_qprep_kernel(const T *__restrict__ Q, T *__restrict__ Qp, long long BT,
                                                          int Hkv, int G, int d) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long total = BT * Hkv * d;
    if (i >= total) return;
    const int e = (int)(i % d);
    const long long r = i / d;   // (bt, j)
    const T *q = Q + (size_t)r * G * d + e;
    float P = 0.f, N = 0.f;
    for (int g = 0; g < G; ++g) {
        const float x = to_f32(q[(size_t)g * d]);
        P += fmaxf(x, 0.f);
        N += fminf(x, 0.f);
    }
    if constexpr (sizeof(T) == 2) {
        const __nv_bfloat16 ph = __float2bfloat16_rn(P), nh = __float2bfloat16_rn(N);
        const __nv_bfloat16 pl = __float2bfloat16_rn(P - __bfloat162float(ph));
        const __nv_bfloat16 nl = __float2bfloat16_rn(N - __bfloat162float(nh));
        T *o = Qp + (size_t)r * 4 * d;   // [2 rows][2d]
        o[e] = ph;
        o[d + e] = nh;
        o[2 * d + e] = pl;
        o[3 * d + e] = nl;
    } else {
        T *o = Qp + (size_t)r * 2 * d;   // [1 row][2d]
        o[e] = from_f32<T>(P);
        o[d + e] = from_f32<T>(N);
    }
}

}  // namespace

Prob quest_select_view(const Prob &p) {
    Prob v = p;
    const int gq = p.dtype == HSA_BF16 ? 2 : 1;
    v.G = gq;
    v.H = p.Hkv * gq;
    v.d = 2 * p.d;
    v.flags &= ~HSA_FLAG_QUEST;
    return v;
}

size_t quest_qprep_bytes(const Prob &p) {
    const size_t es = p.dtype == HSA_BF16 ? 2 : 4;
    const int gq = p.dtype == HSA_BF16 ? 2 : 1;
    return (size_t)p.rows * gq * 2 * p.d * es;
}

cudaError_t launch_quest_qprep(const Prob &p, const void *Q, void *Qp, cudaStream_t st) {
    if (p.rows == 0) return cudaSuccess;
    const long long total = p.rows * p.d;
    const unsigned blocks = (unsigned)((total + 255) / 256);
    const long long BT = (long long)p.B * p.Tq;
    if (p.dtype == HSA_BF16)
        quest_qprep_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>((const __nv_bfloat16 *)Q, (__nv_bfloat16 *)Qp, BT,
                                                                  p.Hkv, p.G, p.d);
    else
        quest_qprep_kernel<float><<<blocks, 256, 0, st>>>((const float *)Q, (float *)Qp, BT, p.Hkv, p.G, p.d);
    return cudaGetLastError();
}

static cudaError_t quest_summaries_range(const Prob &p, const void *K, void *Lq, int c0, int nc, cudaStream_t st) {
    if (p.B == 0 || nc == 0) return cudaSuccess;
    dim3 grid(nc, p.B);
    if (p.dtype == HSA_BF16)
        quest_summary_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)K, (__nv_bfloat16 *)Lq,
                                                                  p.Tcap, p.Hkv, p.d, p.S, p.Lc, c0);
    else
        quest_summary_kernel<float><<<grid, 256, 0, st>>>((const float *)K, (float *)Lq, p.Tcap, p.Hkv, p.d, p.S,
                                                          p.Lc, c0);
    return cudaGetLastError();
}

cudaError_t launch_quest_summaries(const Prob &p, const void *K, void *Lq, cudaStream_t st) {
    return quest_summaries_range(p, K, Lq, 0, p.C, st);
}

cudaError_t launch_quest_summary_chunk(const Prob &p, const void *K, void *Lq, int c, cudaStream_t st) {
    return quest_summaries_range(p, K, Lq, c, 1, st);
}

size_t refine_smem(const Prob &p) {
    return sizeof(float) * ((size_t)p.S * p.d + 5 * (size_t)p.d + p.S + (size_t)(RT / p.d) * p.d);
}

cudaError_t launch_landmarks_refined(const Prob &p, const void *K, const void *WL, const void *Wq, const void *Wk,
                                     const void *Wv, void *L, cudaStream_t st) {
    if (p.B == 0 || p.C == 0) return cudaSuccess;
    dim3 grid(p.C * p.Hkv, p.B);
    const size_t smem = refine_smem(p);
    const float scale = 1.0f / sqrtf((float)p.d);
    if (p.dtype == HSA_BF16) {
        auto k = refine_kernel<__nv_bfloat16>;
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, RT, smem, st>>>((const __nv_bfloat16 *)K, (const __nv_bfloat16 *)WL, (const __nv_bfloat16 *)Wq,
                                  (const __nv_bfloat16 *)Wk, (const __nv_bfloat16 *)Wv, (__nv_bfloat16 *)L, p.Tcap,
                                  p.Hkv, p.d, p.S, p.Lc, scale);
    } else {
        auto k = refine_kernel<float>;
        if (smem > 48 * 1024) cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        k<<<grid, RT, smem, st>>>((const float *)K, (const float *)WL, (const float *)Wq, (const float *)Wk,
                                  (const float *)Wv, (float *)L, p.Tcap, p.Hkv, p.d, p.S, p.Lc, scale);
    }
    return cudaGetLastError();
}

}  // namespace hsa
