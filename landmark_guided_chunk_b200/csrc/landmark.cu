// landmark.cu -- landmark of every complete chunk (HSA summary page,
// Implementation: landmark = encode(mean pooling of the chunk), read here as
// the mean of the chunk's keys times the d x d projection W_L).
//
// One CTA per (chunk c, batch b).  The S x Hkv x d keys of a chunk are one
// contiguous block of K, so the pooling pass streams it with 16-byte loads:
// each thread accumulates 8 (bf16) or 4 (fp32) channels over a share of the S
// rows in fp32, eight rows' loads in flight at a time, and the shares are
// summed in shared memory.  The pooled means stay in shared memory.  Each CTA
// copies W_L into shared memory (cp.async, overlapping the pooling loads; every
// CTA reads the same copy from L2).  The projection is register-blocked: a
// thread forms four output columns for eight kv heads over a slice of the
// input dimension, so each W_L element is read once per chunk, and the slices
// are summed through shared memory.  L is rounded once to the dtype.
#include "common.cuh"

namespace hsa {
namespace {

template <typename T> struct Vec;
template <> struct Vec<float> {
    static constexpr int N = 4;
    __device__ static void add(float *acc, uint4 u) {
        const float *f = reinterpret_cast<const float *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[i] += f[i];
    }
};
template <> struct Vec<__nv_bfloat16> {
    static constexpr int N = 8;
    __device__ static void add(float *acc, uint4 u) {
        const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float2 f = __bfloat1622float2(h[i]);
            acc[2 * i] += f.x;
            acc[2 * i + 1] += f.y;
        }
    }
};

template <typename T> __device__ __forceinline__ void store4(T *dst, float4 o);
template <> __device__ __forceinline__ void store4<float>(float *dst, float4 o) {
    *reinterpret_cast<float4 *>(dst) = o;
}
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *dst, float4 o) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(o.x, o.y), hi = __floats2bfloat162_rn(o.z, o.w);
    uint2 u;
    u.x = *reinterpret_cast<unsigned *>(&lo);
    u.y = *reinterpret_cast<unsigned *>(&hi);
    *reinterpret_cast<uint2 *>(dst) = u;
}

// Four consecutive W_L entries of one row, from shared memory, as fp32.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                       __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ void fma4(float4 &o, float m, float4 w) {
    o.x = fmaf(m, w.x, o.x);
    o.y = fmaf(m, w.y, o.y);
    o.z = fmaf(m, w.z, o.z);
    o.w = fmaf(m, w.w, o.w);
}

constexpr int NT = 256;   // threads per CTA
constexpr int JB = 8;     // kv heads per projection pass (register block)
constexpr int RB = 16;    // rows whose loads a pooling thread issues before summing them

// Row groups of the pooling pass: R groups of nvr threads split a chunk's S rows.
__host__ __device__ __forceinline__ int row_groups(int nvr) { return NT >= nvr ? NT / nvr : 1; }

// Shared memory: W_L [d][d] (dtype T) | pooling partials [R][n] fp32 (row 0 ends
// as the chunk means) | projection partials [NT / (d/4)][JB][d] fp32.
__host__ __device__ __forceinline__ size_t landmark_smem(int n, int d, int nv, int tsize) {
    return (size_t)d * d * tsize + sizeof(float) * ((size_t)n * row_groups(n / nv) + (size_t)NT / (d / 4) * JB * d);
}

// A row of K as 16-byte vectors: through the read-only path, or (for a chunk this
// kernel itself has just completed) with ordinary loads, which see this CTA's writes.
template <bool NC> __device__ __forceinline__ uint4 ld_row(const uint4 *p) {
    if constexpr (NC) return __ldg(p);
    else return *p;
}

// The landmark of chunk c of sequence b, computed by the whole CTA (NT threads; the
// dynamic shared memory is laid out as landmark_smem describes).
template <typename T, bool NC>
__device__ __forceinline__ void landmark_chunk(unsigned char *sm, const T *__restrict__ K, const T *__restrict__ W,
                                               T *__restrict__ L, int b, int c, int Tcap, int Hkv, int d, int S,
                                               int Lc) {
    constexpr int NV = Vec<T>::N;
    const int n = Hkv * d;              // channels of one token row
    const int nvr = n / NV;             // 16-byte vectors of one token row
    const int R = row_groups(nvr);
    T *Ws = reinterpret_cast<T *>(sm);
    float *part = reinterpret_cast<float *>(sm + (size_t)d * d * sizeof(T));
    float *pp = part + (size_t)R * n;

    // W_L (at most 32 KB in bf16) is copied in asynchronously while the chunk streams;
    // every CTA reads the same copy from L2.
    for (int v = threadIdx.x; v < d * d / NV; v += NT)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         (uint32_t)__cvta_generic_to_shared(Ws + v * NV)),
                     "l"(W + v * NV)
                     : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");

    // Pooling: group grp sums rows grp, grp + R, ... with eight rows' loads in flight.
    const T *chunk = K + ((size_t)b * Tcap + (size_t)c * S) * n;
    const float inv = 1.0f / (float)S;
    if ((int)threadIdx.x < R * nvr || R == 1) {
        const int grp = R == 1 ? 0 : (int)threadIdx.x / nvr;
        const int v0 = R == 1 ? (int)threadIdx.x : (int)threadIdx.x % nvr;
        const int vstep = R == 1 ? NT : nvr;
        for (int v = v0; v < nvr; v += vstep) {
            float acc[NV];
#pragma unroll
            for (int i = 0; i < NV; ++i) acc[i] = 0.f;
            const uint4 *src = reinterpret_cast<const uint4 *>(chunk) + v;
            int u = grp;
            for (; u + (RB - 1) * R < S; u += RB * R) {
                uint4 x[RB];
#pragma unroll
                for (int k = 0; k < RB; ++k) x[k] = ld_row<NC>(src + (size_t)(u + k * R) * nvr);
#pragma unroll
                for (int k = 0; k < RB; ++k) Vec<T>::add(acc, x[k]);
            }
            for (; u < S; u += R) Vec<T>::add(acc, ld_row<NC>(src + (size_t)u * nvr));
            const float scl = R == 1 ? inv : 1.0f;
#pragma unroll
            for (int i = 0; i < NV; ++i) part[grp * n + v * NV + i] = acc[i] * scl;
        }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    if (R > 1) {
        for (int i = threadIdx.x; i < n; i += NT) {
            float sum = 0.f;
            for (int g = 0; g < R; ++g) sum += part[g * n + i];
            part[i] = sum * inv;
        }
        __syncthreads();
    }

    // Projection L[j][f] = sum_e mean[j][e] W_L[e][f].  Thread (eg, fq) forms columns
    // 4fq .. 4fq+3 for JB kv heads at once over its own slice of e (one W_L load feeds
    // 4 JB FMAs); the NT / (d/4) slices are then summed through shared memory.
    const int nfq = d >> 2, neg = NT / nfq, epg = d / neg;
    const int fq = (int)threadIdx.x % nfq, eg = (int)threadIdx.x / nfq;
    for (int j0 = 0; j0 < Hkv; j0 += JB) {
        float4 o[JB];
#pragma unroll
        for (int jj = 0; jj < JB; ++jj) o[jj] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int e4 = eg * epg; e4 < (eg + 1) * epg; e4 += 4) {
            const float4 w0 = load4(Ws + (size_t)(e4 + 0) * d + 4 * fq);
            const float4 w1 = load4(Ws + (size_t)(e4 + 1) * d + 4 * fq);
            const float4 w2 = load4(Ws + (size_t)(e4 + 2) * d + 4 * fq);
            const float4 w3 = load4(Ws + (size_t)(e4 + 3) * d + 4 * fq);
#pragma unroll
            for (int jj = 0; jj < JB; ++jj) {
                if (j0 + jj < Hkv) {
                    const float4 m = *reinterpret_cast<const float4 *>(part + (j0 + jj) * d + e4);
                    fma4(o[jj], m.x, w0);
                    fma4(o[jj], m.y, w1);
                    fma4(o[jj], m.z, w2);
                    fma4(o[jj], m.w, w3);
                }
            }
        }
#pragma unroll
        for (int jj = 0; jj < JB; ++jj)
            *reinterpret_cast<float4 *>(pp + ((size_t)eg * JB + jj) * d + 4 * fq) = o[jj];
        __syncthreads();
        for (int q = threadIdx.x; q < JB * nfq; q += NT) {
            const int jj = q / nfq, f4 = q - jj * nfq;
            if (j0 + jj >= Hkv) continue;
            float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int g = 0; g < neg; ++g) {
                const float4 x = *reinterpret_cast<const float4 *>(pp + ((size_t)g * JB + jj) * d + 4 * f4);
                sum.x += x.x;
                sum.y += x.y;
                sum.z += x.z;
                sum.w += x.w;
            }
            store4<T>(L + (((size_t)b * Hkv + j0 + jj) * Lc + c) * d + 4 * f4, sum);
        }
        __syncthreads();
    }
}

template <typename T>
__global__ void __launch_bounds__(NT, 2) landmark_kernel(const T *__restrict__ K, const T *__restrict__ W,
                                                         T *__restrict__ L, int Tcap, int Hkv, int d, int S, int Lc) {
    extern __shared__ __align__(16) unsigned char sm[];
    landmark_chunk<T, true>(sm, K, W, L, blockIdx.y, blockIdx.x, Tcap, Hkv, d, S, Lc);
}

// One decode step's cache update, one CTA per sequence b: the new token's K and V
// rows go to position Tkv, and if that completes a chunk, its landmark follows.
template <typename T>
__global__ void __launch_bounds__(NT, 2) decode_append_kernel(const T *__restrict__ knew, const T *__restrict__ vnew,
                                                              T *__restrict__ K, T *__restrict__ V,
                                                              const T *__restrict__ W, T *__restrict__ L, int Tkv,
                                                              int Tcap, int Hkv, int d, int S, int Lc, int complete) {
    extern __shared__ __align__(16) unsigned char sm[];
    const int b = blockIdx.x;
    const int n = Hkv * d, nv16 = n * (int)sizeof(T) / 16;
    const uint4 *ks = reinterpret_cast<const uint4 *>(knew + (size_t)b * n);
    const uint4 *vs = reinterpret_cast<const uint4 *>(vnew + (size_t)b * n);
    uint4 *kd = reinterpret_cast<uint4 *>(K + ((size_t)b * Tcap + Tkv) * n);
    uint4 *vd = reinterpret_cast<uint4 *>(V + ((size_t)b * Tcap + Tkv) * n);
    for (int v = threadIdx.x; v < nv16; v += NT) {
        kd[v] = ks[v];
        vd[v] = vs[v];
    }
    if (!complete) return;
    __syncthreads();   // the chunk's last row, written above, is read back by the whole CTA
    landmark_chunk<T, false>(sm, K, W, L, b, (Tkv + 1) / S - 1, Tcap, Hkv, d, S, Lc);
}

}  // namespace

cudaError_t launch_landmarks(const Prob &p, const void *K, const void *W, void *L, cudaStream_t st) {
    if (p.B == 0 || p.C == 0) return cudaSuccess;
    dim3 grid(p.C, p.B);
    const bool bf = p.dtype == HSA_BF16;
    const size_t smem = landmark_smem(p.Hkv * p.d, p.d, bf ? 8 : 4, bf ? 2 : 4);
    if (p.dtype == HSA_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(landmark_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        landmark_kernel<__nv_bfloat16><<<grid, NT, smem, st>>>(
            (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)W, (__nv_bfloat16 *)L, p.Tcap, p.Hkv, p.d, p.S, p.Lc);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(landmark_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        landmark_kernel<float><<<grid, NT, smem, st>>>((const float *)K, (const float *)W, (float *)L, p.Tcap,
                                                         p.Hkv, p.d, p.S, p.Lc);
    }
    return cudaGetLastError();
}

cudaError_t launch_decode_append(const Prob &p, const void *knew, const void *vnew, void *K, void *V, const void *W,
                                 void *L, cudaStream_t st) {
    if (p.B == 0) return cudaSuccess;
    const int complete = (p.Tkv + 1) % p.S == 0 ? 1 : 0;
    const bool bf = p.dtype == HSA_BF16;
    const size_t smem = complete ? landmark_smem(p.Hkv * p.d, p.d, bf ? 8 : 4, bf ? 2 : 4) : 0;
    if (bf) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(decode_append_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)smem);
        decode_append_kernel<__nv_bfloat16><<<p.B, NT, smem, st>>>(
            (const __nv_bfloat16 *)knew, (const __nv_bfloat16 *)vnew, (__nv_bfloat16 *)K, (__nv_bfloat16 *)V,
            (const __nv_bfloat16 *)W, (__nv_bfloat16 *)L, p.Tkv, p.Tcap, p.Hkv, p.d, p.S, p.Lc, complete);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(decode_append_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        decode_append_kernel<float><<<p.B, NT, smem, st>>>((const float *)knew, (const float *)vnew, (float *)K,
                                                           (float *)V, (const float *)W, (float *)L, p.Tkv, p.Tcap,
                                                           p.Hkv, p.d, p.S, p.Lc, complete);
    }
    return cudaGetLastError();
}

}  // namespace hsa
