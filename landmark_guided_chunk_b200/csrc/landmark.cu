// landmark.cu -- landmark of every complete chunk (HSA summary page,
// Implementation: landmark = encode(mean pooling of the chunk), read here as
// the mean of the chunk's keys times the d x d projection W_L).
//
// One CTA per (chunk c, batch b).  The S x Hkv x d keys of a chunk are one
// contiguous block of K, so the pooling pass streams it with 16-byte loads.
// Each thread accumulates 8 (bf16) or 4 (fp32) channels over the S rows in
// fp32.  The pooled means stay in shared memory.  The projection reads W_L
// through L1/L2 (it is at most 64 KB and every CTA shares it).  L is rounded
// once to the dtype.
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

template <typename T>
__global__ void __launch_bounds__(256) landmark_kernel(const T *__restrict__ K, const T *__restrict__ W,
                                                       T *__restrict__ L, int Tkv, int Hkv, int d, int S, int C) {
    extern __shared__ float pooled[];   // [Hkv][d]
    constexpr int NV = Vec<T>::N;
    const int c = blockIdx.x, b = blockIdx.y;
    const int n = Hkv * d;              // channels of one token row
    const T *chunk = K + ((size_t)b * Tkv + (size_t)c * S) * n;
    const float inv = 1.0f / (float)S;
    for (int v = threadIdx.x; v < n / NV; v += blockDim.x) {
        float acc[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) acc[i] = 0.f;
        const uint4 *src = reinterpret_cast<const uint4 *>(chunk) + v;
        for (int u = 0; u < S; ++u) Vec<T>::add(acc, __ldg(src + (size_t)u * (n / NV)));
#pragma unroll
        for (int i = 0; i < NV; ++i) pooled[v * NV + i] = acc[i] * inv;
    }
    __syncthreads();
    for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int j = i / d, f = i - j * d;
        const float *m = pooled + j * d;
        float acc = 0.f;
        for (int e = 0; e < d; ++e) acc = fmaf(m[e], to_f32(W[(size_t)e * d + f]), acc);
        L[(((size_t)b * Hkv + j) * C + c) * d + f] = from_f32<T>(acc);
    }
}

}  // namespace

cudaError_t launch_landmarks(const Prob &p, const void *K, const void *W, void *L, cudaStream_t st) {
    if (p.B == 0 || p.C == 0) return cudaSuccess;
    dim3 grid(p.C, p.B);
    size_t smem = sizeof(float) * (size_t)p.Hkv * p.d;
    if (p.dtype == HSA_BF16) {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(landmark_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        landmark_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(
            (const __nv_bfloat16 *)K, (const __nv_bfloat16 *)W, (__nv_bfloat16 *)L, p.Tkv, p.Hkv, p.d, p.S, p.C);
    } else {
        if (smem > 48 * 1024)
            cudaFuncSetAttribute(landmark_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        landmark_kernel<float><<<grid, 256, smem, st>>>((const float *)K, (const float *)W, (float *)L, p.Tkv,
                                                         p.Hkv, p.d, p.S, p.C);
    }
    return cudaGetLastError();
}

}  // namespace hsa
