// decode_mma.cuh -- warp-level pieces shared by the decode kernels (the
// landmark scan, the chunk gather and the fused decode step): ldmatrix and
// mma.sync m16n8k16 wrappers (bf16 in, fp32 accumulate), the 128-byte swizzle
// address of a TMA box, and one chunk's attention for a GQA group
// (HSA summary page, Implementation: standard attention inside each selected
// chunk; the chunk output is weighted by the softmax of the retrieval scores).
#pragma once

#include "common.cuh"

namespace hsa {
namespace decode {

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
// c += a * b for one m16n8k16 tile: a row-major 16x16 bf16, b column-major 16x8 bf16, c 16x8 fp32
__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    mma16816(c, a[0], a[1], a[2], a[3], b0, b1);
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}
// shared-memory address of 16-byte chunk j of row u in a box of 128-byte rows
// written by TMA with the 128-byte swizzle (chunk index XOR row mod 8)
__device__ __forceinline__ uint32_t swz(uint32_t box, int u, int j) {
    return box + (uint32_t)u * 128u + ((uint32_t)(j ^ (u & 7)) << 4);
}

__device__ __forceinline__ void red_add2(float *addr, float x, float y) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(x), "f"(y) : "memory");
}

// Q fragments of one row's group: rows g = lane/4 and lane/4 + 8 of the 16-row
// A tile, rows >= G zero.  Element (g, k) pairs come straight from global memory.
template <int D>
__device__ __forceinline__ void load_q_frags(const __nv_bfloat16 *qb, int G, uint32_t (&qa)[D / 16][4]) {
    const int lane = threadIdx.x & 31;
    const int g0 = lane >> 2, g1 = g0 + 8, q2 = 2 * (lane & 3);
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        const int k0 = 16 * ks + q2;
        qa[ks][0] = g0 < G ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g0 * D + k0) : 0u;
        qa[ks][1] = g1 < G ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g1 * D + k0) : 0u;
        qa[ks][2] = g0 < G ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g0 * D + k0 + 8) : 0u;
        qa[ks][3] = g1 < G ? *reinterpret_cast<const uint32_t *>(qb + (size_t)g1 * D + k0 + 8) : 0u;
    }
}

// One staged chunk (K boxes at sK, V boxes at sV): the group's attention
// output, times w / (softmax denominator), handed to emit(g, col, x, y) for
// the column pair (col, col+1) of head g < G, columns [d0, d0+DW).  wait_v()
// is called between the softmax and the PV product (V may still be landing
// while the scores are computed); if it returns false the product is skipped
// and the function returns false.
template <int D, int S, int DW, typename WaitV, typename Emit>
__device__ __forceinline__ bool chunk_unit(uint32_t sK, uint32_t sV, const uint32_t (&qa)[D / 16][4], int G,
                                           float scale, float w, int d0, Emit emit, WaitV wait_v) {
    constexpr int BOX = S * 128;     // bytes per box
    constexpr int KS = D / 16;       // k-steps of the score MMA
    constexpr int QN = S / 8;        // n-tiles of the score tile
    constexpr int PK = S / 16;       // k-steps of the PV MMA
    constexpr int ON = DW / 8;       // output n-tiles of this warp (even)
    const int lane = threadIdx.x & 31;
    const int g0 = lane >> 2, g1 = g0 + 8, q2 = 2 * (lane & 3);
    const int mi = lane >> 3, r8 = lane & 7;   // ldmatrix: this lane addresses row r8 of matrix mi

    // ---- scores: the 16 x S tile, all of it in every warp
    float sc[QN][4];
#pragma unroll
    for (int n = 0; n < QN; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
        const uint32_t kbox = sK + (uint32_t)(ks / 4) * BOX;
        const int jc = 2 * (ks % 4) + (mi & 1);
#pragma unroll
        for (int p = 0; p < QN / 2; ++p) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(swz(kbox, 16 * p + 8 * (mi >> 1) + r8, jc), b0, b1, b2, b3);
            mma16816(sc[2 * p], qa[ks], b0, b1);
            mma16816(sc[2 * p + 1], qa[ks], b2, b3);
        }
    }
    // ---- softmax per row (fp32): rows g0 (elements 0,1) and g1 (elements 2,3)
    float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
    for (int n = 0; n < QN; ++n) {
        m0 = fmaxf(m0, fmaxf(sc[n][0], sc[n][1]));
        m1 = fmaxf(m1, fmaxf(sc[n][2], sc[n][3]));
    }
    m0 = fmaxf(m0, __shfl_xor_sync(FULL, m0, 1));
    m0 = fmaxf(m0, __shfl_xor_sync(FULL, m0, 2));
    m1 = fmaxf(m1, __shfl_xor_sync(FULL, m1, 1));
    m1 = fmaxf(m1, __shfl_xor_sync(FULL, m1, 2));
    float l0 = 0.f, l1 = 0.f;
#pragma unroll
    for (int n = 0; n < QN; ++n) {
        sc[n][0] = expf((sc[n][0] - m0) * scale);
        sc[n][1] = expf((sc[n][1] - m0) * scale);
        sc[n][2] = expf((sc[n][2] - m1) * scale);
        sc[n][3] = expf((sc[n][3] - m1) * scale);
        l0 += sc[n][0] + sc[n][1];
        l1 += sc[n][2] + sc[n][3];
    }
    l0 += __shfl_xor_sync(FULL, l0, 1);
    l0 += __shfl_xor_sync(FULL, l0, 2);
    l1 += __shfl_xor_sync(FULL, l1, 1);
    l1 += __shfl_xor_sync(FULL, l1, 2);
    if (!wait_v()) return false;
    // ---- PV: columns [d0, d0 + DW)
    float o[ON][4];
#pragma unroll
    for (int n = 0; n < ON; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
#pragma unroll
    for (int kp = 0; kp < PK; ++kp) {
        uint32_t pa[4];
        pa[0] = pack_bf16(sc[2 * kp][0], sc[2 * kp][1]);
        pa[1] = pack_bf16(sc[2 * kp][2], sc[2 * kp][3]);
        pa[2] = pack_bf16(sc[2 * kp + 1][0], sc[2 * kp + 1][1]);
        pa[3] = pack_bf16(sc[2 * kp + 1][2], sc[2 * kp + 1][3]);
#pragma unroll
        for (int pp = 0; pp < ON / 2; ++pp) {
            const int c0 = d0 + 16 * pp;   // two n-tiles, inside one 64-column box
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(swz(sV + (uint32_t)(c0 / 64) * BOX, 16 * kp + 8 * (mi & 1) + r8, (c0 % 64) / 8 + (mi >> 1)), b0,
                      b1, b2, b3);
            mma16816(o[2 * pp], pa, b0, b1);
            mma16816(o[2 * pp + 1], pa, b2, b3);
        }
    }
    const float f0 = w / l0, f1 = w / l1;
#pragma unroll
    for (int n = 0; n < ON; ++n) {
        const int col = d0 + 8 * n + q2;
        if (g0 < G) emit(g0, col, o[n][0] * f0, o[n][1] * f0);
        if (g1 < G) emit(g1, col, o[n][2] * f1, o[n][3] * f1);
    }
    return true;
}

// Convert one row's fp32 accumulator (G*D values, in L2) to bf16 O, one warp.
__device__ __forceinline__ void acc_to_bf16(const float *src, __nv_bfloat16 *out, int n) {
    const int lane = threadIdx.x & 31;
    for (int e = lane * 4; e < n; e += 32 * 4) {
        const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + e));
        uint2 pk;
        pk.x = pack_bf16(v.x, v.y);
        pk.y = pack_bf16(v.z, v.w);
        *reinterpret_cast<uint2 *>(out + e) = pk;
    }
}

}  // namespace decode
}  // namespace hsa
