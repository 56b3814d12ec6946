// attend_gather.cu -- chunk attention and retrieval-weighted fusion for few
// rows with many kept slots (decode), bf16 (HSA summary page, Implementation:
// attend to each selected chunk with standard attention, then fuse the chunk
// outputs weighted by the softmax of their retrieval scores).
//
// A unit is one (row = (b, t, kv head j), kept slot i).  Persistent CTAs (as
// many as fit on the GPU) take units round-robin; one warp reads all of a
// CTA's keff and chunk indices in one round trip, and thread 0 starts TMA
// copies of the chunks -- S rows of K and of V as boxes of 64 columns x S rows
// with the 128-byte swizzle -- into a ring of stages, refilling each stage as
// soon as its unit is done.  So the resident CTAs keep the gather streaming
// from HBM back to back.  The GQA group's G <= 16 query heads are the rows of
// one 16-row MMA tile, so the one staged copy serves the whole group:
//   scores : every warp computes the full 16 x S tile Q_g . K_u with
//            mma.sync m16n8k16 (bf16 in, fp32 accumulate), K fragments read
//            with ldmatrix from the swizzled boxes
//   softmax: fp32 on the accumulator fragments (max subtracted; the four
//            lanes that share a row reduce with two shuffles)
//   PV     : the probabilities, rounded to bf16, are the A fragments of the
//            second MMA as they stand; warp w produces output columns
//            [w*d/4, (w+1)*d/4), V fragments read with ldmatrix.trans
// The chunk output, multiplied by its fusion weight w_i and divided by the
// chunk's softmax denominator, is added (red.add) into the row's fp32
// accumulator in the workspace.  Whichever warp completes a row's last slot
// (per-row counter; counters and accumulators are zeroed with the status word)
// converts the accumulator to bf16 O, so no second launch is needed.
//
// The group's heads are only G rows, far below a tcgen05 tile; the warp-level
// MMA is used because it removes the CUDA-core conversions and FMAs that
// would otherwise bound this HBM-bound step.
#include "common.cuh"
#include "sm100.cuh"

namespace hsa {
namespace {

using namespace sm100;

constexpr int NTG = 128;   // threads per CTA: 4 warps

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
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
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

__device__ __forceinline__ void red_add2(float *addr, float x, float y) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(addr), "f"(x), "f"(y) : "memory");
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

constexpr int MAXW = 8;    // worker warps (= chunk stages) per CTA at most
constexpr int MAXU = 32;   // units per worker at most (the grid is sized for it)

struct GatherArgs {
    int B, Tq, Tcap, H, Hkv, S, C, kmax, G;
    int nunits, nw;     // units = rows * kmax (slot-major within a row); worker warps per CTA
    long long q_pos0;
    float scale;        // 1/sqrt(d)
    uint32_t *status;   // workspace status word
    float *part;        // partial mode: o_i of every (row, slot) [rows][kmax][G][D], unweighted; else null
};

// Every warp is an independent worker with one chunk stage of its own; a CTA is
// just as many workers as one SM's shared memory holds, so that (for decode
// sizes) every unit's chunk is in flight in a single wave.  Worker x + w*grid
// takes units worker, worker + workers, ...  For each unit it loads keff, the
// chunk index, the row's retrieval scores and the group's Q in one round trip,
// starts the TMA copies of the chunk's K and V (separate barriers: the scores
// are computed while V lands), and adds the weighted chunk output into the
// row's fp32 accumulator.  The per-row completion counters are bumped after
// all of the worker's additions, behind a single fence; the warp that
// completes a row converts its accumulator to bf16 O.
template <int D, int S, bool PART>
__global__ void __launch_bounds__(MAXW * 32) attend_gather_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                  const __grid_constant__ CUtensorMap tmV,
                                                                  const __nv_bfloat16 *__restrict__ Q,
                                                                  const int32_t *__restrict__ idx,
                                                                  const float *__restrict__ score,
                                                                  const int32_t *__restrict__ keff,
                                                                  __nv_bfloat16 *__restrict__ O,
                                                                  float *__restrict__ acc, int32_t *__restrict__ cnt,
                                                                  GatherArgs a) {
    constexpr int NB = D / 64;            // boxes per K chunk (and per V chunk)
    constexpr int BOX = S * 128;          // bytes per box
    constexpr int STAGE = 2 * NB * BOX;   // one chunk's K and V
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar[2 * MAXW];   // K and V barrier of each worker
    __shared__ int s_abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int workers = (int)gridDim.x * a.nw, worker = (int)blockIdx.x + warp * (int)gridDim.x;
    uint64_t *mbk = &bar[2 * warp], *mbv = &bar[2 * warp + 1];
    uint8_t *stage = base + (size_t)warp * STAGE;
    if (threadIdx.x == 0) s_abort = 0;
    if (lane == 0) {
        mbar_init(mbk, 1);
        mbar_init(mbv, 1);
        fence_mbar_init();
    }
    __syncthreads();

    // per unit r of this worker, kept by lane r: its row, keff and chunk (-2: slot unused)
    int m_row = 0, m_ke = 0, m_c = -2;
    uint32_t phase = 0;     // parity of the next K (and V) load
    bool pend_k = false, pend_v = false;   // copies issued and not yet consumed
    int nr = 0;
    for (int u = worker; u < a.nunits; u += workers, ++nr) {
        const int row = u / a.kmax, i = u - row * a.kmax;
        const int j = row % a.Hkv, bt = row / a.Hkv, t = bt % a.Tq, b = bt / a.Tq;
        const size_t qrow = (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * D;
        // one round trip: keff, chunk index, retrieval scores, Q fragments
        int ke = 0, c = 0;
        if (lane == 0) {
            ke = keff[row];
            c = idx[(size_t)row * a.kmax + i];
        }
        const float sv = (!PART && lane < a.kmax) ? score[(size_t)row * a.kmax + lane] : -INFINITY;
        uint32_t qa[D / 16][4];
        load_q_frags<D>(Q + qrow, a.G, qa);
        ke = __shfl_sync(FULL, ke, 0);
        c = __shfl_sync(FULL, c, 0);
        bool bad = false;
        if (ke < 0 || ke > a.kmax) {
            bad = true;
            ke = ke < 0 ? 0 : a.kmax;
        }
        if (i >= ke) {
            c = -2;
        } else {
            long long ncl = (a.q_pos0 + t) / a.S;
            if (ncl > a.C) ncl = a.C;
            if (c < 0 || c >= ncl) {
                bad = true;
                c = -1;
            }
        }
        if (bad && lane == 0) atomicOr(a.status, DEV_BAD_INDEX);
        if (lane == nr) {
            m_row = row;
            m_ke = ke;
            m_c = c;
        }
        bool issued = false;
        if (c >= 0 && !s_abort) {
            issued = true;
            if (lane == 0) {
                const int z = b * a.Tcap + c * S;
                mbar_expect_tx(mbk, (uint32_t)(NB * BOX));
                mbar_expect_tx(mbv, (uint32_t)(NB * BOX));
#pragma unroll
                for (int kb = 0; kb < NB; ++kb) tma_load_3d(stage + kb * BOX, &tmK, 64 * kb, j, z, mbk);
#pragma unroll
                for (int kb = 0; kb < NB; ++kb) tma_load_3d(stage + (NB + kb) * BOX, &tmV, 64 * kb, j, z, mbv);
            }
            pend_k = pend_v = true;
        }
        if (c == -2) {
            if (ke == 0 && i == 0 && !PART)   // no candidates: the output is zero
                for (int e = lane; e < a.G * D; e += 32) O[qrow + e] = __float2bfloat16(0.f);
            continue;
        }
        // this slot's fusion weight: softmax over the row's kept retrieval scores
        const float xs = lane < ke ? sv : -INFINITY;
        const float m = warp_max(xs);
        const float ex = lane < ke ? expf(xs - m) : 0.f;
        const float w = __shfl_sync(FULL, ex, i) / warp_sum(ex);
        bool ok = pend_k && mbar_wait(mbk, phase, &s_abort, a.status);
        if (ok) pend_k = false;
        ok = __all_sync(FULL, ok) && !s_abort;
        if (ok) {
            const uint32_t sk = smem_u32(stage);
            auto wait_v = [&]() {
                bool v = mbar_wait(mbv, phase, &s_abort, a.status);
                if (v) pend_v = false;
                return __all_sync(FULL, v) && !s_abort;
            };
            if constexpr (!PART) {
                float *racc = acc + (size_t)row * a.G * D;
                chunk_unit<D, S, D>(sk, sk + NB * BOX, qa, a.G, a.scale, w, 0,
                                    [&](int g, int col, float x, float y) { red_add2(racc + (size_t)g * D + col, x, y); },
                                    wait_v);
            } else {   // partial output of this slot: o_i unweighted, plain stores
                float *po = a.part + ((size_t)row * a.kmax + i) * a.G * D;
                chunk_unit<D, S, D>(sk, sk + NB * BOX, qa, a.G, a.scale, 1.0f, 0,
                                    [&](int g, int col, float x, float y) {
                                        *reinterpret_cast<float2 *>(po + (size_t)g * D + col) = make_float2(x, y);
                                    },
                                    wait_v);
            }
        }
        if (issued && !pend_k && !pend_v) phase ^= 1u;   // both copies consumed (after an expired wait they stay pending)
        __syncwarp();   // the stage is free for the next unit
    }

    // completion counters, behind one fence for all of this worker's additions;
    // whoever completes a row's last slot converts the row's accumulator to O
    if (!PART) __threadfence();
    for (int r = 0; r < nr && !PART; ++r) {
        const int row = __shfl_sync(FULL, m_row, r), ke = __shfl_sync(FULL, m_ke, r), c = __shfl_sync(FULL, m_c, r);
        if (c == -2) continue;
        int last = 0;
        if (lane == 0) last = atomicAdd(&cnt[row], 1) == ke - 1;
        if (!__shfl_sync(FULL, last, 0)) continue;
        __threadfence();
        const int j = row % a.Hkv, bt = row / a.Hkv, t = bt % a.Tq, b = bt / a.Tq;
        __nv_bfloat16 *out = O + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * D;
        const float *src = acc + (size_t)row * a.G * D;
        for (int e = lane * 4; e < a.G * D; e += 32 * 4) {
            const float4 v = __ldcg(reinterpret_cast<const float4 *>(src + e));
            uint2 pk;
            pk.x = pack_bf16(v.x, v.y);
            pk.y = pack_bf16(v.z, v.w);
            *reinterpret_cast<uint2 *>(out + e) = pk;
        }
    }
    // after an expired wait: let the copies still in flight land before the CTA exits
    if (lane == 0 && pend_k) mbar_drain(mbk, phase);
    if (lane == 0 && pend_v) mbar_drain(mbv, phase);
}

template <int D, int S, bool PART>
cudaError_t launch_ds(const Prob &p, GatherArgs a, const CUtensorMap &mk, const CUtensorMap &mv, const void *Q,
                      const int32_t *idx, const float *score, const int32_t *keff, void *O, float *acc, int32_t *cnt,
                      cudaStream_t st) {
    constexpr int STAGE = 2 * (D / 64) * S * 128;
    int nw = (232448 - 2048) / STAGE;   // stages that fit one CTA's shared memory
    a.nw = nw < 1 ? 1 : (nw > MAXW ? MAXW : nw);
    const size_t smem = 1024 + (size_t)a.nw * STAGE;
    cudaError_t e =
        cudaFuncSetAttribute(attend_gather_kernel<D, S, PART>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148, per_sm = 1;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attend_gather_kernel<D, S, PART>, a.nw * 32,
                                                           smem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) per_sm = 1;
    long long grid = (long long)sms * per_sm;
    const long long min_grid = (a.nunits + (long long)MAXU * a.nw - 1) / ((long long)MAXU * a.nw);
    if (grid < min_grid) grid = min_grid;
    const long long max_grid = (a.nunits + a.nw - 1) / a.nw;   // no CTA without units
    if (grid > max_grid) grid = max_grid;
    attend_gather_kernel<D, S, PART><<<(unsigned)grid, a.nw * 32, smem, st>>>(
        mk, mv, (const __nv_bfloat16 *)Q, idx, score, keff, (__nv_bfloat16 *)O, acc, cnt, a);
    return cudaGetLastError();
}

template <int D, bool PART>
cudaError_t launch_d(const Prob &p, const GatherArgs &a, const CUtensorMap &mk, const CUtensorMap &mv, const void *Q,
                     const int32_t *idx, const float *score, const int32_t *keff, void *O, float *acc, int32_t *cnt,
                     cudaStream_t st) {
    switch (p.S) {
        case 32: return launch_ds<D, 32, PART>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
        case 64: return launch_ds<D, 64, PART>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
        case 128: return launch_ds<D, 128, PART>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

bool attend_gather_supported(const Prob &p) {
    return p.dtype == HSA_BF16 && (p.d == 64 || p.d == 128) && (p.S == 32 || p.S == 64 || p.S == 128) &&
           p.G <= 16 && p.kmax <= 32 && (long long)p.B * p.Tcap < (1ll << 31) && p.rows * p.kmax < (1ll << 31);
}

cudaError_t launch_attend_gather(const Prob &p, const void *Q, const void *K, const void *V, const int32_t *idx,
                                 const float *score, const int32_t *keff, void *O, float *acc, int32_t *cnt,
                                 uint32_t *status, cudaStream_t st, float *part) {
    GatherArgs a;
    a.part = part;
    a.B = p.B;
    a.Tq = p.Tq;
    a.Tcap = p.Tcap;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.S = p.S;
    a.C = p.C;
    a.kmax = p.kmax;
    a.G = p.G;
    a.nunits = (int)(p.rows * p.kmax);
    a.nw = 1;
    a.q_pos0 = p.q_pos0;
    a.scale = 1.0f / sqrtf((float)p.d);
    a.status = status;
    // K and V as 3D (d, Hkv, B*Tcap): box (64, 1, S) = S rows of 128 bytes, 128-byte swizzle
    CUtensorMap mk, mv;
    const uint64_t dims[3] = {(uint64_t)p.d, (uint64_t)p.Hkv, (uint64_t)p.B * p.Tcap};
    const uint64_t strides[2] = {(uint64_t)p.d * 2, (uint64_t)p.Hkv * p.d * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)p.S};
    cudaError_t e;
    if ((e = make_tmap_3d(&mk, K, dims, strides, box)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, V, dims, strides, box)) != cudaSuccess) return e;
    if (part != nullptr) {
        if (p.d == 128) return launch_d<128, true>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
        return launch_d<64, true>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
    }
    if (p.d == 128) return launch_d<128, false>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
    return launch_d<64, false>(p, a, mk, mv, Q, idx, score, keff, O, acc, cnt, st);
}

}  // namespace hsa
