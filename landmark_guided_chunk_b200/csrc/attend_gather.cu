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
#include "decode_mma.cuh"
#include "sm100.cuh"

namespace hsa {
namespace {

using namespace sm100;
using namespace decode;

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
        acc_to_bf16(acc + (size_t)row * a.G * D, out, a.G * D);
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
