// select_stream.cu -- chunk selection for decode (one query per sequence over
// a long cached context), bf16 (HSA summary page, Core Technique /
// Implementation: score every landmark of the strictly-past chunks, keep the
// top k; gap router from the value-of-information router page).
//
// The rows (b, kv head j) all have the same candidates, ncand = min(q_pos0/S, C),
// so their landmarks form rows * ceil(ncand/64) tiles of 64 chunks.  Each
// persistent CTA (one per SM) takes a contiguous range of those tiles:
//   warp 6     TMA producer: streams the range's tiles (64 landmark rows x d,
//              boxes of 64 columns with the 128-byte swizzle) through a ring
//              of NST stages, so ~190 KB per SM are always in flight
//   warps 0-5  consumers, tile k -> warp k % 6 (stage k % 12, so each stage
//              has one consumer warp): the group score of 16 chunks
//              per mma.sync m16n8k16 (A = landmark rows via ldmatrix, B = the
//              group's query heads as columns, fp32 accumulate; the products
//              are exact and the group score is the fp32 sum of the head
//              columns), then a warp-wide top-k list per row: a batch of 32
//              candidates with few qualifiers is inserted one by one, one with
//              many is sorted by a bitonic network and merged
// At the end each CTA merges its warps' lists per row (bitonic merges), writes
// one list per (row, CTA), and the CTA that completes a row (per-row counter,
// zeroed with the status word) merges the row's lists and writes its
// selection, with the router's k_eff.
//
// Fused decode step (hsa_forward): the same launch then does the chunk
// attention and the fusion.  The warp that completes a row publishes, per
// kept slot i, a unit descriptor (chunk + 1, fusion weight w_i) with a
// release store (empty slots get a marker), and once a CTA's scan is done all
// of its warps become gather workers with one K/V stage each, carved from the
// now idle ring: a worker claims the next (row, slot) unit from a global
// counter, loads the row's query heads, waits (bounded) for the descriptor,
// stages the chunk's K and V by TMA and adds w_i * o_i / l_i into the row's
// fp32 accumulator; whoever finishes a row's last slot converts it to bf16 O.
// Rows published early are gathered while the slowest CTAs still scan, and the
// gather needs no launch of its own.  Workers wait only on rows, and rows
// depend only on the scan, so the launch is cooperative (every CTA resident)
// and cannot deadlock.
#include <algorithm>

#include "common.cuh"
#include "decode_mma.cuh"
#include "sm100.cuh"

namespace hsa {
namespace {

using namespace sm100;
using namespace decode;

constexpr int TCH = 64;    // chunks per tile
constexpr int NCW = 6;     // consumer warps
constexpr int NST = 12;    // ring stages
constexpr int RMAX = 4;    // rows one CTA may touch
// Tile k goes to warp k % NCW and stage k % NST.  With NST a multiple of NCW
// every stage has a single consumer warp, which waits for the stage's phases
// in order.  (Two warps waiting on one stage for consecutive phases would let
// the later one see the earlier phase's parity as complete.)
static_assert(NST % NCW == 0, "each ring stage must belong to one consumer warp");

struct StreamArgs {
    int Tq, H, Hkv, G, S, C, k, kmax;
    int Lc;               // chunks per (b, kv head) in L's layout
    int ncand, tpr;       // candidates of every row; tiles per row
    long long total;      // rows * tpr
    int grid, maxe;       // CTAs; list slots per row
    float tau;
    uint32_t *status;
    int rows;             // B * Hkv (one query per sequence)
    // fused decode step only
    int B, Tcap, nunits, nwg;   // units = rows * kmax; gather workers per CTA
    float scale;                // 1/sqrt(d)
    unsigned long long *desc;   // [rows][kmax] unit descriptors: (chunk + 1) << 32 | bits(w), EMPTY_SLOT, 0 until published
    int32_t *ctr;               // [0] units claimed
    int32_t *att_cnt;           // [rows] kept slots gathered per row
    float *acc;                 // [rows][G][d] fp32 accumulators
    __nv_bfloat16 *O;
};

struct __align__(8) StreamBars {
    uint64_t full[NST], empty[NST];
    int abort;
};

// A slot or index outside its range (which the grid sizing rules out) is
// recorded in the status word and the access skipped.
__device__ __forceinline__ bool in_range(long long x, long long n, uint32_t *status) {
    if (x >= 0 && x < n) return true;
    atomicOr(status, DEV_INTERNAL);
    return false;
}

__device__ __forceinline__ void st_release_gpu64(unsigned long long *p, unsigned long long v) {
    asm volatile("st.release.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_acquire_gpu64(const unsigned long long *p) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}
constexpr unsigned long long EMPTY_SLOT = 0xffffffff00000000ull;   // a published slot past the row's keff

// Wait until unit descriptor *p is published; 0 if the wait expired or another
// CTA's wait did (the status word carries DEV_TIMEOUT).
__device__ __forceinline__ unsigned long long wait_published(const unsigned long long *p, uint32_t *status,
                                                             volatile int *abort) {
    unsigned long long v = ld_acquire_gpu64(p);
    if (v != 0) return v;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        __nanosleep(128);
        if ((v = ld_acquire_gpu64(p)) != 0) return v;
        if (*abort || (__ldcv(status) & DEV_TIMEOUT)) return 0;
        if (globaltimer_ns() - t0 > WAIT_LIMIT_NS) {
            *abort = 1;
            atomicOr(status, DEV_TIMEOUT);
            return 0;
        }
    }
}

// Order-preserving unsigned code of a float (for atomicMax on scores).
__device__ __forceinline__ unsigned ord_enc(float x) {
    const unsigned u = __float_as_uint(x);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float ord_dec(unsigned e) {
    return __uint_as_float((e & 0x80000000u) ? (e & 0x7fffffffu) : ~e);
}

__device__ __forceinline__ long long cta_lo(const StreamArgs &a, int x) { return (long long)x * a.total / a.grid; }
// the CTA whose range holds tile T
__device__ __forceinline__ int cta_of(const StreamArgs &a, long long T) {
    return (int)(((T + 1) * a.grid - 1) / a.total);
}

// ---------------------------------------------------------------------------- fused gather phase
// Bytes of one gather worker's stage: a chunk's K and V, D/64 boxes of S rows each.
template <int D, int S>
constexpr int gather_stage_bytes() {
    return 2 * (D / 64) * S * 128;
}

// The gather phase of the fused decode step (all of a CTA's warps, after its
// scan): claim units, wait for their descriptors, stage the chunks, accumulate.
template <int D, int S>
__device__ __forceinline__ void gather_phase(const StreamArgs &a, uint8_t *base, uint64_t *gbar, volatile int *abort,
                                             const CUtensorMap &tmK, const CUtensorMap &tmV,
                                             const __nv_bfloat16 *__restrict__ Q) {
    constexpr int NB = D / 64, BOX = S * 128, STAGE = gather_stage_bytes<D, S>();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (warp >= a.nwg) return;
    uint8_t *stage = base + (size_t)warp * STAGE;
    uint64_t *mbk = &gbar[2 * warp], *mbv = &gbar[2 * warp + 1];
    uint32_t phase = 0;                    // parity of the next K (and V) load
    bool pend_k = false, pend_v = false;   // copies issued and not yet consumed
    while (!*abort) {
        int u = 0;
        if (lane == 0) u = atomicAdd(&a.ctr[0], 1);
        u = __shfl_sync(FULL, u, 0);
        if (u >= a.nunits) break;
        const int row = u / a.kmax;
        const int j = row % a.Hkv, b = row / a.Hkv;
        const size_t qrow = ((size_t)b * a.H + (size_t)j * a.G) * D;   // Q [B][1][H][d]
        // the group's query heads while the row's selection may still be in progress
        uint32_t qa[D / 16][4];
        load_q_frags<D>(Q + qrow, a.G, qa);
        unsigned long long dv = 0;
        if (lane == 0) dv = wait_published(&a.desc[u], a.status, abort);
        dv = __shfl_sync(FULL, dv, 0);
        if (dv == 0) break;
        if (dv != EMPTY_SLOT) {
            const int c = (int)(dv >> 32) - 1;
            const float w = __uint_as_float((uint32_t)dv);
            if (in_range(c, a.ncand, a.status)) {
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
                bool ok = mbar_wait(mbk, phase, abort, a.status);
                if (ok) pend_k = false;
                if (!__all_sync(FULL, ok)) break;
                const uint32_t sk = smem_u32(stage);
                float *racc = a.acc + (size_t)row * a.G * D;
                auto wait_v = [&]() {
                    bool v = mbar_wait(mbv, phase, abort, a.status);
                    if (v) pend_v = false;
                    return __all_sync(FULL, v);
                };
                if (!chunk_unit<D, S, D>(sk, sk + NB * BOX, qa, a.G, a.scale, w, 0,
                                         [&](int g, int col, float x, float y) { red_add2(racc + (size_t)g * D + col, x, y); },
                                         wait_v))
                    break;
                phase ^= 1u;   // both copies consumed
            }
        }
        // this slot is done (empty ones too); whoever completes the row's kmax slots converts it to O
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(&a.att_cnt[row], 1) == a.kmax - 1;
        if (__shfl_sync(FULL, last, 0)) {
            __threadfence();
            acc_to_bf16(a.acc + (size_t)row * a.G * D, a.O + qrow, a.G * D);   // zeros for a row without candidates
        }
        __syncwarp();   // the stage is free for the next unit
    }
    // after an expired wait: let the copies still in flight land before the CTA exits
    if (lane == 0 && pend_k) mbar_drain(mbk, phase);
    if (lane == 0 && pend_v) mbar_drain(mbv, phase);
}

constexpr int WL_BYTES = RMAX * NCW * 16 * (int)sizeof(float2);   // the consumer warps' lists

// S is the chunk length of the fused gather phase (0: selection only).
template <int D, int S>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
    select_stream_kernel(const __grid_constant__ CUtensorMap tmL, const __grid_constant__ CUtensorMap tmK,
                         const __grid_constant__ CUtensorMap tmV, const __nv_bfloat16 *__restrict__ Q,
                         float2 *__restrict__ lists, int32_t *__restrict__ idx, float *__restrict__ score,
                         int32_t *__restrict__ keff, int32_t *__restrict__ cnt, StreamArgs a) {
    constexpr bool FUSE = S > 0;
    constexpr int NB = D / 64;          // boxes per tile
    constexpr int BOXB = TCH * 128;     // bytes of one box
    constexpr int STB = NB * BOXB;      // bytes of one stage
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ StreamBars bar;
    __shared__ __align__(8) uint64_t gbar[FUSE ? 2 * (NCW + 1) : 1];   // gather: K and V barrier per worker
    // each consumer warp's list per row slot, after the ring (the gather stages may cover both)
    float2 (*wl)[NCW][16] = reinterpret_cast<float2 (*)[NCW][16]>(base + (size_t)NST * STB);
    __shared__ unsigned s_floor[RMAX];     // best k-th score any warp's list has reached, per row slot
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int x = (int)blockIdx.x;
    const long long lo = cta_lo(a, x), hi = cta_lo(a, x + 1);
    const int ntile = (int)(hi - lo);
    const long long r_lo = lo / a.tpr;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&bar.full[s], 1);
            mbar_init(&bar.empty[s], 1);
        }
        if constexpr (FUSE)
            for (int s = 0; s < 2 * (NCW + 1); ++s) mbar_init(&gbar[s], 1);
        bar.abort = 0;
        fence_mbar_init();
    }
    for (int e = threadIdx.x; e < RMAX * NCW * 16; e += blockDim.x)
        (&wl[0][0][0])[e] = make_float2(-INFINITY, __int_as_float(INT32_MAX));
    if (threadIdx.x < RMAX) s_floor[threadIdx.x] = 0x007fffffu;   // the code of -inf
    __syncthreads();

    if (warp == NCW) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            bool ok = true;
            int k = 0;
            for (; k < ntile; ++k) {
                const int s = k % NST, u = k / NST;
                if (u > 0 && !(ok = mbar_wait(&bar.empty[s], (u - 1) & 1, &bar.abort, a.status))) break;
                const long long T = lo + k, row = dbg_clamp(T / a.tpr, 0, a.rows, a.status);
                const int y = (int)(row * a.Lc + dbg_clamp((T % a.tpr) * TCH, 0, a.ncand, a.status));
                mbar_expect_tx(&bar.full[s], (uint32_t)STB);
#pragma unroll
                for (int kb = 0; kb < NB; ++kb)
                    tma_load_2d(base + (size_t)s * STB + kb * BOXB, &tmL, 64 * kb, y, &bar.full[s]);
            }
            // every load issued has landed before the CTA may exit
            for (int s = 0; s < NST && s < k; ++s) mbar_drain(&bar.full[s], ((k - 1 - s) / NST) & 1);
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int r4 = lane >> 2, q2 = 2 * (lane & 3);
        const int mi = lane >> 3, r8 = lane & 7;   // ldmatrix: this lane addresses row r8 of matrix mi
        uint32_t bq[D / 16][2];
        long long cur = -1;
        float v;
        int id;
        list_init(v, id);
        for (int k = warp; k < ntile; k += NCW) {
            const int s = k % NST, u = k / NST;
            const long long T = lo + k, row = T / a.tpr;
            const int kt = (int)(T % a.tpr);
            if (row != cur) {
                if (cur >= 0 && lane < 16 && in_range(cur - r_lo, RMAX, a.status))
                    wl[cur - r_lo][warp][lane] = make_float2(v, __int_as_float(id));
                list_init(v, id);
                cur = row;
                // the group's query heads as B columns (head lane/4; heads >= G are zero)
                const int j = (int)(row % a.Hkv), b = (int)(row / a.Hkv);
                const __nv_bfloat16 *qh = Q + (((size_t)b * a.Tq) * a.H + (size_t)j * a.G + r4) * D;
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    bq[ks][0] = r4 < a.G ? *reinterpret_cast<const uint32_t *>(qh + 16 * ks + q2) : 0u;
                    bq[ks][1] = r4 < a.G ? *reinterpret_cast<const uint32_t *>(qh + 16 * ks + 8 + q2) : 0u;
                }
            }
            if (!mbar_wait(&bar.full[s], u & 1, &bar.abort, a.status)) break;
            const uint32_t st = smem_u32(base + (size_t)s * STB);
            float sc[TCH / 16][2];
#pragma unroll
            for (int mt = 0; mt < TCH / 16; ++mt) {
                float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int ks = 0; ks < D / 16; ++ks) {
                    uint32_t a0, a1, a2, a3;
                    ldsm_x4(swz(st + (uint32_t)(ks / 4) * BOXB, 16 * mt + 8 * (mi & 1) + r8, 2 * (ks % 4) + (mi >> 1)),
                            a0, a1, a2, a3);
                    mma16816(c, a0, a1, a2, a3, bq[ks][0], bq[ks][1]);
                }
                float s0 = c[0] + c[1], s1 = c[2] + c[3];
                s0 += __shfl_xor_sync(FULL, s0, 1);
                s1 += __shfl_xor_sync(FULL, s1, 1);
                s0 += __shfl_xor_sync(FULL, s0, 2);
                s1 += __shfl_xor_sync(FULL, s1, 2);
                sc[mt][0] = s0;   // chunk 16*mt + r4
                sc[mt][1] = s1;   // chunk 16*mt + r4 + 8
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar.empty[s]);   // the stage may be refilled
            // two offers of 32 chunks: chunk 32h + L sits in m-tile 2h + L/16, half (L/8)&1, quad L%8.
            // A candidate below another warp's k-th best for this row cannot make the row's top k.
            const int rs = (int)(cur - r_lo);
            const float floor = (rs >= 0 && rs < RMAX) ? ord_dec(*(volatile unsigned *)&s_floor[rs]) : -INFINITY;
            const int src = 4 * (lane & 7);
#pragma unroll
            for (int h = 0; h < TCH / 32; ++h) {
                const float x0 = __shfl_sync(FULL, sc[2 * h][0], src), x1 = __shfl_sync(FULL, sc[2 * h][1], src);
                const float x2 = __shfl_sync(FULL, sc[2 * h + 1][0], src), x3 = __shfl_sync(FULL, sc[2 * h + 1][1], src);
                const float mine = lane < 16 ? (lane < 8 ? x0 : x1) : (lane < 24 ? x2 : x3);
                const int c = kt * TCH + 32 * h + lane;
                list_offer16(v, id, mine, c, c < a.ncand, a.kmax, lane, floor);
            }
            // publish this list's k-th best once it holds k entries
            const float vk = __shfl_sync(FULL, v, a.kmax - 1);
            if (lane == 0 && vk != -INFINITY && rs >= 0 && rs < RMAX) atomicMax(&s_floor[rs], ord_enc(vk));
        }
        if (cur >= 0 && lane < 16 && in_range(cur - r_lo, RMAX, a.status))
            wl[cur - r_lo][warp][lane] = make_float2(v, __int_as_float(id));
    }
    __syncthreads();

    // ---- per row slot: merge the consumer warps' lists, publish the CTA's list;
    // the CTA that completes the row merges the row's lists and writes the row
    auto finish_row = [&]() {
        if (ntile == 0 || bar.abort) return;
        const int nrows = (int)((hi - 1) / a.tpr - r_lo + 1);
        if (warp >= nrows || !in_range(warp, RMAX, a.status)) return;
        const long long row = r_lo + warp;
        float v = lane < 16 ? wl[warp][0][lane].x : -INFINITY;
        int id = lane < 16 ? __float_as_int(wl[warp][0][lane].y) : INT32_MAX;
        if (lane >= a.kmax) {
            v = -INFINITY;
            id = INT32_MAX;
        }
        for (int w2 = 1; w2 < NCW; ++w2) {
            const float2 e = lane < 16 ? wl[warp][w2][lane] : make_float2(-INFINITY, __int_as_float(INT32_MAX));
            list_merge16(v, id, e.x, __float_as_int(e.y), a.kmax, lane);
        }
        const long long T0 = row * a.tpr;
        const int x0 = cta_of(a, T0), x1 = cta_of(a, T0 + a.tpr - 1);
        float2 *rl = lists + row * (long long)a.maxe * a.kmax;
        if (!in_range(x - x0, a.maxe, a.status) || !in_range(x1 - x0, a.maxe, a.status)) return;
        if (lane < a.kmax) rl[(x - x0) * a.kmax + lane] = make_float2(v, __int_as_float(id));
        __threadfence();
        int last = 0;
        if (lane == 0) last = atomicAdd(&cnt[row], 1) == x1 - x0;
        if (!__shfl_sync(FULL, last, 0)) return;
        __threadfence();
        list_init(v, id);
        // the row's lists, eight in flight per round trip (then merged in order)
        const int ne = x1 - x0 + 1;
        for (int e0 = 0; e0 < ne; e0 += 8) {
            float2 f[8];
#pragma unroll
            for (int u = 0; u < 8; ++u)
                f[u] = (e0 + u < ne && lane < a.kmax) ? __ldcg(rl + (e0 + u) * a.kmax + lane)
                                                      : make_float2(-INFINITY, __int_as_float(INT32_MAX));
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (e0 + u < ne) list_merge16(v, id, f[u].x, __float_as_int(f[u].y), a.kmax, lane);
        }
        const int ke = list_keff(v, a.ncand, a.k, a.kmax, a.tau);
        if (lane < a.kmax) {
            idx[row * a.kmax + lane] = lane < ke ? id : -1;
            score[row * a.kmax + lane] = lane < ke ? v : -INFINITY;
        }
        if (lane == 0) keff[row] = ke;
        if constexpr (FUSE) {
            // publish each slot's unit: its chunk and its fusion weight (softmax of the kept scores)
            const float m = __shfl_sync(FULL, v, 0);   // the list is sorted: the row's best score
            const float ex = lane < ke ? expf(v - m) : 0.f;
            const float w = ex / warp_sum(ex);
            if (lane < a.kmax)
                st_release_gpu64(&a.desc[row * a.kmax + lane],
                                 lane < ke ? ((unsigned long long)(uint32_t)(id + 1) << 32) | __float_as_uint(w)
                                           : EMPTY_SLOT);
        }
    };
    finish_row();
    if constexpr (FUSE) {
        // the ring and the lists are free: they become the gather stages (TMA
        // writes after this CTA's generic accesses to the same shared memory)
        fence_proxy_async_smem();
        __syncthreads();
        gather_phase<D, S>(a, base, gbar, &bar.abort, tmK, tmV, Q);
    }
}

}  // namespace

// Decode-shaped problems (one query per sequence) with long contexts.
bool select_stream_supported(const Prob &p) {
    const long long ncand = std::min<long long>(p.q_pos0 / p.S, p.C);
    return p.dtype == HSA_BF16 && (p.d == 64 || p.d == 128) && p.Tq == 1 && p.G <= 8 && p.kmax <= 16 &&
           ncand >= 2048 && (long long)p.B * p.Hkv * p.Lc < (1ll << 31);
}

// Grid and list slots of the stream scan (also sizes its workspace).
void select_stream_shape(const Prob &p, int sms, int *grid, int *maxe) {
    const long long ncand = std::min<long long>(p.q_pos0 / p.S, p.C);
    const long long tpr = (ncand + TCH - 1) / TCH, total = p.rows * tpr;
    long long g = sms;
    // a CTA's range may touch at most RMAX rows: at most (RMAX - 1) * tpr + 1 tiles
    const long long need = (total + (RMAX - 1) * tpr) / ((RMAX - 1) * tpr + 1);
    if (g < need) g = need;
    if (g > total) g = total;
    const long long minn = total / g;   // tiles of the smallest range (>= 1)
    long long e = tpr / minn + 2;
    if (e > g) e = g;
    *grid = (int)g;
    *maxe = (int)e;
}

static StreamArgs stream_args(const Prob &p, uint32_t *status, int grid, int maxe) {
    StreamArgs a{};
    a.Tq = p.Tq;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.S = p.S;
    a.C = p.C;
    a.Lc = p.Lc;
    a.k = p.k;
    a.kmax = p.kmax;
    a.ncand = (int)std::min<long long>(p.q_pos0 / p.S, p.C);
    a.tpr = (a.ncand + TCH - 1) / TCH;
    a.rows = (int)p.rows;
    a.total = p.rows * (long long)a.tpr;
    a.grid = grid;
    a.maxe = maxe;
    a.tau = p.tau;
    a.status = status;
    return a;
}

static size_t ring_smem(int d) { return 1024 + (size_t)NST * (d / 64) * TCH * 128 + WL_BYTES; }

cudaError_t launch_select_stream(const Prob &p, const void *Q, const void *L, int32_t *idx, float *score,
                                 int32_t *keff, float2 *lists, int32_t *cnt, uint32_t *status, int grid, int maxe,
                                 cudaStream_t st) {
    StreamArgs a = stream_args(p, status, grid, maxe);
    CUtensorMap ml;
    cudaError_t e = make_tmap_2d(&ml, L, (uint64_t)p.d, (uint64_t)p.B * p.Hkv * p.Lc, 64, TCH);
    if (e != cudaSuccess) return e;
    const size_t smem = ring_smem(p.d);
    // the K/V map arguments are unused without the gather phase
    if (p.d == 128) {
        if ((e = cudaFuncSetAttribute(select_stream_kernel<128, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        select_stream_kernel<128, 0><<<grid, (NCW + 1) * 32, smem, st>>>(ml, ml, ml, (const __nv_bfloat16 *)Q, lists,
                                                                         idx, score, keff, cnt, a);
    } else {
        if ((e = cudaFuncSetAttribute(select_stream_kernel<64, 0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)smem)) != cudaSuccess)
            return e;
        select_stream_kernel<64, 0><<<grid, (NCW + 1) * 32, smem, st>>>(ml, ml, ml, (const __nv_bfloat16 *)Q, lists,
                                                                        idx, score, keff, cnt, a);
    }
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------- fused decode step

bool decode_fused_supported(const Prob &p, int grid, int sms) {
    // one CTA per SM (the ring's shared memory), all resident at once
    return select_stream_supported(p) && !(p.flags & HSA_FLAG_QUEST) && grid <= sms && p.rows * p.kmax < (1ll << 31);
}

template <int D, int S>
static cudaError_t launch_fused_ds(StreamArgs a, const CUtensorMap &ml, const CUtensorMap &mk, const CUtensorMap &mv,
                                   const void *Q, float2 *lists, int32_t *idx, float *score, int32_t *keff,
                                   int32_t *cnt, cudaStream_t st) {
    auto kern = select_stream_kernel<D, S>;
    cudaError_t e;
    int dev = 0, optin = 0;
    cudaFuncAttributes fa;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    constexpr size_t STAGE = gather_stage_bytes<D, S>();
    const long long room = (long long)optin - (long long)fa.sharedSizeBytes - 1024;
    int nwg = (int)std::min<long long>(NCW + 1, room / (long long)STAGE);
    if (nwg < 1) return cudaErrorInvalidConfiguration;
    a.nwg = nwg;
    const size_t smem = std::max(ring_smem(D), 1024 + (size_t)nwg * STAGE);
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    const __nv_bfloat16 *q = (const __nv_bfloat16 *)Q;
    void *args[] = {(void *)&ml, (void *)&mk, (void *)&mv, (void *)&q, (void *)&lists, (void *)&idx,
                    (void *)&score, (void *)&keff, (void *)&cnt, (void *)&a};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)a.grid);
    cfg.blockDim = dim3((NCW + 1) * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: gather workers wait on other CTAs' rows
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, reinterpret_cast<const void *>(kern), args);
}

cudaError_t launch_decode_fused(const Prob &p, const void *Q, const void *K, const void *V, const void *L,
                                int32_t *idx, float *score, int32_t *keff, void *O, float2 *lists, int32_t *cnt,
                                unsigned long long *desc, int32_t *ctr, int32_t *att_cnt, float *acc, uint32_t *status,
                                int grid, int maxe, cudaStream_t st) {
    StreamArgs a = stream_args(p, status, grid, maxe);
    a.B = p.B;
    a.Tcap = p.Tcap;
    a.nunits = (int)(p.rows * p.kmax);
    a.scale = 1.0f / sqrtf((float)p.d);
    a.desc = desc;
    a.ctr = ctr;
    a.att_cnt = att_cnt;
    a.acc = acc;
    a.O = (__nv_bfloat16 *)O;
    CUtensorMap ml, mk, mv;
    cudaError_t e = make_tmap_2d(&ml, L, (uint64_t)p.d, (uint64_t)p.B * p.Hkv * p.Lc, 64, TCH);
    if (e != cudaSuccess) return e;
    // K and V as 3D (d, Hkv, B*Tcap): box (64, 1, S) = S rows of 128 bytes, 128-byte swizzle
    const uint64_t dims[3] = {(uint64_t)p.d, (uint64_t)p.Hkv, (uint64_t)p.B * p.Tcap};
    const uint64_t strides[2] = {(uint64_t)p.d * 2, (uint64_t)p.Hkv * p.d * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)p.S};
    if ((e = make_tmap_3d(&mk, K, dims, strides, box)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, V, dims, strides, box)) != cudaSuccess) return e;
#define HSA_FUSED(D_, S_)                                                                                   \
    if (p.d == D_ && p.S == S_) return launch_fused_ds<D_, S_>(a, ml, mk, mv, Q, lists, idx, score, keff, cnt, st);
    HSA_FUSED(128, 64)
    HSA_FUSED(128, 32)
    HSA_FUSED(128, 128)
    HSA_FUSED(64, 64)
    HSA_FUSED(64, 32)
    HSA_FUSED(64, 128)
#undef HSA_FUSED
    return cudaErrorInvalidValue;
}

}  // namespace hsa
