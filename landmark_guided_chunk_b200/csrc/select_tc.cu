// select_tc.cu -- causal landmark scoring on the tcgen05 tensor cores, fused
// with the per-row top-k and the gap router (HSA summary page, Core Technique
// and Implementation: score every landmark of the strictly-past chunks, keep
// the k best; value-of-information router page: double k on a near-tied cut).
//
// For one (batch b, kv head j) the group score of query row t and chunk c is
//     s[t][c] = sum_{h in group j} q_h[t] . L[c]  =  A[t] . Bcat[c]
// with A[t] = the G*d contiguous values Q[b][t][jG..jG+G-1][:] and Bcat[c] =
// L[c] repeated G times.  So it is one bf16 GEMM with K = G*d, accumulated
// in fp32 in TMEM, and the group sum comes out exact up to fp32 rounding.
// Since B repeats, only the d/64 distinct 64-column blocks of L are staged.
//
// Persistent CTAs walk 128-token M-tiles, heaviest (latest) first.  A tile's
// rows have at most nc_max = floor((q_pos0 + t_last)/S) candidates, so only
// ceil(nc_max/128) N-slices of 128 chunks are computed.  The causal triangle
// is skipped at slice granularity, and the last slice's N is trimmed to a
// multiple of 16.
//
//   warp 0      TMA producer: the A tile (G*d/64 boxes of 128 rows x 64 cols)
//               once per tile, each box reloaded for the next tile as soon as
//               the last slice's MMAs have read it; L slices into a 2-stage ring
//   warp 1      MMA issuer: 4*G*d/64 tcgen05.mma (M128, N<=128, K16) per slice
//               into one of two TMEM accumulators
//   warp 2      TMEM allocator (256 columns)
//   warps 4..7  epilogue: thread = row.  tcgen05.ld 16 scores at a time.
//               Scores of candidate chunks (c < ncand(t)) that beat the
//               row's current k-th best are appended to the row's FIFO (a
//               ring of 32 entries in shared memory, predicated stores).
//               The warp then pops entries in lock-step into sorted register
//               lists (score desc, chunk asc): as many pops as the warp's mean
//               FIFO length, and more if a FIFO could overflow on the next 16
//               columns; everything at the row's end.  Draining by the mean
//               rather than the longest FIFO keeps most lanes busy; an entry
//               that went stale while queued is a no-op push.  Chunks arrive
//               in increasing order, so an entry that equals a listed score
//               goes behind it, which keeps ties on the lower index.
//               The accumulator is released as soon as its last columns are
//               in registers, before that chunk's pops.
#include "common.cuh"
#include "sm100.cuh"

namespace hsa {
namespace {

using namespace sm100;

constexpr int TM = 128;        // tokens per M-tile
constexpr int NSTAGE = 2;      // L-slice ring depth
constexpr int BOX = 64 * 128 * 2;   // one 64-column x 128-row bf16 box of the query tile (16 KB)
constexpr int MAX_KB = 8;      // G*d <= 512
// Chunks per N-slice (NT): 128, or 64 when a landmark row has 256 columns, so
// that the query tile and two slices still fit in shared memory.
constexpr uint64_t TEST_STALL_WAIT_NS = 100000ull;   // wait limit under HSA_FLAG_TEST_STALL (0.1 ms)

struct TcSelArgs {
    int B, Tq, Hkv, G, d, S, C, k, kmax;
    int Lc;                  // chunks per (b, kv head) in L's layout
    int nkb, dkb;            // G*d/64 and d/64
    int mtiles, ntiles;
    long long q_pos0;
    float tau;
    uint32_t *status;
    uint64_t wait_ns;        // limit of every bounded wait
    int stall;               // test hook: the epilogue first waits on a barrier nothing arrives on
};

struct __align__(8) Bars {
    uint64_t a_full[MAX_KB], a_empty[MAX_KB], done, never;
    uint64_t b_full[NSTAGE], b_empty[NSTAGE];
    uint64_t t_full[2], t_empty[2];
    uint32_t tmem_base;
    int abort;
};

struct Tile {
    int b, j, t0, nc_max, nslices;
};

template <int NT>
__device__ __forceinline__ Tile tile_of(const TcSelArgs &a, int tau) {
    Tile T;
    const int bh = a.B * a.Hkv;
    const int mt = a.mtiles - 1 - tau / bh;   // latest (heaviest) tiles first
    const int r = tau % bh;
    T.b = r / a.Hkv;
    T.j = r % a.Hkv;
    T.t0 = mt * TM;
    const int t_last = min(T.t0 + TM - 1, a.Tq - 1);
    long long nc = (a.q_pos0 + t_last) / a.S;
    T.nc_max = (int)(nc < a.C ? nc : a.C);
    T.nslices = (T.nc_max + NT - 1) / NT;
    return T;
}

template <int NT>
__device__ __forceinline__ int slice_n(const Tile &T, int n) {
    int w = min(NT, T.nc_max - n * NT);
    return (w + 15) & ~15;
}

// Insert (x, xi) into the sorted list; xi is larger than every chunk index
// already present, so equal scores already in the list stay ahead of it.
// Entry q keeps its value when v[q] >= x; otherwise it takes x if v[q-1] >= x
// (x lands at q) and v[q-1] otherwise (shifted down).  Going from the tail up,
// v[q-1] still holds its old value when entry q reads it.  x = -inf changes nothing.
template <int KL>
__device__ __forceinline__ void list_push(float (&v)[KL], int (&id)[KL], float x, int xi) {
#pragma unroll
    for (int q = KL - 1; q >= 1; --q) {
        const bool keep = v[q] >= x, here = v[q - 1] >= x;
        v[q] = keep ? v[q] : (here ? x : v[q - 1]);
        id[q] = keep ? id[q] : (here ? xi : id[q - 1]);
    }
    const bool keep0 = v[0] >= x;
    v[0] = keep0 ? v[0] : x;
    id[0] = keep0 ? id[0] : xi;
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

template <int KL, int NT>
__global__ void __launch_bounds__(256, 1)
    select_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmL,
                     int32_t *__restrict__ idx, float *__restrict__ score, int32_t *__restrict__ keff, TcSelArgs a) {
    constexpr int BOXB = 64 * NT * 2;                     // one 64-column x NT-row box of a landmark slice
    constexpr uint32_t TMEM_COLS = 2 * NT;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = base;                                   // nkb boxes
    uint8_t *sB = base + (size_t)a.nkb * BOX;             // NSTAGE x dkb boxes
    // [32][128] queued (score, chunk as int bits): one 8-byte store per queued candidate
    float2 *qvi = reinterpret_cast<float2 *>(sB + (size_t)NSTAGE * a.dkb * BOXB);
    Bars *bar = reinterpret_cast<Bars *>(qvi + 32 * 128);
    volatile int *abort = &bar->abort;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int kb = 0; kb < MAX_KB; ++kb) {
            mbar_init(&bar->a_full[kb], 1);
            mbar_init(&bar->a_empty[kb], 1);
        }
        mbar_init(&bar->done, 1);
        mbar_init(&bar->never, 1);
        for (int s = 0; s < NSTAGE; ++s) {
            mbar_init(&bar->b_full[s], 1);
            mbar_init(&bar->b_empty[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar->t_full[s], 1);
            mbar_init(&bar->t_empty[s], 4);
        }
        bar->abort = 0;
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(&bar->tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQ);
        prefetch_tmap(&tmL);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            int g = 0, ta = 0, kb_part = 0;   // kb_part: boxes issued of a tile cut short
            bool ok = true;
            for (int tau = blockIdx.x; tau < a.ntiles && ok; tau += gridDim.x) {
                const Tile T = tile_of<NT>(a, tau);
                if (T.nslices == 0) continue;
                const int y = (int)dbg_clamp(T.b * a.Tq + T.t0, 0, (long long)a.B * a.Tq, a.status);   // query row
                const int qj = (int)dbg_clamp(T.j, 0, a.Hkv, a.status);
                for (int kb = 0; kb < a.nkb; ++kb) {
                    if (ta > 0 && !(ok = mbar_wait(&bar->a_empty[kb], (ta - 1) & 1, abort, a.status, a.wait_ns))) break;
                    mbar_expect_tx(&bar->a_full[kb], (uint32_t)BOX);
                    tma_load_2d(sA + (size_t)kb * BOX, &tmQ, qj * a.G * a.d + kb * 64, y, &bar->a_full[kb]);
                    kb_part = kb + 1;
                }
                if (!ok) break;
                ++ta;
                kb_part = 0;
                const int ly = (T.b * a.Hkv + qj) * a.Lc;   // the (b, kv head) landmark list
                for (int n = 0; n < T.nslices; ++n, ++g) {
                    const int s = g % NSTAGE, i = g / NSTAGE;
                    if (i > 0 && !(ok = mbar_wait(&bar->b_empty[s], (i - 1) & 1, abort, a.status, a.wait_ns))) break;
                    mbar_expect_tx(&bar->b_full[s], (uint32_t)(a.dkb * BOXB));
                    for (int kd = 0; kd < a.dkb; ++kd)
                        tma_load_2d(sB + (size_t)(s * a.dkb + kd) * BOXB, &tmL, kd * 64,
                                    ly + (int)dbg_clamp(n * NT, 0, a.C, a.status), &bar->b_full[s]);
                }
            }
            // wind down: every load issued has landed before the CTA may exit
            for (int kb = 0; kb < a.nkb; ++kb) {
                const int nload = ta + (kb < kb_part ? 1 : 0);   // loads issued into box kb
                if (nload > 0) mbar_drain(&bar->a_full[kb], (nload - 1) & 1);
            }
            for (int s = 0; s < NSTAGE && s < g; ++s) {
                const int last = (g - 1 - s) / NSTAGE;   // index of the last use of stage s
                mbar_drain(&bar->b_full[s], last & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int g = 0, ta = 0;
            bool ok = true;
            for (int tau = blockIdx.x; tau < a.ntiles && ok; tau += gridDim.x) {
                const Tile T = tile_of<NT>(a, tau);
                if (T.nslices == 0) continue;
                const uint32_t pa = ta & 1;
                ++ta;
                for (int n = 0; n < T.nslices && ok; ++n, ++g) {
                    const int s = g % NSTAGE, i = g / NSTAGE, buf = g & 1, u = g >> 1;
                    if (!(ok = mbar_wait(&bar->b_full[s], i & 1, abort, a.status, a.wait_ns))) break;
                    if (u > 0 && !(ok = mbar_wait(&bar->t_empty[buf], (u - 1) & 1, abort, a.status, a.wait_ns))) break;
                    tc_fence_after();
                    const uint32_t idesc = idesc_bf16_f32(TM, slice_n<NT>(T, n), 0, 0);
                    const uint32_t d_tmem = tmem + (uint32_t)(buf * NT);
                    const uint32_t aBase = smem_u32(sA), bBase = smem_u32(sB + (size_t)s * a.dkb * BOXB);
                    const bool last = n == T.nslices - 1;
                    for (int kb = 0; kb < a.nkb; ++kb) {
                        if (n == 0) {
                            if (!(ok = mbar_wait(&bar->a_full[kb], pa, abort, a.status, a.wait_ns))) break;
                            tc_fence_after();
                        }
                        const uint32_t aK = aBase + kb * BOX, bK = bBase + (kb % a.dkb) * BOXB;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_bf16(d_tmem, desc_kmajor_sw128(aK + kk * 32), desc_kmajor_sw128(bK + kk * 32), idesc,
                                      (kb | kk) != 0);
                        if (last) umma_commit(&bar->a_empty[kb]);   // box kb may be refilled
                    }
                    if (!ok) break;
                    umma_commit(&bar->b_empty[s]);
                    umma_commit(&bar->t_full[buf]);
                }
            }
            umma_commit(&bar->done);
            mbar_drain(&bar->done, 0);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------ epilogue: thread = row
        const int ew = warp - 4;
        const int r = ew * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(ew * 32) << 16);
        int g = 0;
        // test hook: a wait that runs out (nothing arrives on `never`), so the
        // expiry, abort and wind-down of every role run as they would on a stall
        bool ok = !a.stall || mbar_wait(&bar->never, 0, abort, a.status, a.wait_ns);
        for (int tau = blockIdx.x; tau < a.ntiles && ok; tau += gridDim.x) {
            const Tile T = tile_of<NT>(a, tau);
            const int t = T.t0 + r;
            const bool valid = t < a.Tq;
            int nc = 0;
            if (valid) {
                long long x = (a.q_pos0 + t) / a.S;
                nc = (int)(x < a.C ? x : a.C);
            }
            float v[KL];
            int id[KL];
#pragma unroll
            for (int q = 0; q < KL; ++q) {
                v[q] = -INFINITY;
                id[q] = -1;
            }
            int head = 0, tail = 0;   // this row's FIFO of pending (score, chunk): ring of 32 in qvi
            for (int n = 0; n < T.nslices; ++n, ++g) {
                const int buf = g & 1, u = g >> 1;
                if (!(ok = mbar_wait(&bar->t_full[buf], u & 1, abort, a.status, a.wait_ns))) break;
                tc_fence_after();
                const int nch = slice_n<NT>(T, n) / 16;
                const bool last_slice = n == T.nslices - 1;
                for (int q = 0; q < nch; ++q) {
                    uint32_t rr[16];
                    tmem_ld16(lane_base + (uint32_t)(buf * NT + q * 16), rr);
                    tmem_wait_ld();
                    if (q == nch - 1) {   // the accumulator may be overwritten from here on
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&bar->t_empty[buf]);
                    }
                    const int cb = n * NT + q * 16;
                    const float thr = v[KL - 1];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float sv = __uint_as_float(rr[e]);
                        const bool take = (cb + e < nc) && (sv > thr);
                        const int slot = (tail & 31) * 128 + r;
                        if (take) {
                            qvi[slot] = make_float2(sv, __int_as_float(cb + e));
                        }
                        tail += take ? 1 : 0;
                    }
                    const int len = tail - head;
                    const int mx = (int)__reduce_max_sync(FULL, (unsigned)len);
                    int dn = mx;
                    if (!(last_slice && q == nch - 1)) {
                        const int sum = (int)__reduce_add_sync(FULL, (unsigned)len);
                        dn = max((sum + 31) >> 5, mx - 16);   // leaves room for the next 16 columns
                    }
                    for (int it = 0; it < dn; ++it) {
                        const bool has = head < tail;
                        const int slot = (head & 31) * 128 + r;
                        const float2 qe = has ? qvi[slot] : make_float2(-INFINITY, 0.f);
                        const float x = qe.x;
                        const int xi = __float_as_int(qe.y);
                        head += has ? 1 : 0;
                        list_push<KL>(v, id, x, xi);
                    }
                }
            }
            if (!ok || !valid) continue;
            int ke = nc < a.k ? nc : a.k;
            if (a.tau > 0.f && nc > a.k) {
                // entries k-1 and k (k < kmax <= KL) through this thread's column of the
                // drained queue: selecting them from registers by a runtime index would
                // move the whole list into local memory
#pragma unroll
                for (int q = 0; q < KL; ++q) qvi[q * 128 + r].x = v[q];
                const float sk = qvi[(a.k - 1) * 128 + r].x, sk1 = qvi[a.k * 128 + r].x;
                if (sk - sk1 < a.tau * fabsf(sk)) ke = nc < 2 * a.k ? nc : 2 * a.k;
            }
            const long long row = ((long long)T.b * a.Tq + t) * a.Hkv + T.j;
            int32_t *oi = idx + row * a.kmax;
            float *os = score + row * a.kmax;
#pragma unroll
            for (int q = 0; q < KL; ++q) {
                if (q < a.kmax) {
                    oi[q] = q < ke ? id[q] : -1;
                    os[q] = q < ke ? v[q] : -INFINITY;
                }
            }
            keff[row] = ke;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

template <int KL, int NT>
cudaError_t launch_kl(const TcSelArgs &a, const CUtensorMap &mq, const CUtensorMap &ml, int32_t *idx, float *score,
                      int32_t *keff, int grid, size_t smem, cudaStream_t st) {
    cudaError_t e =
        cudaFuncSetAttribute(select_tc_kernel<KL, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    select_tc_kernel<KL, NT><<<grid, 256, smem, st>>>(mq, ml, idx, score, keff, a);
    return cudaGetLastError();
}

template <int NT>
cudaError_t launch_nt(const Prob &p, const TcSelArgs &a, const CUtensorMap &mq, const CUtensorMap &ml, int32_t *idx,
                      float *score, int32_t *keff, int grid, cudaStream_t st) {
    const size_t smem =
        1024 + (size_t)a.nkb * BOX + (size_t)NSTAGE * a.dkb * (64 * NT * 2) + 2 * 32 * 128 * 4 + sizeof(Bars);
    if (p.kmax <= 8) return launch_kl<8, NT>(a, mq, ml, idx, score, keff, grid, smem, st);
    if (p.kmax <= 16) return launch_kl<16, NT>(a, mq, ml, idx, score, keff, grid, smem, st);
    return launch_kl<32, NT>(a, mq, ml, idx, score, keff, grid, smem, st);
}

}  // namespace

bool select_tc_supported(const Prob &p) {
    const int gd = p.G * p.d;
    return p.dtype == HSA_BF16 && (p.d == 64 || p.d == 128 || p.d == 256) && gd % 64 == 0 && gd <= 512 &&
           p.Tq >= 64 && p.C >= 1 && p.kmax <= 32;
}

cudaError_t launch_select_tc(const Prob &p, const void *Q, const void *L, int32_t *idx, float *score, int32_t *keff,
                             uint32_t *status, cudaStream_t st) {
    CUtensorMap mq, ml;
    cudaError_t e = make_tmap_2d(&mq, Q, (uint64_t)p.H * p.d, (uint64_t)p.B * p.Tq, 64, TM);
    if (e != cudaSuccess) return e;
    const int nt = p.d > 128 ? 64 : 128;   // chunks per N-slice
    e = make_tmap_2d(&ml, L, (uint64_t)p.d, (uint64_t)p.B * p.Hkv * p.Lc, 64, (uint32_t)nt);
    if (e != cudaSuccess) return e;
    TcSelArgs a;
    a.B = p.B;
    a.Tq = p.Tq;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.d = p.d;
    a.S = p.S;
    a.C = p.C;
    a.Lc = p.Lc;
    a.k = p.k;
    a.kmax = p.kmax;
    a.nkb = p.G * p.d / 64;
    a.dkb = p.d / 64;
    a.mtiles = (p.Tq + TM - 1) / TM;
    a.ntiles = p.B * p.Hkv * a.mtiles;
    a.q_pos0 = p.q_pos0;
    a.tau = p.tau;
    a.status = status;
    a.stall = (p.flags & HSA_FLAG_TEST_STALL) ? 1 : 0;
    a.wait_ns = a.stall ? TEST_STALL_WAIT_NS : WAIT_LIMIT_NS;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int grid = a.ntiles < sms ? a.ntiles : sms;
    if (nt == 64) return launch_nt<64>(p, a, mq, ml, idx, score, keff, grid, st);
    return launch_nt<128>(p, a, mq, ml, idx, score, keff, grid, st);
}

}  // namespace hsa
