// attend_tc.cu -- chunk attention + retrieval-weighted fusion on the tcgen05
// tensor cores, chunk-major (HSA summary page, Implementation: attend to each
// selected chunk with standard attention, fuse the chunk outputs weighted by
// the softmax of their retrieval scores).
//
// With random selections neighbouring queries share almost no chunks, so a
// query-major schedule would stream k*S keys per query from memory.  Here
// the selection is inverted instead: for every (kv head, chunk) we list the
// (token, slot) pairs that kept it, so K_c and V_c are loaded once per tile of
// up to TOK = 128/G tokens.  The G heads of each token form the 128-row M
// operand:
//     S  = Q_tile . K_c^T / sqrt(d)        tcgen05, M128 x N=S x K=d, TMEM
//     P  = exp(S - rowmax), l = sum P      softmax warps, P -> smem (bf16)
//     O  = P . V_c                          tcgen05, M128 x N=d x K=S, TMEM
//     O_acc[t][h] += (w_slot / l) * O       O-drain warps, fp32 vector reductions (red.v4)
// The kernel is a template on the head dim (D = 64 or 128).  Roles (16 warps,
// 4 per SM sub-partition so each may hold 128 registers): two producer warps
// gather the tile's Q rows (cp.async; for D = 128 through a per-warp table of
// row addresses, so that each 8-lane group copies one whole 128-byte line),
// one loader warp issues the K/V TMA loads, one thread issues the MMAs, four
// softmax warps (one per TMEM lane quadrant) and eight O-drain warps (two per
// quadrant, D/2 columns each) take every tile.  S, P and O are double-buffered
// by tile parity, so the drain of tile i overlaps the softmax of tile i+1 and
// the QK product of tile i+2.
// Since w is known before the attention, the cross-chunk fusion is linear and
// needs no rescaling.
//
// Accumulators.  The pairs are grouped into phases of TB tokens of one (b, kv
// head), and the tiles are ordered phase-major.  The phases are processed in
// batches of NB, one kernel launch per batch.  A batch reduces into NB
// accumulator slots of a ring of 2*NB, which stays resident in L2.  Launch
// beta first finalises batch beta-1 (its slots -> bf16 O, slots zeroed).  Every
// warp of every CTA takes a share of that, and then the CTA moves on to the
// tiles of batch beta, whose slots differ.  The kernel boundary is the only
// synchronisation, so no CTA ever waits for another.
//
// Helper kernels (before the batches): count pairs per (phase, chunk) bucket;
// two-level exclusive scan of pair and tile counts; tile list; scatter of the
// pairs, each with its fusion weight, into their buckets.
#include "common.cuh"
#include "sm100.cuh"

namespace hsa {

namespace {

using namespace sm100;

constexpr int MROWS = 128;       // M of every tile (TOK tokens x G heads)
constexpr int SCAN_BLK = 4096;   // elements per first-level scan block
constexpr int PITCH = 36;        // staging row pitch (floats) for a 32-column slice
constexpr int TB = 16384;        // tokens per phase (larger phases fill the per-chunk tiles better; a multiple of HT)
constexpr int NB = 1;            // phases per batch (= per launch)
constexpr int NT_ATT = 512;      // warps 0-1 Q producers, 2 MMA, 3 K/V loader, 4-7 softmax, 8-15 O drain
constexpr int NPROD = 64;        // producer threads (two tile rows each)

struct AttTcArgs {
    int B, Tq, Tcap, H, Hkv, G, S, C, kmax, tok;
    int ntb, nphase, nbucket, nsq, nskv;
    int batch;                   // batch processed by this launch (== nbatch: finalise only)
    int nbatch;
    long long q_pos0;
    float scale_log2;            // log2(e) / sqrt(d)
    const int32_t *idx;
    const float *score;
    const int32_t *keff;
    float *w8;                   // [rows][kmax] fusion weights (per-pair-atomics path only)
    int32_t *bcount, *bcursor;   // [nbucket]
    int32_t *boff, *btile;       // [nbucket + 1]
    int32_t *blk;                // [2 * nblk] first-level block totals
    int2 *pairs;                 // [rows * kmax]  ((t << 5) | slot, bits of the pair's fusion weight), bucketed
    int4 *tiles;                 // (phase, chunk, first pair, pairs in tile)
    float *ringbuf;              // [2*NB][TB][G][d]
    int d;                       // head dim (64 or 128)
    uint32_t *status;
};

__device__ __forceinline__ int ncand_of(const AttTcArgs &a, int t) {
    long long n = (a.q_pos0 + t) / a.S;
    return (int)(n < a.C ? n : a.C);
}

__device__ __forceinline__ int phase_of(const AttTcArgs &a, int b, int j, int t) {
    return (b * a.Hkv + j) * a.ntb + t / TB;
}

// ring slot of phase p
__device__ __forceinline__ float *slot_of(const AttTcArgs &a, int p) {   // accumulator rows of d floats
    const int s = ((p / NB) & 1) * NB + (p % NB);
    return a.ringbuf + (size_t)s * TB * a.G * a.d;
}

// ---------------------------------------------------------------------------- helper kernels

// One thread per selection row: fusion weights and bucket counts.
__global__ void att_count_kernel(AttTcArgs a) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long rows = (long long)a.B * a.Tq * a.Hkv;
    if (row >= rows) return;
    const int j = (int)(row % a.Hkv);
    const long long bt = row / a.Hkv;
    const int t = (int)(bt % a.Tq), b = (int)(bt / a.Tq);
    int ke = a.keff[row];
    if (ke < 0 || ke > a.kmax) {
        atomicOr(a.status, DEV_BAD_INDEX);
        ke = ke < 0 ? 0 : a.kmax;
    }
    const int nc = ncand_of(a, t);
    const int p = phase_of(a, b, j, t);
    const int32_t *ri = a.idx + row * a.kmax;
    const float *rs = a.score + row * a.kmax;
    float m = -INFINITY;
    for (int i = 0; i < ke; ++i) m = fmaxf(m, rs[i]);
    float z = 0.f;
    for (int i = 0; i < ke; ++i) z += expf(rs[i] - m);
    for (int i = 0; i < ke; ++i) {
        a.w8[row * a.kmax + i] = expf(rs[i] - m) / z;
        const int c = ri[i];
        if (c < 0 || c >= nc) {
            atomicOr(a.status, DEV_BAD_INDEX);
            continue;
        }
        atomicAdd(&a.bcount[(long long)p * a.C + c], 1);
    }
}

// First level of the scan: per block of SCAN_BLK buckets, local exclusive
// prefixes of pair counts (boff) and tile counts (btile), plus block totals.
__global__ void __launch_bounds__(1024) att_scan1_kernel(AttTcArgs a) {
    __shared__ int sp[1024], st[1024];
    const int base = blockIdx.x * SCAN_BLK + threadIdx.x * 4;
    int np[4], nt[4], sp_, st_;
    sp_ = st_ = 0;
    for (int q = 0; q < 4; ++q) {
        const int u = base + q;
        const int n = u < a.nbucket ? a.bcount[u] : 0;
        np[q] = n;
        nt[q] = (n + a.tok - 1) / a.tok;
        sp_ += np[q];
        st_ += nt[q];
    }
    sp[threadIdx.x] = sp_;
    st[threadIdx.x] = st_;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {   // Hillis-Steele inclusive scan
        int vp = threadIdx.x >= o ? sp[threadIdx.x - o] : 0;
        int vt = threadIdx.x >= o ? st[threadIdx.x - o] : 0;
        __syncthreads();
        sp[threadIdx.x] += vp;
        st[threadIdx.x] += vt;
        __syncthreads();
    }
    int ep = sp[threadIdx.x] - sp_, et = st[threadIdx.x] - st_;
    for (int q = 0; q < 4; ++q) {
        const int u = base + q;
        if (u < a.nbucket) {
            a.boff[u] = ep;
            a.btile[u] = et;
        }
        ep += np[q];
        et += nt[q];
    }
    if (threadIdx.x == 1023) {
        a.blk[2 * blockIdx.x] = sp[1023];
        a.blk[2 * blockIdx.x + 1] = st[1023];
    }
}

// Second level: exclusive scan of the block totals (one block, <= 1024 blocks).
__global__ void __launch_bounds__(1024) att_scan2_kernel(AttTcArgs a, int nblk) {
    __shared__ int sp[1024], st[1024];
    const int i = threadIdx.x;
    const int vp0 = i < nblk ? a.blk[2 * i] : 0, vt0 = i < nblk ? a.blk[2 * i + 1] : 0;
    sp[i] = vp0;
    st[i] = vt0;
    __syncthreads();
    for (int o = 1; o < 1024; o <<= 1) {
        int vp = i >= o ? sp[i - o] : 0;
        int vt = i >= o ? st[i - o] : 0;
        __syncthreads();
        sp[i] += vp;
        st[i] += vt;
        __syncthreads();
    }
    if (i < nblk) {
        a.blk[2 * i] = sp[i] - vp0;
        a.blk[2 * i + 1] = st[i] - vt0;
    }
    if (i == 1023) {
        a.boff[a.nbucket] = sp[1023];
        a.btile[a.nbucket] = st[1023];
    }
}

// Global offsets and the tile list (one thread per bucket).
__global__ void att_tiles_kernel(AttTcArgs a) {
    const int u = blockIdx.x * blockDim.x + threadIdx.x;
    if (u >= a.nbucket) return;
    const int blk = u / SCAN_BLK;
    const int op = a.boff[u] + a.blk[2 * blk], ot = a.btile[u] + a.blk[2 * blk + 1];
    a.boff[u] = op;
    a.btile[u] = ot;
    const int n = a.bcount[u];
    for (int q = 0; q * a.tok < n; ++q)
        a.tiles[ot + q] = make_int4(u / a.C, u % a.C, op + q * a.tok, min(a.tok, n - q * a.tok));
}

// One thread per selection row: place its pairs into their buckets.
__global__ void att_scatter_kernel(AttTcArgs a) {
    const long long row = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    const long long rows = (long long)a.B * a.Tq * a.Hkv;
    if (row >= rows) return;
    const int j = (int)(row % a.Hkv);
    const long long bt = row / a.Hkv;
    const int t = (int)(bt % a.Tq), b = (int)(bt / a.Tq);
    int ke = a.keff[row];
    ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
    const int nc = ncand_of(a, t);
    const int p = phase_of(a, b, j, t);
    for (int i = 0; i < ke; ++i) {
        const int c = a.idx[row * a.kmax + i];
        if (c < 0 || c >= nc) continue;
        const long long u = (long long)p * a.C + c;
        const int pos = a.boff[u] + atomicAdd(&a.bcursor[u], 1);
        a.pairs[pos] = make_int2((t << 5) | i, __float_as_int(a.w8[row * a.kmax + i]));
    }
}

// The same two steps with the rows of one CTA taken as HT consecutive tokens of one
// (b, kv head) -- all in one phase, since HT divides TB -- so that a CTA counts its
// pairs per chunk in a shared-memory histogram and touches each of its buckets'
// global counters once, instead of once per pair.  Used when the histogram of C
// counters fits in shared memory (two of them for the scatter).
constexpr int HT = 256;                 // tokens per CTA
constexpr int HIST_MAX_C = 16384;       // chunks whose counters fit in shared memory

__device__ __forceinline__ bool hist_row(const AttTcArgs &a, int &b, int &j, int &t, long long &row) {
    const int tb = (a.Tq + HT - 1) / HT;
    const int blk = (int)blockIdx.x;
    const int bj = blk / tb;
    b = bj / a.Hkv;
    j = bj % a.Hkv;
    t = (blk % tb) * HT + (int)threadIdx.x;
    row = ((long long)b * a.Tq + t) * a.Hkv + j;
    return t < a.Tq;
}

// A row's kept slots: chunk indices, and (val non-null) their scores.  Rows of kmax
// 4-byte entries start on 16-byte boundaries when kmax is a multiple of 4 (the
// buffers are 16-byte aligned), and are then read as 16-byte vectors.
__device__ __forceinline__ void load_row_slots(const int32_t *idx, const float *val, int ke, int kmax,
                                               int (&c)[MAX_KMAX], float (&x)[MAX_KMAX]) {
    if ((kmax & 3) == 0) {
#pragma unroll
        for (int q = 0; q < MAX_KMAX / 4; ++q) {
            if (4 * q < ke) {
                const int4 ci = reinterpret_cast<const int4 *>(idx)[q];
                c[4 * q] = ci.x, c[4 * q + 1] = ci.y, c[4 * q + 2] = ci.z, c[4 * q + 3] = ci.w;
                if (val != nullptr) {
                    const float4 xv = reinterpret_cast<const float4 *>(val)[q];
                    x[4 * q] = xv.x, x[4 * q + 1] = xv.y, x[4 * q + 2] = xv.z, x[4 * q + 3] = xv.w;
                }
            }
        }
    } else {
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) {
                c[i] = idx[i];
                if (val != nullptr) x[i] = val[i];
            }
    }
}

__global__ void __launch_bounds__(HT) att_count_hist_kernel(AttTcArgs a) {
    extern __shared__ int hist[];   // [C]
    for (int c = threadIdx.x; c < a.C; c += HT) hist[c] = 0;
    __syncthreads();
    int b, j, t;
    long long row;
    const bool live = hist_row(a, b, j, t, row);
    if (live) {
        int ke = a.keff[row];
        if (ke < 0 || ke > a.kmax) {
            atomicOr(a.status, DEV_BAD_INDEX);
            ke = ke < 0 ? 0 : a.kmax;
        }
        const int nc = ncand_of(a, t);
        int ci[MAX_KMAX];
        float unused[MAX_KMAX];
        load_row_slots(a.idx + row * a.kmax, nullptr, ke, a.kmax, ci, unused);
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i) {
            if (i >= ke) continue;
            if (ci[i] < 0 || ci[i] >= nc) {
                atomicOr(a.status, DEV_BAD_INDEX);
                continue;
            }
            atomicAdd(&hist[ci[i]], 1);
        }
    }
    __syncthreads();
    const int tb = (a.Tq + HT - 1) / HT;
    const int t0 = ((int)blockIdx.x % tb) * HT;
    const int bj = (int)blockIdx.x / tb;
    const long long p = (long long)bj * a.ntb + t0 / TB;
    for (int c = threadIdx.x; c < a.C; c += HT)
        if (hist[c] > 0) atomicAdd(&a.bcount[p * a.C + c], hist[c]);
}

__global__ void __launch_bounds__(HT) att_scatter_hist_kernel(AttTcArgs a) {
    extern __shared__ int sh[];   // [C] counts, then cursors; [C] bucket bases
    int *cnt = sh, *basep = sh + a.C;
    for (int c = threadIdx.x; c < a.C; c += HT) cnt[c] = 0;
    __syncthreads();
    int b, j, t;
    long long row;
    const bool live = hist_row(a, b, j, t, row);
    int ke = 0, nc = 0;
    int ci[MAX_KMAX];
    float wv[MAX_KMAX];
    if (live) {
        ke = a.keff[row];
        ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
        nc = ncand_of(a, t);
        load_row_slots(a.idx + row * a.kmax, a.score + row * a.kmax, ke, a.kmax, ci, wv);
        // fusion weights: softmax of the kept scores
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) m = fmaxf(m, wv[i]);
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) {
                wv[i] = expf(wv[i] - m);
                z += wv[i];
            }
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) wv[i] /= z;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke && ci[i] >= 0 && ci[i] < nc) atomicAdd(&cnt[ci[i]], 1);
    }
    __syncthreads();
    const int tb = (a.Tq + HT - 1) / HT;
    const int bj = (int)blockIdx.x / tb;
    const long long p = (long long)bj * a.ntb + (((int)blockIdx.x % tb) * HT) / TB;
    for (int c = threadIdx.x; c < a.C; c += HT) {
        const int n = cnt[c];
        if (n > 0) {
            const long long u = p * a.C + c;
            basep[c] = a.boff[u] + atomicAdd(&a.bcursor[u], n);   // this CTA's range in the bucket
        }
        cnt[c] = 0;
    }
    __syncthreads();
    if (live) {
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i) {
            if (i >= ke || ci[i] < 0 || ci[i] >= nc) continue;
            const int pos = basep[ci[i]] + atomicAdd(&cnt[ci[i]], 1);
            a.pairs[pos] = make_int2((t << 5) | i, __float_as_int(wv[i]));
        }
    }
}

// ---------------------------------------------------------------------------- main kernel

constexpr int NINFO = 4;   // tiles of row info (token, weight) the producers may run ahead

struct TileRows {            // one tile's row info, written by the producers, read by the epilogue
    int p, n;
    int off[MROWS];          // row's float offset in its phase's accumulator slot (-1: padding row)
    float w[MROWS];          // fusion weight of each row's (token, slot) pair
};

struct __align__(8) AttBars {
    uint64_t q_full[2], q_empty[2], kv_full[2], kv_empty[2];
    uint64_t s_full[2], p_full[2], p_empty[2], o_full[2], o_empty[2], l_full[2], l_empty[2], done;
    uint64_t info_full[NINFO], info_empty[NINFO];
    float l[2][MROWS];           // softmax row sums of the tiles in the two TMEM/P buffers
    uint32_t tmem_base;
    int abort;
    int tile_lo, tile_hi;
};

struct TileInfo {
    int b, j, c, p, start, n;
};

__device__ __forceinline__ TileInfo tile_info(const AttTcArgs &a, int tau) {
    const int4 e = a.tiles[tau];
    TileInfo T;
    T.p = e.x;
    T.c = e.y;
    const int bj = T.p / a.ntb;
    T.b = bj / a.Hkv;
    T.j = bj % a.Hkv;
    T.start = e.z;
    T.n = e.w;
    return T;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// fp32 vector reduction into global memory with no value returned
__device__ __forceinline__ void red_add_v4(float *addr, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

// Rows (token, head) of the phases in batch `bt`: accumulators -> bf16 O,
// accumulators zeroed.  Warps of the whole grid take groups of 8 consecutive
// rows (2*D float4, D/16 loads in flight per lane).
template <int D>
__device__ void finalize_batch(const AttTcArgs &a, __nv_bfloat16 *__restrict__ O, int bt, int gwarp, int nwarps,
                               int lane) {
    constexpr int RV = D / 4;            // float4 per row
    constexpr int NU = 8 * RV / 32;      // float4 per lane per group of 8 rows
    const int p0 = bt * NB, p1 = min(a.nphase, p0 + NB);
    const int rows_per_phase = TB * a.G;   // a multiple of 8
    const long long ngroups = (long long)(p1 - p0) * rows_per_phase / 8;
    for (long long gi = gwarp; gi < ngroups; gi += nwarps) {
        const long long e0 = gi * 8;
        const int p = p0 + (int)(e0 / rows_per_phase);
        const int rr0 = (int)(e0 % rows_per_phase);
        const int bj = p / a.ntb, tbi = p % a.ntb;
        const int b = bj / a.Hkv, j = bj % a.Hkv;
        float4 *acc = reinterpret_cast<float4 *>(slot_of(a, p) + (size_t)rr0 * D);
        float4 v[NU];
#pragma unroll
        for (int u = 0; u < NU; ++u) v[u] = __ldcg(acc + lane + 32 * u);
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int e = lane + 32 * u;   // float4 e of the group: row rr0 + e / RV, columns 4 (e % RV) ..
            const int rr = rr0 + e / RV;
            const int t = tbi * TB + rr / a.G, g = rr % a.G;
            __stcg(acc + e, make_float4(0.f, 0.f, 0.f, 0.f));
            if (t < a.Tq) {
                __nv_bfloat162 lo = __floats2bfloat162_rn(v[u].x, v[u].y), hi = __floats2bfloat162_rn(v[u].z, v[u].w);
                uint2 pk;
                pk.x = *reinterpret_cast<uint32_t *>(&lo);
                pk.y = *reinterpret_cast<uint32_t *>(&hi);
                reinterpret_cast<uint2 *>(O + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G + g) * D)[e % RV] = pk;
            }
        }
    }
}

template <int D>
__global__ void __launch_bounds__(NT_ATT, 1)
    att_main_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                    const __nv_bfloat16 *__restrict__ Q, __nv_bfloat16 *__restrict__ O, AttTcArgs a) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int S = a.S;
    constexpr int NBX = D / 64;                            // 64-column boxes per row of Q, K, V
    constexpr int QTILE = MROWS * D * 2;                   // one Q tile: NBX boxes of 128 rows x 128 B
    const int kv_bytes = S * 128;                          // one 64-column box of S rows
    const int p_bytes = (S / 64) * 16384;                  // one P tile
    uint8_t *sQ = base;                                    // nsq x QTILE
    uint8_t *sKV = sQ + (size_t)a.nsq * QTILE;             // nskv x (K: NBX boxes, V: NBX boxes)
    uint8_t *sP = sKV + (size_t)a.nskv * 2 * NBX * kv_bytes;   // 2 P buffers x p_bytes
    float *stg = reinterpret_cast<float *>(sP + 2 * (size_t)p_bytes);   // 8 O warps x 32 x PITCH
    TileRows *info = reinterpret_cast<TileRows *>(stg + 8 * 32 * PITCH);      // NINFO stages
    AttBars *bar = reinterpret_cast<AttBars *>(info + NINFO);
    volatile int *abort = &bar->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // finalise the previous batch (its slots are not touched by this batch's tiles)
    if (a.batch > 0)
        finalize_batch<D>(a, O, a.batch - 1, blockIdx.x * (NT_ATT / 32) + warp, gridDim.x * (NT_ATT / 32), lane);
    if (a.batch >= a.nbatch) return;

    if (threadIdx.x == 0) {
        for (int s = 0; s < 2; ++s) {
            mbar_init(&bar->q_full[s], NPROD);
            mbar_init(&bar->q_empty[s], 1);
            mbar_init(&bar->kv_full[s], 1);
            mbar_init(&bar->kv_empty[s], 1);
            mbar_init(&bar->s_full[s], 1);
            mbar_init(&bar->p_full[s], 4);
            mbar_init(&bar->p_empty[s], 1);
            mbar_init(&bar->o_full[s], 1);
            mbar_init(&bar->o_empty[s], 8);
            mbar_init(&bar->l_full[s], 4);
            mbar_init(&bar->l_empty[s], 8);
        }
        for (int s = 0; s < NINFO; ++s) {
            mbar_init(&bar->info_full[s], NPROD);
            mbar_init(&bar->info_empty[s], 8);
        }
        mbar_init(&bar->done, 1);
        bar->abort = 0;
        const int p0 = a.batch * NB, p1 = min(a.nphase, p0 + NB);
        bar->tile_lo = a.btile[p0 * a.C];
        bar->tile_hi = a.btile[p1 * a.C];
        fence_mbar_init();
    }
    if (warp == 2) {
        tmem_alloc(&bar->tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem_base;
    // TMEM columns: S buffers at 0 and 128, O buffers at 256 and 384 (buffer = tile index & 1)
    // each CTA takes a contiguous range of the batch's tiles, so the tiles of one
    // bucket (same chunk) mostly stay together and share one K/V load
    const int per = (bar->tile_hi - bar->tile_lo + (int)gridDim.x - 1) / (int)gridDim.x;
    const int tile_lo = min(bar->tile_hi, bar->tile_lo + (int)blockIdx.x * per);
    const int tile_hi = min(bar->tile_hi, tile_lo + per);

    if (warp < 2) {
        // ------------------------------------------------------------ producers: Q gather (rows r, r+64), K/V TMA
        __shared__ const char *rowsrc[MROWS];   // this tile's row sources (each warp writes and reads its own rows)
        int rr[2], mm[2], gg[2], pr[2];
        float pw[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            rr[h] = threadIdx.x + h * NPROD;
            mm[h] = rr[h] / a.G;
            gg[h] = rr[h] % a.G;
        }
        int i = 0;
        bool ok = true;
        int tau = tile_lo;
        TileInfo T = tau < tile_hi ? tile_info(a, tau) : TileInfo{};
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const bool v = tau < tile_hi && mm[h] < T.n;
            const int2 e = v ? a.pairs[T.start + mm[h]] : make_int2(0, 0);
            pr[h] = e.x;
            pw[h] = __int_as_float(e.y);
        }
        for (; tau < tile_hi && ok; ++i) {
            // prefetch the next tile while this one is issued
            const int tau_n = tau + 1;
            TileInfo Tn = tau_n < tile_hi ? tile_info(a, tau_n) : TileInfo{};
            // row info for the O drain (its slot is free once the drain of tile i - NINFO read it)
            {
                const int si = i % NINFO, ii = i / NINFO;
                if (ii > 0 && !(ok = mbar_wait(&bar->info_empty[si], (ii - 1) & 1, abort, a.status))) break;
                TileRows &ri = info[si];
                if (threadIdx.x == 0) {
                    ri.p = T.p;
                    ri.n = T.n;
                }
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const bool v = mm[h] < T.n;
                    ri.off[rr[h]] = v ? (((pr[h] >> 5) - (T.p % a.ntb) * TB) * a.G + gg[h]) * D : -1;
                    ri.w[rr[h]] = v ? pw[h] : 0.f;
                }
                mbar_arrive(&bar->info_full[si]);
            }
            const int sq = i % a.nsq, iq = i / a.nsq;
            if (iq > 0 && !(ok = mbar_wait(&bar->q_empty[sq], (iq - 1) & 1, abort, a.status))) break;
            // the tile's Q rows: row r of the tile is head gg of token pr >> 5 (padding rows zero-filled)
            const char *srcs[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                srcs[h] = nullptr;
                if (mm[h] < T.n) {
                    const int t0 = (T.p % a.ntb) * TB;   // the tile's phase: tokens t0 .. t0 + TB - 1
                    const int t = (int)dbg_clamp(pr[h] >> 5, t0, min(a.Tq, t0 + TB), a.status);
                    srcs[h] = reinterpret_cast<const char *>(Q) +
                              ((((size_t)T.b * a.Tq + t) * a.H + (size_t)T.j * a.G + gg[h]) * D) * 2;
                }
            }
            const uint32_t qbase = smem_u32(sQ + sq * QTILE);
            if constexpr (D == 128) {
                // each thread puts its two rows' sources in the warp's table; then every copy
                // instruction takes four rows x 128 bytes, each 8-lane group one whole 128-byte line
#pragma unroll
                for (int h = 0; h < 2; ++h) rowsrc[rr[h]] = srcs[h];
                __syncwarp();
                const int cx = lane & 7;
#pragma unroll
                for (int blk = 0; blk < 2; ++blk) {
#pragma unroll
                    for (int g4 = 0; g4 < 8; ++g4) {
                        const int r = warp * 32 + blk * NPROD + g4 * 4 + (lane >> 3);
                        const char *s = rowsrc[r];
                        const uint32_t dq = qbase + (r >> 3) * 1024 + (r & 7) * 128 + ((cx ^ (r & 7)) << 4);
#pragma unroll
                        for (int kb = 0; kb < D / 64; ++kb)
                            cp_async16(dq + kb * 16384, s != nullptr ? s + kb * 128 + cx * 16 : reinterpret_cast<const char *>(Q),
                                       s != nullptr ? 16u : 0u);
                    }
                }
                __syncwarp();   // the table is rewritten for the next tile only after every lane has read it
            } else {
                // 128-byte rows: each thread copies its own two rows (the table measured slower here)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int r = rr[h];
                    const uint32_t dq = qbase + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                    for (int x = 0; x < D / 8; ++x)
                        cp_async16(dq + ((x ^ (r & 7)) << 4),
                                   srcs[h] != nullptr ? srcs[h] + x * 16 : reinterpret_cast<const char *>(Q),
                                   srcs[h] != nullptr ? 16u : 0u);
                }
            }
            cp_async_arrive(&bar->q_full[sq]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const bool v = tau_n < tile_hi && mm[h] < Tn.n;
                const int2 e = v ? a.pairs[Tn.start + mm[h]] : make_int2(0, 0);
                pr[h] = e.x;
                pw[h] = __int_as_float(e.y);
            }
            T = Tn;
            tau = tau_n;
        }
        asm volatile("cp.async.wait_all;" ::: "memory");
    } else if (warp == 3) {
        // ------------------------------------------------------------ K/V loader: one TMA load per bucket run
        // (consecutive tiles of one (phase, chunk) share a load), as far ahead as the stages allow
        if (lane == 0) {
            int nload = 0, prev_p = -1, prev_c = -1;
            bool ok = true;
            for (int tau = tile_lo; tau < tile_hi && ok; ++tau) {
                const int4 e = a.tiles[tau];
                if (e.x == prev_p && e.y == prev_c) continue;
                prev_p = e.x;
                prev_c = e.y;
                const int bj = (int)dbg_clamp(e.x / a.ntb, 0, (long long)a.B * a.Hkv, a.status);
                const int Tb = bj / a.Hkv, Tj = bj % a.Hkv;
                const int cz = (int)dbg_clamp(e.y, 0, a.C, a.status);   // the bucket's chunk
                const int skv = nload % a.nskv, ikv = nload / a.nskv;
                if (ikv > 0 && !(ok = mbar_wait(&bar->kv_empty[skv], (ikv - 1) & 1, abort, a.status))) break;
                mbar_expect_tx(&bar->kv_full[skv], (uint32_t)(2 * NBX * kv_bytes));
                uint8_t *dk = sKV + (size_t)skv * 2 * NBX * kv_bytes;
                const int z = Tb * a.Tcap + cz * S;
#pragma unroll
                for (int kb = 0; kb < NBX; ++kb) {
                    tma_load_3d(dk + kb * kv_bytes, &tmK, 64 * kb, Tj, z, &bar->kv_full[skv]);
                    tma_load_3d(dk + (NBX + kb) * kv_bytes, &tmV, 64 * kb, Tj, z, &bar->kv_full[skv]);
                }
                ++nload;
            }
            // wind down: the K/V loads issued have all landed
            for (int s = 0; s < a.nskv && s < nload; ++s)
                mbar_drain(&bar->kv_full[s], ((nload - 1 - s) / a.nskv) & 1);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ MMA issuer
        // With two K/V stages QK(i+1) is issued before PV(i), so the next tile's softmax
        // overlaps this one's PV; with one stage the order is QK(i), PV(i), ...
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(MROWS, S, 0, 0);
            const uint32_t idesc_o = idesc_bf16_f32(MROWS, D, 0, 1);
            const int n_mine = tile_hi - tile_lo;
            // K/V load index of each tile, derived from the tile records exactly as the loader does;
            // the records come four tiles ahead, so their L2 round trips stay off this loop
            int key_p = -1, key_c = -1, nload = 0;
            auto load_of = [&](int4 e) -> int {   // call with the records of tiles 0, 1, 2, ... in order
                if (e.x != key_p || e.y != key_c) {
                    key_p = e.x;
                    key_c = e.y;
                    ++nload;
                }
                return nload - 1;
            };
            auto rec = [&](int t) -> int4 { return t < n_mine ? a.tiles[tile_lo + t] : make_int4(-1, -1, 0, 0); };
            int4 w1 = rec(1), w2 = rec(2), w3 = rec(3), w4 = rec(4);
            int waited_load = -1;   // last load whose kv_full has been waited on
            // QK(i) writes S buffer i & 1, whose previous tile (i - 2) the softmax has released
            // through p_full before PV(i - 2) was issued, which precedes this call.
            auto issue_qk = [&](int i, int li) -> bool {
                const int sq = i % a.nsq, iq = i / a.nsq, skv = li % a.nskv, ikv = li / a.nskv;
                if (!mbar_wait(&bar->q_full[sq], iq & 1, abort, a.status)) return false;
                if (li != waited_load) {
                    if (!mbar_wait(&bar->kv_full[skv], ikv & 1, abort, a.status)) return false;
                    waited_load = li;
                }
                tc_fence_after();
                const uint32_t s_tmem = tmem + (i & 1) * 128;
                const uint32_t qa = smem_u32(sQ + sq * QTILE);
                const uint32_t kb0 = smem_u32(sKV + (size_t)skv * 2 * NBX * kv_bytes);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t a_addr = qa + (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t b_addr = kb0 + (kk >> 2) * kv_bytes + (kk & 3) * 32;
                    umma_bf16(s_tmem, desc_kmajor_sw128(a_addr), desc_kmajor_sw128(b_addr), idesc_s, kk != 0);
                }
                umma_commit(&bar->s_full[i & 1]);
                umma_commit(&bar->q_empty[sq]);
                return true;
            };
            const bool early = a.nskv >= 2;
            int li = n_mine > 0 ? load_of(rec(0)) : 0;
            bool ok = n_mine > 0 ? issue_qk(0, li) : true;
            for (int i = 0; i < n_mine && ok; ++i) {
                const int b = i & 1, k = i >> 1;
                const int li_next = i + 1 < n_mine ? load_of(w1) : -1;
                w1 = w2;
                w2 = w3;
                w3 = w4;
                w4 = rec(i + 5);
                if (early && li_next >= 0 && !(ok = issue_qk(i + 1, li_next))) break;
                if (!(ok = mbar_wait(&bar->p_full[b], k & 1, abort, a.status))) break;
                if (k > 0 && !(ok = mbar_wait(&bar->o_empty[b], (k - 1) & 1, abort, a.status))) break;
                tc_fence_after();
                const int skv = li % a.nskv;
                const uint32_t o_tmem = tmem + 256 + b * 128;
                const uint32_t pa = smem_u32(sP + b * p_bytes);
                const uint32_t vb = smem_u32(sKV + (size_t)skv * 2 * NBX * kv_bytes) + NBX * kv_bytes;
                for (int kk = 0; kk < S / 16; ++kk) {
                    // P: K-major, k-block kk/4 (64 keys each), 32 B per K=16 step inside it.
                    // V: MN-major, keys kk*16..+15 are two 8-row groups starting (kk*16)*128 B
                    // into each 64-dim box; the two boxes are kv_bytes apart.
                    const uint32_t a_addr = pa + (kk >> 2) * 16384 + (kk & 3) * 32;
                    const uint32_t b_addr = vb + kk * 16 * 128;
                    umma_bf16(o_tmem, desc_kmajor_sw128(a_addr), desc_mnmajor_sw128(b_addr, kv_bytes, 1024), idesc_o,
                              kk != 0);
                }
                umma_commit(&bar->o_full[b]);
                umma_commit(&bar->p_empty[b]);
                // the K/V stage is free once the last tile of its load is done
                if (li_next != li) umma_commit(&bar->kv_empty[skv]);
                if (!early && li_next >= 0 && !(ok = issue_qk(i + 1, li_next))) break;
                li = li_next;
            }
            umma_commit(&bar->done);
            mbar_drain(&bar->done, 0);
        }
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------ softmax: thread = tile row, every tile
        const int ew = warp & 3;               // TMEM lane quadrant
        const int r = ew * 32 + lane;
        const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
        bool ok = true;
        for (int i = 0; tile_lo + i < tile_hi && ok; ++i) {
            const int b = i & 1, k = i >> 1;
            if (!(ok = mbar_wait(&bar->s_full[b], k & 1, abort, a.status))) break;
            tc_fence_after();
            const uint32_t s_base = tmem + lane_off + b * 128;
            uint8_t *myP = sP + b * p_bytes;
            float l = 0.f;
            uint32_t sr[32];
            float mx = -INFINITY;
            for (int q = 0; q < S / 32; ++q) {
                tmem_ld32(s_base + q * 32, sr);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) mx = fmaxf(mx, __uint_as_float(sr[e]));
            }
            // P buffer b is free once PV(i - 2) has read it
            if (k > 0 && !(ok = mbar_wait(&bar->p_empty[b], (k - 1) & 1, abort, a.status))) break;
            for (int q = 0; q < S / 32; ++q) {
                tmem_ld32(s_base + q * 32, sr);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = exp2f((__uint_as_float(sr[2 * e]) - mx) * a.scale_log2);
                    const float p1 = exp2f((__uint_as_float(sr[2 * e + 1]) - mx) * a.scale_log2);
                    __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                    // the MMA sees the rounded probabilities: normalise by their sum
                    const float2 hf = __bfloat1622float2(h);
                    l += hf.x + hf.y;
                    pk[e] = *reinterpret_cast<uint32_t *>(&h);
                }
                uint8_t *prow = myP + (q >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int cx = (q & 1) * 4 + x;
                    *reinterpret_cast<uint4 *>(prow + ((cx ^ (r & 7)) << 4)) =
                        make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->p_full[b]);
            // row sum for the O drain of this tile
            if (k > 0 && !(ok = mbar_wait(&bar->l_empty[b], (k - 1) & 1, abort, a.status))) break;
            bar->l[b][r] = l;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->l_full[b]);
        }
    } else if (warp >= 8) {
        // ------------------------------------------------------------ O drain: thread = tile row, D/2 of its columns
        const int ew = warp & 3;               // TMEM lane quadrant
        const int hf = (warp - 8) >> 2;        // column half
        const int r = ew * 32 + lane;
        const uint32_t lane_off = (uint32_t)(ew * 32) << 16;
        float *wst = stg + (warp - 8) * 32 * PITCH;
        bool ok = true;
        for (int i = 0; tile_lo + i < tile_hi && ok; ++i) {
            const int b = i & 1, k = i >> 1;
            const int si = i % NINFO;
            if (!(ok = mbar_wait(&bar->info_full[si], (i / NINFO) & 1, abort, a.status))) break;
            const int Tp = info[si].p;
            const int myoff = info[si].off[r];
            const float w = info[si].w[r];
            // destinations of the staging rows this lane will reduce (rows rr*4 + lane/8 of the warp)
            int dstoff[8];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) {
                // -1 (padding) or the start of a row of the phase's accumulator slot
                const int o = info[si].off[ew * 32 + rr * 4 + (lane >> 3)];
                dstoff[rr] = o < 0 ? -1 : (int)dbg_clamp(o, 0, (long long)(TB - 1) * a.G * D + 1, a.status);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->info_empty[si]);
            if (!(ok = mbar_wait(&bar->l_full[b], k & 1, abort, a.status))) break;
            const float l = bar->l[b][r];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->l_empty[b]);
            const float f = myoff >= 0 ? w / l : 0.f;
            // O row -> (w/l) * O, reduced into the phase's accumulator slot 32 columns at a time
            if (!(ok = mbar_wait(&bar->o_full[b], k & 1, abort, a.status))) break;
            tc_fence_after();
            float *acc_slot = slot_of(a, Tp) + 4 * (lane & 7);
            const uint32_t o_base = tmem + lane_off + 256 + b * 128 + hf * (D / 2);
            for (int q = 0; q < D / 64; ++q) {
                uint32_t orr[32];
                tmem_ld32(o_base + q * 32, orr);
                tmem_wait_ld();
                if (q == D / 64 - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&bar->o_empty[b]);
                }
                float *mine = wst + lane * PITCH;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(mine + e) =
                        make_float4(__uint_as_float(orr[e]) * f, __uint_as_float(orr[e + 1]) * f,
                                    __uint_as_float(orr[e + 2]) * f, __uint_as_float(orr[e + 3]) * f);
                __syncwarp();
                const int col = hf * (D / 2) + q * 32;
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    if (dstoff[rr] >= 0) {
                        const int lr = rr * 4 + (lane >> 3);
                        red_add_v4(acc_slot + dstoff[rr] + col,
                                   *reinterpret_cast<const float4 *>(wst + lr * PITCH + 4 * (lane & 7)));
                    }
                }
                __syncwarp();
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

}  // namespace

// ---------------------------------------------------------------------------- host side

bool attend_tc_supported(const Prob &p) {
    // G need not divide the 128 tile rows: a tile holds floor(128 / G) tokens and the last rows are padding
    if (!(p.dtype == HSA_BF16 && (p.d == 64 || p.d == 128) && (p.S == 64 || p.S == 128) && p.G <= 16 &&
          p.C >= 1 && p.Tq >= 1 && p.kmax <= 32 && p.Tq < (1 << 26) && (long long)p.B * p.Tcap < (1ll << 31)))
        return false;
    // the second scan level is one block of 1024 threads over SCAN_BLK-bucket blocks
    const long long ntb = (p.Tq + TB - 1) / TB;
    const long long nbucket = (long long)p.B * p.Hkv * ntb * p.C;
    return nbucket <= 1024LL * SCAN_BLK && (long long)p.rows * p.kmax < (1LL << 31);
}

AttTcLayout attend_tc_layout(const Prob &p) {
    AttTcLayout L{};
    L.tb = TB;
    L.ntb = (p.Tq + TB - 1) / TB;
    L.nsub = 0;
    L.nphase = p.B * p.Hkv * L.ntb;
    L.nbucket = L.nphase * p.C;
    L.nblk = (L.nbucket + SCAN_BLK - 1) / SCAN_BLK;
    L.tok = MROWS / p.G;
    L.ring = 2 * NB;
    L.hist = p.C <= HIST_MAX_C;
    const size_t pairs = (size_t)p.rows * p.kmax;
    L.max_tiles = pairs / L.tok + (size_t)L.nbucket + 1;
    L.counter_ints = 2 * (size_t)L.nbucket;
    L.ring_bytes = (size_t)L.ring * TB * p.G * p.d * sizeof(float);
    return L;
}

int attend_tc_launches(const AttTcLayout &L) {
    const int nbatch = (L.nphase + NB - 1) / NB;
    return 5 + nbatch + 1;   // count, scan1, scan2, tiles, scatter, one per batch, final finalise
}

cudaError_t launch_attend_tc(const Prob &p, const AttTcLayout &L, const AttTcBuffers &bf, const void *Q, const void *K,
                             const void *V, const int32_t *idx, const float *score, const int32_t *keff, void *O,
                             cudaStream_t st) {
    AttTcArgs a;
    a.B = p.B;
    a.Tq = p.Tq;
    a.Tcap = p.Tcap;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.S = p.S;
    a.C = p.C;
    a.kmax = p.kmax;
    a.tok = L.tok;
    a.ntb = L.ntb;
    a.nphase = L.nphase;
    a.nbucket = L.nbucket;
    // double-buffered Q and K/V where shared memory allows (d=128, S=128: single, ~200 KB)
    a.nsq = (p.S <= 64 || p.d == 64) ? 2 : 1;
    a.nskv = (p.S <= 64 || p.d == 64) ? 2 : 1;
    a.d = p.d;
    a.nbatch = (L.nphase + NB - 1) / NB;
    a.q_pos0 = p.q_pos0;
    a.scale_log2 = 1.4426950408889634f / sqrtf((float)p.d);
    a.idx = idx;
    a.score = score;
    a.keff = keff;
    a.w8 = bf.w8;
    a.bcount = bf.counters;
    a.bcursor = bf.counters + L.nbucket;
    a.boff = bf.boff;
    a.btile = bf.btile;
    a.blk = bf.blk;
    a.pairs = bf.pairs;
    a.tiles = bf.tiles;
    a.ringbuf = bf.ring;
    a.status = bf.status;

    // bucket counters and the accumulator ring start at zero on every call
    cudaError_t e = cudaMemsetAsync(bf.counters, 0, L.counter_ints * sizeof(int32_t), st);
    if (e == cudaSuccess) e = cudaMemsetAsync(bf.ring, 0, L.ring_bytes, st);
    if (e != cudaSuccess) return e;
    const int rows_blocks = (int)((p.rows + 255) / 256);
    const bool hist = L.hist;
    const int hist_blocks = p.B * p.Hkv * ((p.Tq + HT - 1) / HT);
    if (hist) {
        if ((e = cudaFuncSetAttribute(att_scatter_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(2 * p.C * sizeof(int)))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(att_count_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(p.C * sizeof(int)))) != cudaSuccess)
            return e;
        att_count_hist_kernel<<<hist_blocks, HT, p.C * sizeof(int), st>>>(a);
    } else {
        att_count_kernel<<<rows_blocks, 256, 0, st>>>(a);
    }
    att_scan1_kernel<<<L.nblk, 1024, 0, st>>>(a);
    att_scan2_kernel<<<1, 1024, 0, st>>>(a, L.nblk);
    att_tiles_kernel<<<(L.nbucket + 255) / 256, 256, 0, st>>>(a);
    if (hist)
        att_scatter_hist_kernel<<<hist_blocks, HT, 2 * p.C * sizeof(int), st>>>(a);
    else
        att_scatter_kernel<<<rows_blocks, 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;

    // K and V as 3D (d, Hkv, B*Tcap): box (64, 1, S) = S rows of 128 B
    CUtensorMap mk, mv;
    const uint64_t dims[3] = {(uint64_t)p.d, (uint64_t)p.Hkv, (uint64_t)p.B * p.Tcap};
    const uint64_t strides[2] = {(uint64_t)p.d * 2, (uint64_t)p.Hkv * p.d * 2};
    const uint32_t box[3] = {64, 1, (uint32_t)p.S};
    if ((e = make_tmap_3d(&mk, K, dims, strides, box)) != cudaSuccess) return e;
    if ((e = make_tmap_3d(&mv, V, dims, strides, box)) != cudaSuccess) return e;
    const size_t smem = 1024 + (size_t)a.nsq * 128 * p.d * 2 + (size_t)a.nskv * 2 * (p.d / 64) * p.S * 128 +
                        2 * (size_t)(p.S / 64) * 16384 + 8 * 32 * PITCH * sizeof(float) + NINFO * sizeof(TileRows) +
                        sizeof(AttBars);
    auto kern = p.d == 64 ? att_main_kernel<64> : att_main_kernel<128>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) != cudaSuccess)
        return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    for (int bt = 0; bt <= a.nbatch; ++bt) {
        a.batch = bt;
        kern<<<sms, NT_ATT, smem, st>>>(mk, mv, (const __nv_bfloat16 *)Q, (__nv_bfloat16 *)O, a);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace hsa
