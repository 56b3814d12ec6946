// backward.cu -- gradients of the method with respect to Q, K, V and W_L, with
// the chunk selection of the forward held fixed (HSA summary page,
// Implementation: the retrieval scores weight the chunk outputs, so they carry
// a gradient into the queries and, through the landmarks, into the keys and
// W_L; which chunks are kept is a discrete choice with no gradient).
//
// For a selection row (b, t, kv head j) with kept chunks c_i, fusion weights
// w = softmax(s) and in-chunk probabilities a_hiu of its heads h:
//   e_hi  = dO_h . o_hi = sum_u a_hiu (dO_h . V_u)
//   dz_hiu = w_i a_hiu (dO_h . V_u - e_hi) / sqrt(d)         (in-chunk softmax)
//   dQ_h += sum_u dz_hiu K_u,  dK_u += dz_hiu q_h,  dV_u += w_i a_hiu dO_h
//   ds_i  = w_i (dw_i - sum_i' w_i' dw_i'),  dw_i = sum_h e_hi (fusion softmax)
//   dQ_h += sum_i ds_i L_ci,   dL_ci += ds_i sum_h q_h       (s_i = sum_h q_h . L_ci)
// and through every landmark L_c = mean(K of chunk c) W_L:
//   dW_L += mean_c^T dL_c,     dK_u += (dL_c W_L^T) / S for the S keys of chunk c.
//
// Stages (all on the caller's stream):
//   prep     one thread per selection row: fusion weights, pair count per
//            (b, j, c) bucket, checks of keff and the chunk indices;
//   scan     one CTA: exclusive scans of the bucket counts (pairs) and of
//            their tile counts, the tile list, the scatter cursors;
//   scatter  one thread per selection row: its (row, slot) pairs -> buckets;
//   attend   chunk-major, one CTA per SM over a contiguous range of tiles of
//            query-head rows that kept one chunk; K_c and V_c are staged once
//            per bucket run and dK_c, dV_c stay on chip until the bucket
//            changes.  Per tile: Z = q K^T, GV = dO V^T, the row softmax and
//            e, then dQ = dZ K and the dK/dV updates; e goes to the
//            workspace.  bf16 with d = 128 runs on tcgen05 (bwd_tcw_kernel
//            for S = 64, bwd_tc_kernel for S = 128); everything else, and any
//            problem with HSA_FLAG_SIMT, on CUDA cores (bwd_attend_kernel).
//   fuse     one warp per selection row: dw, ds, the score path into dQ and dL;
//   landmark one pass over all complete chunks: chunk means, dW_L partials per
//            CTA, and dL W_L^T / S added to the chunk's key gradients.
// Accumulation is fp32 everywhere and the gradients are fp32 buffers; the
// stored inputs (fp32 or bf16) are read exactly.  The tensor-core kernels
// round dZ and w P to bf16 before the dQ, dK and dV products, as the forward
// rounds P; the CUDA-core kernel rounds nothing.
#include "common.cuh"
#include "sm100.cuh"

namespace hsa {
namespace {

constexpr int RT = 32;          // query-head rows per tile
constexpr int NT_BWD = 512;     // threads of the attend kernel (16 warps)
constexpr int NT_SCAN = 1024;

struct BwdArgs {
    int B, Tq, Tcap, H, Hkv, G, d, S, C, kmax, pt;   // pt: pairs per tile = RT / G
    long long q_pos0, rows;
    long long nbucket;
    float scale;                // 1/sqrt(d)
    const int32_t *idx, *keff;
    const float *score;
    float *w;                   // [rows][kmax] fusion weights
    float *e;                   // [rows][kmax][G]  dO_h . o_hi
    int32_t *bcount;            // [nbucket] pair counts, then scatter cursors
    int32_t *boff;              // [nbucket + 1] first pair of each bucket
    int32_t *btile;             // [nbucket + 1] first tile of each bucket
    int32_t *pairs;             // [rows * kmax] row * kmax + slot, bucket-major
    float *pair_w;              // [rows * kmax] fusion weight of each pair, bucket-major
    int4 *tiles;                // (bucket, first pair, pairs, 0)
    int32_t *ntiles;            // number of tiles (written by the scan)
    float *dL;                  // [B][Hkv][C][d] landmark gradients
    uint32_t *status;
};

__device__ __forceinline__ void red_add4(float *p, float4 v) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(p), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}
__device__ __forceinline__ void red_add2(float *p, float2 v) {
    asm volatile("red.global.add.v2.f32 [%0], {%1, %2};" ::"l"(p), "f"(v.x), "f"(v.y) : "memory");
}

// number of candidate chunks of a query row
__device__ __forceinline__ long long ncand_of(const BwdArgs &a, int t) {
    long long nc = (a.q_pos0 + t) / a.S;
    return nc > a.C ? a.C : nc;
}

// ---------------------------------------------------------------------------- prep, scan, scatter

__global__ void bwd_prep_kernel(BwdArgs a) {
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= a.rows) return;
    const int j = (int)(r % a.Hkv);
    const long long bt = r / a.Hkv;
    const int t = (int)(bt % a.Tq), b = (int)(bt / a.Tq);
    int ke = a.keff[r];
    if (ke < 0 || ke > a.kmax) {
        atomicOr(a.status, DEV_BAD_INDEX);
        ke = ke < 0 ? 0 : a.kmax;
    }
    const float *sc = a.score + r * a.kmax;
    float m = -INFINITY;
    for (int i = 0; i < ke; ++i) m = fmaxf(m, sc[i]);
    float z = 0.f;
    for (int i = 0; i < ke; ++i) z += expf(sc[i] - m);
    const long long nc = ncand_of(a, t);
    for (int i = 0; i < a.kmax; ++i) {
        const float wi = i < ke ? expf(sc[i] - m) / z : 0.f;
        a.w[r * a.kmax + i] = wi;
        if (i >= ke) continue;
        const int c = a.idx[r * a.kmax + i];
        if (c < 0 || c >= nc) {
            atomicOr(a.status, DEV_BAD_INDEX);
            continue;
        }
        atomicAdd(a.bcount + ((long long)b * a.Hkv + j) * a.C + c, 1);
    }
}

// Exclusive scans of pair counts and tile counts over the buckets, in blocks
// of NT_SCAN with a running carry; each bucket's count becomes its scatter
// cursor.  The tile records are written by bwd_tiles_kernel, one thread per
// bucket over the whole grid.
__global__ void __launch_bounds__(NT_SCAN) bwd_scan_kernel(BwdArgs a) {
    __shared__ int wp[NT_SCAN / 32], wt[NT_SCAN / 32];
    __shared__ int carry_p, carry_t;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (threadIdx.x == 0) {
        carry_p = 0;
        carry_t = 0;
    }
    __syncthreads();
    for (long long base = 0; base < a.nbucket; base += NT_SCAN) {
        const long long i = base + threadIdx.x;
        const int cnt = i < a.nbucket ? a.bcount[i] : 0;
        const int nt = (cnt + a.pt - 1) / a.pt;
        int ip = cnt, it = nt;   // inclusive warp scans
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int xp = __shfl_up_sync(FULL, ip, o), xt = __shfl_up_sync(FULL, it, o);
            if (lane >= o) {
                ip += xp;
                it += xt;
            }
        }
        if (lane == 31) {
            wp[warp] = ip;
            wt[warp] = it;
        }
        __syncthreads();
        if (warp == 0) {
            int sp = wp[lane], st = wt[lane];
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int xp = __shfl_up_sync(FULL, sp, o), xt = __shfl_up_sync(FULL, st, o);
                if (lane >= o) {
                    sp += xp;
                    st += xt;
                }
            }
            wp[lane] = sp;   // inclusive prefix over warps
            wt[lane] = st;
        }
        __syncthreads();
        const int ep = carry_p + (warp ? wp[warp - 1] : 0) + ip - cnt;
        const int et = carry_t + (warp ? wt[warp - 1] : 0) + it - nt;
        if (i < a.nbucket) {
            a.boff[i] = ep;
            a.btile[i] = et;
            a.bcount[i] = ep;   // scatter cursor
        }
        __syncthreads();
        if (threadIdx.x == NT_SCAN - 1) {
            carry_p = ep + cnt;
            carry_t = et + nt;
        }
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        a.boff[a.nbucket] = carry_p;
        a.btile[a.nbucket] = carry_t;
        *a.ntiles = carry_t;
    }
}

// Each bucket's tile records: (bucket, first pair, pairs, 0), pt pairs per tile.
__global__ void bwd_tiles_kernel(BwdArgs a) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= a.nbucket) return;
    const int ep = a.boff[i], cnt = a.boff[i + 1] - ep, et = a.btile[i], nt = a.btile[i + 1] - et;
    for (int q = 0; q < nt; ++q) a.tiles[et + q] = make_int4((int)i, ep + q * a.pt, min(a.pt, cnt - q * a.pt), 0);
}

__global__ void bwd_scatter_kernel(BwdArgs a) {
    const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (r >= a.rows) return;
    const int j = (int)(r % a.Hkv);
    const long long bt = r / a.Hkv;
    const int t = (int)(bt % a.Tq), b = (int)(bt / a.Tq);
    int ke = a.keff[r];
    ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
    const long long nc = ncand_of(a, t);
    for (int i = 0; i < ke; ++i) {
        const int c = a.idx[r * a.kmax + i];
        if (c < 0 || c >= nc) continue;
        const int pos = atomicAdd(a.bcount + ((long long)b * a.Hkv + j) * a.C + c, 1);
        a.pairs[pos] = (int)(r * a.kmax + i);
        a.pair_w[pos] = a.w[r * a.kmax + i];
    }
}

// The same two steps with the rows of one CTA taken as BHT consecutive tokens
// of one (b, kv head): the CTA counts its pairs per chunk in a shared-memory
// histogram and touches each of its buckets' global counters once, instead of
// once per pair.  Used when the C counters (two arrays for the scatter) fit in
// shared memory.  Rows are read as 16-byte vectors when kmax is a multiple of 4.
constexpr int BHT = 256;
constexpr int BHIST_MAX_C = 16384;

__device__ __forceinline__ bool bhist_row(const BwdArgs &a, int &b, int &j, int &t, long long &r) {
    const int tb = (a.Tq + BHT - 1) / BHT;
    const int bj = (int)blockIdx.x / tb;
    b = bj / a.Hkv;
    j = bj % a.Hkv;
    t = ((int)blockIdx.x % tb) * BHT + (int)threadIdx.x;
    r = ((long long)b * a.Tq + t) * a.Hkv + j;
    return t < a.Tq;
}

// A row's first ke slots of an int and a float array (rows of kmax entries).
__device__ __forceinline__ void bwd_row_slots(const int32_t *ip, const float *fp, int ke, int kmax,
                                              int (&c)[MAX_KMAX], float (&x)[MAX_KMAX]) {
    if ((kmax & 3) == 0) {
#pragma unroll
        for (int q = 0; q < MAX_KMAX / 4; ++q)
            if (4 * q < ke) {
                const int4 ci = reinterpret_cast<const int4 *>(ip)[q];
                const float4 xv = reinterpret_cast<const float4 *>(fp)[q];
                c[4 * q] = ci.x, c[4 * q + 1] = ci.y, c[4 * q + 2] = ci.z, c[4 * q + 3] = ci.w;
                x[4 * q] = xv.x, x[4 * q + 1] = xv.y, x[4 * q + 2] = xv.z, x[4 * q + 3] = xv.w;
            }
    } else {
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) {
                c[i] = ip[i];
                x[i] = fp[i];
            }
    }
}

__global__ void __launch_bounds__(BHT) bwd_prep_hist_kernel(BwdArgs a) {
    extern __shared__ int hist[];   // [C]
    for (int c = threadIdx.x; c < a.C; c += BHT) hist[c] = 0;
    __syncthreads();
    int b, j, t;
    long long r;
    if (bhist_row(a, b, j, t, r)) {
        int ke = a.keff[r];
        if (ke < 0 || ke > a.kmax) {
            atomicOr(a.status, DEV_BAD_INDEX);
            ke = ke < 0 ? 0 : a.kmax;
        }
        int ci[MAX_KMAX];
        float sv[MAX_KMAX];
        bwd_row_slots(a.idx + r * a.kmax, a.score + r * a.kmax, ke, a.kmax, ci, sv);
        float m = -INFINITY;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) m = fmaxf(m, sv[i]);
        float z = 0.f;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke) {
                sv[i] = expf(sv[i] - m);
                z += sv[i];
            }
        const long long nc = ncand_of(a, t);
        float *wr = a.w + r * a.kmax;
        for (int i = 0; i < a.kmax; ++i) wr[i] = 0.f;
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i) {
            if (i >= ke) continue;
            wr[i] = sv[i] / z;
            if (ci[i] < 0 || ci[i] >= nc) {
                atomicOr(a.status, DEV_BAD_INDEX);
                continue;
            }
            atomicAdd(&hist[ci[i]], 1);
        }
    }
    __syncthreads();
    const int tb = (a.Tq + BHT - 1) / BHT;
    const long long bj = (int)blockIdx.x / tb;
    for (int c = threadIdx.x; c < a.C; c += BHT)
        if (hist[c] > 0) atomicAdd(a.bcount + bj * a.C + c, hist[c]);
}

__global__ void __launch_bounds__(BHT) bwd_scatter_hist_kernel(BwdArgs a) {
    extern __shared__ int sh[];   // [C] counts, then cursors; [C] this CTA's base in each bucket
    int *cnt = sh, *basep = sh + a.C;
    for (int c = threadIdx.x; c < a.C; c += BHT) cnt[c] = 0;
    __syncthreads();
    int b, j, t;
    long long r;
    const bool live = bhist_row(a, b, j, t, r);
    int ke = 0;
    long long nc = 0;
    int ci[MAX_KMAX];
    float wv[MAX_KMAX];
    if (live) {
        ke = a.keff[r];
        ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
        nc = ncand_of(a, t);
        bwd_row_slots(a.idx + r * a.kmax, a.w + r * a.kmax, ke, a.kmax, ci, wv);
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i)
            if (i < ke && ci[i] >= 0 && ci[i] < nc) atomicAdd(&cnt[ci[i]], 1);
    }
    __syncthreads();
    const int tb = (a.Tq + BHT - 1) / BHT;
    const long long bj = (int)blockIdx.x / tb;
    for (int c = threadIdx.x; c < a.C; c += BHT) {
        const int n = cnt[c];
        if (n > 0) basep[c] = atomicAdd(a.bcount + bj * a.C + c, n);   // this CTA's run in the bucket
        cnt[c] = 0;
    }
    __syncthreads();
    if (live) {
#pragma unroll
        for (int i = 0; i < MAX_KMAX; ++i) {
            if (i >= ke || ci[i] < 0 || ci[i] >= nc) continue;
            const int pos = basep[ci[i]] + atomicAdd(&cnt[ci[i]], 1);
            a.pairs[pos] = (int)(r * a.kmax + i);
            a.pair_w[pos] = wv[i];
        }
    }
}

// ---------------------------------------------------------------------------- chunk-major attention backward

// 16 bytes of stored values -> fp32 in shared memory
__device__ __forceinline__ void cvt16(const float *src, float *dst) {
    *reinterpret_cast<float4 *>(dst) = __ldg(reinterpret_cast<const float4 *>(src));
}
__device__ __forceinline__ void cvt16(const __nv_bfloat16 *src, float *dst) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(src));
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
    const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
    const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
    reinterpret_cast<float4 *>(dst)[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
    reinterpret_cast<float4 *>(dst)[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
}

template <int CPL> struct Cols;   // CPL consecutive fp32 values of one lane
template <> struct Cols<4> {
    float v[4];
    __device__ __forceinline__ void load(const float *p) {
        const float4 x = *reinterpret_cast<const float4 *>(p);
        v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    }
    __device__ __forceinline__ void red(float *p) const { red_add4(p, make_float4(v[0], v[1], v[2], v[3])); }
};
template <> struct Cols<2> {
    float v[2];
    __device__ __forceinline__ void load(const float *p) {
        const float2 x = *reinterpret_cast<const float2 *>(p);
        v[0] = x.x; v[1] = x.y;
    }
    __device__ __forceinline__ void red(float *p) const { red_add2(p, make_float2(v[0], v[1])); }
};

template <int S, int D> struct BwdShape {
    static constexpr int KP = D + 4;       // K, V, q, dO row pitch (floats): float4 rows, conflict-free
    static constexpr int SP = S + 4;       // dZ, w*P row pitch
    static constexpr int KPT = S / 32;     // keys per lane in the row pass
    static constexpr int UPW = S / 16;     // keys per warp in the dK/dV pass
    static constexpr int CPL = D / 32;     // columns per lane
    static constexpr size_t smem = sizeof(float) * (2 * (size_t)S * KP + 2 * (size_t)RT * KP + 2 * (size_t)RT * SP) +
                                   RT * (sizeof(long long) + sizeof(float) + sizeof(int));
};

template <typename T, int S, int D>
__global__ void __launch_bounds__(NT_BWD, 1)
    bwd_attend_kernel(BwdArgs a, const T *__restrict__ Q, const T *__restrict__ K, const T *__restrict__ V,
                      const T *__restrict__ dO, float *__restrict__ dQ, float *__restrict__ dK,
                      float *__restrict__ dV) {
    using SH = BwdShape<S, D>;
    constexpr int KP = SH::KP, SP = SH::SP, KPT = SH::KPT, UPW = SH::UPW, CPL = SH::CPL;
    constexpr int EPS = 16 / (int)sizeof(T);   // stored elements per 16-byte load
    constexpr int SEGS = D / EPS;
    extern __shared__ float4 smem4[];
    float *sK = reinterpret_cast<float *>(smem4);
    float *sV = sK + S * KP;
    float *sq = sV + S * KP;
    float *sg = sq + RT * KP;
    float *sZ = sg + RT * KP;     // dZ (scaled in-chunk softmax gradient)
    float *sPw = sZ + RT * SP;    // w * P
    long long *s_qoff = reinterpret_cast<long long *>(sPw + RT * SP);
    float *s_w = reinterpret_cast<float *>(s_qoff + RT);
    int *s_e = reinterpret_cast<int *>(s_w + RT);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = *a.ntiles;
    const int lo = (int)((long long)ntiles * blockIdx.x / gridDim.x);
    const int hi = (int)((long long)ntiles * (blockIdx.x + 1) / gridDim.x);
    const float scale_log2 = a.scale * 1.4426950408889634f;

    float accK[UPW][CPL], accV[UPW][CPL];   // keys warp + 16 m, columns lane * CPL + x
#pragma unroll
    for (int m = 0; m < UPW; ++m)
#pragma unroll
        for (int x = 0; x < CPL; ++x) accK[m][x] = accV[m][x] = 0.f;
    int cur = -1, cb = 0, cj = 0, cc = 0;

    auto flush = [&]() {
#pragma unroll
        for (int m = 0; m < UPW; ++m) {
            const int u = warp + 16 * m;
            const long long off = (((long long)cb * a.Tcap + (long long)cc * S + u) * a.Hkv + cj) * D + lane * CPL;
            Cols<CPL> k, v;
#pragma unroll
            for (int x = 0; x < CPL; ++x) {
                k.v[x] = accK[m][x];
                v.v[x] = accV[m][x];
                accK[m][x] = accV[m][x] = 0.f;
            }
            k.red(dK + off);
            v.red(dV + off);
        }
    };

    for (int ti = lo; ti < hi; ++ti) {
        const int4 tr = a.tiles[ti];
        const int nrow = tr.z * a.G;
        if (tr.x != cur) {
            if (cur >= 0) flush();
            cur = tr.x;
            cc = cur % a.C;
            const int bj = cur / a.C;
            cj = bj % a.Hkv;
            cb = bj / a.Hkv;
            const long long row0 = ((long long)cb * a.Tcap + (long long)cc * S) * a.Hkv + cj;
            for (int i = threadIdx.x; i < S * SEGS; i += NT_BWD) {
                const int u = i / SEGS, sgm = i - u * SEGS;
                const long long off = (row0 + (long long)u * a.Hkv) * D + sgm * EPS;
                cvt16(K + off, sK + u * KP + sgm * EPS);
                cvt16(V + off, sV + u * KP + sgm * EPS);
            }
        }
        if (threadIdx.x < RT) {
            const int rr = threadIdx.x;
            if (rr < nrow) {
                const int pc = (int)dbg_clamp(a.pairs[tr.y + rr / a.G], 0, a.rows * a.kmax, a.status), g = rr % a.G;
                const long long bt = (long long)(pc / a.kmax) / a.Hkv;
                s_qoff[rr] = (bt * a.H + (long long)cj * a.G + g) * D;
                s_w[rr] = a.w[pc];
                s_e[rr] = pc * a.G + g;
            }
        }
        __syncthreads();
        for (int i = threadIdx.x; i < RT * SEGS; i += NT_BWD) {
            const int rr = i / SEGS, sgm = i - rr * SEGS;
            float *qd = sq + rr * KP + sgm * EPS, *gd = sg + rr * KP + sgm * EPS;
            if (rr < nrow) {
                cvt16(Q + s_qoff[rr] + sgm * EPS, qd);
                cvt16(dO + s_qoff[rr] + sgm * EPS, gd);
            } else {
#pragma unroll
                for (int x = 0; x < EPS; ++x) qd[x] = gd[x] = 0.f;
            }
        }
        __syncthreads();

        // ---- rows warp and warp + 16: Z = q K^T and GV = dO V^T over keys lane + 32 m
        if (warp < nrow) {
            float z0[KPT], z1[KPT], v0[KPT], v1[KPT];
#pragma unroll
            for (int m = 0; m < KPT; ++m) z0[m] = z1[m] = v0[m] = v1[m] = 0.f;
            const float *qa = sq + warp * KP, *qb = sq + (warp + 16) * KP;
            const float *ga = sg + warp * KP, *gb = sg + (warp + 16) * KP;
#pragma unroll 4
            for (int x = 0; x < D; x += 4) {
                const float4 q0 = *reinterpret_cast<const float4 *>(qa + x);
                const float4 q1 = *reinterpret_cast<const float4 *>(qb + x);
                const float4 g0 = *reinterpret_cast<const float4 *>(ga + x);
                const float4 g1 = *reinterpret_cast<const float4 *>(gb + x);
#pragma unroll
                for (int m = 0; m < KPT; ++m) {
                    const float4 k = *reinterpret_cast<const float4 *>(sK + (lane + 32 * m) * KP + x);
                    const float4 v = *reinterpret_cast<const float4 *>(sV + (lane + 32 * m) * KP + x);
                    z0[m] = fmaf(q0.x, k.x, fmaf(q0.y, k.y, fmaf(q0.z, k.z, fmaf(q0.w, k.w, z0[m]))));
                    z1[m] = fmaf(q1.x, k.x, fmaf(q1.y, k.y, fmaf(q1.z, k.z, fmaf(q1.w, k.w, z1[m]))));
                    v0[m] = fmaf(g0.x, v.x, fmaf(g0.y, v.y, fmaf(g0.z, v.z, fmaf(g0.w, v.w, v0[m]))));
                    v1[m] = fmaf(g1.x, v.x, fmaf(g1.y, v.y, fmaf(g1.z, v.z, fmaf(g1.w, v.w, v1[m]))));
                }
            }
            // softmax over the chunk's keys, e = sum_u P_u GV_u, dZ and w P of one row
            auto finish = [&](float (&z)[KPT], const float (&gv)[KPT], int rr) {
                float mx = z[0];
#pragma unroll
                for (int m = 1; m < KPT; ++m) mx = fmaxf(mx, z[m]);
                mx = warp_max(mx);
                float l = 0.f;
#pragma unroll
                for (int m = 0; m < KPT; ++m) {
                    z[m] = exp2f((z[m] - mx) * scale_log2);
                    l += z[m];
                }
                const float inv = 1.f / warp_sum(l);
                float ev = 0.f;
#pragma unroll
                for (int m = 0; m < KPT; ++m) {
                    z[m] *= inv;
                    ev = fmaf(z[m], gv[m], ev);
                }
                ev = warp_sum(ev);
                const float w = s_w[rr], ws = w * a.scale;
#pragma unroll
                for (int m = 0; m < KPT; ++m) {
                    sZ[rr * SP + lane + 32 * m] = ws * z[m] * (gv[m] - ev);
                    sPw[rr * SP + lane + 32 * m] = w * z[m];
                }
                if (lane == 0) a.e[s_e[rr]] = ev;
            };
            finish(z0, v0, warp);
            if (warp + 16 < nrow) finish(z1, v1, warp + 16);
        }
        __syncthreads();

        // ---- dQ of rows warp, warp + 16 (columns lane * CPL ..)
        if (warp < nrow) {
            float d0[CPL], d1[CPL];
#pragma unroll
            for (int x = 0; x < CPL; ++x) d0[x] = d1[x] = 0.f;
            const bool two = warp + 16 < nrow;
#pragma unroll 4
            for (int u = 0; u < S; ++u) {
                Cols<CPL> k;
                k.load(sK + u * KP + lane * CPL);
                const float za = sZ[warp * SP + u], zb = two ? sZ[(warp + 16) * SP + u] : 0.f;
#pragma unroll
                for (int x = 0; x < CPL; ++x) {
                    d0[x] = fmaf(za, k.v[x], d0[x]);
                    d1[x] = fmaf(zb, k.v[x], d1[x]);
                }
            }
            Cols<CPL> o;
#pragma unroll
            for (int x = 0; x < CPL; ++x) o.v[x] = d0[x];
            o.red(dQ + s_qoff[warp] + lane * CPL);
            if (two) {
#pragma unroll
                for (int x = 0; x < CPL; ++x) o.v[x] = d1[x];
                o.red(dQ + s_qoff[warp + 16] + lane * CPL);
            }
        }
        // ---- dK_u += sum_r dZ[r][u] q_r, dV_u += sum_r wP[r][u] dO_r  (keys warp + 16 m)
        for (int rr = 0; rr < nrow; ++rr) {
            Cols<CPL> qv, gv;
            qv.load(sq + rr * KP + lane * CPL);
            gv.load(sg + rr * KP + lane * CPL);
#pragma unroll
            for (int m = 0; m < UPW; ++m) {
                const float zz = sZ[rr * SP + warp + 16 * m], pw = sPw[rr * SP + warp + 16 * m];
#pragma unroll
                for (int x = 0; x < CPL; ++x) {
                    accK[m][x] = fmaf(zz, qv.v[x], accK[m][x]);
                    accV[m][x] = fmaf(pw, gv.v[x], accV[m][x]);
                }
            }
        }
        __syncthreads();
    }
    if (cur >= 0) flush();
}

// ---------------------------------------------------------------------------- fusion softmax backward

constexpr int NT_FUSE = 256;   // 8 warps, one selection row each

// CPL consecutive stored values of a row (this lane's columns) as fp32, one vector load.
template <int CPL> __device__ __forceinline__ void load_cols(const float *p, float (&o)[CPL]) {
    if constexpr (CPL == 4) {
        const float4 v = __ldg(reinterpret_cast<const float4 *>(p));
        o[0] = v.x, o[1] = v.y, o[2] = v.z, o[3] = v.w;
    } else {
        const float2 v = __ldg(reinterpret_cast<const float2 *>(p));
        o[0] = v.x, o[1] = v.y;
    }
}
template <int CPL> __device__ __forceinline__ void load_cols(const __nv_bfloat16 *p, float (&o)[CPL]) {
    if constexpr (CPL == 4) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.x));
        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v.y));
        o[0] = f0.x, o[1] = f0.y, o[2] = f1.x, o[3] = f1.y;
    } else {
        const uint32_t v = __ldg(reinterpret_cast<const unsigned int *>(p));
        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&v));
        o[0] = f0.x, o[1] = f0.y;
    }
}

// Per selection row: dw_i = sum_h e_hi, ds_i = w_i (dw_i - sum w dw); then
// dQ_h += sum_i ds_i L_ci for every head of the group, dL_ci += ds_i sum_h q_h.
template <typename T, int D>
__global__ void __launch_bounds__(NT_FUSE) bwd_fuse_kernel(BwdArgs a, int Lc, const T *__restrict__ Q,
                                                           const T *__restrict__ L, float *__restrict__ dQ) {
    constexpr int CPL = D / 32;
    const int lane = threadIdx.x & 31;
    const long long r = (long long)blockIdx.x * (NT_FUSE / 32) + (threadIdx.x >> 5);
    if (r >= a.rows) return;
    const int j = (int)(r % a.Hkv);
    const long long bt = r / a.Hkv;
    const int t = (int)(bt % a.Tq), b = (int)(bt / a.Tq);
    int ke = a.keff[r];
    ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
    if (ke == 0) return;
    const long long nc = ncand_of(a, t);
    float w = 0.f, dw = 0.f;
    int c = -1;
    if (lane < ke) {
        c = a.idx[r * a.kmax + lane];
        if (c >= 0 && c < nc) {
            w = a.w[r * a.kmax + lane];
            const float *e = a.e + (r * a.kmax + lane) * a.G;
            for (int g = 0; g < a.G; ++g) dw += e[g];
        } else {
            c = -1;
        }
    }
    const float wdw = warp_sum(w * dw);
    const float ds = w * (dw - wdw);
    // sum of the group's query rows, this lane's columns
    float qs[CPL];
#pragma unroll
    for (int x = 0; x < CPL; ++x) qs[x] = 0.f;
    // (one row at a time: the kernel relies on occupancy, eight CTAs of low register use per SM,
    // to hide the loads' latency; batching them in registers measured slower)
    const T *qrow = Q + (bt * a.H + (long long)j * a.G) * D + lane * CPL;
    for (int g = 0; g < a.G; ++g) {
        float qv[CPL];
        load_cols<CPL>(qrow + (long long)g * D, qv);
#pragma unroll
        for (int x = 0; x < CPL; ++x) qs[x] += qv[x];
    }
    float dq[CPL];
#pragma unroll
    for (int x = 0; x < CPL; ++x) dq[x] = 0.f;
    for (int i = 0; i < ke; ++i) {
        const float dsi = __shfl_sync(FULL, ds, i);
        const int ci = __shfl_sync(FULL, c, i);
        if (ci < 0) continue;   // warp-uniform
        float lv[CPL];
        load_cols<CPL>(L + (((long long)b * a.Hkv + j) * Lc + ci) * D + lane * CPL, lv);
        Cols<CPL> o;
#pragma unroll
        for (int x = 0; x < CPL; ++x) {
            dq[x] = fmaf(dsi, lv[x], dq[x]);
            o.v[x] = dsi * qs[x];
        }
        o.red(a.dL + (((long long)b * a.Hkv + j) * a.C + ci) * D + lane * CPL);
    }
    Cols<CPL> o;
#pragma unroll
    for (int x = 0; x < CPL; ++x) o.v[x] = dq[x];
    for (int g = 0; g < a.G; ++g) o.red(dQ + (bt * a.H + (long long)j * a.G + g) * D + lane * CPL);
}

// ---------------------------------------------------------------------------- landmark backward

constexpr int NT_LM = 256;

template <int D> struct LmShape {
    static constexpr int WP = D + 1;   // W_L row pitch in shared memory (conflict-free column walks)
    static constexpr int PARTS = NT_LM / D;
    static constexpr size_t smem = sizeof(float) * ((size_t)D * WP + 3 * (size_t)D + (size_t)PARTS * D);
};

// Every complete chunk (b, j, c) with a nonzero landmark gradient: its key
// mean m_c, dW_L += m_c^T dL_c (a per-CTA partial in registers, added once),
// and dL_c W_L^T / S added to the gradients of its S keys.  Each chunk has one
// CTA, and the attention kernels that also add into dK have finished, so the
// key gradients are updated with plain loads and stores.
template <typename T, int D>
__global__ void __launch_bounds__(NT_LM) bwd_landmark_kernel(BwdArgs a, const T *__restrict__ K,
                                                             const T *__restrict__ W, float *__restrict__ dK,
                                                             float *__restrict__ dW) {
    using SH = LmShape<D>;
    constexpr int WP = SH::WP, PARTS = SH::PARTS, CPL = D / 32, XPW = D / (NT_LM / 32);
    extern __shared__ float4 smem4[];
    float *sW = reinterpret_cast<float *>(smem4);
    float *sdl = sW + D * WP;
    float *sm = sdl + D;
    float *sdm = sm + D;
    float *spart = sdm + D;   // [PARTS][D]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = threadIdx.x; i < D * D; i += NT_LM) sW[(i / D) * WP + (i % D)] = to_f32(W[i]);
    float acc[XPW][CPL];   // dW_L rows warp + 8 a, columns lane * CPL + x
#pragma unroll
    for (int q = 0; q < XPW; ++q)
#pragma unroll
        for (int x = 0; x < CPL; ++x) acc[q][x] = 0.f;
    const long long nch = (long long)a.B * a.Hkv * a.C;
    const long long lo = nch * blockIdx.x / gridDim.x, hi = nch * (blockIdx.x + 1) / gridDim.x;
    const int xcol = threadIdx.x % D, part = threadIdx.x / D;
    __syncthreads();
    for (long long ch = lo; ch < hi; ++ch) {
        const int c = (int)(ch % a.C);
        const long long bj = ch / a.C;
        const int j = (int)(bj % a.Hkv), b = (int)(bj / a.Hkv);
        float v = 0.f;
        if (threadIdx.x < D) {
            v = a.dL[ch * D + threadIdx.x];
            sdl[threadIdx.x] = v;
        }
        if (!__syncthreads_or(v != 0.f)) continue;   // never kept by any row: nothing to add
        const long long row0 = ((long long)b * a.Tcap + (long long)c * a.S) * a.Hkv + j;
        float ps = 0.f, pm = 0.f;
        // this thread's column of the chunk's keys, eight rows' loads in flight (summed in row order)
        for (int u0 = part; u0 < a.S; u0 += 8 * PARTS) {
            float kv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int u = u0 + q * PARTS;
                kv[q] = u < a.S ? to_f32(K[(row0 + (long long)u * a.Hkv) * D + xcol]) : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q)
                if (u0 + q * PARTS < a.S) ps += kv[q];
        }
        for (int f = part; f < D; f += PARTS) pm = fmaf(sdl[f], sW[xcol * WP + f], pm);
        spart[part * D + xcol] = ps;
        __syncthreads();
        if (threadIdx.x < D) {
            float m = 0.f;
            for (int q = 0; q < PARTS; ++q) m += spart[q * D + threadIdx.x];
            sm[threadIdx.x] = m / (float)a.S;
        }
        __syncthreads();
        spart[part * D + xcol] = pm;
        __syncthreads();
        if (threadIdx.x < D) {
            float m = 0.f;
            for (int q = 0; q < PARTS; ++q) m += spart[q * D + threadIdx.x];
            sdm[threadIdx.x] = m / (float)a.S;
        }
        __syncthreads();
        // the keys' gradients += dL_c W_L^T / S, eight read-modify-writes in flight per thread
        for (int i0 = threadIdx.x; i0 < a.S * D; i0 += 8 * NT_LM) {
            float kv[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = i0 + q * NT_LM, u = i / D, x = i - u * D;
                kv[q] = i < a.S * D ? dK[(row0 + (long long)u * a.Hkv) * D + x] : 0.f;
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = i0 + q * NT_LM, u = i / D, x = i - u * D;
                if (i < a.S * D) dK[(row0 + (long long)u * a.Hkv) * D + x] = kv[q] + sdm[x];
            }
        }
#pragma unroll
        for (int q = 0; q < XPW; ++q) {
            const float mx = sm[warp + 8 * q];
#pragma unroll
            for (int x = 0; x < CPL; ++x) acc[q][x] = fmaf(mx, sdl[lane * CPL + x], acc[q][x]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int q = 0; q < XPW; ++q) {
        Cols<CPL> o;
#pragma unroll
        for (int x = 0; x < CPL; ++x) o.v[x] = acc[q][x];
        o.red(dW + (long long)(warp + 8 * q) * D + lane * CPL);
    }
}

// ---------------------------------------------------------------------------- tensor-core attention backward
//
// bf16, d = 128, used for S = 128 (S = 64 runs the warp-specialized bwd_tcw_kernel below, which
// needs TMEM columns this one spends on S = 128).  One CTA of 128 threads per SM; thread r is
// tile row r and TMEM lane r.  A tile is up to 128 query-head rows that kept
// one chunk (128 / G pairs).  Per tile, issued by thread 0 on tcgen05 with
// fp32 accumulators in TMEM:
//   Z   = Q K^T,  GV = dO V^T          M128 x N=S x K=d   (both operands K-major)
//   (threads: P = softmax(Z / sqrt d), e = P . GV, dZ = w P (GV - e) / sqrt d, wP;
//    dZ and wP rounded to bf16 into shared memory, as P is in the forward)
//   dQ   = dZ K                        M128 x N=d x K=S   (dZ K-major, K MN-major)
//   dK^T += Q^T dZ,  dV^T += dO^T wP   M=d x N=S x K=128 rows (both MN-major: the
//                                      same swizzled tiles read transposed)
// dK^T and dV^T stay in TMEM for a bucket's run of tiles and are added to
// memory (fp32 reductions, one key per column) when the bucket changes; dQ
// is added per tile through a staging buffer so each reduction covers whole
// 128-byte row segments.  TMEM columns: Z [0, S), GV [S, 2S), dQ [0, 128)
// (over Z and GV, which are read before dQ is issued), dK^T [2S, 3S), dV^T
// [3S, 4S).  Shared tiles use the 128-byte swizzle of the forward kernel
// (rows of 64 bf16, 8-row groups 1024 B apart, 16-byte chunk c of row r at
// c ^ (r & 7)).  With one Q / dO buffer (S = 128) the next tile is gathered
// after this tile's MMAs have read its rows.

constexpr int BT_ROWS = 128;
constexpr int BT_PITCH = 36;   // dQ staging pitch (floats)

struct BwdTcBars {
    uint64_t zg, mma2, done;
    uint32_t tmem;
    int abort;
};

template <int S> struct BwdTcShape {
    static constexpr int NQB = S == 64 ? 2 : 1;   // Q / dO buffers
    static constexpr int KVB = S * 128;           // one 64-column box of S rows
    static constexpr int PB = (S / 64) * 16384;   // one [128][S] bf16 tile
    static constexpr int TMEM_COLS = 4 * S;
    static constexpr size_t smem = 1024 + (size_t)NQB * 2 * 32768 + 4 * (size_t)KVB + 2 * (size_t)PB +
                                   4 * 32 * BT_PITCH * sizeof(float) + (size_t)NQB * BT_ROWS * sizeof(long long) +
                                   sizeof(BwdTcBars);
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
// arrive on *bar once this thread's earlier cp.async copies have landed (no pending-count increment)
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(sm100::smem_u32(bar)) : "memory");
}

// (batch, kv head, chunk) of a bucket index (b * Hkv + j) * C + c
struct BucketPos {
    int b, j, c;
};
__device__ __forceinline__ BucketPos bucket_pos(const BwdArgs &a, int bucket) {
    BucketPos q;
    q.c = bucket % a.C;
    const int bj = bucket / a.C;
    q.j = bj % a.Hkv;
    q.b = bj / a.Hkv;
    return q;
}

template <int S>
__global__ void __launch_bounds__(BT_ROWS, 1)
    bwd_tc_kernel(BwdArgs a, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                  const __nv_bfloat16 *__restrict__ V, const __nv_bfloat16 *__restrict__ dO,
                  float *__restrict__ dQ, float *__restrict__ dK, float *__restrict__ dV) {
    using namespace sm100;
    using SH = BwdTcShape<S>;
    constexpr int NQB = SH::NQB, KVB = SH::KVB, PB = SH::PB, D = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                       // NQB x 32 KB: two 64-dim boxes of 128 rows
    uint8_t *sG = sQ + NQB * 32768;           // dO, same layout
    uint8_t *sK = sG + NQB * 32768;           // two boxes of S rows
    uint8_t *sV = sK + 2 * KVB;
    uint8_t *sZ = sV + 2 * KVB;               // dZ, bf16 [128][S]
    uint8_t *sP = sZ + PB;                    // w P, bf16 [128][S]
    float *stg = reinterpret_cast<float *>(sP + PB);                          // 4 warps x 32 x BT_PITCH
    long long *s_qoff = reinterpret_cast<long long *>(stg + 4 * 32 * BT_PITCH);   // [NQB][128]
    BwdTcBars *bar = reinterpret_cast<BwdTcBars *>(s_qoff + NQB * BT_ROWS);
    volatile int *abort = &bar->abort;
    const int r = threadIdx.x, warp = r >> 5, lane = r & 31;
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    const int ntiles = *a.ntiles;
    const int lo = (int)((long long)ntiles * blockIdx.x / gridDim.x);
    const int hi = (int)((long long)ntiles * (blockIdx.x + 1) / gridDim.x);
    if (lo >= hi) return;
    const float scale_log2 = a.scale * 1.4426950408889634f;

    if (r == 0) {
        mbar_init(&bar->zg, 1);
        mbar_init(&bar->mma2, 1);
        mbar_init(&bar->done, 1);
        bar->abort = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        tmem_alloc(&bar->tmem, SH::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem;

    // Tile ti's Q / dO rows into buffer qb (zero rows past the tile).  Each thread first looks up
    // its own row (and keeps that row's fusion weight and e slot); then the copies are dealt so
    // that 16 consecutive lanes copy one row's 256 contiguous bytes, two rows per warp
    // instruction, instead of one row per lane.
    auto gather = [&](int ti, int qb, float &w_o, int &e_o) {
        const int4 tr = a.tiles[ti];
        const int nrow = tr.z * a.G;
        const int j = (tr.x / a.C) % a.Hkv;
        long long qoff = -1;
        w_o = 0.f;
        e_o = -1;
        if (r < nrow) {
            const int pc = (int)dbg_clamp(a.pairs[tr.y + r / a.G], 0, a.rows * a.kmax, a.status), g = r % a.G;
            const long long bt = (long long)(pc / a.kmax) / a.Hkv;
            qoff = (bt * a.H + (long long)j * a.G + g) * D;
            w_o = a.w[pc];
            e_o = pc * a.G + g;
        }
        s_qoff[qb * BT_ROWS + r] = qoff;
        __syncthreads();
        const char *q8 = reinterpret_cast<const char *>(Q), *g8 = reinterpret_cast<const char *>(dO);
        const uint32_t bq = smem_u32(sQ + qb * 32768), bg = smem_u32(sG + qb * 32768);
#pragma unroll 4
        for (int k = 0; k < 16; ++k) {
            const int idx = r + BT_ROWS * k, row = idx >> 4, x = idx & 15;
            const long long off = s_qoff[qb * BT_ROWS + row];
            const uint32_t nb = off >= 0 ? 16u : 0u;
            const long long src = off >= 0 ? off * 2 + x * 16 : 0;
            const uint32_t o = (x >> 3) * 16384 + (row >> 3) * 1024 + (row & 7) * 128 + (((x & 7) ^ (row & 7)) << 4);
            cp_async16(bq + o, q8 + src, nb);
            cp_async16(bg + o, g8 + src, nb);
        }
    };
    // K_c and V_c of a bucket into the two box pairs
    auto load_kv = [&](int bucket) {
        const int c = bucket % a.C, bj = bucket / a.C, j = bj % a.Hkv, b = bj / a.Hkv;
        const long long row0 = ((long long)b * a.Tcap + (long long)c * S) * a.Hkv + j;
        for (int i = r; i < S * 16; i += BT_ROWS) {
            const int u = i >> 4, x = i & 15;
            const uint32_t o = (x >> 3) * KVB + (u >> 3) * 1024 + (u & 7) * 128 + (((x & 7) ^ (u & 7)) << 4);
            const long long src = (row0 + (long long)u * a.Hkv) * D + x * 8;
            cp_async16(smem_u32(sK) + o, K + src, 16u);
            cp_async16(smem_u32(sV) + o, V + src, 16u);
        }
    };
    // dK^T and dV^T of the finished bucket -> memory (lane r = dimension r; one key per column)
    auto drain_kv = [&](int bucket) {
        const int c = bucket % a.C, bj = bucket / a.C, j = bj % a.Hkv, b = bj / a.Hkv;
        const long long row0 = ((long long)b * a.Tcap + (long long)c * S) * a.Hkv + j;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
            float *dst = h ? dV : dK;
#pragma unroll 1
            for (int q = 0; q < S / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + (2 + h) * S + q * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float *pd = dst + (row0 + (long long)(q * 32 + e) * a.Hkv) * D + r;
                    asm volatile("red.global.add.f32 [%0], %1;" ::"l"(pd), "f"(__uint_as_float(v[e])) : "memory");
                }
            }
        }
    };

    const uint32_t idesc_zg = idesc_bf16_f32(128, S, 0, 0);
    const uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
    const uint32_t idesc_kv = idesc_bf16_f32(128, S, 1, 1);
    float w_c, w_n = 0.f;
    int e_c, e_n = -1;
    int bucket = a.tiles[lo].x;
    load_kv(bucket);
    gather(lo, 0, w_c, e_c);
    cp_async_wait_all();
    fence_proxy_async_smem();
    __syncthreads();
    bool first = true;   // first tile of the bucket run: dK^T / dV^T start from zero
    int i = 0;
    for (int ti = lo; ti < hi; ++ti, ++i) {
        const int qb = NQB == 2 ? (i & 1) : 0;
        const bool has_next = ti + 1 < hi;
        const int nbucket = has_next ? a.tiles[ti + 1].x : -1;
        // ---- Z = Q K^T, GV = dO V^T
        if (r == 0) {
            tc_fence_after();
            const uint32_t qa = smem_u32(sQ + qb * 32768), ga = smem_u32(sG + qb * 32768);
            const uint32_t kb = smem_u32(sK), vb = smem_u32(sV);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32, bo = (kk >> 2) * KVB + (kk & 3) * 32;
                umma_bf16(tmem, desc_kmajor_sw128(qa + ao), desc_kmajor_sw128(kb + bo), idesc_zg, kk != 0);
                umma_bf16(tmem + S, desc_kmajor_sw128(ga + ao), desc_kmajor_sw128(vb + bo), idesc_zg, kk != 0);
            }
            umma_commit(&bar->zg);
        }
        if (NQB == 2 && has_next) gather(ti + 1, qb ^ 1, w_n, e_n);
        if (!__syncthreads_and(mbar_wait(&bar->zg, i & 1, abort, a.status))) break;
        tc_fence_after();
        // ---- row softmax, e, dZ and w P (this thread's row)
        {
            float p[S];
            float mx = -INFINITY;
#pragma unroll
            for (int q = 0; q < S / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + q * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    p[q * 32 + e] = __uint_as_float(v[e]);
                    mx = fmaxf(mx, p[q * 32 + e]);
                }
            }
            float l = 0.f;
#pragma unroll
            for (int u = 0; u < S; ++u) {
                p[u] = exp2f((p[u] - mx) * scale_log2);
                l += p[u];
            }
            const float inv = 1.f / l;
            float ev = 0.f;
#pragma unroll
            for (int q = 0; q < S / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + S + q * 32, v);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    p[q * 32 + e] *= inv;
                    ev = fmaf(p[q * 32 + e], __uint_as_float(v[e]), ev);
                }
            }
            if (e_c >= 0) a.e[e_c] = ev;
            const float ws = w_c * a.scale;
#pragma unroll
            for (int q = 0; q < S / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + S + q * 32, v);
                tmem_wait_ld();
                uint32_t zk[16], pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float p0 = p[q * 32 + 2 * e], p1 = p[q * 32 + 2 * e + 1];
                    __nv_bfloat162 hz = __floats2bfloat162_rn(ws * p0 * (__uint_as_float(v[2 * e]) - ev),
                                                              ws * p1 * (__uint_as_float(v[2 * e + 1]) - ev));
                    __nv_bfloat162 hp = __floats2bfloat162_rn(w_c * p0, w_c * p1);
                    zk[e] = *reinterpret_cast<uint32_t *>(&hz);
                    pk[e] = *reinterpret_cast<uint32_t *>(&hp);
                }
                const int ro = (q >> 1) * 16384 + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int cx = (q & 1) * 4 + x, o = ro + ((cx ^ (r & 7)) << 4);
                    *reinterpret_cast<uint4 *>(sZ + o) = make_uint4(zk[4 * x], zk[4 * x + 1], zk[4 * x + 2], zk[4 * x + 3]);
                    *reinterpret_cast<uint4 *>(sP + o) = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        // ---- dQ = dZ K, dK^T += Q^T dZ, dV^T += dO^T wP
        if (r == 0) {
            tc_fence_after();
            const uint32_t za = smem_u32(sZ), pa = smem_u32(sP), kb = smem_u32(sK);
            const uint32_t qa = smem_u32(sQ + qb * 32768), ga = smem_u32(sG + qb * 32768);
#pragma unroll
            for (int kk = 0; kk < S / 16; ++kk)
                umma_bf16(tmem, desc_kmajor_sw128(za + (kk >> 2) * 16384 + (kk & 3) * 32),
                          desc_mnmajor_sw128(kb + kk * 2048, KVB, 1024), idesc_dq, kk != 0);
#pragma unroll
            for (int kk = 0; kk < BT_ROWS / 16; ++kk) {
                const uint32_t acc = (kk != 0 || !first) ? 1u : 0u;
                umma_bf16(tmem + 2 * S, desc_mnmajor_sw128(qa + kk * 2048, 16384, 1024),
                          desc_mnmajor_sw128(za + kk * 2048, 16384, 1024), idesc_kv, acc);
                umma_bf16(tmem + 3 * S, desc_mnmajor_sw128(ga + kk * 2048, 16384, 1024),
                          desc_mnmajor_sw128(pa + kk * 2048, 16384, 1024), idesc_kv, acc);
            }
            umma_commit(&bar->mma2);
        }
        if (!__syncthreads_and(mbar_wait(&bar->mma2, i & 1, abort, a.status))) break;
        tc_fence_after();
        // ---- dQ rows -> memory, 32 columns at a time through the warp's staging rows
        {
            float *wst = stg + warp * 32 * BT_PITCH;
            long long dst[8];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) dst[rr] = s_qoff[qb * BT_ROWS + warp * 32 + rr * 4 + (lane >> 3)];
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + q * 32, v);
                tmem_wait_ld();
                float *mine = wst + lane * BT_PITCH;
#pragma unroll
                for (int e = 0; e < 32; e += 4)
                    *reinterpret_cast<float4 *>(mine + e) = make_float4(__uint_as_float(v[e]), __uint_as_float(v[e + 1]),
                                                                        __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    if (dst[rr] >= 0) {
                        const int lr = rr * 4 + (lane >> 3);
                        red_add4(dQ + dst[rr] + q * 32 + 4 * (lane & 7),
                                 *reinterpret_cast<const float4 *>(wst + lr * BT_PITCH + 4 * (lane & 7)));
                    }
                }
                __syncwarp();
            }
        }
        first = nbucket != bucket;
        if (first) drain_kv(bucket);
        if (has_next) {
            if (NQB == 1) gather(ti + 1, 0, w_n, e_n);
            if (nbucket != bucket) load_kv(nbucket);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        bucket = nbucket;
        w_c = w_n;
        e_c = e_n;
    }
    cp_async_wait_all();
    // wind down: every MMA issued has completed before TMEM is released
    if (r == 0) {
        umma_commit(&bar->done);
        mbar_drain(&bar->done, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, SH::TMEM_COLS);
    }
}

// ---------------------------------------------------------------------------- warp-specialized tensor-core backward (S = 64)
//
// The tile steps of bwd_tc_kernel, with roles that overlap from tile to tile:
//   warps 0-3   producers: each tile's row info (query offset, fusion weight, e slot) into a ring
//               of NWI slots, the Q / dO rows into one of two buffers (16 lanes per 256-byte row),
//               and K / V once per chunk run
//   warps 4-7   softmax: P, e, dZ and w P of tile i (thread = TMEM lane = row)
//   warps 8-11  drain: dQ of every tile through the staging rows, dK^T / dV^T at a run's end
//   warp 12     one thread issues the MMAs
// TMEM: Z [0, 64), GV [64, 128), dQ of tile parity b at [128 + 128 b, 256 + 128 b), dK^T
// [384, 448), dV^T [448, 512).  dQ is double-buffered, so the MMAs of tile i+1 need not wait for
// the drain of tile i: the softmax of tile i+1 runs while the drain reduces dQ of tile i and the
// producers gather tile i+2.  Each barrier has one group of waiters that waits its phases in
// order, and every wait is bounded.

constexpr int NW_P = 4, NW_S = 4, NW_D = 4;
constexpr int NT_W = 32 * (NW_P + NW_S + NW_D + 1);
constexpr int NWI = 4;   // row-info ring slots

struct BwInfo {
    long long qoff[BT_ROWS];
    float w[BT_ROWS];
    int e[BT_ROWS];
};

struct BwBars {
    uint64_t q_full[2], q_empty[2], kv_full, kv_empty, zg_full, zg_empty, ds_full, ds_empty, dq_full[2], dq_empty[2];
    uint64_t info_full[NWI], info_empty[NWI], done;
    uint32_t tmem;
    int abort;
};

constexpr size_t BW_SMEM = 1024 + 4 * 32768 + 4 * 8192 + 2 * 16384 + NW_D * 32 * BT_PITCH * sizeof(float) +
                           NWI * sizeof(BwInfo) + sizeof(BwBars);

__global__ void __launch_bounds__(NT_W, 1)
    bwd_tcw_kernel(BwdArgs a, const __nv_bfloat16 *__restrict__ Q, const __nv_bfloat16 *__restrict__ K,
                   const __nv_bfloat16 *__restrict__ V, const __nv_bfloat16 *__restrict__ dO,
                   float *__restrict__ dQ, float *__restrict__ dK, float *__restrict__ dV) {
    using namespace sm100;
    constexpr int S = 64, D = 128, KVB = S * 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sQ = base;                    // 2 x 32 KB
    uint8_t *sG = sQ + 2 * 32768;          // 2 x 32 KB
    uint8_t *sK = sG + 2 * 32768;          // two boxes of S rows
    uint8_t *sV = sK + 2 * KVB;
    uint8_t *sZ = sV + 2 * KVB;            // dZ, bf16 [128][64]
    uint8_t *sP = sZ + 16384;              // w P
    float *stg = reinterpret_cast<float *>(sP + 16384);
    BwInfo *info = reinterpret_cast<BwInfo *>(stg + NW_D * 32 * BT_PITCH);
    BwBars *bar = reinterpret_cast<BwBars *>(info + NWI);
    volatile int *abort = &bar->abort;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ntiles = *a.ntiles;
    const int lo = (int)((long long)ntiles * blockIdx.x / gridDim.x);
    const int hi = (int)((long long)ntiles * (blockIdx.x + 1) / gridDim.x);
    const int n = hi - lo;
    if (n <= 0) return;
    const float scale_log2 = a.scale * 1.4426950408889634f;

    if (threadIdx.x == 0) {
        for (int q = 0; q < 2; ++q) {
            mbar_init(&bar->q_full[q], 32 * NW_P);
            mbar_init(&bar->q_empty[q], 1);
            mbar_init(&bar->dq_full[q], 1);
            mbar_init(&bar->dq_empty[q], NW_D);
        }
        mbar_init(&bar->zg_full, 1);
        mbar_init(&bar->zg_empty, NW_S);
        mbar_init(&bar->kv_full, 32 * NW_P);
        mbar_init(&bar->kv_empty, 1);
        mbar_init(&bar->ds_full, NW_S);
        mbar_init(&bar->ds_empty, 1);
        for (int q = 0; q < NWI; ++q) {
            mbar_init(&bar->info_full[q], NW_P);
            mbar_init(&bar->info_empty[q], NW_D);
        }
        mbar_init(&bar->done, 1);
        bar->abort = 0;
        fence_mbar_init();
    }
    if (warp == NW_P + NW_S + NW_D) {
        tmem_alloc(&bar->tmem, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = bar->tmem;
    auto bucket_at = [&](int i) -> int { return i < n ? a.tiles[lo + i].x : -1; };
    auto wait_all = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(FULL, mbar_wait(b, par, abort, a.status) ? 1 : 0) != 0;
    };

    if (warp < NW_P) {
        // ------------------------------------------------------------ producers
        const int pr = threadIdx.x;   // this thread's row of each tile
        int prev = -1, nload = 0;
        int4 tr_next = a.tiles[lo];
        for (int i = 0; i < n; ++i) {
            const int b = i & 1, si = i % NWI;
            const int4 tr = tr_next;
            if (i + 1 < n) tr_next = a.tiles[lo + i + 1];   // read a tile ahead
            if (tr.x != prev) {
                // K / V of a new chunk run, once the previous run's last MMAs have released them
                if (nload > 0 && !wait_all(&bar->kv_empty, (nload - 1) & 1)) break;
                const BucketPos bp = bucket_pos(a, tr.x);
                const long long row0 = ((long long)bp.b * a.Tcap + (long long)bp.c * S) * a.Hkv + bp.j;
                for (int q = pr; q < S * 16; q += 32 * NW_P) {
                    const int u = q >> 4, x = q & 15;
                    const uint32_t o = (x >> 3) * KVB + (u >> 3) * 1024 + (u & 7) * 128 + (((x & 7) ^ (u & 7)) << 4);
                    const long long src = (row0 + (long long)u * a.Hkv) * D + x * 8;
                    cp_async16(smem_u32(sK) + o, K + src, 16u);
                    cp_async16(smem_u32(sV) + o, V + src, 16u);
                }
                cp_async_arrive(&bar->kv_full);
                ++nload;
                prev = tr.x;
            }
            if (i >= 2 && !wait_all(&bar->q_empty[b], ((i >> 1) - 1) & 1)) break;
            if (i >= NWI && !wait_all(&bar->info_empty[si], ((i / NWI) - 1) & 1)) break;
            long long qoff = -1;
            float w = 0.f;
            int e = -1;
            if (pr < tr.z * a.G) {
                const int pc = (int)dbg_clamp(a.pairs[tr.y + pr / a.G], 0, a.rows * a.kmax, a.status), g = pr % a.G;
                w = a.pair_w[tr.y + pr / a.G];
                const long long bt = (long long)(pc / a.kmax) / a.Hkv;
                qoff = (bt * a.H + (long long)bucket_pos(a, tr.x).j * a.G + g) * D;
                e = pc * a.G + g;
            }
            info[si].qoff[pr] = qoff;
            info[si].w[pr] = w;
            info[si].e[pr] = e;
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->info_full[si]);
            // this warp's 32 rows, 16 lanes per row
            const char *q8 = reinterpret_cast<const char *>(Q), *g8 = reinterpret_cast<const char *>(dO);
            const uint32_t bq = smem_u32(sQ + b * 32768), bg = smem_u32(sG + b * 32768);
#pragma unroll 4
            for (int k = 0; k < 16; ++k) {
                const int rr = 2 * k + (lane >> 4), x = lane & 15;
                const long long off = __shfl_sync(FULL, qoff, rr);
                const int row = warp * 32 + rr;
                const uint32_t nb = off >= 0 ? 16u : 0u;
                const long long src = off >= 0 ? off * 2 + x * 16 : 0;
                const uint32_t o = (x >> 3) * 16384 + (row >> 3) * 1024 + (row & 7) * 128 + (((x & 7) ^ (row & 7)) << 4);
                cp_async16(bq + o, q8 + src, nb);
                cp_async16(bg + o, g8 + src, nb);
            }
            cp_async_arrive(&bar->q_full[b]);
        }
        cp_async_wait_all();
    } else if (warp < NW_P + NW_S) {
        // ------------------------------------------------------------ softmax
        const int quad = warp & 3, row = quad * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        for (int i = 0; i < n; ++i) {
            const int b = i & 1, si = i % NWI;
            if (!wait_all(&bar->info_full[si], (i / NWI) & 1)) break;
            const float w = info[si].w[row];
            const int eslot = info[si].e[row];
            if (!wait_all(&bar->zg_full, i & 1)) break;
            tc_fence_after();
            const uint32_t zt = tmem + lane_off, gt = zt + 64;
            float p[S];
            float mx = -INFINITY;
            {
                uint32_t v0[32], v1[32];
                tmem_ld32(zt, v0);
                tmem_ld32(zt + 32, v1);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    p[x] = __uint_as_float(v0[x]);
                    p[32 + x] = __uint_as_float(v1[x]);
                    mx = fmaxf(mx, fmaxf(p[x], p[32 + x]));
                }
            }
            float l = 0.f;
#pragma unroll
            for (int u = 0; u < S; ++u) {
                p[u] = exp2f((p[u] - mx) * scale_log2);
                l += p[u];
            }
            const float inv = 1.f / l;
            float ev = 0.f;
            {
                uint32_t v0[32], v1[32];
                tmem_ld32(gt, v0);
                tmem_ld32(gt + 32, v1);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) {
                    p[x] *= inv;
                    p[32 + x] *= inv;
                    ev = fmaf(p[x], __uint_as_float(v0[x]), ev);
                    ev = fmaf(p[32 + x], __uint_as_float(v1[x]), ev);
                }
            }
            if (eslot >= 0) a.e[eslot] = ev;
            // dZ / w P buffer: free once the previous tile's MMAs have read it
            if (i >= 1 && !wait_all(&bar->ds_empty, (i - 1) & 1)) break;
            const float ws = w * a.scale;
#pragma unroll
            for (int q = 0; q < S / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(gt + q * 32, v);
                tmem_wait_ld();
                uint32_t zk[16], pk[16];
#pragma unroll
                for (int x = 0; x < 16; ++x) {
                    const float p0 = p[q * 32 + 2 * x], p1 = p[q * 32 + 2 * x + 1];
                    __nv_bfloat162 hz = __floats2bfloat162_rn(ws * p0 * (__uint_as_float(v[2 * x]) - ev),
                                                              ws * p1 * (__uint_as_float(v[2 * x + 1]) - ev));
                    __nv_bfloat162 hp = __floats2bfloat162_rn(w * p0, w * p1);
                    zk[x] = *reinterpret_cast<uint32_t *>(&hz);
                    pk[x] = *reinterpret_cast<uint32_t *>(&hp);
                }
                const int ro = (row >> 3) * 1024 + (row & 7) * 128;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int cx = q * 4 + x, o = ro + ((cx ^ (row & 7)) << 4);
                    *reinterpret_cast<uint4 *>(sZ + o) = make_uint4(zk[4 * x], zk[4 * x + 1], zk[4 * x + 2], zk[4 * x + 3]);
                    *reinterpret_cast<uint4 *>(sP + o) = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
                }
            }
            tc_fence_before();
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&bar->zg_empty);
                mbar_arrive(&bar->ds_full);
            }
        }
    } else if (warp < NW_P + NW_S + NW_D) {
        // ------------------------------------------------------------ drain
        const int quad = warp & 3;
        const uint32_t lane_off = (uint32_t)(quad * 32) << 16;
        float *wst = stg + quad * 32 * BT_PITCH;
        int bk_next = bucket_at(0);
        for (int i = 0; i < n; ++i) {
            const int si = i % NWI, bk = bk_next;
            bk_next = bucket_at(i + 1);
            if (!wait_all(&bar->info_full[si], (i / NWI) & 1)) break;
            long long dst[8];
#pragma unroll
            for (int rr = 0; rr < 8; ++rr) dst[rr] = info[si].qoff[quad * 32 + rr * 4 + (lane >> 3)];
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->info_empty[si]);
            if (!wait_all(&bar->dq_full[i & 1], (i >> 1) & 1)) break;
            tc_fence_after();
#pragma unroll 1
            for (int q = 0; q < D / 32; ++q) {
                uint32_t v[32];
                tmem_ld32(tmem + lane_off + 128 + 128 * (i & 1) + q * 32, v);
                tmem_wait_ld();
                float *mine = wst + lane * BT_PITCH;
#pragma unroll
                for (int x = 0; x < 32; x += 4)
                    *reinterpret_cast<float4 *>(mine + x) = make_float4(__uint_as_float(v[x]), __uint_as_float(v[x + 1]),
                                                                        __uint_as_float(v[x + 2]), __uint_as_float(v[x + 3]));
                __syncwarp();
#pragma unroll
                for (int rr = 0; rr < 8; ++rr) {
                    if (dst[rr] >= 0) {
                        const int lr = rr * 4 + (lane >> 3);
                        red_add4(dQ + dst[rr] + q * 32 + 4 * (lane & 7),
                                 *reinterpret_cast<const float4 *>(wst + lr * BT_PITCH + 4 * (lane & 7)));
                    }
                }
                __syncwarp();
            }
            if (bk_next != bk) {
                // end of this CTA's run of the chunk: dK^T / dV^T (lane = dimension) -> memory
                const BucketPos bp = bucket_pos(a, bk);
                const long long row0 = ((long long)bp.b * a.Tcap + (long long)bp.c * S) * a.Hkv + bp.j;
#pragma unroll 1
                for (int h = 0; h < 2; ++h) {
                    float *dstp = h ? dV : dK;
#pragma unroll 1
                    for (int q = 0; q < S / 32; ++q) {
                        uint32_t v[32];
                        tmem_ld32(tmem + lane_off + 384 + h * 64 + q * 32, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 32; ++x) {
                            float *pd = dstp + (row0 + (long long)(q * 32 + x) * a.Hkv) * D + quad * 32 + lane;
                            asm volatile("red.global.add.f32 [%0], %1;" ::"l"(pd), "f"(__uint_as_float(v[x])) : "memory");
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar->dq_empty[i & 1]);
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc_zg = idesc_bf16_f32(128, S, 0, 0);
        const uint32_t idesc_dq = idesc_bf16_f32(128, D, 0, 1);
        const uint32_t idesc_kv = idesc_bf16_f32(128, S, 1, 1);
        const uint32_t kb = smem_u32(sK), vb = smem_u32(sV), za = smem_u32(sZ), pa = smem_u32(sP);
        auto mma1 = [&](int i, bool newc, int li) -> bool {
            const int b = i & 1;
            if (!mbar_wait(&bar->q_full[b], (i >> 1) & 1, abort, a.status)) return false;
            if (newc && !mbar_wait(&bar->kv_full, li & 1, abort, a.status)) return false;
            if (i >= 1 && !mbar_wait(&bar->zg_empty, (i - 1) & 1, abort, a.status)) return false;
            tc_fence_after();
            const uint32_t qa = smem_u32(sQ + b * 32768), ga = smem_u32(sG + b * 32768);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ao = (kk >> 2) * 16384 + (kk & 3) * 32, bo = (kk >> 2) * KVB + (kk & 3) * 32;
                umma_bf16(tmem, desc_kmajor_sw128(qa + ao), desc_kmajor_sw128(kb + bo), idesc_zg, kk != 0);
                umma_bf16(tmem + 64, desc_kmajor_sw128(ga + ao), desc_kmajor_sw128(vb + bo), idesc_zg, kk != 0);
            }
            umma_commit(&bar->zg_full);
            return true;
        };
        auto mma2 = [&](int i, bool first, bool endc) -> bool {
            const int b = i & 1;
            if (!mbar_wait(&bar->ds_full, i & 1, abort, a.status)) return false;
            if (i >= 2 && !mbar_wait(&bar->dq_empty[b], ((i >> 1) - 1) & 1, abort, a.status)) return false;
            tc_fence_after();
            const uint32_t qa = smem_u32(sQ + b * 32768), ga = smem_u32(sG + b * 32768);
#pragma unroll
            for (int kk = 0; kk < S / 16; ++kk)
                umma_bf16(tmem + 128 + 128 * b, desc_kmajor_sw128(za + (kk & 3) * 32),
                          desc_mnmajor_sw128(kb + kk * 2048, KVB, 1024), idesc_dq, kk != 0);
#pragma unroll
            for (int kk = 0; kk < BT_ROWS / 16; ++kk) {
                const uint32_t acc = (kk != 0 || !first) ? 1u : 0u;
                umma_bf16(tmem + 384, desc_mnmajor_sw128(qa + kk * 2048, 16384, 1024),
                          desc_mnmajor_sw128(za + kk * 2048, 16384, 1024), idesc_kv, acc);
                umma_bf16(tmem + 448, desc_mnmajor_sw128(ga + kk * 2048, 16384, 1024),
                          desc_mnmajor_sw128(pa + kk * 2048, 16384, 1024), idesc_kv, acc);
            }
            umma_commit(&bar->dq_full[b]);
            umma_commit(&bar->ds_empty);
            umma_commit(&bar->q_empty[b]);
            if (endc) umma_commit(&bar->kv_empty);
            return true;
        };
        bool ok = true, first_prev = false, end_prev = false;
        int prev = -1, li = -1, bk_next = bucket_at(0), bk_next2 = bucket_at(1);
        for (int i = 0; i < n && ok; ++i) {
            const int bk = bk_next;
            bk_next = bk_next2;
            bk_next2 = bucket_at(i + 2);   // read two tiles ahead
            const bool newc = bk != prev, endc = bk_next != bk;
            if (newc) ++li;
            // at a run boundary the previous tile's MMAs release K / V before the new run's land
            if (i >= 1 && newc) ok = mma2(i - 1, first_prev, end_prev);
            if (ok) ok = mma1(i, newc, li);
            if (ok && i >= 1 && !newc) ok = mma2(i - 1, first_prev, end_prev);
            first_prev = newc;
            end_prev = endc;
            prev = bk;
        }
        if (ok) mma2(n - 1, first_prev, end_prev);
        umma_commit(&bar->done);
        mbar_drain(&bar->done, 0);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == NW_P + NW_S + NW_D) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

template <typename T, int S, int D>
cudaError_t launch_attend_t(const BwdArgs &a, int grid, const void *Q, const void *K, const void *V, const void *dO,
                            float *dQ, float *dK, float *dV, cudaStream_t st) {
    const size_t smem = BwdShape<S, D>::smem;
    cudaError_t e = cudaFuncSetAttribute(bwd_attend_kernel<T, S, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    bwd_attend_kernel<T, S, D><<<grid, NT_BWD, smem, st>>>(a, (const T *)Q, (const T *)K, (const T *)V,
                                                            (const T *)dO, dQ, dK, dV);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_attend_s(const BwdArgs &a, int grid, const void *Q, const void *K, const void *V, const void *dO,
                            float *dQ, float *dK, float *dV, cudaStream_t st) {
    switch (a.S) {
        case 32: return launch_attend_t<T, 32, D>(a, grid, Q, K, V, dO, dQ, dK, dV, st);
        case 64: return launch_attend_t<T, 64, D>(a, grid, Q, K, V, dO, dQ, dK, dV, st);
        default: return launch_attend_t<T, 128, D>(a, grid, Q, K, V, dO, dQ, dK, dV, st);
    }
}

template <typename T, int D>
cudaError_t launch_tail_t(const BwdArgs &a, int Lc, int lm_grid, const void *Q, const void *K, const void *W,
                          const void *L, float *dQ, float *dK, float *dW, cudaStream_t st) {
    const unsigned fuse_grid = (unsigned)((a.rows + NT_FUSE / 32 - 1) / (NT_FUSE / 32));
    bwd_fuse_kernel<T, D><<<fuse_grid, NT_FUSE, 0, st>>>(a, Lc, (const T *)Q, (const T *)L, dQ);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const size_t smem = LmShape<D>::smem;
    e = cudaFuncSetAttribute(bwd_landmark_kernel<T, D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    bwd_landmark_kernel<T, D><<<lm_grid, NT_LM, smem, st>>>(a, (const T *)K, (const T *)W, dK, dW);
    return cudaGetLastError();
}

}  // namespace

BwdLayout backward_layout(const Prob &p) {
    BwdLayout w{};
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += (bytes + 255) & ~(size_t)255;
        return o;
    };
    const size_t pairs = (size_t)p.rows * p.kmax;
    w.tc = p.dtype == HSA_BF16 && p.d == 128 && (p.S == 64 || p.S == 128) && !(p.flags & HSA_FLAG_SIMT);
    w.pt = (w.tc ? BT_ROWS : RT) / p.G;
    w.nbucket = (long long)p.B * p.Hkv * p.C;
    w.max_tiles = (long long)((pairs + w.pt - 1) / w.pt) + w.nbucket;
    w.hdr = take(256);   // status word at 0, tile count at 16
    w.bcount = take((size_t)w.nbucket * sizeof(int32_t));
    w.dL = take((size_t)w.nbucket * p.d * sizeof(float));
    w.clear_bytes = off;
    w.w = take(pairs * sizeof(float));
    w.e = take(pairs * p.G * sizeof(float));
    w.boff = take(((size_t)w.nbucket + 1) * sizeof(int32_t));
    w.btile = take(((size_t)w.nbucket + 1) * sizeof(int32_t));
    w.pairs = take(pairs * sizeof(int32_t));
    w.pair_w = take(pairs * sizeof(float));
    w.tiles = take((size_t)w.max_tiles * sizeof(int4));
    w.total = off;
    return w;
}

bool backward_supported(const Prob &p) {
    const BwdLayout w = backward_layout(p);
    return (long long)p.rows * p.kmax * p.G < (1ll << 31) && w.max_tiles < (1ll << 31) && p.G <= RT;
}

int backward_launches(const Prob &p) { return p.rows > 0 && p.C > 0 ? 7 : 0; }

cudaError_t launch_backward(const Prob &p, const BwdLayout &w, char *ws, int sms, const void *Q, const void *K,
                            const void *V, const void *W, const void *L, const int32_t *idx, const float *score,
                            const int32_t *keff, const void *dO, float *dQ, float *dK, float *dV, float *dW,
                            cudaStream_t st) {
    cudaError_t e;
    const size_t kv_bytes = (size_t)p.B * p.Tcap * p.Hkv * p.d * sizeof(float);
    const size_t q_bytes = (size_t)p.B * p.Tq * p.H * p.d * sizeof(float);
    if (q_bytes && (e = cudaMemsetAsync(dQ, 0, q_bytes, st)) != cudaSuccess) return e;
    if (kv_bytes && (e = cudaMemsetAsync(dK, 0, kv_bytes, st)) != cudaSuccess) return e;
    if (kv_bytes && (e = cudaMemsetAsync(dV, 0, kv_bytes, st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(dW, 0, (size_t)p.d * p.d * sizeof(float), st)) != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(ws, 0, w.clear_bytes, st)) != cudaSuccess) return e;
    if (p.rows == 0 || p.C == 0) return cudaSuccess;
    BwdArgs a;
    a.B = p.B;
    a.Tq = p.Tq;
    a.Tcap = p.Tcap;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.d = p.d;
    a.S = p.S;
    a.C = p.C;
    a.kmax = p.kmax;
    a.pt = w.pt;
    a.q_pos0 = p.q_pos0;
    a.rows = p.rows;
    a.nbucket = w.nbucket;
    a.scale = 1.f / sqrtf((float)p.d);
    a.idx = idx;
    a.keff = keff;
    a.score = score;
    a.w = reinterpret_cast<float *>(ws + w.w);
    a.e = reinterpret_cast<float *>(ws + w.e);
    a.bcount = reinterpret_cast<int32_t *>(ws + w.bcount);
    a.boff = reinterpret_cast<int32_t *>(ws + w.boff);
    a.btile = reinterpret_cast<int32_t *>(ws + w.btile);
    a.pairs = reinterpret_cast<int32_t *>(ws + w.pairs);
    a.pair_w = reinterpret_cast<float *>(ws + w.pair_w);
    a.tiles = reinterpret_cast<int4 *>(ws + w.tiles);
    a.ntiles = reinterpret_cast<int32_t *>(ws + w.hdr + 16);
    a.dL = reinterpret_cast<float *>(ws + w.dL);
    a.status = reinterpret_cast<uint32_t *>(ws + w.hdr);
    const unsigned row_grid = (unsigned)((p.rows + 255) / 256);
    const bool hist = p.C <= BHIST_MAX_C;
    const unsigned hist_grid = (unsigned)(p.B * p.Hkv * ((p.Tq + BHT - 1) / BHT));
    if (hist) {
        if ((e = cudaFuncSetAttribute(bwd_prep_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(p.C * sizeof(int)))) != cudaSuccess ||
            (e = cudaFuncSetAttribute(bwd_scatter_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)(2 * p.C * sizeof(int)))) != cudaSuccess)
            return e;
        bwd_prep_hist_kernel<<<hist_grid, BHT, p.C * sizeof(int), st>>>(a);
    } else {
        bwd_prep_kernel<<<row_grid, 256, 0, st>>>(a);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_scan_kernel<<<1, NT_SCAN, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    bwd_tiles_kernel<<<(unsigned)((w.nbucket + 255) / 256), 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (hist)
        bwd_scatter_hist_kernel<<<hist_grid, BHT, 2 * p.C * sizeof(int), st>>>(a);
    else
        bwd_scatter_kernel<<<row_grid, 256, 0, st>>>(a);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int grid = (int)(w.max_tiles < sms ? w.max_tiles : sms);
    const bool bf = p.dtype == HSA_BF16;
    if (w.tc) {
        const size_t smem = p.S == 64 ? BW_SMEM : BwdTcShape<128>::smem;
        if (p.S == 64) {
            e = cudaFuncSetAttribute(bwd_tcw_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess)
                bwd_tcw_kernel<<<grid, NT_W, smem, st>>>(a, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                                         (const __nv_bfloat16 *)V, (const __nv_bfloat16 *)dO, dQ, dK,
                                                         dV);
        } else {
            e = cudaFuncSetAttribute(bwd_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
            if (e == cudaSuccess)
                bwd_tc_kernel<128><<<grid, BT_ROWS, smem, st>>>(a, (const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)K,
                                                                (const __nv_bfloat16 *)V, (const __nv_bfloat16 *)dO,
                                                                dQ, dK, dV);
        }
        if (e == cudaSuccess) e = cudaGetLastError();
    } else if (p.d == 64)
        e = bf ? launch_attend_s<__nv_bfloat16, 64>(a, grid, Q, K, V, dO, dQ, dK, dV, st)
               : launch_attend_s<float, 64>(a, grid, Q, K, V, dO, dQ, dK, dV, st);
    else
        e = bf ? launch_attend_s<__nv_bfloat16, 128>(a, grid, Q, K, V, dO, dQ, dK, dV, st)
               : launch_attend_s<float, 128>(a, grid, Q, K, V, dO, dQ, dK, dV, st);
    if (e != cudaSuccess) return e;
    const long long nch = w.nbucket;
    const int lm_grid = (int)(nch < 2ll * sms ? nch : 2ll * sms);
    if (p.d == 64)
        return bf ? launch_tail_t<__nv_bfloat16, 64>(a, p.Lc, lm_grid, Q, K, W, L, dQ, dK, dW, st)
                  : launch_tail_t<float, 64>(a, p.Lc, lm_grid, Q, K, W, L, dQ, dK, dW, st);
    return bf ? launch_tail_t<__nv_bfloat16, 128>(a, p.Lc, lm_grid, Q, K, W, L, dQ, dK, dW, st)
              : launch_tail_t<float, 128>(a, p.Lc, lm_grid, Q, K, W, L, dQ, dK, dW, st);
}

}  // namespace hsa
