// select_simt.cu -- chunk selection on CUDA cores (HSA summary page, Core
// Technique / Implementation: score every landmark of the strictly-past
// chunks, keep the top k; gap router from the value-of-information router
// page).  Works for every supported shape and dtype.  fp32 problems always
// use it, and bf16 problems whose shape the tensor-core kernel does not cover.
//
// Score of chunk c for a (b, t, kv head j) row: s_c = sum_{h in group j} q_h . L_c,
// computed as qbar . L_c with qbar = sum_h q_h formed in fp32 (the same sum,
// up to fp32 rounding).  Each lane scores its own chunk of a 32-chunk batch.
// Lanes whose score beats the current k-th entry are inserted, in chunk
// order, into a warp-distributed sorted list.
//
//  * select_rows_kernel   : one warp per row, scans all candidates (prefill).
//  * select_split_kernel  : (split, row) CTAs, each scanning a chunk range with
//                           8 warps and emitting one merged list (decode: few
//                           rows, very long scans).
//  * select_merge_kernel  : one warp per row merges the split lists.
//  * select_split_mma_kernel : the split scan for bf16 with G <= 8, scoring 16
//                           chunks per tensor-core instruction; the CTA that
//                           completes a row's last split merges the row, so
//                           there is no separate merge launch.
#include "common.cuh"

namespace hsa {
namespace {

struct SelArgs {
    int Tq, H, Hkv, d, S, C, k, kmax, G;
    int Lc;               // chunks per (b, kv head) in L's layout
    long long q_pos0, rows;
    float tau;
};

__device__ __forceinline__ void row_coords(const SelArgs &a, long long row, int &b, int &t, int &j) {
    j = (int)(row % a.Hkv);
    long long bt = row / a.Hkv;
    t = (int)(bt % a.Tq);
    b = (int)(bt / a.Tq);
}

__device__ __forceinline__ int row_ncand(const SelArgs &a, int t) {
    long long n = (a.q_pos0 + t) / a.S;
    return (int)(n < a.C ? n : a.C);
}

// qbar[e] = sum over the group's heads of Q[b][t][h][e], into shared memory.
template <typename T>
__device__ __forceinline__ void load_qbar(const T *Q, const SelArgs &a, int b, int t, int j, float *qs, int lane) {
    const T *q = Q + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * a.d;
    for (int e = lane; e < a.d; e += 32) {
        float s = 0.f;
        for (int g = 0; g < a.G; ++g) s += to_f32(q[(size_t)g * a.d + e]);
        qs[e] = s;
    }
    __syncwarp();
}

template <typename T>
__device__ __forceinline__ void scan_range(const float *qs, const T *Lj, const SelArgs &a, int c0, int c1, int step,
                                           float &v, int &id, int lane) {
    for (int base = c0; base < c1; base += step) {
        int c = base + lane;
        bool valid = c < c1;
        float s = valid ? dot_row(qs, Lj + (size_t)c * a.d, a.d) : -INFINITY;
        list_offer(v, id, s, c, valid, a.kmax, lane);
    }
}

// Same scan, but with a row of L spread over SEGS lanes (16 bytes each), so a
// warp's load instruction covers 32/SEGS whole rows contiguously.  The
// partial dots are summed with xor-shuffles, and each score is handed to the
// lane that owns its chunk in the 32-chunk batch offered to the list.
template <typename T, int SEGS>
__device__ __forceinline__ void scan_range_rows(const float *qs, const T *Lj, const SelArgs &a, int c0, int c1,
                                                int step, float &v, int &id, int lane) {
    constexpr int EPS = 16 / (int)sizeof(T);   // elements per 16-byte segment
    constexpr int CPR = 32 / SEGS;             // rows per load instruction
    const int seg = lane % SEGS, sub = lane / SEGS;
    float qv[EPS];
#pragma unroll
    for (int e = 0; e < EPS; ++e) qv[e] = qs[seg * EPS + e];
    for (int base = c0; base < c1; base += step) {
        float mine = -INFINITY;
#pragma unroll
        for (int r = 0; r < 32 / CPR; ++r) {
            const int c = base + r * CPR + sub;
            float part = 0.f;
            if (c < c1) {
                const uint4 u = __ldg(reinterpret_cast<const uint4 *>(Lj + (size_t)c * a.d) + seg);
                if (sizeof(T) == 2) {
                    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 f = __bfloat1622float2(h[e]);
                        part = fmaf(qv[2 * e], f.x, part);
                        part = fmaf(qv[2 * e + 1], f.y, part);
                    }
                } else {
                    const float *f = reinterpret_cast<const float *>(&u);
#pragma unroll
                    for (int e = 0; e < 4; ++e) part = fmaf(qv[e], f[e], part);
                }
            }
#pragma unroll
            for (int o = SEGS / 2; o > 0; o >>= 1) part += __shfl_xor_sync(FULL, part, o);
            // the score of row r*CPR + x sits in lanes x*SEGS .. x*SEGS+SEGS-1
            const float got = __shfl_sync(FULL, part, (lane % CPR) * SEGS);
            if (lane / CPR == r) mine = got;
        }
        const int c = base + lane;
        list_offer(v, id, mine, c, c < c1, a.kmax, lane);
    }
}

template <typename T>
__device__ __forceinline__ void scan_range_fast(const float *qs, const T *Lj, const SelArgs &a, int c0, int c1,
                                                int step, float &v, int &id, int lane) {
    const int segs = a.d * (int)sizeof(T) / 16;
    if (segs == 16) scan_range_rows<T, 16>(qs, Lj, a, c0, c1, step, v, id, lane);
    else if (segs == 8) scan_range_rows<T, 8>(qs, Lj, a, c0, c1, step, v, id, lane);
    else if (segs == 32) scan_range_rows<T, 32>(qs, Lj, a, c0, c1, step, v, id, lane);
    else scan_range(qs, Lj, a, c0, c1, step, v, id, lane);
}

// ---------------------------------------------------------------------------- tensor-core scan (bf16)
// Scores of 16 consecutive chunks for the whole GQA group with mma.sync
// m16n8k16: A = 16 landmark rows (M = chunk, K = d), B = the group's query
// heads (K = d, N = head, G <= 8 of the 8 columns; the others zero), fp32
// accumulation.  Each product is exact, and the group score is the fp32 sum
// of a row's head columns.  Because the contraction runs over d in any order,
// the k index is permuted so that every fragment a lane needs is one 16-byte
// piece of a row: lane (r, q) = (lane/4, lane%4) reads d = 32p + 8q .. +7 of
// landmark rows r and r+8 (A) and of head r (B) for k-steps 2p and 2p+1.

__device__ __forceinline__ void mma_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Group scores of chunks cb .. cb+15 of Lj (rows >= c_end read as zero): on
// return every lane of quad r holds chunk cb+r in s0 and chunk cb+r+8 in s1.
template <int D>
__device__ __forceinline__ void tile_scores(const __nv_bfloat16 *Lj, int cb, int c_end, const uint4 (&bq)[D / 32],
                                            float &s0, float &s1) {
    const int lane = threadIdx.x & 31, r = lane >> 2, q = lane & 3;
    const bool ra = cb + r < c_end, rb = cb + r + 8 < c_end;
    uint4 ua[D / 32], ub[D / 32];
#pragma unroll
    for (int p = 0; p < D / 32; ++p) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        ua[p] = ra ? __ldg(reinterpret_cast<const uint4 *>(Lj + (size_t)(cb + r) * D + 32 * p + 8 * q)) : z;
        ub[p] = rb ? __ldg(reinterpret_cast<const uint4 *>(Lj + (size_t)(cb + r + 8) * D + 32 * p + 8 * q)) : z;
    }
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int p = 0; p < D / 32; ++p) {
        mma_16816(c, ua[p].x, ub[p].x, ua[p].y, ub[p].y, bq[p].x, bq[p].y);
        mma_16816(c, ua[p].z, ub[p].z, ua[p].w, ub[p].w, bq[p].z, bq[p].w);
    }
    s0 = c[0] + c[1];
    s1 = c[2] + c[3];
    s0 += __shfl_xor_sync(FULL, s0, 1);
    s1 += __shfl_xor_sync(FULL, s1, 1);
    s0 += __shfl_xor_sync(FULL, s0, 2);
    s1 += __shfl_xor_sync(FULL, s1, 2);
}

// Scan chunks [c0, c1) of Lj into the warp list, 32 chunks per offer.
template <int D>
__device__ __forceinline__ void scan_range_mma(const uint4 (&bq)[D / 32], const __nv_bfloat16 *Lj, const SelArgs &a,
                                               int c0, int c1, float &v, int &id, int lane) {
    for (int base = c0; base < c1; base += 32) {
        float s00, s01, s10, s11;
        tile_scores<D>(Lj, base, c1, bq, s00, s01);
        tile_scores<D>(Lj, base + 16, c1, bq, s10, s11);
        // chunk base + lane: tile lane/16, half (lane/8)&1, row lane%8, held by lane 4*(lane%8)
        const int src = 4 * (lane & 7);
        const float x00 = __shfl_sync(FULL, s00, src), x01 = __shfl_sync(FULL, s01, src);
        const float x10 = __shfl_sync(FULL, s10, src), x11 = __shfl_sync(FULL, s11, src);
        const float mine = lane < 16 ? (lane < 8 ? x00 : x01) : (lane < 24 ? x10 : x11);
        const int c = base + lane;
        if (a.kmax <= 16)
            list_offer16(v, id, mine, c, c < c1, a.kmax, lane);
        else
            list_offer(v, id, mine, c, c < c1, a.kmax, lane);
    }
}

__device__ __forceinline__ void write_row(const SelArgs &a, long long row, float v, int id, int ke, int32_t *idx,
                                          float *score, int32_t *keff, int lane) {
    if (lane < a.kmax) {
        idx[row * a.kmax + lane] = lane < ke ? id : -1;
        score[row * a.kmax + lane] = lane < ke ? v : -INFINITY;
    }
    if (lane == 0) keff[row] = ke;
}

template <typename T>
__global__ void __launch_bounds__(256) select_rows_kernel(const T *__restrict__ Q, const T *__restrict__ L,
                                                          int32_t *__restrict__ idx, float *__restrict__ score,
                                                          int32_t *__restrict__ keff, SelArgs a) {
    extern __shared__ float qsm[];   // [8 warps][d]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + warp;
    if (row >= a.rows) return;
    int b, t, j;
    row_coords(a, row, b, t, j);
    float *qs = qsm + warp * a.d;
    load_qbar(Q, a, b, t, j, qs, lane);
    const int ncand = row_ncand(a, t);
    const T *Lj = L + ((size_t)b * a.Hkv + j) * (size_t)a.Lc * a.d;
    float v;
    int id;
    list_init(v, id);
    scan_range(qs, Lj, a, 0, ncand, 32, v, id, lane);
    write_row(a, row, v, id, list_keff(v, ncand, a.k, a.kmax, a.tau), idx, score, keff, lane);
}

// One CTA = one (split, row).  Warps interleave over 32-chunk batches of the
// split's range; their lists are merged by warp 0 into the split's list.
template <typename T>
__global__ void __launch_bounds__(256) select_split_kernel(const T *__restrict__ Q, const T *__restrict__ L,
                                                           float2 *__restrict__ lists, SelArgs a, int chunks_per_split,
                                                           int nsplit) {
    extern __shared__ float qsm[];   // [d] qbar, then 8 x kmax (v, id) pairs
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.y;
    const int split = blockIdx.x;
    int b, t, j;
    row_coords(a, row, b, t, j);
    float *qs = qsm;
    float2 *wl = reinterpret_cast<float2 *>(qsm + a.d);
    if (warp == 0) load_qbar(Q, a, b, t, j, qs, lane);
    __syncthreads();
    const int ncand = row_ncand(a, t);
    const int c0 = split * chunks_per_split;
    const int c1 = min(ncand, c0 + chunks_per_split);
    const T *Lj = L + ((size_t)b * a.Hkv + j) * (size_t)a.Lc * a.d;
    float v;
    int id;
    list_init(v, id);
    if (c0 < c1) scan_range_fast(qs, Lj, a, c0 + 32 * warp, c1, 256, v, id, lane);
    if (lane < a.kmax) wl[warp * a.kmax + lane] = make_float2(v, __int_as_float(id));
    __syncthreads();
    if (warp == 0) {
        float mv;
        int mid;
        list_init(mv, mid);
        const int n = 8 * a.kmax;
        for (int base = 0; base < n; base += 32) {
            int e = base + lane;
            float2 x = e < n ? wl[e] : make_float2(-INFINITY, __int_as_float(INT32_MAX));
            int xi = __float_as_int(x.y);
            list_offer(mv, mid, x.x, xi, xi != INT32_MAX, a.kmax, lane);
        }
        if (lane < a.kmax) lists[(row * nsplit + split) * a.kmax + lane] = make_float2(mv, __int_as_float(mid));
    }
}

// Merge a warp-list set: n entries (v, id) from src (global, read through L2)
// into the warp list, then write the row (lane k < kmax holds entry k).
__device__ __forceinline__ void merge_lists_to_row(const float2 *src, int n, const SelArgs &a, long long row,
                                                   int ncand, int32_t *idx, float *score, int32_t *keff, int lane) {
    float v;
    int id;
    list_init(v, id);
    if (a.kmax <= 16) {   // n / kmax sorted lists: bitonic merges, one list at a time
        for (int base = 0; base < n; base += a.kmax) {
            const float2 x = lane < a.kmax ? __ldcg(src + base + lane) : make_float2(-INFINITY, __int_as_float(INT32_MAX));
            list_merge16(v, id, x.x, __float_as_int(x.y), a.kmax, lane);
        }
        write_row(a, row, v, id, list_keff(v, ncand, a.k, a.kmax, a.tau), idx, score, keff, lane);
        return;
    }
    for (int base = 0; base < n; base += 32) {
        const int e = base + lane;
        const float2 x = e < n ? __ldcg(src + e) : make_float2(-INFINITY, __int_as_float(INT32_MAX));
        const int xi = __float_as_int(x.y);
        list_offer(v, id, x.x, xi, xi != INT32_MAX, a.kmax, lane);
    }
    write_row(a, row, v, id, list_keff(v, ncand, a.k, a.kmax, a.tau), idx, score, keff, lane);
}

// Decode scan, bf16, G <= 8: one CTA = one (split, row); each warp scans a
// contiguous part of the split's range with the tensor-core tile scores, the
// warp lists are merged into the split's list, and the CTA that completes the
// row's last split (per-row counter, zeroed with the status word) merges the
// row's split lists and writes the row's selection.
template <int D>
__global__ void __launch_bounds__(256) select_split_mma_kernel(const __nv_bfloat16 *__restrict__ Q,
                                                               const __nv_bfloat16 *__restrict__ L,
                                                               float2 *__restrict__ lists, int32_t *__restrict__ idx,
                                                               float *__restrict__ score, int32_t *__restrict__ keff,
                                                               int32_t *__restrict__ cnt, SelArgs a,
                                                               int chunks_per_split, int nsplit) {
    __shared__ float2 wl[8 * MAX_KMAX];
    __shared__ int s_last;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = blockIdx.y;
    const int split = blockIdx.x;
    int b, t, j;
    row_coords(a, row, b, t, j);
    const int ncand = row_ncand(a, t);
    const int c0 = split * chunks_per_split;
    const int c1 = min(ncand, c0 + chunks_per_split);
    float v;
    int id;
    list_init(v, id);
    if (c0 < c1) {
        // the group's query heads as B fragments (head lane/4; heads >= G are zero)
        uint4 bq[D / 32];
        const int hr = lane >> 2, q = lane & 3;
        const __nv_bfloat16 *qh = Q + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G + hr) * D;
#pragma unroll
        for (int p = 0; p < D / 32; ++p)
            bq[p] = hr < a.G ? __ldg(reinterpret_cast<const uint4 *>(qh + 32 * p + 8 * q)) : make_uint4(0u, 0u, 0u, 0u);
        const int per = ((c1 - c0 + 8 * 32 - 1) / (8 * 32)) * 32;   // a multiple of 32 per warp
        const int w0 = c0 + warp * per, w1 = min(c1, w0 + per);
        const __nv_bfloat16 *Lj = L + ((size_t)b * a.Hkv + j) * (size_t)a.Lc * D;
        if (w0 < w1) scan_range_mma<D>(bq, Lj, a, w0, w1, v, id, lane);
    }
    if (lane < a.kmax) wl[warp * a.kmax + lane] = make_float2(v, __int_as_float(id));
    __syncthreads();
    if (warp == 0) {
        float mv;
        int mid;
        list_init(mv, mid);
        const int n = 8 * a.kmax;
        if (a.kmax <= 16) {   // eight sorted lists: bitonic merges
            for (int w2 = 0; w2 < 8; ++w2) {
                const float2 x = lane < a.kmax ? wl[w2 * a.kmax + lane] : make_float2(-INFINITY, __int_as_float(INT32_MAX));
                list_merge16(mv, mid, x.x, __float_as_int(x.y), a.kmax, lane);
            }
        } else {
            for (int base = 0; base < n; base += 32) {
                const int e = base + lane;
                const float2 x = e < n ? wl[e] : make_float2(-INFINITY, __int_as_float(INT32_MAX));
                const int xi = __float_as_int(x.y);
                list_offer(mv, mid, x.x, xi, xi != INT32_MAX, a.kmax, lane);
            }
        }
        if (lane < a.kmax) lists[(row * nsplit + split) * a.kmax + lane] = make_float2(mv, __int_as_float(mid));
        __threadfence();
    }
    __syncthreads();
    if (threadIdx.x == 0) s_last = atomicAdd(&cnt[row], 1) == nsplit - 1;
    __syncthreads();
    if (s_last && warp == 0) {
        __threadfence();
        merge_lists_to_row(lists + row * nsplit * a.kmax, nsplit * a.kmax, a, row, ncand, idx, score, keff, lane);
    }
}

__global__ void __launch_bounds__(256) select_merge_kernel(const float2 *__restrict__ lists, int32_t *__restrict__ idx,
                                                           float *__restrict__ score, int32_t *__restrict__ keff,
                                                           SelArgs a, int nsplit) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long row = (long long)blockIdx.x * 8 + warp;
    if (row >= a.rows) return;
    int b, t, j;
    row_coords(a, row, b, t, j);
    const float2 *src = lists + row * nsplit * a.kmax;
    const int n = nsplit * a.kmax;
    float v;
    int id;
    list_init(v, id);
    for (int base = 0; base < n; base += 32) {
        int e = base + lane;
        float2 x = e < n ? src[e] : make_float2(-INFINITY, __int_as_float(INT32_MAX));
        int xi = __float_as_int(x.y);
        list_offer(v, id, x.x, xi, xi != INT32_MAX, a.kmax, lane);
    }
    write_row(a, row, v, id, list_keff(v, row_ncand(a, t), a.k, a.kmax, a.tau), idx, score, keff, lane);
}

SelArgs make_args(const Prob &p) {
    SelArgs a;
    a.Tq = p.Tq;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.d = p.d;
    a.S = p.S;
    a.C = p.C;
    a.Lc = p.Lc;
    a.k = p.k;
    a.kmax = p.kmax;
    a.G = p.G;
    a.q_pos0 = p.q_pos0;
    a.rows = p.rows;
    a.tau = p.tau;
    return a;
}

template <typename T>
cudaError_t launch_typed(const Prob &p, const WsLayout &w, const void *Q, const void *L, int32_t *idx, float *score,
                         int32_t *keff, char *ws, cudaStream_t st) {
    SelArgs a = make_args(p);
    if (w.split_select && w.mma_select) {
        float2 *lists = reinterpret_cast<float2 *>(ws + w.split_lists);
        int32_t *cnt = reinterpret_cast<int32_t *>(ws + w.sel_cnt);
        dim3 grid(w.nsplit, (unsigned)p.rows);
        if (p.d == 128)
            select_split_mma_kernel<128><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)L, lists,
                                                               idx, score, keff, cnt, a, w.chunks_per_split, w.nsplit);
        else
            select_split_mma_kernel<64><<<grid, 256, 0, st>>>((const __nv_bfloat16 *)Q, (const __nv_bfloat16 *)L, lists,
                                                              idx, score, keff, cnt, a, w.chunks_per_split, w.nsplit);
        return cudaGetLastError();
    }
    if (!w.split_select) {
        unsigned blocks = (unsigned)((p.rows + 7) / 8);
        select_rows_kernel<T><<<blocks, 256, 8 * p.d * sizeof(float), st>>>((const T *)Q, (const T *)L, idx, score,
                                                                            keff, a);
        return cudaGetLastError();
    }
    float2 *lists = reinterpret_cast<float2 *>(ws + w.split_lists);
    dim3 grid(w.nsplit, (unsigned)p.rows);
    size_t smem = p.d * sizeof(float) + 8 * p.kmax * sizeof(float2);
    select_split_kernel<T><<<grid, 256, smem, st>>>((const T *)Q, (const T *)L, lists, a, w.chunks_per_split,
                                                    w.nsplit);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    select_merge_kernel<<<(unsigned)((p.rows + 7) / 8), 256, 0, st>>>(lists, idx, score, keff, a, w.nsplit);
    return cudaGetLastError();
}

}  // namespace

bool select_mma_supported(const Prob &p) {
    return p.dtype == HSA_BF16 && (p.d == 64 || p.d == 128) && p.G <= 8 && p.kmax <= MAX_KMAX;
}

cudaError_t launch_select(const Prob &p, const WsLayout &w, const void *Q, const void *L, int32_t *idx,
                          float *score, int32_t *keff, char *ws, cudaStream_t st) {
    if (p.rows == 0) return cudaSuccess;
    if (w.tc_select) return launch_select_tc(p, Q, L, idx, score, keff, reinterpret_cast<uint32_t *>(ws + w.hdr), st);
    if (w.stream_select)
        return launch_select_stream(p, Q, L, idx, score, keff, reinterpret_cast<float2 *>(ws + w.split_lists),
                                    reinterpret_cast<int32_t *>(ws + w.sel_cnt), reinterpret_cast<uint32_t *>(ws + w.hdr),
                                    w.stream_grid, w.stream_maxe, st);
    if (p.dtype == HSA_BF16) return launch_typed<__nv_bfloat16>(p, w, Q, L, idx, score, keff, ws, st);
    return launch_typed<float>(p, w, Q, L, idx, score, keff, ws, st);
}

}  // namespace hsa
