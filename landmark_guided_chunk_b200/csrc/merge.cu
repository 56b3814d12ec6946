// merge.cu -- the merge step of context-sharded decode (HSA summary page,
// Implementation: keep the top k chunks by retrieval score, fuse the chunk
// outputs weighted by the softmax of those scores).
//
// With the chunks split over nshard shards (contiguous ranges, each with its
// own K, V and landmarks), every shard keeps its local top kmax chunks and the
// unweighted attention output o_i of each of them (hsa_attend_partials).  The
// global top kmax is contained in the union of the local ones, so merging the
// shards' lists under the same order (score descending, lower chunk first)
// reproduces the selection of one device holding the whole context; the gap
// router is then applied to the merged list, and since the fusion weights are
// a softmax over the kept scores, the output is sum_i w_i o_i over the kept
// (shard, slot) pairs.
//
// One CTA of four warps per selection row.  Warp 0 ranks the row's
// nshard*kmax <= 256 candidates (8 per lane in registers): the kmax winners are
// found one per round by a warp arg-max on (score, -chunk) and recorded in
// shared memory.  Then every thread owns float4 columns of the G*d outputs and
// sums the kept slots' partial outputs into them, with the loads of 8 slots in
// flight before their FMAs (the partials were just written by another kernel or
// received from other ranks, so each round trip is a full memory latency).
#include "common.cuh"

namespace hsa {
namespace {

constexpr int MT = 128;      // threads per CTA (one row)
constexpr int MPL = 8;       // candidates per lane of warp 0 (nshard * kmax <= 256)
constexpr int MAXO4 = 4;     // float4 outputs per thread (G * d <= 2048)
constexpr int SB = 8;        // slots whose loads are in flight together

struct MergeArgs {
    int Tq, H, Hkv, G, d, k, kmax, nshard;
    long long rows;
    float tau;
};

// ranking order: score descending, then lower chunk index
__device__ __forceinline__ bool ranks_before(float s1, int c1, float s2, int c2) {
    return s1 > s2 || (s1 == s2 && c1 < c2);
}

__device__ __forceinline__ void store_out4(float *o, float4 v) { *reinterpret_cast<float4 *>(o) = v; }
__device__ __forceinline__ void store_out4(__nv_bfloat16 *o, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(o) = u;
}

template <typename T>
__global__ void __launch_bounds__(MT) merge_kernel(MergeArgs a, const float *__restrict__ score,
                                                            const int32_t *__restrict__ idx,
                                                            const int32_t *__restrict__ keff,
                                                            const float *__restrict__ part, T *__restrict__ O,
                                                            int32_t *__restrict__ idx_out, float *__restrict__ score_out,
                                                            int32_t *__restrict__ keff_out) {
    __shared__ float s_score[MAX_KMAX];
    __shared__ float s_w[MAX_KMAX];    // fusion weight of each kept slot
    __shared__ int s_cand[MAX_KMAX];   // winning candidate e = shard * kmax + slot
    __shared__ int s_ke;
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const long long row = blockIdx.x;
    const int n = a.nshard * a.kmax;

    if (wid == 0) {
        // this lane's candidates e = lane + 32u
        float cs[MPL];
        int cc[MPL];
#pragma unroll
        for (int u = 0; u < MPL; ++u) {
            const int e = lane + 32 * u;
            cs[u] = -INFINITY;
            cc[u] = -1;
            if (e < n) {
                const int sh = e / a.kmax, i = e - sh * a.kmax;
                int ke = keff[(long long)sh * a.rows + row];
                ke = ke < 0 ? 0 : (ke > a.kmax ? a.kmax : ke);
                const long long at = ((long long)sh * a.rows + row) * a.kmax + i;
                const int c = idx[at];
                if (i < ke && c >= 0) {
                    cs[u] = score[at];
                    cc[u] = c;
                }
            }
        }
        // kmax rounds of warp arg-max; taken candidates drop out
        unsigned taken = 0;
        int total = 0;
        for (int r = 0; r < a.kmax; ++r) {
            float bs = -INFINITY;
            int bc = 0x7fffffff, bu = -1;
#pragma unroll
            for (int u = 0; u < MPL; ++u) {
                const bool live = cc[u] >= 0 && !((taken >> u) & 1u);
                if (live && ranks_before(cs[u], cc[u], bs, bc)) {
                    bs = cs[u];
                    bc = cc[u];
                    bu = u;
                }
            }
            float ws = bs;
            int wc = bc;
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) {
                const float os = __shfl_xor_sync(FULL, ws, off);
                const int oc = __shfl_xor_sync(FULL, wc, off);
                if (ranks_before(os, oc, ws, wc)) {
                    ws = os;
                    wc = oc;
                }
            }
            if (wc == 0x7fffffff) break;   // no candidate left (warp-uniform)
            // chunk indices are distinct across shards: exactly one lane holds the winner
            const bool mine = bu >= 0 && bc == wc;
            const unsigned who = __ballot_sync(FULL, mine);
            const int src = __ffs(who) - 1;
            const int e = __shfl_sync(FULL, lane + 32 * (bu < 0 ? 0 : bu), src);
            if (mine) taken |= 1u << bu;
            if (lane == 0) {
                s_score[r] = ws;
                s_cand[r] = e;
            }
            ++total;
        }
        int ke = total < a.k ? total : a.k;
        if (a.tau > 0.f && total > a.k) {
            __syncwarp();
            const float sk = s_score[a.k - 1], sk1 = s_score[a.k];
            if (sk - sk1 < a.tau * fabsf(sk)) ke = total < 2 * a.k ? total : 2 * a.k;
        }
        // fusion weights: softmax over the kept scores
        __syncwarp();
        const float xs = lane < ke ? s_score[lane] : -INFINITY;
        float m = xs;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(FULL, m, off));
        const float ex = lane < ke ? expf(xs - m) : 0.f;
        float z = ex;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) z += __shfl_xor_sync(FULL, z, off);
        if (lane < ke) s_w[lane] = ex / z;
        if (lane == 0) s_ke = ke;
    }
    __syncthreads();
    const int ke = s_ke;
    // O[g][:] = sum_i w_i o_i[g][:], this thread's float4 columns
    const int gd = a.G * a.d;
    const long long bt = row / a.Hkv;
    const int j = (int)(row - bt * a.Hkv);
    T *out = O + (bt * a.H + (long long)j * a.G) * a.d;
#pragma unroll
    for (int q = 0; q < MAXO4; ++q) {
        const int x = 4 * ((int)threadIdx.x + MT * q);
        if (x >= gd) break;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int i0 = 0; i0 < ke; i0 += SB) {
            float4 v[SB];
            float w[SB];
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                const int i = i0 + u;
                w[u] = 0.f;
                v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (i < ke) {
                    w[u] = s_w[i];
                    const int e = s_cand[i];
                    const int sh = e / a.kmax, slot = e - sh * a.kmax;
                    v[u] = *reinterpret_cast<const float4 *>(
                        part + (((long long)sh * a.rows + row) * a.kmax + slot) * gd + x);
                }
            }
#pragma unroll
            for (int u = 0; u < SB; ++u) {
                if (i0 + u < ke) {
                    acc.x = fmaf(w[u], v[u].x, acc.x);
                    acc.y = fmaf(w[u], v[u].y, acc.y);
                    acc.z = fmaf(w[u], v[u].z, acc.z);
                    acc.w = fmaf(w[u], v[u].w, acc.w);
                }
            }
        }
        store_out4(out + x, acc);
    }
    if (threadIdx.x < a.kmax) {
        const int r = threadIdx.x;
        if (idx_out != nullptr) {
            int c = -1;
            if (r < ke) {
                const int e = s_cand[r];
                const int sh = e / a.kmax;
                c = idx[((long long)sh * a.rows + row) * a.kmax + (e - sh * a.kmax)];
            }
            idx_out[row * a.kmax + r] = c;
        }
        if (score_out != nullptr) score_out[row * a.kmax + r] = r < ke ? s_score[r] : -INFINITY;
    }
    if (keff_out != nullptr && threadIdx.x == 0) keff_out[row] = ke;
}

}  // namespace

cudaError_t launch_merge_partials(const Prob &p, int nshard, const float *score, const int32_t *idx,
                                  const int32_t *keff, const float *part, void *O, int32_t *idx_out, float *score_out,
                                  int32_t *keff_out, cudaStream_t st) {
    if (p.rows == 0) return cudaSuccess;
    MergeArgs a;
    a.Tq = p.Tq;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.G = p.G;
    a.d = p.d;
    a.k = p.k;
    a.kmax = p.kmax;
    a.nshard = nshard;
    a.rows = p.rows;
    a.tau = p.tau;
    const long long grid = p.rows;
    if (p.dtype == HSA_BF16)
        merge_kernel<__nv_bfloat16><<<(unsigned)grid, MT, 0, st>>>(a, score, idx, keff, part,
                                                                            (__nv_bfloat16 *)O, idx_out, score_out,
                                                                            keff_out);
    else
        merge_kernel<float><<<(unsigned)grid, MT, 0, st>>>(a, score, idx, keff, part, (float *)O, idx_out,
                                                                    score_out, keff_out);
    return cudaGetLastError();
}

bool merge_supported(const Prob &p, int nshard) {
    return nshard >= 1 && (long long)nshard * p.kmax <= 32 * MPL && (long long)p.G * p.d <= 4 * MT * MAXO4 &&
           p.rows < (1ll << 31);
}

}  // namespace hsa
