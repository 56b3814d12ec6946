// common.cuh -- shared device helpers and the internal launch interface of the
// HSA library.  Host code outside this library never includes it.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "hsa.h"

namespace hsa {

constexpr unsigned FULL = 0xffffffffu;
constexpr int MAX_KMAX = 32;   // selection slots per row (2k with the router)
constexpr int MAX_G = 16;      // query heads per kv head

// Validated problem with the derived quantities every stage uses.
struct Prob {
    int B, Tq, Tkv, H, Hkv, d, S, k, G, C, kmax, dtype;
    int Tcap;         // K/V token stride: tokens each sequence's buffers hold (>= Tkv)
    int Lc;           // L chunk stride: floor(Tcap / S) (>= C)
    long long q_pos0;
    float tau;
    unsigned flags;
    long long rows;   // B * Tq * Hkv selection rows
};

// Sizes of the chunk-major tensor-core attention's workspace pieces.
struct AttTcLayout {
    int tb, ntb, nsub, nphase, nbucket, nblk, tok, ring;
    bool hist;   // buckets counted through shared-memory histograms (C small enough); else per-pair atomics
    size_t max_tiles, counter_ints, ring_bytes;
};

struct AttTcBuffers {
    float *w8;                 // per-pair-atomics path only: fusion weights [rows][kmax]
    int2 *pairs;               // bucketed (token << 5 | slot, fusion weight bits)
    int32_t *counters, *boff, *btile, *blk;
    int4 *tiles;
    float *ring;
    uint32_t *status;
};

// Byte offsets inside the caller's workspace (all 256-byte aligned).
struct WsLayout {
    size_t hdr;          // device-status word (uint32) + padding
    size_t sel_idx, sel_score, sel_keff;   // selection outputs when hsa_forward gets NULLs
    size_t split_lists;  // decode split scan: rows x nsplit x kmax (score, id)
    size_t partials;     // decode split attend: rows x kmax x G x d fp32
    size_t sel_cnt;      // split select (tensor-core scan): per-row completion counters, right after the header
    size_t att_cnt;      // gather attend: per-row completion counters, right after the header
    size_t att_acc;      // gather attend: per-row fp32 accumulators (rows x G x d), right after the counters
    size_t dec_desc;     // fused decode step: unit descriptors (rows x kmax x 8 B), zeroed with the status word
    size_t dec_ctr;      // fused decode step: units claimed (int32), zeroed likewise
    bool fused_decode;   // hsa_forward runs the decode scan and the gather as one launch
    size_t clear_bytes;  // bytes from the workspace start zeroed before every call (status word, counters)
    size_t total;
    int nsplit, chunks_per_split;
    bool split_select, mma_select, stream_select, split_attend, gather_attend, tc_select, tc_attend;
    int stream_grid, stream_maxe;   // stream scan: CTAs and list slots per row
    AttTcLayout att;
    bool quest;          // Quest scoring: the select fields above describe quest_select_view(p)
    size_t quest_q;      // Quest scoring: the transformed query rows (quest_qprep_bytes)
    size_t att_w8, att_pairs, att_counters, att_boff, att_btile, att_blk, att_tiles, att_ring;
    hsa_plan_t plan;     // kernel paths and launch counts per stage
};

WsLayout ws_layout(const Prob &p);

// Host-side helpers of the entry points (hsa_api.cu): record the detail for
// hsa_last_error() and return the status; validate a problem; check a pointer.
hsa_status_t fail(hsa_status_t s, const char *fmt, ...);
hsa_status_t cuda_fail(cudaError_t e, const char *what);
hsa_status_t validate(const hsa_problem_t *in, Prob *p);
hsa_status_t need(const void *x, bool required, const char *name);

// status word values (workspace header)
constexpr uint32_t DEV_OK = 0;
constexpr uint32_t DEV_TIMEOUT = 1;      // a bounded wait expired
constexpr uint32_t DEV_BAD_INDEX = 2;    // hsa_attend got a chunk index / keff outside its row's range
constexpr uint32_t DEV_INTERNAL = 4;     // a kernel's own slot/index check failed; the access was skipped

// Debug builds (compiled with -DHSA_DEBUG into libhsa_b200_debug.so) check the
// indices a kernel derives itself before it uses them: gathered token and
// chunk indices, TMA coordinates, accumulator offsets.  An index outside its
// range is recorded in the status word (DEV_INTERNAL, HSA_ERR_CUDA from
// hsa_get_device_status) and clamped into the range, so the access stays
// inside its tensor and no wait is left without its data.  Release builds
// compile the checks away.
#ifdef HSA_DEBUG
constexpr bool kDebugChecks = true;
#else
constexpr bool kDebugChecks = false;
#endif
__device__ __forceinline__ long long dbg_clamp(long long x, long long lo, long long hi, uint32_t *status) {
    if constexpr (kDebugChecks) {
        if (x < lo || x >= hi) {
            atomicOr(status, DEV_INTERNAL);
            return x < lo ? lo : hi - 1;
        }
    }
    return x;
}

// ---------------------------------------------------------------------------- element access

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Dot product of an fp32 vector in shared memory with one stored row (16-byte aligned),
// accumulated in fp32 in index order.
__device__ __forceinline__ float dot_row(const float *__restrict__ q, const float *__restrict__ row, int d) {
    float acc = 0.f;
    const float4 *r4 = reinterpret_cast<const float4 *>(row);
    for (int x = 0; x < d / 4; ++x) {
        float4 v = __ldg(r4 + x);
        acc = fmaf(q[4 * x + 0], v.x, acc);
        acc = fmaf(q[4 * x + 1], v.y, acc);
        acc = fmaf(q[4 * x + 2], v.z, acc);
        acc = fmaf(q[4 * x + 3], v.w, acc);
    }
    return acc;
}

__device__ __forceinline__ float dot_row(const float *__restrict__ q, const __nv_bfloat16 *__restrict__ row, int d) {
    float acc = 0.f;
    const uint4 *r4 = reinterpret_cast<const uint4 *>(row);
    for (int x = 0; x < d / 8; ++x) {
        uint4 u = __ldg(r4 + x);
        const __nv_bfloat162 *h2 = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
        for (int y = 0; y < 4; ++y) {
            float2 f = __bfloat1622float2(h2[y]);
            acc = fmaf(q[8 * x + 2 * y + 0], f.x, acc);
            acc = fmaf(q[8 * x + 2 * y + 1], f.y, acc);
        }
    }
    return acc;
}

// ---------------------------------------------------------------------------- warp top-k list
// A sorted list of up to kmax (<= 32) entries spread over a warp: lane i holds
// entry i as (v, id).  Order: v descending, id ascending.  Empty entries are
// (-inf, INT32_MAX) and rank after every real candidate.

__device__ __forceinline__ bool ranks_before(float v1, int id1, float v2, int id2) {
    return v1 > v2 || (v1 == v2 && id1 < id2);
}

__device__ __forceinline__ void list_init(float &v, int &id) {
    v = -INFINITY;
    id = INT32_MAX;
}

// Insert (s, c) (the same on every lane) if it ranks before entry kmax-1.
__device__ __forceinline__ void list_insert(float &v, int &id, float s, int c, int kmax, int lane) {
    float vl = __shfl_sync(FULL, v, kmax - 1);
    int il = __shfl_sync(FULL, id, kmax - 1);
    if (!ranks_before(s, c, vl, il)) return;
    unsigned before = __ballot_sync(FULL, lane < kmax && ranks_before(v, id, s, c));
    int pos = __popc(before);
    float vu = __shfl_up_sync(FULL, v, 1);
    int iu = __shfl_up_sync(FULL, id, 1);
    if (lane < kmax) {
        if (lane == pos) {
            v = s;
            id = c;
        } else if (lane > pos) {
            v = vu;
            id = iu;
        }
    }
}

// Offer one candidate per lane (valid lanes only); inserts those that qualify,
// in lane order.
__device__ __forceinline__ void list_offer(float &v, int &id, float s, int c, bool valid, int kmax, int lane) {
    float vl = __shfl_sync(FULL, v, kmax - 1);
    int il = __shfl_sync(FULL, id, kmax - 1);
    unsigned m = __ballot_sync(FULL, valid && ranks_before(s, c, vl, il));
    while (m) {
        int src = __ffs(m) - 1;
        m &= m - 1;
        float sv = __shfl_sync(FULL, s, src);
        int cv = __shfl_sync(FULL, c, src);
        list_insert(v, id, sv, cv, kmax, lane);
    }
}

// ---- bitonic forms of the same list (kmax <= 16).  One (v, id) per lane;
// "better" is ranks_before; sentinels (-inf, INT32_MAX) rank last.

// Compare-exchange with the lane at distance `stride`: the lower lane of the
// pair keeps the better entry when `desc` holds for it, the worse otherwise.
__device__ __forceinline__ void bitonic_step(float &v, int &id, int stride, bool desc, int lane) {
    const float pv = __shfl_xor_sync(FULL, v, stride);
    const int pid = __shfl_xor_sync(FULL, id, stride);
    const bool lower = (lane & stride) == 0;
    const bool take = (lower == desc) ? ranks_before(pv, pid, v, id) : ranks_before(v, id, pv, pid);
    if (take) {
        v = pv;
        id = pid;
    }
}

// Sort the 32 lanes' entries, best first.
__device__ __forceinline__ void bitonic_sort32(float &v, int &id, int lane) {
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
        const bool desc = (lane & size) == 0;   // direction of this lane's block
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) bitonic_step(v, id, stride, desc, lane);
    }
}

// Lanes 0..15 hold a sorted list A (best first), lanes 16..31 a sorted list B
// in reverse (worst first): the sequence is bitonic; afterwards all 32 lanes
// are sorted best first, so lanes 0..15 hold the best 16 of A and B.
__device__ __forceinline__ void bitonic_merge32(float &v, int &id, int lane) {
#pragma unroll
    for (int stride = 16; stride > 0; stride >>= 1) bitonic_step(v, id, stride, true, lane);
}

// Merge a sorted list held the same way (lane < kmax <= 16: entry lane) into
// the warp list.
__device__ __forceinline__ void list_merge16(float &v, int &id, float bv, int bid, int kmax, int lane) {
    // lane 16 + i takes B's entry 15 - i
    const float rv = __shfl_sync(FULL, bv, 31 - lane);
    const int rid = __shfl_sync(FULL, bid, 31 - lane);
    float x = lane < 16 ? (lane < kmax ? v : -INFINITY) : (31 - lane < kmax ? rv : -INFINITY);
    int xi = lane < 16 ? (lane < kmax ? id : INT32_MAX) : (31 - lane < kmax ? rid : INT32_MAX);
    bitonic_merge32(x, xi, lane);
    v = lane < kmax ? x : -INFINITY;
    id = lane < kmax ? xi : INT32_MAX;
}

// Offer one candidate per lane (valid lanes only), kmax <= 16: few qualifying
// candidates are inserted one by one; many are sorted as a batch and merged.
// `floor`: candidates scoring below it are known to be out of the row's top k
// (another list already holds k entries at or above it), so they are skipped.
__device__ __forceinline__ void list_offer16(float &v, int &id, float s, int c, bool valid, int kmax, int lane,
                                             float floor = -INFINITY) {
    const float vl = __shfl_sync(FULL, v, kmax - 1);
    const int il = __shfl_sync(FULL, id, kmax - 1);
    const bool pass = valid && s >= floor && ranks_before(s, c, vl, il);
    unsigned m = __ballot_sync(FULL, pass);
    if (__popc(m) <= 3) {
        while (m) {
            const int src = __ffs(m) - 1;
            m &= m - 1;
            list_insert(v, id, __shfl_sync(FULL, s, src), __shfl_sync(FULL, c, src), kmax, lane);
        }
        return;
    }
    float x = pass ? s : -INFINITY;
    int xi = pass ? c : INT32_MAX;
    bitonic_sort32(x, xi, lane);
    list_merge16(v, id, x, xi, kmax, lane);
}

// keff for a row from its sorted list (entries k-1 and k), with the gap router.
__device__ __forceinline__ int list_keff(float v, int ncand, int k, int kmax, float tau) {
    int ke = ncand < k ? ncand : k;
    float sk = __shfl_sync(FULL, v, k - 1);
    float sk1 = __shfl_sync(FULL, v, kmax > k ? k : k - 1);
    if (tau > 0.f && ncand > k && (sk - sk1) < tau * fabsf(sk)) ke = ncand < 2 * k ? ncand : 2 * k;
    return ke;
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
    return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}

// ---------------------------------------------------------------------------- launchers
// Each returns a cudaError_t from the launch; shapes are already validated.

// bf16 TMA tensor maps (128-byte swizzle); strides in bytes, box in elements.
cudaError_t make_tmap_2d(CUtensorMap *m, const void *base, uint64_t inner, uint64_t outer, uint32_t box_inner,
                         uint32_t box_outer);
cudaError_t make_tmap_3d(CUtensorMap *m, const void *base, const uint64_t dims3[3], const uint64_t strides_bytes[2],
                         const uint32_t box3[3]);

bool select_tc_supported(const Prob &p);
cudaError_t launch_select_tc(const Prob &p, const void *Q, const void *L, int32_t *idx, float *score, int32_t *keff,
                             uint32_t *status, cudaStream_t st);

bool attend_tc_supported(const Prob &p);
bool attend_gather_supported(const Prob &p);
bool select_mma_supported(const Prob &p);
bool select_stream_supported(const Prob &p);
void select_stream_shape(const Prob &p, int sms, int *grid, int *maxe);
cudaError_t launch_select_stream(const Prob &p, const void *Q, const void *L, int32_t *idx, float *score,
                                 int32_t *keff, float2 *lists, int32_t *cnt, uint32_t *status, int grid, int maxe,
                                 cudaStream_t st);
// The fused decode step: the stream scan, then (same launch, cooperative) the chunk
// gather of each published row (select_stream.cu).  grid is the scan's grid.
bool decode_fused_supported(const Prob &p, int grid, int sms);
cudaError_t launch_decode_fused(const Prob &p, const void *Q, const void *K, const void *V, const void *L,
                                int32_t *idx, float *score, int32_t *keff, void *O, float2 *lists, int32_t *cnt,
                                unsigned long long *desc, int32_t *ctr, int32_t *att_cnt, float *acc, uint32_t *status,
                                int grid, int maxe, cudaStream_t st);
// part != null: partial mode (o_i of every (row, slot) into part [rows][kmax][G][d]; no fusion, O unused)
cudaError_t launch_attend_gather(const Prob &p, const void *Q, const void *K, const void *V, const int32_t *idx,
                                 const float *score, const int32_t *keff, void *O, float *acc, int32_t *cnt,
                                 uint32_t *status, cudaStream_t st, float *part = nullptr);
// The merge of per-shard selections and partial outputs into one row's output (merge.cu).
cudaError_t launch_merge_partials(const Prob &p, int nshard, const float *score, const int32_t *idx,
                                  const int32_t *keff, const float *part, void *O, int32_t *idx_out, float *score_out,
                                  int32_t *keff_out, cudaStream_t st);
bool merge_supported(const Prob &p, int nshard);
AttTcLayout attend_tc_layout(const Prob &p);
int attend_tc_launches(const AttTcLayout &L);
cudaError_t launch_attend_tc(const Prob &p, const AttTcLayout &L, const AttTcBuffers &bf, const void *Q, const void *K,
                             const void *V, const int32_t *idx, const float *score, const int32_t *keff, void *O,
                             cudaStream_t st);

cudaError_t launch_landmarks(const Prob &p, const void *K, const void *W, void *L, cudaStream_t st);

// Selection variants (variants.cu): the landmark refiner and Quest scoring.
cudaError_t launch_landmarks_refined(const Prob &p, const void *K, const void *WL, const void *Wq, const void *Wk,
                                     const void *Wv, void *L, cudaStream_t st);
cudaError_t launch_quest_summaries(const Prob &p, const void *K, void *Lq, cudaStream_t st);
cudaError_t launch_quest_summary_chunk(const Prob &p, const void *K, void *Lq, int c, cudaStream_t st);
// The problem the selection kernels see under Quest scoring: d' = 2d, G' = 2 (bf16) or 1 (fp32).
Prob quest_select_view(const Prob &p);
size_t quest_qprep_bytes(const Prob &p);
cudaError_t launch_quest_qprep(const Prob &p, const void *Q, void *Qp, cudaStream_t st);

// Backward (backward.cu): workspace layout, support check, kernel count, launch.
struct BwdLayout {
    size_t hdr, bcount, dL, clear_bytes, w, e, boff, btile, pairs, pair_w, tiles, total;
    long long nbucket, max_tiles;
    int pt;    // pairs per tile
    bool tc;   // tensor-core attention backward (bf16, d 128, S 64 / 128)
};
BwdLayout backward_layout(const Prob &p);
bool backward_supported(const Prob &p);
int backward_launches(const Prob &p);
cudaError_t launch_backward(const Prob &p, const BwdLayout &w, char *ws, int sms, const void *Q, const void *K,
                            const void *V, const void *W, const void *L, const int32_t *idx, const float *score,
                            const int32_t *keff, const void *dO, float *dQ, float *dK, float *dV, float *dW,
                            cudaStream_t st);
cudaError_t launch_decode_append(const Prob &p, const void *knew, const void *vnew, void *K, void *V, const void *W,
                                 void *L, cudaStream_t st);
cudaError_t launch_select(const Prob &p, const WsLayout &w, const void *Q, const void *L, int32_t *idx,
                          float *score, int32_t *keff, char *ws, cudaStream_t st);
cudaError_t launch_attend(const Prob &p, const WsLayout &w, const void *Q, const void *K, const void *V,
                          const int32_t *idx, const float *score, const int32_t *keff, void *O, char *ws,
                          cudaStream_t st);

}  // namespace hsa
