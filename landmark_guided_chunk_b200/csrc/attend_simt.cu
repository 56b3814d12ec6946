// attend_simt.cu -- chunk attention and retrieval-weighted fusion on CUDA cores
// (HSA summary page, Implementation: attend to each selected chunk with
// standard attention, then fuse the chunk outputs weighted by the retrieval
// scores, read as their softmax).  Works for every supported shape and dtype.
//
//  * attend_rows_kernel  : one CTA per (b, t, kv head) row.  It loops over the
//                          kept chunks and keeps one accumulator per (head, dim)
//                          in registers.  Used for many rows (prefill).
//  * attend_split_kernel : one CTA per (slot i, row), writing the normalised
//                          chunk output o_i of the group's heads to the
//                          workspace.  attend_combine_kernel then sums
//                          w_i o_i.  Used for few rows (decode), where
//                          parallelism has to come from the slots.
//
// A chunk's K and V rows are staged in shared memory as fp32, with a padded
// pitch for K, so that thread u's dot product and thread e's value sum are
// both conflict-free.  Softmax is fp32 with the running max subtracted.
#include "common.cuh"

namespace hsa {
namespace {

struct AttArgs {
    int Tq, Tcap, H, Hkv, d, S, C, kmax, G;
    long long q_pos0, rows;
    float scale;        // 1/sqrt(d)
    uint32_t *status;   // workspace status word
};

// keff and chunk indices come from the caller: out-of-range values are skipped
// (never dereferenced) and reported through the status word.
__device__ __forceinline__ int checked_keff(const AttArgs &a, int ke) {
    if (ke < 0 || ke > a.kmax) {
        atomicOr(a.status, DEV_BAD_INDEX);
        return ke < 0 ? 0 : a.kmax;
    }
    return ke;
}
__device__ __forceinline__ bool valid_chunk(const AttArgs &a, int t, int c) {
    long long nc = (a.q_pos0 + t) / a.S;
    if (nc > a.C) nc = a.C;
    if (c < 0 || c >= nc) {
        if (threadIdx.x == 0) atomicOr(a.status, DEV_BAD_INDEX);
        return false;
    }
    return true;
}

constexpr int NT = 128;   // threads per CTA (>= S and >= d)

struct Smem {
    float *q;    // [G][d]
    float *Ks;   // [S][d+1]
    float *Vs;   // [S][d]
    float *p;    // [S]
    float *red;  // [8]
    float *w;    // [kmax]
};

__device__ __forceinline__ Smem carve(float *base, const AttArgs &a) {
    Smem s;
    s.q = base;
    s.Ks = s.q + a.G * a.d;
    s.Vs = s.Ks + a.S * (a.d + 1);
    s.p = s.Vs + a.S * a.d;
    s.red = s.p + a.S;
    s.w = s.red + 8;
    return s;
}

__host__ __device__ inline size_t smem_bytes(int G, int d, int S, int kmax) {
    return sizeof(float) * ((size_t)G * d + (size_t)S * (d + 1) + (size_t)S * d + S + 8 + kmax);
}

__device__ __forceinline__ float block_max(float x, float *red) {
    x = warp_max(x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = red[0];
    for (int i = 1; i < NT / 32; ++i) r = fmaxf(r, red[i]);
    return r;
}
__device__ __forceinline__ float block_sum(float x, float *red) {
    x = warp_sum(x);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();
    if (lane == 0) red[warp] = x;
    __syncthreads();
    float r = 0.f;
    for (int i = 0; i < NT / 32; ++i) r += red[i];
    return r;
}

__device__ __forceinline__ void row_coords(const AttArgs &a, long long row, int &b, int &t, int &j) {
    j = (int)(row % a.Hkv);
    long long bt = row / a.Hkv;
    t = (int)(bt % a.Tq);
    b = (int)(bt / a.Tq);
}

// Stage chunk c of kv head j (batch b) into shared memory as fp32, reading
// the S rows of K and V with 16-byte loads.
template <typename T>
__device__ __forceinline__ void stage_chunk(const T *K, const T *V, const AttArgs &a, int b, int j, int c,
                                            const Smem &s) {
    constexpr int EPS = 16 / (int)sizeof(T);
    const int segs = a.d / EPS;
    const size_t row0 = ((size_t)b * a.Tcap + (size_t)c * a.S) * a.Hkv + j;
    for (int i = threadIdx.x; i < a.S * segs; i += NT) {
        const int u = i / segs, sg = i - u * segs;
        const size_t off = (row0 + (size_t)u * a.Hkv) * a.d + (size_t)sg * EPS;
        const uint4 kk = __ldg(reinterpret_cast<const uint4 *>(K + off));
        const uint4 vv = __ldg(reinterpret_cast<const uint4 *>(V + off));
        const T *kt = reinterpret_cast<const T *>(&kk);
        const T *vt = reinterpret_cast<const T *>(&vv);
        float *kd = s.Ks + u * (a.d + 1) + sg * EPS;
        float *vd = s.Vs + u * a.d + sg * EPS;
#pragma unroll
        for (int e = 0; e < EPS; ++e) {
            kd[e] = to_f32(kt[e]);
            vd[e] = to_f32(vt[e]);
        }
    }
}

// Normalised attention output of query head g over the staged chunk; thread
// e < d returns o[e].
__device__ __forceinline__ float chunk_attention(const AttArgs &a, const Smem &s, int g) {
    const int tid = threadIdx.x;
    float x = -INFINITY;
    if (tid < a.S) {
        const float *q = s.q + g * a.d;
        const float *kr = s.Ks + tid * (a.d + 1);
        float acc = 0.f;
        for (int e = 0; e < a.d; ++e) acc = fmaf(q[e], kr[e], acc);
        x = acc * a.scale;
    }
    const float m = block_max(x, s.red);
    const float pe = tid < a.S ? expf(x - m) : 0.f;
    if (tid < a.S) s.p[tid] = pe;
    const float l = block_sum(pe, s.red);   // its barriers also publish s.p
    float o = 0.f;
    if (tid < a.d) {
        for (int u = 0; u < a.S; ++u) o = fmaf(s.p[u], s.Vs[u * a.d + tid], o);
        o = o / l;
    }
    __syncthreads();   // s.p and s.red are reused by the next call
    return o;
}

template <typename T>
__device__ __forceinline__ void load_q(const T *Q, const AttArgs &a, int b, int t, int j, const Smem &s) {
    const T *q = Q + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * a.d;
    for (int i = threadIdx.x; i < a.G * a.d; i += NT) s.q[i] = to_f32(q[i]);
}

// Fusion weights w_i = softmax over the kept slots of the retrieval scores.
__device__ __forceinline__ void fusion_weights(const float *score, int ke, const Smem &s) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float x = lane < ke ? score[lane] : -INFINITY;
        float m = warp_max(x);
        float e = lane < ke ? expf(x - m) : 0.f;
        float z = warp_sum(e);
        if (lane < ke) s.w[lane] = e / z;
    }
}

template <typename T>
__global__ void __launch_bounds__(NT) attend_rows_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                         const T *__restrict__ V, const int32_t *__restrict__ idx,
                                                         const float *__restrict__ score,
                                                         const int32_t *__restrict__ keff, T *__restrict__ O,
                                                         AttArgs a) {
    extern __shared__ float smem[];
    const Smem s = carve(smem, a);
    const long long row = blockIdx.x;
    int b, t, j;
    row_coords(a, row, b, t, j);
    const int ke = checked_keff(a, keff[row]);
    T *out = O + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * a.d;
    float acc[MAX_G];
#pragma unroll
    for (int g = 0; g < MAX_G; ++g) acc[g] = 0.f;
    if (ke > 0) {
        load_q(Q, a, b, t, j, s);
        fusion_weights(score + row * a.kmax, ke, s);
        for (int i = 0; i < ke; ++i) {
            const int c = idx[row * a.kmax + i];
            if (!valid_chunk(a, t, c)) continue;   // uniform over the block
            __syncthreads();
            stage_chunk(K, V, a, b, j, c, s);
            __syncthreads();
            const float wi = s.w[i];
#pragma unroll
            for (int g = 0; g < MAX_G; ++g)
                if (g < a.G) acc[g] = fmaf(wi, chunk_attention(a, s, g), acc[g]);
        }
    }
    if (threadIdx.x < a.d) {
#pragma unroll
        for (int g = 0; g < MAX_G; ++g)
            if (g < a.G) out[(size_t)g * a.d + threadIdx.x] = from_f32<T>(acc[g]);
    }
}

template <typename T>
__global__ void __launch_bounds__(NT) attend_split_kernel(const T *__restrict__ Q, const T *__restrict__ K,
                                                          const T *__restrict__ V, const int32_t *__restrict__ idx,
                                                          const int32_t *__restrict__ keff,
                                                          float *__restrict__ part, AttArgs a) {
    extern __shared__ float smem[];
    const Smem s = carve(smem, a);
    const int i = blockIdx.x;
    const long long row = blockIdx.y;
    if (i >= checked_keff(a, keff[row])) return;
    int b, t, j;
    row_coords(a, row, b, t, j);
    const int c = idx[row * a.kmax + i];
    float *dst = part + (row * a.kmax + i) * (size_t)a.G * a.d;
    if (!valid_chunk(a, t, c)) {
        for (int x = threadIdx.x; x < a.G * a.d; x += NT) dst[x] = 0.f;
        return;
    }
    load_q(Q, a, b, t, j, s);
    stage_chunk(K, V, a, b, j, c, s);
    __syncthreads();
    for (int g = 0; g < a.G; ++g) {
        const float o = chunk_attention(a, s, g);
        if (threadIdx.x < a.d) dst[(size_t)g * a.d + threadIdx.x] = o;
    }
}

template <typename T>
__global__ void __launch_bounds__(NT) attend_combine_kernel(const float *__restrict__ part,
                                                            const float *__restrict__ score,
                                                            const int32_t *__restrict__ keff, T *__restrict__ O,
                                                            AttArgs a) {
    __shared__ float wbuf[MAX_KMAX];
    Smem s{};
    s.w = wbuf;
    const long long row = blockIdx.x;
    int b, t, j;
    row_coords(a, row, b, t, j);
    const int ke = checked_keff(a, keff[row]);
    fusion_weights(score + row * a.kmax, ke, s);
    __syncthreads();
    T *out = O + (((size_t)b * a.Tq + t) * a.H + (size_t)j * a.G) * a.d;
    const float *src = part + row * a.kmax * (size_t)a.G * a.d;
    for (int x = threadIdx.x; x < a.G * a.d; x += NT) {
        float acc = 0.f;
        for (int i = 0; i < ke; ++i) acc = fmaf(s.w[i], src[(size_t)i * a.G * a.d + x], acc);
        out[x] = from_f32<T>(acc);
    }
}

template <typename T>
cudaError_t launch_typed(const Prob &p, const WsLayout &w, const void *Q, const void *K, const void *V,
                         const int32_t *idx, const float *score, const int32_t *keff, void *O, char *ws,
                         cudaStream_t st) {
    AttArgs a;
    a.Tq = p.Tq;
    a.Tcap = p.Tcap;
    a.H = p.H;
    a.Hkv = p.Hkv;
    a.d = p.d;
    a.S = p.S;
    a.C = p.C;
    a.kmax = p.kmax;
    a.G = p.G;
    a.q_pos0 = p.q_pos0;
    a.rows = p.rows;
    a.scale = 1.0f / sqrtf((float)p.d);
    a.status = reinterpret_cast<uint32_t *>(ws + w.hdr);
    const size_t smem = smem_bytes(p.G, p.d, p.S, p.kmax);
    if (!w.split_attend) {
        cudaFuncSetAttribute(attend_rows_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        attend_rows_kernel<T><<<(unsigned)p.rows, NT, smem, st>>>((const T *)Q, (const T *)K, (const T *)V, idx,
                                                                  score, keff, (T *)O, a);
        return cudaGetLastError();
    }
    float *part = reinterpret_cast<float *>(ws + w.partials);
    cudaFuncSetAttribute(attend_split_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attend_split_kernel<T><<<dim3(p.kmax, (unsigned)p.rows), NT, smem, st>>>((const T *)Q, (const T *)K,
                                                                              (const T *)V, idx, keff, part, a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attend_combine_kernel<T><<<(unsigned)p.rows, NT, 0, st>>>(part, score, keff, (T *)O, a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const Prob &p, const WsLayout &w, const void *Q, const void *K, const void *V,
                          const int32_t *idx, const float *score, const int32_t *keff, void *O, char *ws,
                          cudaStream_t st) {
    if (p.rows == 0) return cudaSuccess;
    if (w.tc_attend) {
        AttTcBuffers bf;
        bf.w8 = w.att.hist ? nullptr : reinterpret_cast<float *>(ws + w.att_w8);
        bf.pairs = reinterpret_cast<int2 *>(ws + w.att_pairs);
        bf.counters = reinterpret_cast<int32_t *>(ws + w.att_counters);
        bf.boff = reinterpret_cast<int32_t *>(ws + w.att_boff);
        bf.btile = reinterpret_cast<int32_t *>(ws + w.att_btile);
        bf.blk = reinterpret_cast<int32_t *>(ws + w.att_blk);
        bf.tiles = reinterpret_cast<int4 *>(ws + w.att_tiles);
        bf.ring = reinterpret_cast<float *>(ws + w.att_ring);
        bf.status = reinterpret_cast<uint32_t *>(ws + w.hdr);
        return launch_attend_tc(p, w.att, bf, Q, K, V, idx, score, keff, O, st);
    }
    if (w.gather_attend)
        return launch_attend_gather(p, Q, K, V, idx, score, keff, O, reinterpret_cast<float *>(ws + w.att_acc),
                                    reinterpret_cast<int32_t *>(ws + w.att_cnt), reinterpret_cast<uint32_t *>(ws + w.hdr),
                                    st);
    if (p.dtype == HSA_BF16) return launch_typed<__nv_bfloat16>(p, w, Q, K, V, idx, score, keff, O, ws, st);
    return launch_typed<float>(p, w, Q, K, V, idx, score, keff, O, ws, st);
}

}  // namespace hsa
