// hsa_api.cu -- the C ABI declared in include/hsa.h: host-side validation,
// workspace layout and stage dispatch.  No entry point allocates memory,
// throws, or keeps global mutable state (the last-error text is per host
// thread).
#include <stdarg.h>
#include <stdio.h>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace hsa {

static thread_local char g_err[512] = "";

// An NVTX range around each launching entry point, named after it, so that a
// timeline (nsys, ncu's range filters) shows the library's calls.  Header-only
// NVTX: without an attached tool a range costs a null check.
struct NvtxRange {
    explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
};

hsa_status_t fail(hsa_status_t s, const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof g_err, fmt, ap);
    va_end(ap);
    return s;
}

hsa_status_t cuda_fail(cudaError_t e, const char *what) {
    return fail(HSA_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

static inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// SMs of the current device (148 if it cannot be queried); kernels sized by it
// and their workspace layouts use the same value.
static int device_sms() {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms <= 0) {
        cudaGetLastError();
        return 148;
    }
    return sms;
}


WsLayout ws_layout(const Prob &p) {
    WsLayout w{};
    // Under Quest scoring the selection kernels run on a transformed problem
    // (query rows [P | N], landmarks = chunk summaries, width 2d); every select
    // decision below is taken on that view.
    w.quest = (p.flags & HSA_FLAG_QUEST) != 0;
    const Prob ps = w.quest ? quest_select_view(p) : p;
    size_t off = 0;
    auto take = [&](size_t bytes) {
        size_t o = off;
        off += align256(bytes);
        return o;
    };
    const size_t rows = (size_t)p.rows;
    w.hdr = take(256);
    // Many rows: tensor-core scoring.  Few rows with long scans: split each
    // row's chunk range over CTAs -- for decode in bf16 (one query per row,
    // G <= 8, kmax <= 16) one CTA per SM streams its share of all rows' landmarks
    // through a TMA ring; otherwise in bf16 with G <= 8 (split) CTAs score with
    // the tensor cores and fold the merge in.  Otherwise one warp per row.
    w.tc_select = rows > 0 && !(p.flags & HSA_FLAG_SIMT) && select_tc_supported(ps);
    w.split_select = !w.tc_select && rows > 0 && rows <= 4096 && p.C >= 2048;
    w.stream_select = w.split_select && !(p.flags & HSA_FLAG_SIMT) && select_stream_supported(ps);
    w.mma_select = w.split_select && !w.stream_select && !(p.flags & HSA_FLAG_SIMT) && select_mma_supported(ps);
    if (w.stream_select) select_stream_shape(ps, device_sms(), &w.stream_grid, &w.stream_maxe);
    // Few rows: the kept slots are spread over CTAs too (split attend); in bf16
    // the gather kernel does it in one launch.
    w.split_attend = rows > 0 && rows <= 2048;
    w.gather_attend = w.split_attend && !(p.flags & HSA_FLAG_SIMT) && attend_gather_supported(p);
    // Per-row completion counters and fp32 accumulators of those single-launch
    // kernels sit right after the header, so that the one memset of the status
    // word that starts every call clears them too.
    if (w.mma_select || w.stream_select) w.sel_cnt = take(rows * sizeof(int32_t));
    if (w.gather_attend) {
        w.att_cnt = take(rows * sizeof(int32_t));
        w.att_acc = take(rows * (size_t)p.G * p.d * sizeof(float));
    }
    // Decode with both of those kernels: hsa_forward fuses them into one launch.
    w.fused_decode = w.stream_select && w.gather_attend && decode_fused_supported(p, w.stream_grid, device_sms());
    if (w.fused_decode) {
        w.dec_desc = take(rows * (size_t)p.kmax * sizeof(unsigned long long));
        w.dec_ctr = take(sizeof(int32_t));
    }
    w.clear_bytes = off > 256 ? off : sizeof(uint32_t);
    w.sel_idx = take(rows * p.kmax * sizeof(int32_t));
    w.sel_score = take(rows * p.kmax * sizeof(float));
    w.sel_keff = take(rows * sizeof(int32_t));
    if (w.quest) w.quest_q = take(quest_qprep_bytes(p));
    if (w.split_select) {
        const long long target = 148 * 8;
        long long per_row = (target + (long long)rows - 1) / (long long)rows;
        long long cps = ((long long)p.C + per_row - 1) / per_row;
        cps = ((cps + 255) / 256) * 256;
        if (cps < 256) cps = 256;
        w.chunks_per_split = (int)cps;
        w.nsplit = (int)(((long long)p.C + cps - 1) / cps);
        const size_t slots = w.stream_select ? (size_t)w.stream_maxe : (size_t)w.nsplit;
        w.split_lists = take(rows * slots * p.kmax * sizeof(float2));
    }
    // Many rows: chunk-major tensor-core attention.
    w.tc_attend = !w.split_attend && rows > 0 && !(p.flags & HSA_FLAG_SIMT) && attend_tc_supported(p);
    if (w.split_attend && !w.gather_attend) w.partials = take(rows * (size_t)p.kmax * p.G * p.d * sizeof(float));
    if (w.tc_attend) {
        w.att = attend_tc_layout(p);
        if (!w.att.hist) w.att_w8 = take(rows * p.kmax * sizeof(float));
        w.att_pairs = take(rows * p.kmax * sizeof(int2));
        w.att_counters = take(w.att.counter_ints * sizeof(int32_t));
        w.att_boff = take(((size_t)w.att.nbucket + 1) * sizeof(int32_t));
        w.att_btile = take(((size_t)w.att.nbucket + 1) * sizeof(int32_t));
        w.att_blk = take(2 * (size_t)w.att.nblk * sizeof(int32_t));
        w.att_tiles = take(w.att.max_tiles * sizeof(int4));
        w.att_ring = take(w.att.ring_bytes);
    }
    w.total = off;
    const bool has_chunks = (long long)p.B * p.C > 0;
    w.plan.landmark_path = has_chunks ? HSA_PATH_SIMT_ROWS : HSA_PATH_NONE;
    w.plan.landmark_kernels = has_chunks ? 1 : 0;
    w.plan.select_path = rows == 0 ? HSA_PATH_NONE
                         : w.tc_select  ? HSA_PATH_TENSOR
                         : (w.stream_select || w.mma_select) ? HSA_PATH_MMA_SPLIT
                         : (w.split_select ? HSA_PATH_SIMT_SPLIT : HSA_PATH_SIMT_ROWS);
    w.plan.select_kernels = rows == 0 ? 0 : (w.split_select && !w.mma_select && !w.stream_select ? 2 : 1) + (w.quest ? 1 : 0);
    w.plan.attend_path = rows == 0 ? HSA_PATH_NONE
                         : w.tc_attend  ? HSA_PATH_TENSOR
                         : w.gather_attend ? HSA_PATH_MMA_SPLIT
                         : (w.split_attend ? HSA_PATH_SIMT_SPLIT : HSA_PATH_SIMT_ROWS);
    // tensor path: count, scan (2 levels), tile list, scatter, one main kernel per phase batch + 1
    w.plan.attend_kernels = rows == 0 ? 0
                            : w.tc_attend ? attend_tc_launches(w.att)
                                          : (w.split_attend && !w.gather_attend ? 2 : 1);
    w.plan.forward_fused = w.fused_decode ? 1 : 0;
    return w;
}

hsa_status_t validate(const hsa_problem_t *in, Prob *p) {
    if (!in) return fail(HSA_ERR_INVALID_ARG, "problem pointer is NULL");
    if (in->B < 0 || in->Tq < 0 || in->Tkv < 0)
        return fail(HSA_ERR_INVALID_ARG, "negative size (B=%d Tq=%d Tkv=%d)", in->B, in->Tq, in->Tkv);
    if (in->H < 1 || in->Hkv < 1 || in->d < 1 || in->S < 1 || in->k < 1)
        return fail(HSA_ERR_INVALID_ARG, "H, Hkv, d, S, k must be >= 1 (H=%d Hkv=%d d=%d S=%d k=%d)", in->H, in->Hkv,
                    in->d, in->S, in->k);
    if (in->H % in->Hkv != 0) return fail(HSA_ERR_INVALID_ARG, "H=%d is not a multiple of Hkv=%d", in->H, in->Hkv);
    if (in->dtype != HSA_F32 && in->dtype != HSA_BF16) return fail(HSA_ERR_INVALID_ARG, "unknown dtype %d", in->dtype);
    if (!(in->tau >= 0.0f) || isinf(in->tau)) return fail(HSA_ERR_INVALID_ARG, "tau must be finite and >= 0");
    if (in->q_pos0 < 0) return fail(HSA_ERR_INVALID_ARG, "q_pos0 must be >= 0");
    if (in->flags & ~(HSA_FLAG_LANDMARKS_READY | HSA_FLAG_SIMT | HSA_FLAG_TEST_STALL | HSA_FLAG_QUEST))
        return fail(HSA_ERR_INVALID_ARG, "unknown flags 0x%x", in->flags);
    if (in->d != 64 && in->d != 128) return fail(HSA_ERR_UNSUPPORTED, "d=%d (supported: 64, 128)", in->d);
    if (in->S != 32 && in->S != 64 && in->S != 128)
        return fail(HSA_ERR_UNSUPPORTED, "S=%d (supported: 32, 64, 128)", in->S);
    const int kmax = in->tau > 0.0f ? 2 * in->k : in->k;
    if (kmax > MAX_KMAX) return fail(HSA_ERR_UNSUPPORTED, "k=%d gives %d slots (max %d)", in->k, kmax, MAX_KMAX);
    if (in->H / in->Hkv > MAX_G) return fail(HSA_ERR_UNSUPPORTED, "G=%d (max %d)", in->H / in->Hkv, MAX_G);
    if (in->B > 65535) return fail(HSA_ERR_UNSUPPORTED, "B=%d (max 65535)", in->B);
    if (in->kv_cap != 0 && in->kv_cap < in->Tkv)
        return fail(HSA_ERR_INVALID_ARG, "kv_cap=%d is below Tkv=%d", in->kv_cap, in->Tkv);
    p->B = in->B;
    p->Tq = in->Tq;
    p->Tkv = in->Tkv;
    p->H = in->H;
    p->Hkv = in->Hkv;
    p->d = in->d;
    p->S = in->S;
    p->k = in->k;
    p->G = in->H / in->Hkv;
    p->C = in->Tkv / in->S;
    p->Tcap = in->kv_cap != 0 ? in->kv_cap : in->Tkv;
    p->Lc = p->Tcap / in->S;
    p->kmax = kmax;
    p->dtype = in->dtype;
    p->q_pos0 = in->q_pos0;
    p->tau = in->tau;
    p->flags = in->flags;
    p->rows = (long long)in->B * in->Tq * in->Hkv;
    return HSA_OK;
}

static bool aligned16(const void *x) { return ((uintptr_t)x & 15u) == 0; }

hsa_status_t need(const void *x, bool required, const char *name) {
    if (!required) return HSA_OK;
    if (!x) return fail(HSA_ERR_INVALID_ARG, "%s is NULL", name);
    if (!aligned16(x)) return fail(HSA_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return HSA_OK;
}

#define HSA_TRY(expr)                       \
    do {                                    \
        hsa_status_t s_ = (expr);           \
        if (s_ != HSA_OK) return s_;        \
    } while (0)

static hsa_status_t check_ws(const WsLayout &w, void *ws, size_t ws_bytes) {
    if (ws_bytes < w.total) return fail(HSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, w.total);
    if (!ws) return fail(HSA_ERR_WORKSPACE, "workspace is NULL");
    if ((uintptr_t)ws & 255u) return fail(HSA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    return HSA_OK;
}

// The selection stage as the caller's problem asks: under Quest scoring the
// query rows are transformed into the workspace first and the selection
// kernels run on the transformed problem.
static cudaError_t run_selection(const Prob &p, const WsLayout &w, const void *Q, const void *L, int32_t *idx,
                                 float *score, int32_t *keff, char *ws, cudaStream_t st) {
    if (!w.quest) return launch_select(p, w, Q, L, idx, score, keff, ws, st);
    if (p.rows == 0) return cudaSuccess;
    void *Qp = ws + w.quest_q;
    cudaError_t e = launch_quest_qprep(p, Q, Qp, st);
    if (e != cudaSuccess) return e;
    return launch_select(quest_select_view(p), w, Qp, L, idx, score, keff, ws, st);
}

// Landmarks, or the Quest chunk summaries under HSA_FLAG_QUEST.
static cudaError_t run_landmarks(const Prob &p, const void *K, const void *W_L, void *L, cudaStream_t st) {
    if (p.flags & HSA_FLAG_QUEST) return launch_quest_summaries(p, K, L, st);
    return launch_landmarks(p, K, W_L, L, st);
}

static hsa_status_t clear_status(char *ws, const WsLayout &w, cudaStream_t st) {
    cudaError_t e = cudaMemsetAsync(ws, 0, w.clear_bytes, st);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "clearing the device-status word");
}

// Device copies that hsa_forward_host keeps in the caller's buffer: byte
// offsets (256-aligned) and sizes of Q, K, V, W_L, the landmarks and O.
struct HostLayout {
    size_t q, k, v, w, l, o, total;
    size_t q_bytes, kv_bytes, w_bytes, l_bytes;
};

static HostLayout host_layout(const Prob &p) {
    const size_t es = p.dtype == HSA_BF16 ? 2 : 4;
    const bool quest = (p.flags & HSA_FLAG_QUEST) != 0;
    HostLayout h{};
    size_t off = 0;
    auto take = [&](size_t n) {
        const size_t o = off;
        off += (n + 255) & ~size_t(255);
        return o;
    };
    h.q_bytes = (size_t)p.B * p.Tq * p.H * p.d * es;
    h.kv_bytes = (size_t)p.B * p.Tcap * p.Hkv * p.d * es;
    h.w_bytes = quest ? 0 : (size_t)p.d * p.d * es;
    h.l_bytes = (size_t)p.B * p.Hkv * p.Lc * (quest ? 2 : 1) * p.d * es;
    h.q = take(h.q_bytes);
    h.k = take(h.kv_bytes);
    h.v = take(h.kv_bytes);
    h.w = take(h.w_bytes);
    h.l = take(h.l_bytes);
    h.o = take(h.q_bytes);
    h.total = off > 256 ? off : 256;
    return h;
}

}  // namespace hsa

using namespace hsa;

extern "C" {

int hsa_abi_version(void) { return HSA_ABI_VERSION; }

int hsa_debug_checks(void) { return kDebugChecks ? 1 : 0; }

const char *hsa_last_error(void) { return g_err; }

const char *hsa_status_string(hsa_status_t s) {
    switch (s) {
        case HSA_OK: return "HSA_OK";
        case HSA_ERR_INVALID_ARG: return "HSA_ERR_INVALID_ARG: invalid argument";
        case HSA_ERR_UNSUPPORTED: return "HSA_ERR_UNSUPPORTED: shape not implemented";
        case HSA_ERR_WORKSPACE: return "HSA_ERR_WORKSPACE: workspace missing or too small";
        case HSA_ERR_CUDA: return "HSA_ERR_CUDA: CUDA call failed";
        case HSA_ERR_TIMEOUT: return "HSA_ERR_TIMEOUT: a device-side wait expired";
    }
    return "unknown hsa_status_t";
}

hsa_status_t hsa_workspace_size(const hsa_problem_t *prob, size_t *bytes) {
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (!bytes) return fail(HSA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = ws_layout(p).total;
    return HSA_OK;
}

hsa_status_t hsa_plan(const hsa_problem_t *prob, hsa_plan_t *plan) {
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (!plan) return fail(HSA_ERR_INVALID_ARG, "plan is NULL");
    *plan = ws_layout(p).plan;
    return HSA_OK;
}

hsa_status_t hsa_landmarks(const hsa_problem_t *prob, const void *K, const void *W_L, void *L, void *stream) {
    NvtxRange nvtx_("hsa_landmarks");
    Prob p;
    HSA_TRY(validate(prob, &p));
    const bool any = (long long)p.B * p.C > 0;
    HSA_TRY(need(K, any, "K"));
    HSA_TRY(need(W_L, any && !(p.flags & HSA_FLAG_QUEST), "W_L"));
    HSA_TRY(need(L, any, "L"));
    cudaError_t e = run_landmarks(p, K, W_L, L, (cudaStream_t)stream);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "landmark kernel launch");
}

hsa_status_t hsa_landmarks_refined(const hsa_problem_t *prob, const void *K, const void *W_L, const void *W_q,
                                   const void *W_k, const void *W_v, void *L, void *stream) {
    NvtxRange nvtx_("hsa_landmarks_refined");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.flags & HSA_FLAG_QUEST) return fail(HSA_ERR_INVALID_ARG, "the refiner makes landmarks, not Quest summaries");
    const bool any = (long long)p.B * p.C > 0;
    HSA_TRY(need(K, any, "K"));
    HSA_TRY(need(W_L, any, "W_L"));
    HSA_TRY(need(W_q, any, "W_q"));
    HSA_TRY(need(W_k, any, "W_k"));
    HSA_TRY(need(W_v, any, "W_v"));
    HSA_TRY(need(L, any, "L"));
    cudaError_t e = launch_landmarks_refined(p, K, W_L, W_q, W_k, W_v, L, (cudaStream_t)stream);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "refined landmark kernel launch");
}

hsa_status_t hsa_decode_append(const hsa_problem_t *prob, const void *k_new, const void *v_new, void *K, void *V,
                               const void *W_L, void *L, void *stream) {
    NvtxRange nvtx_("hsa_decode_append");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.B > 0 && p.Tkv >= p.Tcap)
        return fail(HSA_ERR_INVALID_ARG, "no room to append: Tkv=%d, kv_cap=%d", p.Tkv, p.Tcap);
    const bool any = p.B > 0;
    const bool completes = any && (p.Tkv + 1) % p.S == 0;
    HSA_TRY(need(k_new, any, "k_new"));
    HSA_TRY(need(v_new, any, "v_new"));
    HSA_TRY(need(K, any, "K"));
    HSA_TRY(need(V, any, "V"));
    const bool quest = (p.flags & HSA_FLAG_QUEST) != 0;
    HSA_TRY(need(W_L, completes && !quest, "W_L"));
    HSA_TRY(need(L, completes, "L"));
    cudaStream_t st = (cudaStream_t)stream;
    if (quest) {
        // the append alone, then the completed chunk's summary (stream-ordered after the append)
        Prob pa = p;
        pa.S = p.Tcap + 1;   // no chunk completes for the append kernel
        cudaError_t e = launch_decode_append(pa, k_new, v_new, K, V, nullptr, nullptr, st);
        if (e == cudaSuccess && completes) e = launch_quest_summary_chunk(p, K, L, (p.Tkv + 1) / p.S - 1, st);
        return e == cudaSuccess ? HSA_OK : cuda_fail(e, "decode append kernel launch");
    }
    cudaError_t e = launch_decode_append(p, k_new, v_new, K, V, W_L, L, st);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "decode append kernel launch");
}

hsa_status_t hsa_select(const hsa_problem_t *prob, const void *Q, const void *L, int32_t *idx, float *score,
                        int32_t *keff, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange nvtx_("hsa_select");
    Prob p;
    HSA_TRY(validate(prob, &p));
    const bool rows = p.rows > 0;
    HSA_TRY(need(Q, rows, "Q"));
    HSA_TRY(need(L, rows && p.C > 0, "L"));
    HSA_TRY(need(idx, rows, "idx"));
    HSA_TRY(need(score, rows, "score"));
    HSA_TRY(need(keff, rows, "keff"));
    const WsLayout w = ws_layout(p);
    HSA_TRY(check_ws(w, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    HSA_TRY(clear_status((char *)ws, w, st));
    cudaError_t e = run_selection(p, w, Q, L, idx, score, keff, (char *)ws, st);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "selection kernel launch");
}

hsa_status_t hsa_attend(const hsa_problem_t *prob, const void *Q, const void *K, const void *V, const int32_t *idx,
                        const float *score, const int32_t *keff, void *O, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange nvtx_("hsa_attend");
    Prob p;
    HSA_TRY(validate(prob, &p));
    const bool rows = p.rows > 0;
    HSA_TRY(need(Q, rows, "Q"));
    HSA_TRY(need(K, rows && p.C > 0, "K"));
    HSA_TRY(need(V, rows && p.C > 0, "V"));
    HSA_TRY(need(idx, rows, "idx"));
    HSA_TRY(need(score, rows, "score"));
    HSA_TRY(need(keff, rows, "keff"));
    HSA_TRY(need(O, rows, "O"));
    const WsLayout w = ws_layout(p);
    HSA_TRY(check_ws(w, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    HSA_TRY(clear_status((char *)ws, w, st));
    cudaError_t e = launch_attend(p, w, Q, K, V, idx, score, keff, O, (char *)ws, st);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "attention kernel launch");
}

hsa_status_t hsa_attend_partials(const hsa_problem_t *prob, const void *Q, const void *K, const void *V,
                                 const int32_t *idx, const int32_t *keff, float *o_part, void *ws, size_t ws_bytes,
                                 void *stream) {
    NvtxRange nvtx_("hsa_attend_partials");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.rows > 0 && !attend_gather_supported(p))
        return fail(HSA_ERR_UNSUPPORTED, "partial outputs need the chunk-gather path (bf16, d 64/128, G <= 16)");
    const bool rows = p.rows > 0;
    HSA_TRY(need(Q, rows, "Q"));
    HSA_TRY(need(K, rows && p.C > 0, "K"));
    HSA_TRY(need(V, rows && p.C > 0, "V"));
    HSA_TRY(need(idx, rows, "idx"));
    HSA_TRY(need(keff, rows, "keff"));
    HSA_TRY(need(o_part, rows, "o_part"));
    const WsLayout w = ws_layout(p);
    HSA_TRY(check_ws(w, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    HSA_TRY(clear_status((char *)ws, w, st));
    if (!rows || p.C == 0) return HSA_OK;
    cudaError_t e = launch_attend_gather(p, Q, K, V, idx, nullptr, keff, nullptr, nullptr, nullptr,
                                         reinterpret_cast<uint32_t *>((char *)ws + w.hdr), st, o_part);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "partial attention kernel launch");
}

hsa_status_t hsa_merge_partials(const hsa_problem_t *prob, int nshard, const float *score, const int32_t *idx,
                                const int32_t *keff, const float *o_part, void *O, int32_t *idx_out,
                                float *score_out, int32_t *keff_out, void *stream) {
    NvtxRange nvtx_("hsa_merge_partials");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (nshard < 1) return fail(HSA_ERR_INVALID_ARG, "nshard=%d", nshard);
    if (!merge_supported(p, nshard))
        return fail(HSA_ERR_UNSUPPORTED, "merge of %d shards x %d slots, G*d=%d (max 256 candidates, G*d <= 2048)",
                    nshard, p.kmax, p.G * p.d);
    const bool rows = p.rows > 0;
    HSA_TRY(need(score, rows, "score"));
    HSA_TRY(need(idx, rows, "idx"));
    HSA_TRY(need(keff, rows, "keff"));
    HSA_TRY(need(o_part, rows, "o_part"));
    HSA_TRY(need(O, rows, "O"));
    cudaError_t e = launch_merge_partials(p, nshard, score, idx, keff, o_part, O, idx_out, score_out, keff_out,
                                          (cudaStream_t)stream);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "merge kernel launch");
}

hsa_status_t hsa_forward(const hsa_problem_t *prob, const void *Q, const void *K, const void *V, const void *W_L,
                         void *L, int32_t *idx, float *score, int32_t *keff, void *O, void *ws, size_t ws_bytes,
                         void *stream) {
    NvtxRange nvtx_("hsa_forward");
    Prob p;
    HSA_TRY(validate(prob, &p));
    const bool rows = p.rows > 0;
    const bool ready = (p.flags & HSA_FLAG_LANDMARKS_READY) != 0;
    const bool chunks = (long long)p.B * p.C > 0;
    HSA_TRY(need(Q, rows, "Q"));
    HSA_TRY(need(K, (rows && p.C > 0) || (chunks && !ready), "K"));
    HSA_TRY(need(V, rows && p.C > 0, "V"));
    HSA_TRY(need(W_L, chunks && !ready && !(p.flags & HSA_FLAG_QUEST), "W_L"));
    HSA_TRY(need(L, chunks, "L"));
    if (idx && !aligned16(idx)) return fail(HSA_ERR_INVALID_ARG, "idx is not 16-byte aligned");
    if (score && !aligned16(score)) return fail(HSA_ERR_INVALID_ARG, "score is not 16-byte aligned");
    if (keff && !aligned16(keff)) return fail(HSA_ERR_INVALID_ARG, "keff is not 16-byte aligned");
    HSA_TRY(need(O, rows, "O"));
    const WsLayout w = ws_layout(p);
    HSA_TRY(check_ws(w, ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    char *wsb = (char *)ws;
    HSA_TRY(clear_status(wsb, w, st));
    cudaError_t e;
    if (!ready) {
        e = run_landmarks(p, K, W_L, L, st);
        if (e != cudaSuccess) return cuda_fail(e, "landmark kernel launch");
    }
    int32_t *sidx = idx ? idx : reinterpret_cast<int32_t *>(wsb + w.sel_idx);
    float *ssc = score ? score : reinterpret_cast<float *>(wsb + w.sel_score);
    int32_t *skf = keff ? keff : reinterpret_cast<int32_t *>(wsb + w.sel_keff);
    if (w.fused_decode && p.C > 0) {
        e = launch_decode_fused(p, Q, K, V, L, sidx, ssc, skf, O, reinterpret_cast<float2 *>(wsb + w.split_lists),
                                reinterpret_cast<int32_t *>(wsb + w.sel_cnt), reinterpret_cast<unsigned long long *>(wsb + w.dec_desc),
                                reinterpret_cast<int32_t *>(wsb + w.dec_ctr), reinterpret_cast<int32_t *>(wsb + w.att_cnt),
                                reinterpret_cast<float *>(wsb + w.att_acc), reinterpret_cast<uint32_t *>(wsb + w.hdr),
                                w.stream_grid, w.stream_maxe, st);
        if (e != cudaErrorCooperativeLaunchTooLarge)
            return e == cudaSuccess ? HSA_OK : cuda_fail(e, "fused decode kernel launch");
        // the device cannot hold every CTA at once right now: the same two kernels, one after the other
        cudaGetLastError();
    }
    e = run_selection(p, w, Q, L, sidx, ssc, skf, wsb, st);
    if (e != cudaSuccess) return cuda_fail(e, "selection kernel launch");
    e = launch_attend(p, w, Q, K, V, sidx, ssc, skf, O, wsb, st);
    if (e != cudaSuccess) return cuda_fail(e, "attention kernel launch");
    return HSA_OK;
}

hsa_status_t hsa_forward_host_bytes(const hsa_problem_t *prob, size_t *bytes) {
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (!bytes) return fail(HSA_ERR_INVALID_ARG, "bytes is NULL");
    *bytes = host_layout(p).total;
    return HSA_OK;
}

hsa_status_t hsa_forward_host(const hsa_problem_t *prob, const void *Q, const void *K, const void *V,
                              const void *W_L, void *O, void *dev, size_t dev_bytes, void *ws, size_t ws_bytes,
                              void *stream) {
    NvtxRange nvtx_("hsa_forward_host");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.flags & HSA_FLAG_LANDMARKS_READY)
        return fail(HSA_ERR_INVALID_ARG, "hsa_forward_host makes the landmarks from K: HSA_FLAG_LANDMARKS_READY "
                    "is not accepted (use hsa_forward)");
    // the host tensors hsa_forward will read (landmarks are always made here)
    const bool rows = p.rows > 0;
    const bool chunks = (long long)p.B * p.C > 0;
    const bool need_k = (rows && p.C > 0) || chunks;
    const bool need_v = rows && p.C > 0;
    const bool need_w = chunks && !(p.flags & HSA_FLAG_QUEST);
    if (rows && !Q) return fail(HSA_ERR_INVALID_ARG, "Q is NULL");
    if (need_k && !K) return fail(HSA_ERR_INVALID_ARG, "K is NULL");
    if (need_v && !V) return fail(HSA_ERR_INVALID_ARG, "V is NULL");
    if (need_w && !W_L) return fail(HSA_ERR_INVALID_ARG, "W_L is NULL");
    if (rows && !O) return fail(HSA_ERR_INVALID_ARG, "O is NULL");
    const HostLayout h = host_layout(p);
    if (!dev) return fail(HSA_ERR_INVALID_ARG, "device buffer is NULL");
    if ((uintptr_t)dev & 255u) return fail(HSA_ERR_INVALID_ARG, "device buffer is not 256-byte aligned");
    if (dev_bytes < h.total)
        return fail(HSA_ERR_INVALID_ARG, "device buffer has %zu bytes, needs %zu", dev_bytes, h.total);
    HSA_TRY(check_ws(ws_layout(p), ws, ws_bytes));
    cudaStream_t st = (cudaStream_t)stream;
    char *db = (char *)dev;
    cudaError_t e = cudaSuccess;
    auto up = [&](size_t off, const void *src, size_t n, bool needed) {
        if (e == cudaSuccess && needed && n > 0) e = cudaMemcpyAsync(db + off, src, n, cudaMemcpyHostToDevice, st);
    };
    up(h.q, Q, h.q_bytes, rows);
    up(h.k, K, h.kv_bytes, need_k);
    up(h.v, V, h.kv_bytes, need_v);
    up(h.w, W_L, h.w_bytes, need_w);
    if (e != cudaSuccess) return cuda_fail(e, "host-to-device copy of the inputs");
    HSA_TRY(hsa_forward(prob, db + h.q, db + h.k, db + h.v, db + h.w, db + h.l, nullptr, nullptr, nullptr, db + h.o,
                        ws, ws_bytes, stream));
    if (rows && h.q_bytes > 0) {
        e = cudaMemcpyAsync(O, db + h.o, h.q_bytes, cudaMemcpyDeviceToHost, st);
        if (e != cudaSuccess) return cuda_fail(e, "device-to-host copy of O");
    }
    return HSA_OK;
}

hsa_status_t hsa_backward_workspace_size(const hsa_problem_t *prob, size_t *bytes) {
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.flags & HSA_FLAG_QUEST) return fail(HSA_ERR_UNSUPPORTED, "backward of Quest scoring is not implemented");
    if (!bytes) return fail(HSA_ERR_INVALID_ARG, "bytes is NULL");
    if (!backward_supported(p)) return fail(HSA_ERR_UNSUPPORTED, "backward: problem too large for 32-bit pair indices");
    *bytes = backward_layout(p).total;
    return HSA_OK;
}

hsa_status_t hsa_backward(const hsa_problem_t *prob, const void *Q, const void *K, const void *V, const void *W_L,
                          const void *L, const int32_t *idx, const float *score, const int32_t *keff, const void *dO,
                          float *dQ, float *dK, float *dV, float *dW_L, void *ws, size_t ws_bytes, void *stream) {
    NvtxRange nvtx_("hsa_backward");
    Prob p;
    HSA_TRY(validate(prob, &p));
    if (p.flags & HSA_FLAG_QUEST) return fail(HSA_ERR_UNSUPPORTED, "backward of Quest scoring is not implemented");
    if (!backward_supported(p)) return fail(HSA_ERR_UNSUPPORTED, "backward: problem too large for 32-bit pair indices");
    const bool rows = p.rows > 0;
    const bool work = rows && p.C > 0;
    const bool kv = (long long)p.B * p.Tcap > 0;
    HSA_TRY(need(Q, rows, "Q"));
    HSA_TRY(need(K, work, "K"));
    HSA_TRY(need(V, work, "V"));
    HSA_TRY(need(W_L, work, "W_L"));
    HSA_TRY(need(L, work, "L"));
    HSA_TRY(need(idx, work, "idx"));
    HSA_TRY(need(score, work, "score"));
    HSA_TRY(need(keff, work, "keff"));
    HSA_TRY(need(dO, rows, "dO"));
    HSA_TRY(need(dQ, rows, "dQ"));
    HSA_TRY(need(dK, kv, "dK"));
    HSA_TRY(need(dV, kv, "dV"));
    HSA_TRY(need(dW_L, true, "dW_L"));
    const BwdLayout w = backward_layout(p);
    if (ws_bytes < w.total) return fail(HSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, w.total);
    if (!ws) return fail(HSA_ERR_WORKSPACE, "workspace is NULL");
    if ((uintptr_t)ws & 255u) return fail(HSA_ERR_WORKSPACE, "workspace is not 256-byte aligned");
    cudaError_t e = launch_backward(p, w, (char *)ws, device_sms(), Q, K, V, W_L, L, idx, score, keff, dO, dQ, dK,
                                    dV, dW_L, (cudaStream_t)stream);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "backward kernel launch");
}

hsa_status_t hsa_get_device_status(void *ws, size_t ws_bytes, void *stream) {
    if (!ws || ws_bytes < 256) return fail(HSA_ERR_WORKSPACE, "workspace missing or smaller than its header");
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, ws, sizeof word, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device-status word");
    if (word == DEV_OK) return HSA_OK;
    e = cudaMemsetAsync(ws, 0, sizeof word, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the device-status word");
    if (word & DEV_TIMEOUT) return fail(HSA_ERR_TIMEOUT, "device-status word 0x%x: a bounded device wait expired", word);
    if (word & DEV_INTERNAL)
        return fail(HSA_ERR_CUDA, "device-status word 0x%x: a kernel's internal index check failed (the access was "
                    "skipped or, in the debug build, clamped; results of that call are incomplete)", word);
    return fail(HSA_ERR_INVALID_ARG, "device-status word 0x%x: hsa_attend got a keff or chunk index outside "
                "its row's candidates (those slots were skipped)", word);
}

}  // extern "C"
