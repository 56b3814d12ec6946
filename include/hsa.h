/*
 * hsa.h -- C ABI of the B200 (sm_100a) Hierarchical Sparse Attention forward path and its backward.
 *
 * Method: "Every Token Counts 16m Context" (HSA summary page), sections Core
 * Technique and Implementation.  The key sequence is cut into fixed-length,
 * non-overlapping chunks of S tokens.  Every chunk gets a landmark: the mean of
 * its keys, projected by a learned d x d matrix W_L.  Every query scores the
 * landmarks of the chunks strictly before its own and keeps the k best.  It
 * attends inside each kept chunk with standard softmax attention.  The k chunk
 * outputs are then fused, weighted by the softmax of their retrieval scores.
 * The optional gap router (value-of-information router page, abstract) doubles
 * k for rows whose top-k cut is nearly tied.
 *
 * Conventions shared by every entry point:
 *   - All tensor arguments are DEVICE pointers, except the tensors of
 *     hsa_forward_host, which live in host memory.  The caller allocates them,
 *     and also the workspace.  The library never allocates, keeps no global
 *     mutable state, and is safe to call from several host threads on
 *     different streams, each with its own workspace.
 *   - Calls are asynchronous and ordered on `stream` (a cudaStream_t; NULL =
 *     the legacy default stream).  Host-side validation runs before any launch.
 *     An invalid call launches nothing and returns a status.
 *   - Layouts (row-major, contiguous, every device pointer 16-byte aligned):
 *       Q, O   [B][Tq][H][d]       K, V  [B][Tcap][Hkv][d]
 *       W_L    [d][d]  (row = input dim: landmark = mean_row * W_L)
 *       L      [B][Hkv][Ccap][d],  C = floor(Tkv / S) of them valid
 *     Tkv is the number of cached tokens; Tcap >= Tkv (hsa_problem_t.kv_cap,
 *     0 = Tkv) the tokens the K/V buffers hold per sequence, and
 *     Ccap = floor(Tcap / S) the chunks L holds per (b, kv head).  A decode
 *     loop keeps Tcap fixed while Tkv grows (hsa_decode_append).
 *       idx    [B][Tq][Hkv][kmax] int32   score [B][Tq][Hkv][kmax] float
 *       keff   [B][Tq][Hkv] int32,        kmax = (tau > 0 ? 2k : k)
 *     Q, K, V, W_L, L and O all have the problem's dtype.  Scores are fp32 and
 *     indices int32.
 *   - Query head h reads kv head floor(h / G), with G = H / Hkv.  One chunk
 *     selection is made per (batch, query, kv head).  It ranks chunks by the
 *     sum, over the G query heads, of the raw dot products q_h . L_c.
 *   - The query at row t sits at absolute position p = q_pos0 + t.  Its
 *     candidates are the complete chunks c < min(floor(p / S), C).  A trailing
 *     partial chunk (Tkv mod S tokens) has no landmark and is never a
 *     candidate.  Prefill: Tq == Tkv and q_pos0 = 0.  Decode: Tq = 1 and
 *     q_pos0 = Tkv.
 *   - Ranking: score descending, equal scores to the lower chunk index.
 *     keff = min(k, #candidates).  With the router on, when #candidates > k
 *     and (s_k - s_{k+1}) < tau * |s_k|: keff = min(2k, #candidates).
 *     Unused slots hold idx = -1 and score = -inf.  A row with keff = 0
 *     outputs zeros.
 *   - Arithmetic: products of stored values, fp32 accumulation, fp32
 *     softmax.  L and O are rounded once (to nearest, ties to even) to the
 *     dtype.
 *   - Errors are status codes only.  Nothing is thrown across the ABI.  A CUDA
 *     launch failure maps to HSA_ERR_CUDA.  A kernel whose bounded wait expired
 *     records HSA_ERR_TIMEOUT in the workspace header.
 *     hsa_get_device_status() reports it.  Inputs are assumed finite.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define HSA_ABI_VERSION 6

#if defined(__GNUC__)
#define HSA_API __attribute__((visibility("default")))
#else
#define HSA_API
#endif

typedef enum {
    HSA_OK = 0,
    HSA_ERR_INVALID_ARG = 1,   /* null pointer, bad shape, misaligned pointer, bad tau */
    HSA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels implement (d, S, k) */
    HSA_ERR_WORKSPACE = 3,     /* workspace missing or smaller than hsa_workspace_size() */
    HSA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed */
    HSA_ERR_TIMEOUT = 5        /* a device-side bounded wait expired (read via hsa_get_device_status) */
} hsa_status_t;

typedef enum { HSA_F32 = 0, HSA_BF16 = 1 } hsa_dtype_t;

/* hsa_problem_t.flags */
#define HSA_FLAG_LANDMARKS_READY 1u  /* hsa_forward: L already holds the landmarks; skip that stage (W_L may be NULL) */
#define HSA_FLAG_SIMT 2u             /* use the CUDA-core kernels even where a tensor-core kernel exists (testing) */
/* Testing only: the tcgen05 scoring kernel (hsa_select on the HSA_PATH_TENSOR select path;
 * other paths ignore the flag) runs with a 0.1 ms wait limit, and its epilogue first waits on a
 * barrier that nothing arrives on.  That wait expires, every role of the kernel winds down
 * (in-flight loads drained, MMAs committed, TMEM freed) and the call's status word records
 * HSA_ERR_TIMEOUT; idx/score/keff are left incomplete.  It exercises the failure path that a
 * real stall would take, without faulting or hanging the device. */
#define HSA_FLAG_TEST_STALL 4u
/* Quest block scoring in place of the landmark dot product (value-of-information router page,
 * abstract: the router stacks on block scorers such as Quest).  "Landmarks" are then the Quest
 * chunk summaries Lq [B][Hkv][Ccap][2d]: the channel-wise max of the chunk's keys, then the
 * channel-wise min (exact stored values; hsa_landmarks computes them and takes no W_L).  A query
 * row's score of chunk c is sum_{h in group} sum_e max(q_h[e] Lq_c[e], q_h[e] Lq_c[d + e]);
 * candidates, ranking, ties, keff, router and the fusion weights (softmax of these scores) are
 * unchanged.  Honoured by hsa_landmarks, hsa_decode_append, hsa_select, hsa_forward and
 * hsa_workspace_size; hsa_backward and hsa_select_noalloc return HSA_ERR_UNSUPPORTED. */
#define HSA_FLAG_QUEST 8u

typedef struct {
    int32_t B, Tq, Tkv, H, Hkv, d, S, k;
    int64_t q_pos0;      /* absolute position of query row 0 */
    float tau;           /* gap-router threshold; 0 disables it, > 0 enables it (then 2k <= 32) */
    int32_t dtype;       /* hsa_dtype_t */
    uint32_t flags;      /* HSA_FLAG_* */
    int32_t kv_cap;      /* Tcap: tokens per sequence the K/V buffers hold (0 = Tkv; else >= Tkv) */
} hsa_problem_t;

/* Supported shapes: d in {64, 128}; S in {32, 64, 128}; 1 <= k <= 32 (2k <= 32 with the
 * router); H % Hkv == 0 and G = H / Hkv <= 16.  B, Tq or Tkv may be 0 (nothing to do). */

/*
 * Bytes of device workspace that hsa_select / hsa_attend / hsa_forward need for
 * problem *p.  The workspace must be 256-byte aligned.  A call may use all of it
 * and leaves no state in it that a later call depends on, except the
 * device-status word that hsa_get_device_status() reads and clears.  Calls
 * that overlap on the GPU must use distinct workspaces.
 * Returns HSA_ERR_INVALID_ARG / HSA_ERR_UNSUPPORTED for a bad problem.
 */
HSA_API hsa_status_t hsa_workspace_size(const hsa_problem_t *p, size_t *bytes);

/*
 * Landmarks (summary page, Implementation: landmark = encode(mean pool of the
 * chunk), with encode read as the d x d projection W_L):
 *   L[b][j][c][:] = ( (1/S) sum_{u<S} K[b][cS+u][j][:] ) * W_L
 * for every complete chunk c < C.  The mean and the projection are done in
 * fp32, and the result is rounded once to the dtype.  Needs no workspace.
 * Q-side fields (Tq, q_pos0, k, tau) are validated but not used.
 */
HSA_API hsa_status_t hsa_landmarks(const hsa_problem_t *p, const void *K, const void *W_L, void *L,
                           void *stream);

/*
 * Refined landmarks (HSA summary page, Implementation: a learned layer with
 * cross-attention refines the mean-pooled landmark).  For every complete chunk
 * c and kv head j, one head of cross-attention whose query is the pooled
 * landmark and whose keys and values are the chunk's own keys, added back:
 *   L0 = ( (1/S) sum_{u<S} K[b][cS+u][j][:] ) * W_L
 *   a_u = softmax_u( (L0 W_q) . (K[b][cS+u][j][:] W_k) / sqrt(d) )
 *   L[b][j][c][:] = L0 + sum_u a_u K[b][cS+u][j][:] W_v
 * W_L, W_q, W_k, W_v are d x d (row = input dim) in the dtype.  fp32 throughout,
 * one rounding of L to the dtype.  The result replaces hsa_landmarks' output:
 * pass it to hsa_select / hsa_forward (HSA_FLAG_LANDMARKS_READY).  Needs no
 * workspace; one launch.  HSA_FLAG_QUEST is rejected (HSA_ERR_INVALID_ARG).
 * hsa_backward differentiates the plain landmark only and does not apply.
 */
HSA_API hsa_status_t hsa_landmarks_refined(const hsa_problem_t *p, const void *K, const void *W_L, const void *W_q,
                                           const void *W_k, const void *W_v, void *L, void *stream);

/*
 * One step of a decode loop on a cache that grows in place (summary page,
 * Implementation: every chunk gets its landmark; a decode step that completes
 * a chunk therefore has to produce that chunk's landmark before a later query
 * can retrieve it).  With Tkv = the tokens cached before the step (< Tcap):
 *   K[b][Tkv][:][:] = k_new[b][:][:],  V[b][Tkv][:][:] = v_new[b][:][:]
 * for every sequence b (k_new, v_new are [B][Hkv][d]), and, if Tkv + 1 is a
 * multiple of S, the landmark of the chunk c = (Tkv + 1) / S - 1 that the new
 * token completes is written to L[b][:][c][:] exactly as hsa_landmarks
 * computes it (the same kernel code, so the two agree bit for bit).  The next
 * step's problem has Tkv + 1 (and, for its query, q_pos0 = Tkv + 1).  Only
 * B, Tkv, Hkv, d, S, dtype and kv_cap are used; Tkv must be < Tcap.  One
 * launch; needs no workspace.  W_L and L may be NULL when no chunk completes.
 */
HSA_API hsa_status_t hsa_decode_append(const hsa_problem_t *p, const void *k_new, const void *v_new, void *K,
                                       void *V, const void *W_L, void *L, void *stream);

/*
 * Chunk selection (summary page, Core Technique and Implementation: score all
 * landmarks, keep the top k; router page: gap router).  Writes idx, score and
 * keff as described above.  score holds the group-summed retrieval score of
 * each kept chunk (fp32).
 */
HSA_API hsa_status_t hsa_select(const hsa_problem_t *p, const void *Q, const void *L, int32_t *idx,
                        float *score, int32_t *keff, void *ws, size_t ws_bytes, void *stream);

/*
 * Chunk attention and fusion (summary page, Implementation: attend to each
 * selected chunk with standard attention, then fuse the results weighted by
 * the retrieval scores).  For each (b, t, kv head j) and each head h of the
 * group:
 *   w_i  = softmax_{i < keff}(score_i)
 *   o_i  = softmax_u(q_h . K[c_i S + u] / sqrt(d)) . V[c_i S + u]     (u < S)
 *   O[h] = sum_i w_i o_i                                              (0 when keff = 0)
 * idx/score/keff are as hsa_select writes them.  Every idx[i] for i < keff
 * must be a candidate chunk of its row and keff must lie in [0, kmax].  An
 * out-of-range value is never dereferenced: its slot is skipped, and
 * hsa_get_device_status() then reports HSA_ERR_INVALID_ARG.
 */
HSA_API hsa_status_t hsa_attend(const hsa_problem_t *p, const void *Q, const void *K, const void *V,
                        const int32_t *idx, const float *score, const int32_t *keff, void *O,
                        void *ws, size_t ws_bytes, void *stream);

/*
 * hsa_select without a workspace, for callers that cannot allocate device
 * memory at the point of the call: code that runs under an allocator that
 * must not be re-entered, a runtime whose memory pool is already carved up, or
 * an embedding that only owns the tensors it passes in.  It computes exactly
 * what hsa_select computes; the paper has no counterpart for this entry point.
 *   - Its scratch (the status word and, for few rows with long scans, the
 *     per-split candidate lists) is a 1 MiB array inside the library.  Every
 *     GPU that loads the library holds that array until the process exits.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress), so make that first call before any stream
 *     capture.  Later calls reuse the address.
 *   - Problems whose scratch would exceed 1 MiB are rejected with
 *     HSA_ERR_WORKSPACE before anything is launched (e.g. 64 decode rows over
 *     16384 chunks with k = 16 need ~0.13 MiB; prefill problems need only the
 *     status word; 4096 decode rows with 32 slots each need just over 1 MiB).
 *   - It calls no cudaMalloc, cudaFree or allocating library routine.
 *   - Every call on a device shares the one array, which keeps the last
 *     call's contents: calls that overlap on the GPU (other streams, other
 *     host threads) race on it and must be serialised by the caller.  A
 *     device-side timeout of this call is recorded in that array, not in any
 *     workspace: hsa_noalloc_status() reports it.
 */
HSA_API hsa_status_t hsa_select_noalloc(const hsa_problem_t *p, const void *Q, const void *L, int32_t *idx,
                                        float *score, int32_t *keff, void *stream);

/*
 * Device status of the latest hsa_select_noalloc call on the current device:
 * synchronises `stream`, then reads and clears the status word at the start of
 * the library's static scratch (every hsa_select_noalloc call clears it when it
 * starts).  Returns HSA_OK, HSA_ERR_TIMEOUT (a bounded device wait expired; the
 * call's idx/score/keff are incomplete) or HSA_ERR_CUDA (a kernel's own index
 * check failed and skipped the access).  Allocates nothing.
 */
HSA_API hsa_status_t hsa_noalloc_status(void *stream);

/*
 * Context-sharded decode, per shard (summary page, Implementation: the
 * retrieval scores rank the chunks and weight their outputs).  The chunks of
 * a sequence may be split into contiguous ranges held by different devices
 * (shards): each shard selects its own top kmax chunks (hsa_select with
 * k = kmax and tau = 0, so its list is never cut by the router) and computes
 * here, for every selection row and kept slot i < keff, the chunk's attention
 * output for each of the G query heads, without the fusion weight:
 *   o_part[b][t][j][i][g][:] = softmax_u(q_{jG+g} . K[c_i S + u] / sqrt(d)) . V[c_i S + u]
 * (fp32, [B][Tq][Hkv][kmax][G][d]; slots i >= keff are not written).  idx holds
 * the shard's local chunk indices.  bf16 only, d 64/128; the rows' chunks are
 * all gathered at once, which suits decode (few rows).  Uses the workspace's
 * status word only (hsa_workspace_size of the same problem suffices).
 */
HSA_API hsa_status_t hsa_attend_partials(const hsa_problem_t *p, const void *Q, const void *K, const void *V,
                                         const int32_t *idx, const int32_t *keff, float *o_part, void *ws,
                                         size_t ws_bytes, void *stream);

/*
 * Context-sharded decode, the merge: from the nshard shards' selections and
 * partial outputs, concatenated shard-major as an all-gather leaves them --
 *   score, idx [nshard][B][Tq][Hkv][kmax] (idx: GLOBAL chunk indices),
 *   keff [nshard][B][Tq][Hkv], o_part [nshard][B][Tq][Hkv][kmax][G][d] --
 * the rows' selection over the whole context (the top kmax of the union, same
 * order and ties as hsa_select; then keff = min(k, #kept), doubled by the gap
 * router as in hsa_select) and the output
 *   O[b][t][jG+g][:] = sum_{i < keff} softmax_i(score_i) o_part[shard_i][b][t][j][slot_i][g][:].
 * The problem describes one shard's rows (B, Tq, H, Hkv, d, k, tau, dtype);
 * its Tkv is not used.  idx_out, score_out ([B][Tq][Hkv][kmax]) and keff_out
 * may each be NULL.  Needs nshard * kmax <= 256 and G * d <= 2048.  No
 * workspace.
 */
HSA_API hsa_status_t hsa_merge_partials(const hsa_problem_t *p, int nshard, const float *score,
                                        const int32_t *idx, const int32_t *keff, const float *o_part, void *O,
                                        int32_t *idx_out, float *score_out, int32_t *keff_out, void *stream);

/*
 * The whole path: hsa_landmarks (unless HSA_FLAG_LANDMARKS_READY), then
 * hsa_select, then hsa_attend.  L is an output (or an input with the flag).
 * idx, score and keff may each be NULL.  The selection then lives only in the
 * workspace.  For decode shapes (one query per sequence over a long context,
 * hsa_plan_t.forward_fused = 1) the selection and the attention run as one
 * cooperative launch: each row's chunks are gathered as soon as its selection
 * is complete, while other rows are still being scored.  The results are
 * those of hsa_select followed by hsa_attend (O up to fp32 summation order).
 */
HSA_API hsa_status_t hsa_forward(const hsa_problem_t *p, const void *Q, const void *K, const void *V,
                         const void *W_L, void *L, int32_t *idx, float *score, int32_t *keff,
                         void *O, void *ws, size_t ws_bytes, void *stream);

/*
 * hsa_forward for a caller whose tensors live in HOST memory.  On `stream` it
 * enqueues the copies of the inputs into the device buffer `dev`, the whole
 * forward of hsa_forward there (landmarks, selection, chunk attention and
 * fusion), and the copy of O back to host memory; each copy is one
 * cudaMemcpyAsync.  Host layouts are those of hsa_forward: Q and O
 * [B][Tq][H][d], K and V [B][Tcap][Hkv][d] (copied whole), W_L [d][d] (not
 * read under HSA_FLAG_QUEST).  A host pointer may be NULL only where
 * hsa_forward would not read the tensor (e.g. K and V with no chunks); host
 * pointers need no alignment.
 * dev: a device buffer of hsa_forward_host_bytes(p) bytes, 256-byte aligned,
 * that receives the device copies of Q, K, V, W_L, the landmarks and O; it is
 * the caller's and may be reused once the stream has passed this call.  ws:
 * the workspace of hsa_workspace_size(p).  Every argument is checked before
 * anything is enqueued.  The call returns once the work is enqueued: O is
 * complete when the stream reaches this point, and the host buffers must stay
 * valid until then.  With page-locked host memory the copies are
 * asynchronous, so calls on several streams (each with its own dev and ws)
 * overlap one call's uploads with another's compute and download.
 * HSA_FLAG_LANDMARKS_READY is refused: the landmarks are made here from K.
 */
HSA_API hsa_status_t hsa_forward_host_bytes(const hsa_problem_t *p, size_t *bytes);
HSA_API hsa_status_t hsa_forward_host(const hsa_problem_t *p, const void *Q, const void *K, const void *V,
                                      const void *W_L, void *O, void *dev, size_t dev_bytes, void *ws,
                                      size_t ws_bytes, void *stream);

/*
 * Backward pass: gradients of the method with respect to Q, K, V and W_L,
 * with the forward's chunk selection held fixed (HSA summary page,
 * Implementation: the kept chunks' retrieval scores weight their outputs, so
 * the scores carry a gradient; which chunks are kept is a discrete choice and
 * has none).  With w = softmax(score) over the kept slots of a selection row,
 * a the in-chunk attention probabilities and o the per-chunk outputs, it
 * returns the exact gradients of O = sum_i w_i o_i, for the upstream gradient
 * dO, through the in-chunk softmax attention, the fusion softmax, the group
 * scores s_i = sum_h q_h . L_ci, and the landmarks L_c = mean(K of chunk c) W_L.
 *
 * Inputs (the problem's dtype unless noted): Q, K, V, W_L and L as given to
 * hsa_forward (L: the landmarks the scores were taken from); idx, score, keff:
 * the selection the forward returned (score fp32: it sets the fusion
 * weights); dO [B][Tq][H][d].
 * Outputs, fp32, OVERWRITTEN (the call zeroes them first): dQ [B][Tq][H][d],
 * dK and dV [B][Tcap][Hkv][d] (the K/V layout; tokens past Tkv, and those of a
 * trailing partial chunk, get 0), dW_L [d][d].
 * L enters the scores as stored: its rounding to the dtype counts as the
 * identity in the chain rule.  A chunk index or keff outside its row's
 * candidates is skipped and recorded in the status word (HSA_ERR_INVALID_ARG
 * from hsa_get_device_status).  Workspace: hsa_backward_workspace_size (its
 * header is the status word).  The adds into dQ, dK, dV and dW_L are fp32
 * atomic reductions, so their order, and the last bits of the result, vary
 * from call to call.
 * Paths: bf16 with d = 128 and S = 64 or 128 uses the tcgen05 tensor cores,
 * with dZ (the in-chunk softmax gradient) and w P rounded to bf16 before the
 * dQ, dK and dV products; fp32, d = 64, S = 32, or HSA_FLAG_SIMT in p->flags
 * use fp32 CUDA-core arithmetic throughout.  Six kernel launches (plus the
 * zeroing of the outputs), all on `stream`.
 */
HSA_API hsa_status_t hsa_backward_workspace_size(const hsa_problem_t *p, size_t *bytes);
HSA_API hsa_status_t hsa_backward(const hsa_problem_t *p, const void *Q, const void *K, const void *V,
                                  const void *W_L, const void *L, const int32_t *idx, const float *score,
                                  const int32_t *keff, const void *dO, float *dQ, float *dK, float *dV,
                                  float *dW_L, void *ws, size_t ws_bytes, void *stream);

/*
 * Synchronises `stream`, then reads and clears the device-status word in the
 * workspace header.  Every call that takes a workspace clears that word when it
 * starts (stream-ordered), so the word describes the latest such call.
 * Returns HSA_OK, HSA_ERR_TIMEOUT (a bounded device wait expired),
 * HSA_ERR_INVALID_ARG (hsa_attend skipped an out-of-range chunk index or keff)
 * or HSA_ERR_CUDA (a CUDA call failed, or a kernel's own index check failed and
 * skipped the access, leaving that call's results incomplete).
 */
HSA_API hsa_status_t hsa_get_device_status(void *ws, size_t ws_bytes, void *stream);

/* Kernel paths a stage can take (hsa_plan_t.*_path). */
typedef enum {
    HSA_PATH_NONE = 0,         /* stage has nothing to do for this problem */
    HSA_PATH_SIMT_ROWS = 1,    /* CUDA cores, one warp / CTA per selection row (landmarks: per chunk) */
    HSA_PATH_SIMT_SPLIT = 2,   /* CUDA cores, each row split over CTAs, then merged */
    HSA_PATH_TENSOR = 3,       /* tcgen05 tensor-core kernel (TMEM accumulators), many rows per tile */
    HSA_PATH_MMA_SPLIT = 4     /* warp-level mma.sync tensor-core kernel for few rows: each row's chunks
                                  split over CTAs (decode scan, chunk gather), merged in the same launch */
} hsa_path_t;

typedef struct {
    int32_t landmark_path, select_path, attend_path;        /* hsa_path_t */
    int32_t landmark_kernels, select_kernels, attend_kernels; /* kernel launches per call of each stage */
    int32_t forward_fused;   /* 1: hsa_forward runs selection and attention as one launch (select_kernels
                                counts it; the attention stage adds none) */
} hsa_plan_t;

/*
 * Which kernels hsa_landmarks / hsa_select / hsa_attend launch for problem *p
 * (a pure function of the problem; nothing is launched).  hsa_forward launches
 * the sum of the three (minus the landmark stage with HSA_FLAG_LANDMARKS_READY,
 * and minus attend_kernels when forward_fused is 1).
 */
HSA_API hsa_status_t hsa_plan(const hsa_problem_t *p, hsa_plan_t *plan);

/* Static description of a status code. */
HSA_API const char *hsa_status_string(hsa_status_t s);

/* Detail of the last failing call on this host thread (which argument, which CUDA error). */
HSA_API const char *hsa_last_error(void);

/* 1 if the loaded library is the debug build (compiled with HSA_DEBUG): every
 * kernel checks the indices it derives itself -- gathered token and chunk
 * indices, TMA coordinates, accumulator offsets -- and a failed check is
 * recorded in the status word (hsa_get_device_status: HSA_ERR_CUDA, "internal
 * index check") with the index clamped into its range.  0 for release builds. */
HSA_API int hsa_debug_checks(void);

/* HSA_ABI_VERSION of the loaded library. */
HSA_API int hsa_abi_version(void);

#ifdef __cplusplus
}
#endif
#endif /* HSA_H_ */
