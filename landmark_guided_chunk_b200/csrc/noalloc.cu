// noalloc.cu -- hsa_select_noalloc: the chunk-selection stage with its scratch
// memory in a fixed device array, for callers that cannot allocate device
// memory (see include/hsa.h).
//
// The scratch is a file-scope __device__ array, so every GPU that loads this
// library holds it until the process exits.  In host code its name is only a
// host-side stand-in; the device address is fetched once per device with
// cudaGetSymbolAddress (with that device current) and passed to the kernels.
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace hsa {
namespace {

constexpr size_t NOALLOC_BYTES = 1u << 20;   // 1 MiB
__device__ __align__(256) unsigned char g_noalloc_scratch[NOALLOC_BYTES];

constexpr int MAX_DEVICES = 64;
std::mutex g_mu;
void *g_scratch_ptr[MAX_DEVICES] = {};

// Device address of the scratch on the current device (fetched on first use).
hsa_status_t scratch_on_current_device(void **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= MAX_DEVICES) return fail(HSA_ERR_UNSUPPORTED, "device ordinal %d (max %d)", dev, MAX_DEVICES - 1);
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the static scratch");
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HSA_OK;
}

}  // namespace
}  // namespace hsa

using namespace hsa;

static hsa_status_t select_noalloc_impl(const hsa_problem_t *prob, const void *Q, const void *L, int32_t *idx,
                                        float *score, int32_t *keff, void *stream);

extern "C" HSA_API hsa_status_t hsa_select_noalloc(const hsa_problem_t *prob, const void *Q, const void *L,
                                                   int32_t *idx, float *score, int32_t *keff, void *stream) {
    nvtxRangePushA("hsa_select_noalloc");
    const hsa_status_t r = select_noalloc_impl(prob, Q, L, idx, score, keff, stream);
    nvtxRangePop();
    return r;
}

static hsa_status_t select_noalloc_impl(const hsa_problem_t *prob, const void *Q, const void *L, int32_t *idx,
                                        float *score, int32_t *keff, void *stream) {
    Prob p;
    hsa_status_t s = validate(prob, &p);
    if (s != HSA_OK) return s;
    if (p.flags & HSA_FLAG_QUEST)
        return fail(HSA_ERR_UNSUPPORTED, "hsa_select_noalloc: Quest scoring needs a caller workspace (use hsa_select)");
    const bool rows = p.rows > 0;
    if ((s = need(Q, rows, "Q")) != HSA_OK) return s;
    if ((s = need(L, rows && p.C > 0, "L")) != HSA_OK) return s;
    if ((s = need(idx, rows, "idx")) != HSA_OK) return s;
    if ((s = need(score, rows, "score")) != HSA_OK) return s;
    if ((s = need(keff, rows, "keff")) != HSA_OK) return s;
    // The selection stage needs the status word and, on the split path, the
    // per-row counters of the tensor-core scan and the per-split candidate
    // lists; nothing else of the full workspace layout.
    const WsLayout full = ws_layout(p);
    WsLayout w{};
    w.tc_select = full.tc_select;
    w.split_select = full.split_select;
    w.mma_select = full.mma_select;
    w.stream_select = full.stream_select;
    w.stream_grid = full.stream_grid;
    w.stream_maxe = full.stream_maxe;
    w.nsplit = full.nsplit;
    w.chunks_per_split = full.chunks_per_split;
    w.hdr = 0;
    // after the status word: the per-row counters of the split scan (zeroed
    // with it), then the per-split candidate lists
    const size_t counters =
        (w.mma_select || w.stream_select) ? (((size_t)p.rows * sizeof(int32_t) + 255) & ~(size_t)255) : 0;
    w.sel_cnt = 256;
    w.split_lists = 256 + counters;
    const size_t slots = w.stream_select ? (size_t)w.stream_maxe : (size_t)w.nsplit;
    const size_t lists = w.split_select ? (size_t)p.rows * slots * p.kmax * sizeof(float2) : 0;
    const size_t needed = 256 + counters + lists;
    if (needed > NOALLOC_BYTES)
        return fail(HSA_ERR_WORKSPACE,
                    "hsa_select_noalloc: this problem needs %zu bytes of scratch; the static scratch holds %zu "
                    "(use hsa_select with a caller workspace)",
                    needed, NOALLOC_BYTES);
    if (!rows) return HSA_OK;
    void *scratch = nullptr;
    if ((s = scratch_on_current_device(&scratch)) != HSA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    // status word (and the split scan's counters) start clear
    cudaError_t e = cudaMemsetAsync(scratch, 0, counters ? 256 + counters : sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch status word");
    e = launch_select(p, w, Q, L, idx, score, keff, (char *)scratch, st);
    return e == cudaSuccess ? HSA_OK : cuda_fail(e, "selection kernel launch");
}

// Status of the latest hsa_select_noalloc call on the current device: the word
// at the start of the static scratch, read and cleared after `stream` drains.
extern "C" HSA_API hsa_status_t hsa_noalloc_status(void *stream) {
    void *scratch = nullptr;
    hsa_status_t s = scratch_on_current_device(&scratch);
    if (s != HSA_OK) return s;
    cudaStream_t st = (cudaStream_t)stream;
    uint32_t word = 0;
    cudaError_t e = cudaMemcpyAsync(&word, scratch, sizeof word, cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the static scratch status word");
    if (word == DEV_OK) return HSA_OK;
    e = cudaMemsetAsync(scratch, 0, sizeof word, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "clearing the static scratch status word");
    if (word & DEV_TIMEOUT)
        return fail(HSA_ERR_TIMEOUT, "static scratch status word 0x%x: a bounded device wait expired", word);
    return fail(HSA_ERR_CUDA, "static scratch status word 0x%x: a kernel's internal index check failed", word);
}
