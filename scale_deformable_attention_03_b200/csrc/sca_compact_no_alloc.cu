// sca_compact_no_alloc: the bev_mask compaction of sca_compact for callers
// that cannot allocate device memory.
//
// The two compaction passes need one int of scratch per (batch item, camera,
// 1024-query chunk): the number of seeing queries in that chunk.  sca_compact
// takes that scratch from a caller workspace.  Some callers cannot provide
// one: the framework around them owns all device memory and hands out no
// scratch for this step, or the pipeline forbids allocation once it is
// running, because cudaMalloc can block and cudaFree synchronises the device.
// This entry point keeps the scratch in a fixed array that the library itself
// owns, so the caller passes only its inputs and outputs.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "msda.h"
#include "msda_launch.h"

namespace {

// The per-chunk counts.  Its size is fixed at MSDA_NO_ALLOC_COUNT_SLOTS ints
// (256 KiB); every GPU that loads the library holds it until the process
// exits.  In host code this name is only a stand-in for the array, not a
// device address: the address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) int32_t g_chunk_counts[MSDA_NO_ALLOC_COUNT_SLOTS];

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_address[kMaxDevices] = {nullptr};  // device address of g_chunk_counts, per device

// The array's address on the current device, looked up the first time this
// device calls in (with the device current) and remembered afterwards.
cudaError_t chunk_counts_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_address[dev] == nullptr) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_chunk_counts);
        if (e != cudaSuccess) return e;
        g_address[dev] = p;
    }
    *out = g_address[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" msda_status_t sca_compact_no_alloc(const uint8_t* bev_mask, msda_dims_t d,
                                              int32_t* idx, int32_t* count, int32_t* pos,
                                              int32_t* hits, msda_stream_t stream)
{
    char msg[256];
    if (d.B < 0 || d.Nq < 0) {
        snprintf(msg, sizeof(msg), "B (%d) and Nq (%d) must be >= 0", d.B, d.Nq);
        return msda::api_fail(MSDA_ERR_INVALID_ARG, msg);
    }
    if (d.Ncam < 1 || d.Ncam > MSDA_MAX_CAMERAS) {
        snprintf(msg, sizeof(msg), "Ncam = %d outside 1..%d", d.Ncam, MSDA_MAX_CAMERAS);
        return msda::api_fail(MSDA_ERR_UNSUPPORTED, msg);
    }
    if (d.R < 1) {
        snprintf(msg, sizeof(msg), "R = %d must be >= 1", d.R);
        return msda::api_fail(MSDA_ERR_INVALID_ARG, msg);
    }
    if ((int64_t)d.B * d.Ncam > MSDA_MAX_BATCH_CAMERAS ||
        (int64_t)d.B * d.Ncam * d.Nq > INT32_MAX) {
        return msda::api_fail(MSDA_ERR_UNSUPPORTED,
                              "B * Ncam or B * Ncam * Nq exceeds the supported range");
    }
    if (d.B == 0) return msda::api_ok();
    const int64_t chunks = d.Nq > 0 ? ((int64_t)d.Nq + msda::kCompactChunk - 1) / msda::kCompactChunk : 1;
    const int64_t slots = (int64_t)d.B * d.Ncam * chunks;
    if (slots > MSDA_NO_ALLOC_COUNT_SLOTS) {
        snprintf(msg, sizeof(msg),
                 "needs %lld count slots (B * Ncam * ceil(Nq / 1024)); the fixed array holds %d",
                 (long long)slots, MSDA_NO_ALLOC_COUNT_SLOTS);
        return msda::api_fail(MSDA_ERR_UNSUPPORTED, msg);
    }
    if (count == nullptr || ((uintptr_t)count & 3)) return msda::api_fail(MSDA_ERR_INVALID_ARG, "count is null or misaligned");
    if (d.Nq > 0) {
        if (bev_mask == nullptr) return msda::api_fail(MSDA_ERR_INVALID_ARG, "bev_mask is null");
        if (idx == nullptr || pos == nullptr || hits == nullptr ||
            (((uintptr_t)idx | (uintptr_t)pos | (uintptr_t)hits) & 3))
            return msda::api_fail(MSDA_ERR_INVALID_ARG, "idx, pos or hits is null or misaligned");
    }
    void* scratch = nullptr;
    const cudaError_t e = chunk_counts_address(&scratch);
    if (e != cudaSuccess) return msda::api_cuda(e, "sca_compact_no_alloc: cudaGetSymbolAddress");
    // The first pass writes every count the second pass reads, so nothing in
    // the array has to start at zero.
    return msda::api_cuda(msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, idx, count,
                                                   pos, hits, static_cast<int32_t*>(scratch),
                                                   (cudaStream_t)stream),
                          "sca_compact_no_alloc");
}
