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
#include <cuda.h>
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

// The array's device address is a property of the CUDA context that loaded
// the module, not of the device ordinal: after cudaDeviceReset, or with
// another context current, the old address is stale.  So each remembered
// address carries the unique id of the context it was looked up in
// (cuCtxGetId), and a lookup in any other context asks again.
struct Remembered {
    unsigned long long ctx_id;
    void* address;
};
Remembered g_remembered[kMaxDevices] = {};

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

// Unique id of the current context; 0 when there is none yet or the driver
// entry points are unavailable (then nothing is remembered).
unsigned long long current_context_id()
{
    static CtxGetCurrentFn get_current = nullptr;
    static CtxGetIdFn get_id = nullptr;
    static bool looked_up = false;
    if (!looked_up) {
        cudaDriverEntryPointQueryResult q1, q2;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", reinterpret_cast<void**>(&get_current),
                                    cudaEnableDefault, &q1) != cudaSuccess ||
            q1 != cudaDriverEntryPointSuccess)
            get_current = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", reinterpret_cast<void**>(&get_id),
                                    cudaEnableDefault, &q2) != cudaSuccess ||
            q2 != cudaDriverEntryPointSuccess)
            get_id = nullptr;
        looked_up = true;
    }
    if (get_current == nullptr || get_id == nullptr) return 0;
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

// The array's address in the current context of the current device: looked
// up (cudaGetSymbolAddress, with that device current) the first time a
// context calls in, and remembered for that context afterwards.
cudaError_t chunk_counts_address(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mutex);
    const unsigned long long id = current_context_id();
    Remembered& r = g_remembered[dev];
    if (id != 0 && r.ctx_id == id && r.address != nullptr) {
        *out = r.address;
        return cudaSuccess;
    }
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_chunk_counts);  // also creates the context if needed
    if (e != cudaSuccess) return e;
    r.ctx_id = current_context_id();
    r.address = r.ctx_id != 0 ? p : nullptr;
    *out = p;
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
