// The C ABI of libmsda.so (declared in include/msda.h): argument validation,
// workspace carving and kernel dispatch.  Host code only; no allocation.
#include <cuda_runtime.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "msda.h"
#include "msda_launch.h"

namespace {

thread_local char g_error[512] = "";

msda_status_t fail(msda_status_t code, const char* fmt, ...)
{
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_error, sizeof(g_error), fmt, ap);
    va_end(ap);
    return code;
}

msda_status_t ok()
{
    g_error[0] = '\0';
    return MSDA_OK;
}

msda_status_t cuda_status(cudaError_t e, const char* where)
{
    if (e == cudaSuccess) return ok();
    return fail(MSDA_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

#define MSDA_CHECK(cond, code, ...)                                                              \
    do {                                                                                         \
        if (!(cond)) return fail(code, __VA_ARGS__);                                             \
    } while (0)

// Sizes common to every call; `sca` adds the camera checks.
msda_status_t check_dims(const msda_dims_t& d, bool sca)
{
    MSDA_CHECK(d.B >= 0 && d.Nq >= 0, MSDA_ERR_INVALID_ARG, "B (%d) and Nq (%d) must be >= 0",
               d.B, d.Nq);
    MSDA_CHECK(d.Nv >= 1 && d.H >= 1, MSDA_ERR_INVALID_ARG, "Nv (%d) and H (%d) must be >= 1",
               d.Nv, d.H);
    MSDA_CHECK(d.L >= 1 && d.L <= MSDA_MAX_LEVELS, MSDA_ERR_UNSUPPORTED, "L = %d outside 1..%d",
               d.L, MSDA_MAX_LEVELS);
    MSDA_CHECK(d.P >= 1 && d.P <= MSDA_MAX_POINTS, MSDA_ERR_UNSUPPORTED, "P = %d outside 1..%d",
               d.P, MSDA_MAX_POINTS);
    MSDA_CHECK(d.R >= 1 && d.P % d.R == 0, MSDA_ERR_INVALID_ARG,
               "R = %d must be >= 1 and divide P = %d", d.R, d.P);
    // per-(batch, camera) value element offsets are 32-bit inside the kernels
    MSDA_CHECK((int64_t)d.Nv * d.H * MSDA_HEAD_DIM <= INT32_MAX, MSDA_ERR_UNSUPPORTED,
               "Nv * H * 32 = %lld exceeds the 32-bit index range",
               (long long)d.Nv * d.H * MSDA_HEAD_DIM);
    if (sca) {
        MSDA_CHECK(d.Ncam >= 1 && d.Ncam <= MSDA_MAX_CAMERAS, MSDA_ERR_UNSUPPORTED,
                   "Ncam = %d outside 1..%d", d.Ncam, MSDA_MAX_CAMERAS);
        MSDA_CHECK((int64_t)d.B * d.Ncam * d.Nq <= INT32_MAX, MSDA_ERR_UNSUPPORTED,
                   "B * Ncam * Nq exceeds the 32-bit row range");
    }
    return MSDA_OK;
}

msda_status_t check_levels(const msda_dims_t& d, const int64_t* shapes, const int64_t* starts,
                           msda::Levels& lv)
{
    MSDA_CHECK(shapes != nullptr && starts != nullptr, MSDA_ERR_INVALID_ARG,
               "spatial_shapes and level_start_index must be host arrays");
    std::memset(&lv, 0, sizeof(lv));
    for (int l = 0; l < d.L; ++l) {
        const int64_t Hl = shapes[2 * l], Wl = shapes[2 * l + 1], st = starts[l];
        MSDA_CHECK(Hl >= 1 && Wl >= 1 && Hl <= (1 << 24) && Wl <= (1 << 24), MSDA_ERR_INVALID_ARG,
                   "level %d has shape %lld x %lld", l, (long long)Hl, (long long)Wl);
        MSDA_CHECK(st >= 0 && st + Hl * Wl <= d.Nv, MSDA_ERR_INVALID_ARG,
                   "level %d (start %lld, %lld x %lld) does not fit in Nv = %d", l, (long long)st,
                   (long long)Hl, (long long)Wl, d.Nv);
        lv.h[l] = (int)Hl;
        lv.w[l] = (int)Wl;
        lv.start[l] = (int)st;
    }
    return MSDA_OK;
}

msda_status_t check_dtype(msda_dtype_t vdt)
{
    MSDA_CHECK(vdt == MSDA_F32 || vdt == MSDA_BF16, MSDA_ERR_INVALID_ARG, "unknown value dtype %d",
               (int)vdt);
    return MSDA_OK;
}

msda_status_t check_value(const void* value)
{
    MSDA_CHECK(value != nullptr, MSDA_ERR_INVALID_ARG, "value is null");
    MSDA_CHECK(aligned(value, 16), MSDA_ERR_INVALID_ARG, "value must be 16-byte aligned");
    return MSDA_OK;
}

#define MSDA_TRY(expr)                                                                           \
    do {                                                                                         \
        msda_status_t st_ = (expr);                                                              \
        if (st_ != MSDA_OK) return st_;                                                          \
    } while (0)

#define MSDA_PTR(p, align)                                                                       \
    do {                                                                                         \
        MSDA_CHECK((p) != nullptr, MSDA_ERR_INVALID_ARG, #p " is null");                         \
        MSDA_CHECK(aligned((p), (align)), MSDA_ERR_INVALID_ARG,                                  \
                   #p " must be " #align "-byte aligned");                                       \
    } while (0)

msda::Problem make_problem(const void* value, msda_dtype_t vdt, const msda_dims_t& d,
                           const msda::Levels& lv)
{
    msda::Problem p;
    p.value = value;
    p.bf16 = vdt == MSDA_BF16;
    p.B = d.B;
    p.Ncam = d.Ncam;
    p.Nq = d.Nq;
    p.Nv = d.Nv;
    p.H = d.H;
    p.L = d.L;
    p.P = d.P;
    p.R = d.R;
    p.lv = lv;
    return p;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

namespace msda {

int device_sm_count()
{
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
            n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

size_t compact_scratch_bytes(int B, int Ncam, int Nq)
{
    const size_t nbc = (size_t)B * Ncam;
    const size_t nchunks = Nq > 0 ? ((size_t)Nq + kCompactChunk - 1) / kCompactChunk : 1;
    return align256(sizeof(int32_t) * nbc * nchunks);
}

CompactScratch compact_scratch_carve(void* base, int, int, int)
{
    CompactScratch c;
    c.chunk_counts = static_cast<int32_t*>(base);
    return c;
}

size_t sca_workspace_bytes(int B, int Ncam, int Nq, int H, bool with_rows)
{
    const size_t nbc = (size_t)B * Ncam;
    size_t n = compact_scratch_bytes(B, Ncam, Nq);
    n += align256(sizeof(int32_t) * nbc * Nq);        // idx
    n += align256(sizeof(int32_t) * nbc * Nq);        // pos
    n += align256(sizeof(int32_t) * nbc);             // count
    n += align256(sizeof(int32_t) * (size_t)B * Nq);  // hits
    if (with_rows) n += align256(sizeof(float) * nbc * Nq * (size_t)H * kHeadDim);
    return n;
}

ScaWorkspace sca_workspace_carve(void* base, int B, int Ncam, int Nq, int H, bool with_rows)
{
    const size_t nbc = (size_t)B * Ncam;
    const CompactScratch cs = compact_scratch_carve(base, B, Ncam, Nq);
    char* p = static_cast<char*>(base) + compact_scratch_bytes(B, Ncam, Nq);
    ScaWorkspace w;
    w.chunk_counts = cs.chunk_counts;
    w.idx = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * nbc * Nq);
    w.pos = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * nbc * Nq);
    w.count = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * nbc);
    w.hits = reinterpret_cast<int32_t*>(p);
    p += align256(sizeof(int32_t) * (size_t)B * Nq);
    w.out_rb = with_rows ? reinterpret_cast<float*>(p) : nullptr;
    return w;
}

}  // namespace msda

extern "C" {

int32_t msda_version(void) { return 10200; }  // 1.2.0: sca_backward_full, precise TSA chain, four-lane gather

const char* msda_status_string(msda_status_t status)
{
    switch (status) {
        case MSDA_OK: return "success";
        case MSDA_ERR_INVALID_ARG: return "invalid argument";
        case MSDA_ERR_UNSUPPORTED: return "unsupported size";
        case MSDA_ERR_WORKSPACE: return "workspace missing or too small";
        case MSDA_ERR_CUDA: return "CUDA error";
    }
    return "unknown status";
}

const char* msda_last_error(void) { return g_error; }

msda_status_t msda_forward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                           const int64_t* level_start_index, const float* sampling_locations,
                           const float* attention_weights, msda_dims_t d, float* out,
                           msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_TRY(check_value(value));
    MSDA_PTR(sampling_locations, 8);
    MSDA_PTR(attention_weights, 4);
    MSDA_PTR(out, 16);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    return cuda_status(msda::launch_msda_forward(p, sampling_locations, attention_weights, out,
                                                 (cudaStream_t)stream),
                       "msda_forward");
}

msda_status_t msda_forward_fused(const void* value, msda_dtype_t vdt,
                                 const int64_t* spatial_shapes, const int64_t* level_start_index,
                                 const float* reference_points, const float* sampling_offsets,
                                 const float* attention_logits, msda_dims_t d, float* out,
                                 msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_TRY(check_value(value));
    MSDA_PTR(reference_points, 8);
    MSDA_PTR(sampling_offsets, 8);
    MSDA_PTR(attention_logits, 4);
    MSDA_PTR(out, 16);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    return cuda_status(msda::launch_msda_forward_fused(p, reference_points, sampling_offsets,
                                                       attention_logits, out,
                                                       (cudaStream_t)stream),
                       "msda_forward_fused");
}

msda_status_t tsa_reference_points(const float* ego_motion, int32_t B, int32_t num_queues,
                                   int32_t bev_h, int32_t bev_w, double grid_length_y,
                                   double grid_length_x, float* reference_points,
                                   msda_stream_t stream)
{
    MSDA_CHECK(B >= 0 && num_queues >= 1, MSDA_ERR_INVALID_ARG,
               "B (%d) must be >= 0 and num_queues (%d) >= 1", B, num_queues);
    MSDA_CHECK(bev_h >= 1 && bev_w >= 1 && (int64_t)bev_h * bev_w <= INT32_MAX,
               MSDA_ERR_INVALID_ARG, "BEV grid %d x %d is empty or too large", bev_h, bev_w);
    MSDA_CHECK(grid_length_y > 0.0 && grid_length_x > 0.0 && grid_length_y < 1e30 &&
                   grid_length_x < 1e30,
               MSDA_ERR_INVALID_ARG, "grid lengths (%g, %g) must be finite and > 0",
               grid_length_y, grid_length_x);
    if (B == 0) return ok();
    MSDA_PTR(ego_motion, 4);
    MSDA_PTR(reference_points, 8);
    return cuda_status(msda::launch_tsa_reference(ego_motion, B, num_queues, bev_h, bev_w,
                                                  grid_length_x, grid_length_y, reference_points,
                                                  (cudaStream_t)stream),
                       "tsa_reference_points");
}

msda_status_t tsa_forward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                          const int64_t* level_start_index, const float* reference_points,
                          const float* sampling_offsets, const float* attention_logits,
                          int32_t num_queues, msda_dims_t d, float* out, msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    MSDA_CHECK(num_queues >= 1 && num_queues <= MSDA_MAX_QUEUES, MSDA_ERR_UNSUPPORTED,
               "num_queues = %d outside 1..%d", num_queues, MSDA_MAX_QUEUES);
    MSDA_CHECK((int64_t)d.B * num_queues <= INT32_MAX, MSDA_ERR_UNSUPPORTED,
               "B * num_queues exceeds the 32-bit range");
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_TRY(check_value(value));
    MSDA_PTR(reference_points, 8);
    MSDA_PTR(sampling_offsets, 8);
    MSDA_PTR(attention_logits, 4);
    MSDA_PTR(out, 16);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    return cuda_status(msda::launch_tsa_forward(p, num_queues, reference_points, sampling_offsets,
                                                attention_logits, out, (cudaStream_t)stream),
                       "tsa_forward");
}

static msda_status_t check_workspace(const void* ws, size_t have, size_t need);

size_t tsa_backward_workspace_size(msda_dims_t d, int32_t num_queues)
{
    if (d.B < 0 || d.Nq < 0 || d.H < 1 || d.L < 1 || d.P < 1 || num_queues < 1) return 0;
    const size_t rows = (size_t)d.B * num_queues * d.Nq;
    const size_t S = (size_t)d.H * d.L * d.P;
    // per queue row: location gradients, their fp32 rounding residuals, weight gradients
    return 2 * align256(sizeof(float) * rows * S * 2) + align256(sizeof(float) * rows * S);
}

msda_status_t tsa_backward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                           const int64_t* level_start_index, const float* reference_points,
                           const float* sampling_offsets, const float* attention_logits,
                           int32_t num_queues, const float* grad_out, msda_dims_t d,
                           void* workspace, size_t workspace_bytes, float* grad_value,
                           float* grad_sampling_offsets, float* grad_attention_logits,
                           float* grad_reference_points, msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    MSDA_CHECK(num_queues >= 1 && num_queues <= MSDA_MAX_QUEUES, MSDA_ERR_UNSUPPORTED,
               "num_queues = %d outside 1..%d", num_queues, MSDA_MAX_QUEUES);
    MSDA_CHECK((int64_t)d.B * num_queues * d.Nq <= INT32_MAX, MSDA_ERR_UNSUPPORTED,
               "B * num_queues * Nq exceeds the 32-bit range");
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if (d.B == 0) return ok();
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_TRY(check_value(value));
        MSDA_PTR(reference_points, 8);
        MSDA_PTR(sampling_offsets, 8);
        MSDA_PTR(attention_logits, 4);
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(grad_sampling_offsets, 8);
        MSDA_PTR(grad_attention_logits, 4);
        MSDA_PTR(grad_reference_points, 8);
    }
    MSDA_TRY(check_workspace(workspace, workspace_bytes, tsa_backward_workspace_size(d, num_queues)));
    const cudaStream_t s = (cudaStream_t)stream;
    const int BT = d.B * num_queues;
    const size_t S = (size_t)d.H * d.L * d.P;
    const size_t loc_bytes = align256(sizeof(float) * (size_t)BT * d.Nq * S * 2);
    float* gl = static_cast<float*>(workspace);
    float* gl_lo = reinterpret_cast<float*>(static_cast<char*>(workspace) + loc_bytes);
    float* gw = reinterpret_cast<float*>(static_cast<char*>(workspace) + 2 * loc_bytes);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    cudaError_t e = msda::launch_zero(grad_value, (int64_t)BT * d.Nv * d.H * MSDA_HEAD_DIM, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_tsa_backward(p, num_queues, reference_points, sampling_offsets,
                                      attention_logits, grad_out, grad_value, gl, gl_lo, gw, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_sca_input_grads(attention_logits, nullptr, gl, gw, BT, 1, d.Nq, d.H, d.L,
                                         d.P, d.R, lv, grad_sampling_offsets,
                                         grad_attention_logits, grad_reference_points, s, gl_lo);
    return cuda_status(e, "tsa_backward");
}

msda_status_t msda_backward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                            const int64_t* level_start_index, const float* sampling_locations,
                            const float* attention_weights, const float* grad_out, msda_dims_t d,
                            float* grad_value, float* grad_sampling_locations,
                            float* grad_attention_weights, msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if (d.B == 0) return ok();
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_TRY(check_value(value));
        MSDA_PTR(sampling_locations, 8);
        MSDA_PTR(attention_weights, 4);
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(grad_sampling_locations, 8);
        MSDA_PTR(grad_attention_weights, 4);
    }
    const cudaStream_t s = (cudaStream_t)stream;
    const msda::Problem p = make_problem(value, vdt, d, lv);
    cudaError_t e = msda::launch_zero(grad_value, (int64_t)d.B * d.Nv * d.H * MSDA_HEAD_DIM, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_msda_backward(p, sampling_locations, attention_weights, grad_out,
                                       grad_value, nullptr, grad_sampling_locations,
                                       grad_attention_weights, s);
    return cuda_status(e, "msda_backward");
}

size_t msda_backward_deterministic_workspace_size(msda_dims_t d)
{
    if (d.B < 0 || d.Nv < 1 || d.H < 1) return 0;
    return align256(sizeof(long long) * (size_t)d.B * d.Nv * d.H * MSDA_HEAD_DIM);
}

msda_status_t msda_backward_deterministic(const void* value, msda_dtype_t vdt,
                                          const int64_t* spatial_shapes,
                                          const int64_t* level_start_index,
                                          const float* sampling_locations,
                                          const float* attention_weights, const float* grad_out,
                                          msda_dims_t d, void* workspace, size_t workspace_bytes,
                                          float* grad_value, float* grad_sampling_locations,
                                          float* grad_attention_weights, msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, false));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if (d.B == 0) return ok();
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_TRY(check_value(value));
        MSDA_PTR(sampling_locations, 8);
        MSDA_PTR(attention_weights, 4);
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(grad_sampling_locations, 8);
        MSDA_PTR(grad_attention_weights, 4);
    }
    MSDA_TRY(check_workspace(workspace, workspace_bytes,
                             msda_backward_deterministic_workspace_size(d)));
    const cudaStream_t s = (cudaStream_t)stream;
    const msda::Problem p = make_problem(value, vdt, d, lv);
    const int64_t n = (int64_t)d.B * d.Nv * d.H * MSDA_HEAD_DIM;
    long long* acc = static_cast<long long*>(workspace);
    cudaError_t e = msda::launch_zero(reinterpret_cast<float*>(acc), 2 * n, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_msda_backward(p, sampling_locations, attention_weights, grad_out,
                                       grad_value, acc, grad_sampling_locations,
                                       grad_attention_weights, s);
    if (e == cudaSuccess) e = msda::launch_fix_to_float(acc, grad_value, n, s);
    return cuda_status(e, "msda_backward_deterministic");
}

size_t msda_workspace_size(msda_dims_t d)
{
    if (d.B < 0 || d.Ncam < 1 || d.Nq < 0 || d.H < 1) return 0;
    return msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, true);
}

size_t sca_compact_workspace_size(msda_dims_t d)
{
    if (d.B < 0 || d.Ncam < 1 || d.Nq < 0) return 0;
    return msda::compact_scratch_bytes(d.B, d.Ncam, d.Nq);
}

static msda_status_t check_compact(const msda_dims_t& d)
{
    MSDA_CHECK(d.B >= 0 && d.Nq >= 0, MSDA_ERR_INVALID_ARG, "B (%d) and Nq (%d) must be >= 0",
               d.B, d.Nq);
    MSDA_CHECK(d.Ncam >= 1 && d.Ncam <= MSDA_MAX_CAMERAS, MSDA_ERR_UNSUPPORTED,
               "Ncam = %d outside 1..%d", d.Ncam, MSDA_MAX_CAMERAS);
    MSDA_CHECK(d.R >= 1, MSDA_ERR_INVALID_ARG, "R = %d must be >= 1", d.R);
    MSDA_CHECK((int64_t)d.B * d.Ncam <= MSDA_MAX_BATCH_CAMERAS, MSDA_ERR_UNSUPPORTED,
               "B * Ncam = %lld exceeds %d", (long long)d.B * d.Ncam, MSDA_MAX_BATCH_CAMERAS);
    MSDA_CHECK((int64_t)d.B * d.Ncam * d.Nq <= INT32_MAX, MSDA_ERR_UNSUPPORTED,
               "B * Ncam * Nq exceeds the 32-bit row range");
    return MSDA_OK;
}

static msda_status_t check_workspace(const void* ws, size_t have, size_t need)
{
    MSDA_CHECK(ws != nullptr && have >= need, MSDA_ERR_WORKSPACE,
               "workspace %p of %zu bytes, %zu needed", ws, have, need);
    MSDA_CHECK(aligned(ws, 16), MSDA_ERR_WORKSPACE, "workspace must be 16-byte aligned");
    return MSDA_OK;
}

msda_status_t sca_compact(const uint8_t* bev_mask, msda_dims_t d, void* workspace,
                          size_t workspace_bytes, int32_t* idx, int32_t* count, int32_t* pos,
                          int32_t* hits, msda_stream_t stream)
{
    MSDA_TRY(check_compact(d));
    if (d.B == 0) return ok();
    MSDA_TRY(check_workspace(workspace, workspace_bytes,
                             msda::compact_scratch_bytes(d.B, d.Ncam, d.Nq)));
    MSDA_PTR(count, 4);
    if (d.Nq > 0) {
        MSDA_PTR(bev_mask, 1);
        MSDA_PTR(idx, 4);
        MSDA_PTR(pos, 4);
        MSDA_PTR(hits, 4);
    }
    const msda::CompactScratch cs = msda::compact_scratch_carve(workspace, d.B, d.Ncam, d.Nq);
    return cuda_status(msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, idx, count, pos,
                                                hits, cs.chunk_counts, (cudaStream_t)stream),
                       "sca_compact");
}

static msda_status_t check_sca_inputs(const void* value, msda_dtype_t vdt, const msda_dims_t& d,
                                      const int64_t* spatial_shapes,
                                      const int64_t* level_start_index,
                                      const float* reference_points_cam,
                                      const float* sampling_offsets,
                                      const float* attention_logits, msda::Levels& lv)
{
    MSDA_TRY(check_dims(d, true));
    MSDA_TRY(check_compact(d));
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if ((int64_t)d.B * d.Nq > 0) {
        MSDA_TRY(check_value(value));
        MSDA_PTR(reference_points_cam, 8);
        MSDA_PTR(sampling_offsets, 8);
        MSDA_PTR(attention_logits, 4);
    }
    return MSDA_OK;
}

msda_status_t sca_rebatched_forward(const void* value, msda_dtype_t vdt,
                                    const int64_t* spatial_shapes,
                                    const int64_t* level_start_index,
                                    const float* reference_points_cam,
                                    const float* sampling_offsets, const float* attention_logits,
                                    const int32_t* idx, const int32_t* count, msda_dims_t d,
                                    float* out_rb, msda_stream_t stream)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_PTR(idx, 4);
    MSDA_PTR(count, 4);
    MSDA_PTR(out_rb, 16);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    return cuda_status(msda::launch_sca_gather(p, reference_points_cam, sampling_offsets,
                                               attention_logits, idx, count, out_rb,
                                               (cudaStream_t)stream),
                       "sca_rebatched_forward");
}

msda_status_t sca_camera_average(const float* out_rb, const int32_t* pos, const int32_t* hits,
                                 msda_dims_t d, float* out, msda_stream_t stream)
{
    MSDA_TRY(check_compact(d));
    MSDA_CHECK(d.H >= 1, MSDA_ERR_INVALID_ARG, "H (%d) must be >= 1", d.H);
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_PTR(out_rb, 16);
    MSDA_PTR(pos, 4);
    MSDA_PTR(hits, 4);
    MSDA_PTR(out, 16);
    return cuda_status(msda::launch_sca_average(out_rb, pos, hits, d.B, d.Ncam, d.Nq, d.H, out,
                                                false, (cudaStream_t)stream),
                       "sca_camera_average");
}

msda_status_t sca_camera_average_linear(const float* out_rb, const int32_t* pos,
                                        const int32_t* hits, msda_dims_t d, const void* w,
                                        const float* bias, const float* residual, int32_t N,
                                        msda_dtype_t y_dtype, void* y, float dropout_p,
                                        uint64_t dropout_seed, msda_stream_t stream)
{
    MSDA_TRY(check_compact(d));
    MSDA_CHECK(d.H >= 1 && d.H <= 8, MSDA_ERR_UNSUPPORTED,
               "H = %d: the projection takes rows of 64 .. 256 channels (H in 2..8)", d.H);
    return msda::average_linear_impl(out_rb, pos, hits, d.B, d.Ncam, d.Nq, w, bias, residual, N,
                                     d.H * MSDA_HEAD_DIM, y_dtype, y, dropout_p, dropout_seed,
                                     (cudaStream_t)stream);
}

msda_status_t sca_forward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                          const int64_t* level_start_index, const float* reference_points_cam,
                          const uint8_t* bev_mask, const float* sampling_offsets,
                          const float* attention_logits, msda_dims_t d, void* workspace,
                          size_t workspace_bytes, float* out, msda_stream_t stream)
{
    return msda::sca_forward_to(value, vdt, spatial_shapes, level_start_index,
                                reference_points_cam, bev_mask, sampling_offsets,
                                attention_logits, d, workspace, workspace_bytes, out, false,
                                (cudaStream_t)stream);
}

msda_status_t sca_forward_query_major(const void* value, msda_dtype_t vdt,
                                      const int64_t* spatial_shapes,
                                      const int64_t* level_start_index,
                                      const float* reference_points_cam, const uint8_t* bev_mask,
                                      const float* sampling_offsets,
                                      const float* attention_logits, msda_dims_t d, float* out,
                                      msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, true));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    MSDA_TRY(check_dtype(vdt));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_TRY(check_value(value));
    MSDA_PTR(reference_points_cam, 8);
    MSDA_PTR(bev_mask, 1);
    MSDA_PTR(sampling_offsets, 8);
    MSDA_PTR(attention_logits, 4);
    MSDA_PTR(out, 16);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    return cuda_status(msda::launch_sca_query_major(p, reference_points_cam, bev_mask,
                                                    sampling_offsets, attention_logits, out, false,
                                                    (cudaStream_t)stream),
                       "sca_forward_query_major");
}

msda_status_t sca_rebatched_backward(const void* value, msda_dtype_t vdt,
                                     const int64_t* spatial_shapes,
                                     const int64_t* level_start_index,
                                     const float* reference_points_cam,
                                     const float* sampling_offsets,
                                     const float* attention_logits, const float* grad_out,
                                     const int32_t* idx, const int32_t* count,
                                     const int32_t* hits, msda_dims_t d, float* grad_value,
                                     float* grad_sampling_locations_rb,
                                     float* grad_attention_weights_rb, msda_stream_t stream)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    if (d.B == 0) return ok();
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(idx, 4);
        MSDA_PTR(count, 4);
        MSDA_PTR(hits, 4);
        MSDA_PTR(grad_sampling_locations_rb, 8);
        MSDA_PTR(grad_attention_weights_rb, 4);
    }
    return msda::sca_rebatched_backward_to(value, vdt, d, lv, reference_points_cam,
                                           sampling_offsets, attention_logits, grad_out, idx,
                                           count, hits, grad_value, nullptr,
                                           grad_sampling_locations_rb, grad_attention_weights_rb,
                                           (cudaStream_t)stream);
}

msda_status_t sca_backward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                           const int64_t* level_start_index, const float* reference_points_cam,
                           const uint8_t* bev_mask, const float* sampling_offsets,
                           const float* attention_logits, const float* grad_out, msda_dims_t d,
                           void* workspace, size_t workspace_bytes, float* grad_value,
                           float* grad_sampling_locations_rb, float* grad_attention_weights_rb,
                           msda_stream_t stream)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    if (d.B == 0) return ok();
    if (d.Nq > 0) MSDA_PTR(bev_mask, 1);
    MSDA_TRY(check_workspace(workspace, workspace_bytes,
                             msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, false)));
    const msda::ScaWorkspace w = msda::sca_workspace_carve(workspace, d.B, d.Ncam, d.Nq, d.H, false);
    if (d.Nq > 0) {
        const cudaError_t e = msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, w.idx,
                                                       w.count, w.pos, w.hits, w.chunk_counts,
                                                       (cudaStream_t)stream);
        if (e != cudaSuccess) return cuda_status(e, "sca_backward");
    }
    return sca_rebatched_backward(value, vdt, spatial_shapes, level_start_index,
                                  reference_points_cam, sampling_offsets, attention_logits,
                                  grad_out, w.idx, w.count, w.hits, d, grad_value,
                                  grad_sampling_locations_rb, grad_attention_weights_rb, stream);
}

size_t sca_backward_deterministic_workspace_size(msda_dims_t d)
{
    if (d.B < 0 || d.Ncam < 1 || d.Nq < 0 || d.Nv < 1 || d.H < 1) return 0;
    return msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, false) +
           align256(sizeof(long long) * (size_t)d.B * d.Ncam * d.Nv * d.H * MSDA_HEAD_DIM);
}

msda_status_t sca_backward_deterministic(const void* value, msda_dtype_t vdt,
                                         const int64_t* spatial_shapes,
                                         const int64_t* level_start_index,
                                         const float* reference_points_cam,
                                         const uint8_t* bev_mask, const float* sampling_offsets,
                                         const float* attention_logits, const float* grad_out,
                                         msda_dims_t d, void* workspace, size_t workspace_bytes,
                                         float* grad_value, float* grad_sampling_locations_rb,
                                         float* grad_attention_weights_rb, msda_stream_t stream)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    if (d.B == 0) return ok();
    if (d.Nq > 0) MSDA_PTR(bev_mask, 1);
    MSDA_TRY(check_workspace(workspace, workspace_bytes,
                             sca_backward_deterministic_workspace_size(d)));
    const cudaStream_t s = (cudaStream_t)stream;
    const size_t lists = msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, false);
    const msda::ScaWorkspace w = msda::sca_workspace_carve(workspace, d.B, d.Ncam, d.Nq, d.H, false);
    long long* acc = reinterpret_cast<long long*>(static_cast<char*>(workspace) + lists);
    if (d.Nq > 0) {
        const cudaError_t e = msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, w.idx,
                                                       w.count, w.pos, w.hits, w.chunk_counts, s);
        if (e != cudaSuccess) return cuda_status(e, "sca_backward_deterministic");
    }
    return msda::sca_rebatched_backward_to(value, vdt, d, lv, reference_points_cam,
                                           sampling_offsets, attention_logits, grad_out, w.idx,
                                           w.count, w.hits, grad_value, acc,
                                           grad_sampling_locations_rb, grad_attention_weights_rb,
                                           s);
}

}  // extern "C"

extern "C" size_t sca_backward_full_workspace_size(msda_dims_t d)
{
    if (d.B < 0 || d.Ncam < 1 || d.Nq < 0 || d.H < 1 || d.L < 1 || d.P < 1) return 0;
    const size_t rows = (size_t)d.B * d.Ncam * d.Nq;
    const size_t S = (size_t)d.H * d.L * d.P;
    return msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, false) +
           2 * align256(sizeof(float) * rows * S * 2) + align256(sizeof(float) * rows * S);
}

extern "C" msda_status_t sca_backward_full(
    const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
    const int64_t* level_start_index, const float* reference_points_cam, const uint8_t* bev_mask,
    const float* sampling_offsets, const float* attention_logits, const float* grad_out,
    msda_dims_t d, void* workspace, size_t workspace_bytes, float* grad_value,
    float* grad_sampling_offsets, float* grad_attention_logits, float* grad_reference_points_cam,
    msda_stream_t stream)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    MSDA_TRY(check_compact(d));
    if (d.B == 0) return ok();
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_PTR(bev_mask, 1);
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(grad_sampling_offsets, 8);
        MSDA_PTR(grad_attention_logits, 4);
        MSDA_PTR(grad_reference_points_cam, 4);
    }
    MSDA_TRY(check_workspace(workspace, workspace_bytes, sca_backward_full_workspace_size(d)));
    const cudaStream_t s = (cudaStream_t)stream;
    const msda::ScaWorkspace w = msda::sca_workspace_carve(workspace, d.B, d.Ncam, d.Nq, d.H, false);
    const size_t rows = (size_t)d.B * d.Ncam * d.Nq;
    const size_t S = (size_t)d.H * d.L * d.P;
    char* rest = static_cast<char*>(workspace) +
                 msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, false);
    const size_t loc_bytes = align256(sizeof(float) * rows * S * 2);
    float* gl = reinterpret_cast<float*>(rest);
    float* gl_lo = reinterpret_cast<float*>(rest + loc_bytes);
    float* gw = reinterpret_cast<float*>(rest + 2 * loc_bytes);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    cudaError_t e = msda::launch_zero(grad_value,
                                      (int64_t)d.B * d.Ncam * d.Nv * d.H * MSDA_HEAD_DIM, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, w.idx, w.count, w.pos,
                                     w.hits, w.chunk_counts, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_sca_backward_rows(p, reference_points_cam, sampling_offsets,
                                           attention_logits, grad_out, w.idx, w.hits, w.count,
                                           grad_value, nullptr, gl, gw, s, gl_lo);
    if (e == cudaSuccess && d.Nq > 0)
        e = msda::launch_sca_input_grads(attention_logits, w.pos, gl, gw, d.B, d.Ncam, d.Nq, d.H,
                                         d.L, d.P, d.R, lv, grad_sampling_offsets,
                                         grad_attention_logits, grad_reference_points_cam, s,
                                         gl_lo);
    return cuda_status(e, "sca_backward_full");
}

extern "C" msda_status_t sca_backward_inputs(const int64_t* spatial_shapes,
                                             const int64_t* level_start_index,
                                             const float* attention_logits, const int32_t* pos,
                                             const float* grad_sampling_locations_rb,
                                             const float* grad_attention_weights_rb,
                                             msda_dims_t d, float* grad_sampling_offsets,
                                             float* grad_attention_logits,
                                             float* grad_reference_points_cam,
                                             msda_stream_t stream)
{
    MSDA_TRY(check_dims(d, true));
    MSDA_TRY(check_compact(d));
    msda::Levels lv;
    MSDA_TRY(check_levels(d, spatial_shapes, level_start_index, lv));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_PTR(attention_logits, 4);
    MSDA_PTR(pos, 4);
    MSDA_PTR(grad_sampling_locations_rb, 8);
    MSDA_PTR(grad_attention_weights_rb, 4);
    MSDA_PTR(grad_sampling_offsets, 8);
    MSDA_PTR(grad_attention_logits, 4);
    MSDA_PTR(grad_reference_points_cam, 4);
    return cuda_status(msda::launch_sca_input_grads(
                           attention_logits, pos, grad_sampling_locations_rb,
                           grad_attention_weights_rb, d.B, d.Ncam, d.Nq, d.H, d.L, d.P, d.R, lv,
                           grad_sampling_offsets, grad_attention_logits,
                           grad_reference_points_cam, (cudaStream_t)stream),
                       "sca_backward_inputs");
}

// Status helpers for entry points defined in other translation units (they
// share this file's per-thread error message).
namespace msda {
msda_status_t api_fail(msda_status_t code, const char* message) { return fail(code, "%s", message); }
msda_status_t api_ok() { return ok(); }
msda_status_t api_cuda(cudaError_t e, const char* where) { return cuda_status(e, where); }
}  // namespace msda

namespace msda {

// 1: bf16 value takes the query-major kernel (one pass: no compaction,
// rebatched rows or average kernel; the camera mean formed in registers).
// On the BEVFormer-base step the rebatched kernels are faster for both value
// types (bf16: 0.377 against 0.390 ms), so both take them.
#ifndef MSDA_SCA_FORWARD_QM_BF16
#define MSDA_SCA_FORWARD_QM_BF16 0
#endif

msda_status_t sca_forward_to(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                             const int64_t* level_start_index, const float* reference_points_cam,
                             const uint8_t* bev_mask, const float* sampling_offsets,
                             const float* attention_logits, msda_dims_t d, void* workspace,
                             size_t workspace_bytes, void* out, bool out_bf16, cudaStream_t s,
                             ScaWorkspace* rows)
{
    msda::Levels lv;
    MSDA_TRY(check_sca_inputs(value, vdt, d, spatial_shapes, level_start_index,
                              reference_points_cam, sampling_offsets, attention_logits, lv));
    if ((int64_t)d.B * d.Nq == 0) return ok();
    MSDA_PTR(bev_mask, 1);
    if (rows == nullptr) MSDA_PTR(out, 16);
    MSDA_TRY(check_workspace(workspace, workspace_bytes,
                             msda::sca_workspace_bytes(d.B, d.Ncam, d.Nq, d.H, true)));
    const msda::ScaWorkspace w = msda::sca_workspace_carve(workspace, d.B, d.Ncam, d.Nq, d.H, true);
    const msda::Problem p = make_problem(value, vdt, d, lv);
    if (rows) {
        *rows = w;
        cudaError_t e = msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, w.idx, w.count,
                                                 w.pos, w.hits, w.chunk_counts, s);
        if (e == cudaSuccess)
            e = msda::launch_sca_gather(p, reference_points_cam, sampling_offsets,
                                        attention_logits, w.idx, w.count, w.out_rb, s);
        return cuda_status(e, "sca_forward");
    }
    // the query-major kernel computes the same function (the camera mean is
    // stored once, as fp32 or, for the SCA module, as the bf16 operand of the
    // output projection)
    if (MSDA_SCA_FORWARD_QM_BF16 && vdt == MSDA_BF16)
        return cuda_status(msda::launch_sca_query_major(p, reference_points_cam, bev_mask,
                                                        sampling_offsets, attention_logits, out,
                                                        out_bf16, s),
                           "sca_forward");
    cudaError_t e = msda::launch_sca_compact(bev_mask, d.B, d.Ncam, d.Nq, d.R, w.idx, w.count,
                                             w.pos, w.hits, w.chunk_counts, s);
    if (e == cudaSuccess)
        e = msda::launch_sca_gather(p, reference_points_cam, sampling_offsets, attention_logits,
                                    w.idx, w.count, w.out_rb, s);
    if (e == cudaSuccess)
        e = msda::launch_sca_average(w.out_rb, w.pos, w.hits, d.B, d.Ncam, d.Nq, d.H, out,
                                     out_bf16, s);
    return cuda_status(e, "sca_forward");
}

}  // namespace msda

namespace msda {

// sca_rebatched_backward after its input checks; acc non-null: the
// deterministic fixed-point accumulation (acc zeroed here, then rounded into
// grad_value).
msda_status_t sca_rebatched_backward_to(const void* value, msda_dtype_t vdt, const msda_dims_t& d,
                                        const Levels& lv, const float* reference_points_cam,
                                        const float* sampling_offsets,
                                        const float* attention_logits, const float* grad_out,
                                        const int32_t* idx, const int32_t* count,
                                        const int32_t* hits, float* grad_value, long long* acc,
                                        float* grad_loc_rb, float* grad_attn_rb, cudaStream_t s)
{
    MSDA_PTR(grad_value, 16);
    if (d.Nq > 0) {
        MSDA_PTR(grad_out, 16);
        MSDA_PTR(idx, 4);
        MSDA_PTR(count, 4);
        MSDA_PTR(hits, 4);
        MSDA_PTR(grad_loc_rb, 8);
        MSDA_PTR(grad_attn_rb, 4);
    }
    const Problem p = make_problem(value, vdt, d, lv);
    const int64_t n = (int64_t)d.B * d.Ncam * d.Nv * d.H * MSDA_HEAD_DIM;
    cudaError_t e = acc ? launch_zero(reinterpret_cast<float*>(acc), 2 * n, s)
                        : launch_zero(grad_value, n, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = launch_sca_backward_rows(p, reference_points_cam, sampling_offsets, attention_logits,
                                     grad_out, idx, hits, count, grad_value, acc, grad_loc_rb,
                                     grad_attn_rb, s);
    if (e == cudaSuccess && d.Nq > 0)
        e = launch_sca_zero_tail(count, d.B, d.Ncam, d.Nq, d.H * d.L * d.P, grad_loc_rb,
                                 grad_attn_rb, s);
    if (e == cudaSuccess && acc) e = launch_fix_to_float(acc, grad_value, n, s);
    return cuda_status(e, acc ? "sca_backward_deterministic" : "sca_rebatched_backward");
}

}  // namespace msda
