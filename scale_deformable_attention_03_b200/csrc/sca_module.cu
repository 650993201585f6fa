// sca_module_forward: the whole BEVFormer Spatial Cross-Attention module
// forward of "BEV(三) BEVFormer: how the Query interacts with the 8 Heads of
// the Feature" (sections 3, 4, 10-14; the Tencent Cloud walkthrough's
// listings), on the GPU end to end:
//   q~    = q + pos                      (bf16, the projections' operand)
//   V     = F~ W_v^T + b_v               (section 3; tensor cores; with
//           F~ = F + e_cam + e_level, the embeddings enter as a bias per
//           (camera, level): (e_cam + e_level) W_v^T + b_v)
//   Delta = q~ W_Delta^T + b_Delta       (4.1)
//   a     = q~ W_alpha^T + b_alpha       (4.2)
//   g     = SCA(V, Delta, a, rho, mask)  (5-10: compaction, fused MSDA, average)
//   q_hat = q + dropout(g W_o^T + b_o)   (11-13; dropout in the projection's
//                                         epilogue, the identity when p = 0)
// The SCA runs compaction, the rebatched gather and the camera average, which
// stores g as the projection's bf16 operand.  Built with
// MSDA_MODULE_FUSED_AVERAGE = 1, fp32 value forms the camera average inside
// the output projection instead (its X tiles built from the rebatched rows,
// g never stored), which measured slower on the BEVFormer-base module.
// It composes the library's own kernels; the only new one is the element-wise
// q + pos conversion below.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "msda.h"
#include "msda_launch.h"

#ifndef MSDA_MODULE_FUSED_AVERAGE
#define MSDA_MODULE_FUSED_AVERAGE 0
#endif

namespace msda {
namespace {

// out = bf16(a + b) (b may be null), four elements per thread.
__global__ void add_to_bf16_kernel(const float4* __restrict__ a, const float4* __restrict__ b,
                                   uint2* __restrict__ out, int64_t n4)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
         i += (int64_t)gridDim.x * blockDim.x) {
        float4 v = __ldcs(a + i);
        if (b) {
            const float4 u = __ldcs(b + i);
            v.x += u.x;
            v.y += u.y;
            v.z += u.z;
            v.w += u.w;
        }
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
        uint2 o;
        o.x = *reinterpret_cast<const uint32_t*>(&lo);
        o.y = *reinterpret_cast<const uint32_t*>(&hi);
        __stcs(out + i, o);
    }
}

cudaError_t launch_add_to_bf16(const float* a, const float* b, void* out, int64_t n, cudaStream_t s)
{
    if (n == 0) return cudaSuccess;
    const int64_t n4 = n / 4;  // n is a multiple of 256 here
    const int64_t blocks = std::min<int64_t>((n4 + 255) / 256, (int64_t)device_sm_count() * 8);
    add_to_bf16_kernel<<<(unsigned)blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(a),
                                                        reinterpret_cast<const float4*>(b),
                                                        reinterpret_cast<uint2*>(out), n4);
    return cudaGetLastError();
}

size_t a256(size_t x) { return (x + 255) & ~(size_t)255; }

struct ModuleWs {
    void* qt;          // [B * Nq, C] bf16
    void* value;       // [B * Ncam * Nv, C] value dtype
    float* offsets;    // [B * Nq, H L P 2]
    float* logits;     // [B * Nq, H L P]
    void* g16;         // [B * Nq, C] bf16
    float* embed_bias; // [Ncam * L, C]: the embedding prologue's bias rows
    void* sca;         // sca_forward workspace
    size_t sca_bytes;
    size_t total;
};

ModuleWs module_carve(void* base, const msda_dims_t& d, msda_dtype_t vdt)
{
    const size_t C = (size_t)d.H * MSDA_HEAD_DIM, S = (size_t)d.H * d.L * d.P;
    const size_t rows_q = (size_t)d.B * d.Nq, rows_v = (size_t)d.B * d.Ncam * d.Nv;
    ModuleWs w;
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) {
        char* r = p ? p + off : nullptr;
        off += a256(bytes);
        return r;
    };
    w.qt = take(rows_q * C * 2);
    w.value = take(rows_v * C * (vdt == MSDA_BF16 ? 2 : 4));
    w.offsets = reinterpret_cast<float*>(take(rows_q * S * 2 * 4));
    w.logits = reinterpret_cast<float*>(take(rows_q * S * 4));
    w.g16 = take(rows_q * C * 2);
    w.embed_bias = reinterpret_cast<float*>(take((size_t)d.Ncam * d.L * C * 4));
    w.sca_bytes = msda_workspace_size(d);
    w.sca = take(w.sca_bytes);
    w.total = off;
    return w;
}

}  // namespace
}  // namespace msda

extern "C" size_t sca_module_workspace_size(msda_dims_t d, msda_dtype_t value_dtype)
{
    if (d.B < 0 || d.Ncam < 1 || d.Nq < 0 || d.Nv < 1 || d.H < 1 || d.L < 1 || d.P < 1) return 0;
    return msda::module_carve(nullptr, d, value_dtype).total;
}

extern "C" msda_status_t sca_module_forward(const sca_module_params_t* p,
                                            const int64_t* spatial_shapes,
                                            const int64_t* level_start_index, msda_dims_t d,
                                            void* workspace, size_t workspace_bytes,
                                            float* q_hat, msda_stream_t stream)
{
    using namespace msda;
    if (p == nullptr) return api_fail(MSDA_ERR_INVALID_ARG, "params is null");
    if (p->value_dtype != MSDA_F32 && p->value_dtype != MSDA_BF16)
        return api_fail(MSDA_ERR_INVALID_ARG, "unknown value dtype");
    if (d.B < 0 || d.Nq < 0 || d.Ncam < 1 || d.Nv < 1 || d.H < 1)
        return api_fail(MSDA_ERR_INVALID_ARG, "bad sizes");
    const int C = d.H * MSDA_HEAD_DIM, S = d.H * d.L * d.P;
    if ((int64_t)d.B * d.Nq == 0) return api_ok();
    const ModuleWs need = module_carve(nullptr, d, p->value_dtype);
    if (workspace == nullptr || workspace_bytes < need.total || ((uintptr_t)workspace & 255))
        return api_fail(MSDA_ERR_WORKSPACE, "workspace missing, too small or not 256-byte aligned");
    if (!p->query || !p->features || !p->w_value || !p->w_offsets || !p->w_weights ||
        !p->w_output || !q_hat)
        return api_fail(MSDA_ERR_INVALID_ARG, "a required pointer is null");
    const ModuleWs w = module_carve(workspace, d, p->value_dtype);
    const cudaStream_t s = (cudaStream_t)stream;
    const int64_t rows_q = (int64_t)d.B * d.Nq, rows_v = (int64_t)d.B * d.Ncam * d.Nv;
    if (rows_q > INT32_MAX || rows_v > INT32_MAX)
        return api_fail(MSDA_ERR_UNSUPPORTED, "too many rows for one projection");

    cudaError_t e = launch_add_to_bf16(p->query, p->query_pos, w.qt, rows_q * C, s);
    if (e != cudaSuccess) return api_cuda(e, "sca_module_forward: query + pos");
    msda_status_t st;
    if (p->camera_embeds || p->level_embeds) {
        if (d.L > 8 || ((uintptr_t)p->camera_embeds & 3) || ((uintptr_t)p->level_embeds & 3))
            return api_fail(MSDA_ERR_INVALID_ARG, "embeddings: L <= 8, 4-byte aligned arrays");
        e = launch_embed_bias(p->camera_embeds, p->level_embeds, p->w_value, p->b_value, d.Ncam,
                              d.L, C, C, w.embed_bias, s);
        if (e != cudaSuccess) return api_cuda(e, "sca_module_forward: embedding bias");
        RowBiasArgs rb;
        rb.table = w.embed_bias;
        rb.nv = d.Nv;
        rb.ncam = d.Ncam;
        rb.L = d.L;
        for (int l = 0; l < 8; ++l) rb.start[l] = l < d.L ? (int)level_start_index[l] : 0;
        st = linear_impl(p->features, p->w_value, nullptr, nullptr, (int32_t)rows_v, C, C,
                         p->value_dtype, w.value, 0.f, 0, &rb, s);
    } else {
        st = msda_linear(p->features, p->w_value, p->b_value, nullptr, (int32_t)rows_v, C, C,
                         p->value_dtype, w.value, stream);
    }
    if (st != MSDA_OK) return st;
    if ((st = msda_linear(w.qt, p->w_offsets, p->b_offsets, nullptr, (int32_t)rows_q, S * 2, C,
                          MSDA_F32, w.offsets, stream)) != MSDA_OK)
        return st;
    if ((st = msda_linear(w.qt, p->w_weights, p->b_weights, nullptr, (int32_t)rows_q, S, C,
                          MSDA_F32, w.logits, stream)) != MSDA_OK)
        return st;
    // MSDA_MODULE_FUSED_AVERAGE with fp32 value: the compaction and the
    // rebatched gather, then the camera average formed inside the output
    // projection (g never stored); otherwise the SCA stores g as bf16, then
    // the projection
    if (MSDA_MODULE_FUSED_AVERAGE && p->value_dtype == MSDA_F32 && d.Ncam <= 8) {
        ScaWorkspace rows;
        if ((st = sca_forward_to(w.value, p->value_dtype, spatial_shapes, level_start_index,
                                 p->reference_points_cam, p->bev_mask, w.offsets, w.logits, d,
                                 w.sca, w.sca_bytes, nullptr, false, s, &rows)) != MSDA_OK)
            return st;
        return average_linear_impl(rows.out_rb, rows.pos, rows.hits, d.B, d.Ncam, d.Nq,
                                   p->w_output, p->b_output, p->query, C, C, MSDA_F32, q_hat,
                                   p->dropout_p, p->dropout_seed, s);
    }
    if ((st = sca_forward_to(w.value, p->value_dtype, spatial_shapes, level_start_index,
                             p->reference_points_cam, p->bev_mask, w.offsets, w.logits, d, w.sca,
                             w.sca_bytes, w.g16, true, s)) != MSDA_OK)
        return st;
    return msda_linear_dropout(w.g16, p->w_output, p->b_output, p->query, (int32_t)rows_q, C, C,
                               MSDA_F32, q_hat, p->dropout_p, p->dropout_seed, stream);
}
