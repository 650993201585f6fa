// Internal launcher interface between the C ABI (msda_api.cu) and the kernel
// translation units.  Arguments are already validated when these are called.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "msda_device.cuh"

namespace msda {

struct Problem {
    const void* value;   // [B, (Ncam,) Nv, H, 32]
    bool bf16;
    int B, Ncam, Nq, Nv, H, L, P, R;
    Levels lv;
};

// Workspace layout of sca_forward / sca_backward: compaction scratch, the
// compaction lists, then (forward only) the rebatched rows.
struct ScaWorkspace {
    int32_t* idx;           // [B, Ncam, Nq]
    int32_t* pos;           // [B, Ncam, Nq]
    int32_t* count;         // [B, Ncam]
    int32_t* hits;          // [B, Nq]
    int32_t* chunk_counts;  // [B, Ncam, nchunks]
    float* out_rb;          // [B, Ncam, Nq, H * 32] (forward only)
};

constexpr int kCompactChunk = 1024;  // queries per compaction CTA

struct CompactScratch {
    int32_t* chunk_counts;  // [B, Ncam, nchunks]
};

size_t compact_scratch_bytes(int B, int Ncam, int Nq);
CompactScratch compact_scratch_carve(void* base, int B, int Ncam, int Nq);
size_t sca_workspace_bytes(int B, int Ncam, int Nq, int H, bool with_rows);
ScaWorkspace sca_workspace_carve(void* base, int B, int Ncam, int Nq, int H, bool with_rows);

int device_sm_count();

// Programmatic dependent launch: the kernel may begin while the kernel before
// it in the stream is still running, once every CTA of that kernel has
// executed pdl_trigger() (or exited).  The kernel must call pdl_wait(), which
// returns when that grid has completed and its writes are visible, before it
// reads anything an earlier kernel wrote or writes anything an earlier kernel
// reads.  After a kernel that never triggers, it starts as an ordinary launch.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// K1 / K1f: msda_forward (given locations, weights) and msda_forward_fused.
cudaError_t launch_msda_forward(const Problem& p, const float* loc, const float* attn,
                                float* out, cudaStream_t s);
cudaError_t launch_msda_forward_fused(const Problem& p, const float* ref, const float* off,
                                      const float* logits, float* out, cudaStream_t s);

// K2: compaction (two launches; three above 64 chunks of 1024 queries).
cudaError_t launch_sca_compact(const uint8_t* mask, int B, int Ncam, int Nq, int R,
                               int32_t* idx, int32_t* count, int32_t* pos, int32_t* hits,
                               int32_t* chunk_counts, cudaStream_t s);

// K3: fused MSDA over the rebatched rows of every (batch, camera).
cudaError_t launch_sca_gather(const Problem& p, const float* ref_cam, const float* off,
                              const float* logits, const int32_t* idx, const int32_t* count,
                              float* out_rb, cudaStream_t s);

// K3 with four lanes per (row, head) for rows of up to 32 samples
// (sca_gather_quad.cu); sca_gather_quad_fits says whether a problem qualifies.
bool sca_gather_quad_fits(const Problem& p);
cudaError_t launch_sca_gather_quad(const Problem& p, const float* ref_cam, const float* off,
                                   const float* logits, const int32_t* idx, const int32_t* count,
                                   float* out_rb, cudaStream_t s);

// K3q: the whole SCA forward, query-major (no compaction, no rebatched rows).
// out_bf16: the result stored as bf16 (bf16 value only).
cudaError_t launch_sca_query_major(const Problem& p, const float* ref_cam, const uint8_t* mask,
                                   const float* off, const float* logits, void* out,
                                   bool out_bf16, cudaStream_t s);

// K4: deterministic camera average; fp32 or (out_bf16) bf16 output.
cudaError_t launch_sca_average(const float* out_rb, const int32_t* pos, const int32_t* hits,
                               int B, int Ncam, int Nq, int H, void* out, bool out_bf16,
                               cudaStream_t s);

// Backward.
cudaError_t launch_zero(float* p, int64_t n, cudaStream_t s);
// grad_value_fix non-null: deterministic fixed-point accumulation into it
// (zeroed by the caller) instead of fp32 reductions into grad_value.
cudaError_t launch_msda_backward(const Problem& p, const float* loc, const float* attn,
                                 const float* grad_out, float* grad_value,
                                 long long* grad_value_fix, float* grad_loc, float* grad_attn,
                                 cudaStream_t s);
// grad_loc_lo_rb non-null: the precise location gradients (softmax and
// location gradient in double), with the fp32 rounding residual of each
// location gradient written there (not with grad_value_fix).
cudaError_t launch_sca_backward_rows(const Problem& p, const float* ref_cam, const float* off,
                                     const float* logits, const float* grad_out,
                                     const int32_t* idx, const int32_t* hits,
                                     const int32_t* count, float* grad_value,
                                     long long* grad_value_fix, float* grad_loc_rb,
                                     float* grad_attn_rb, cudaStream_t s,
                                     float* grad_loc_lo_rb = nullptr);
cudaError_t launch_fix_to_float(const long long* acc, float* out, int64_t n, cudaStream_t s);
cudaError_t launch_sca_zero_tail(const int32_t* count, int B, int Ncam, int Nq, int S,
                                 float* grad_loc_rb, float* grad_attn_rb, cudaStream_t s);

}  // namespace msda

#include "msda.h"

namespace msda {
// Gradients of offsets, logits and reference points (sca_input_grads.cu);
// pos == null: Ncam = 1 and row i is query i.  grad_loc_lo_rb (may be null):
// the fp32 rounding residuals of grad_loc_rb, added in double.
cudaError_t launch_sca_input_grads(const float* logits, const int32_t* pos,
                                   const float* grad_loc_rb, const float* grad_attn_rb, int B,
                                   int Ncam, int Nq, int H, int L, int P, int R, const Levels& lv,
                                   float* grad_off, float* grad_logits, float* grad_ref_cam,
                                   cudaStream_t s, const float* grad_loc_lo_rb = nullptr);

// TSA (tsa.cu): ego-motion reference points and the queue-mean fused forward.
cudaError_t launch_tsa_reference(const float* ego, int B, int T, int bev_h, int bev_w, double gx,
                                 double gy, float* ref, cudaStream_t s);
cudaError_t launch_tsa_forward(const Problem& p, int T, const float* ref, const float* off,
                               const float* logits, float* out, cudaStream_t s);

// The projection with a bias per (camera, level) row group (the embedding
// prologue of the SCA module): row r is pixel r mod nv of camera
// (r div nv) mod ncam, level = last l with start[l] <= pixel.
struct RowBiasArgs {
    const float* table;  // [ncam * L, N]
    int nv, ncam, L;
    int start[8];
};
msda_status_t linear_impl(const void* x, const void* w, const float* bias, const float* residual,
                          int32_t M, int32_t N, int32_t K, msda_dtype_t y_dtype, void* y,
                          float dropout_p, uint64_t dropout_seed, const RowBiasArgs* rb,
                          cudaStream_t stream);
// The projection of the camera average: y = residual + dropout(X W^T + bias)
// with X[b * Nq + q] = bf16(sum over c ascending with pos[b, c, q] >= 0 of
// out_rb[b, c, pos[b, c, q]] / max(1, hits[b, q])), formed inside the
// projection kernel (Ncam <= 8; K = the rows' width).
msda_status_t average_linear_impl(const float* out_rb, const int32_t* pos, const int32_t* hits,
                                  int32_t B, int32_t Ncam, int32_t Nq, const void* w,
                                  const float* bias, const float* residual, int32_t N, int32_t K,
                                  msda_dtype_t y_dtype, void* y, float dropout_p,
                                  uint64_t dropout_seed, cudaStream_t stream);
cudaError_t launch_embed_bias(const float* e_cam, const float* e_lvl, const void* w,
                              const float* b, int ncam, int L, int N, int K, float* table,
                              cudaStream_t s);

// sca_forward with its output stored as fp32 or (out_bf16) bf16; validates
// like sca_forward.  rows non-null: only the compaction and the rebatched
// gather run (out unused) and *rows receives the workspace's lists and rows,
// for a consumer that averages the cameras itself.
msda_status_t sca_forward_to(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                             const int64_t* level_start_index, const float* reference_points_cam,
                             const uint8_t* bev_mask, const float* sampling_offsets,
                             const float* attention_logits, msda_dims_t d, void* workspace,
                             size_t workspace_bytes, void* out, bool out_bf16,
                             cudaStream_t stream, ScaWorkspace* rows = nullptr);

// sca_rebatched_backward after its input checks (acc: see msda_api.cu).
msda_status_t sca_rebatched_backward_to(const void* value, msda_dtype_t vdt, const msda_dims_t& d,
                                        const Levels& lv, const float* reference_points_cam,
                                        const float* sampling_offsets,
                                        const float* attention_logits, const float* grad_out,
                                        const int32_t* idx, const int32_t* count,
                                        const int32_t* hits, float* grad_value, long long* acc,
                                        float* grad_loc_rb, float* grad_attn_rb, cudaStream_t s);

// TSA backward rows (msda_backward.cu): location and weight gradients of
// every queue row, grad_value accumulated (zeroed by the caller); p.B counts
// BEV samples, the value holds p.B * T items.
cudaError_t launch_tsa_backward(const Problem& p, int T, const float* ref, const float* off,
                                const float* logits, const float* grad_out, float* grad_value,
                                float* grad_loc, float* grad_loc_lo, float* grad_attn,
                                cudaStream_t s);

// Set the per-thread error message of msda_last_error() and return the code.
msda_status_t api_fail(msda_status_t code, const char* message);
msda_status_t api_ok();
msda_status_t api_cuda(cudaError_t e, const char* where);
}  // namespace msda
