/*
 * msda.h - C ABI of libmsda.so: multi-scale deformable attention (MSDA) and
 * BEVFormer Spatial Cross-Attention (SCA) on NVIDIA B200 (sm_100a).
 *
 * Sources of the operations (pages this library was written from):
 *   [BQ]  "BEV(三) BEVFormer: how the Query interacts with the 8 Heads of the
 *         Feature" (leheavengame.com repost of a CSDN article).
 *   [SCA] "Spatial Cross-Attention" walkthrough, Tencent Cloud developer
 *         article 2321140 (rebatch listing, scatter-add / average listing).
 *   [TS]  "【论文阅读】BEVFormer论文解析及Temporal Self-Attention、Spatial
 *         Cross-Attention注意力机制详解及代码示例" (wsisp.com): section 二.2
 *         (TSA) and the BEV encoder listing (ego motion from the CAN bus,
 *         0.512 m BEV cells).
 *
 * What one MSDA output row computes ([BQ] sections 4.2, 5, 6, 8, 9):
 *   alpha_{h,l,k} = softmax over the L*P logits of head h        (4.2)
 *   s_{h,l,k}     = rho_{m(k)} + (dx / W_l, dy / H_l), m(k) = k mod R (5)
 *   x = W_l s_x - 1/2, y = H_l s_y - 1/2; bilinear read of the 32-channel
 *   head-h slice at (x, y), four neighbours, zero outside the map  (6)
 *   g^(h) = sum_{l,k} alpha_{h,l,k} * read_{h,l,k};  out = concat_h g^(h) (8, 9)
 * The corner decision (x, then floor) is made in IEEE binary32 with
 * round-to-nearest and no fused multiply-add; a location with x <= -1,
 * x >= W_l (same for y) or a non-finite coordinate reads nothing.
 *
 * Conventions of every call:
 *   - Tensor pointers are caller-owned DEVICE memory, contiguous, row-major
 *     in the shapes given.  spatial_shapes and level_start_index are HOST
 *     arrays (read during the call, not kept).
 *   - The library allocates no memory and keeps no pointer after returning.
 *     Its only state: a per-thread error message, a per-device cache of the
 *     SM count, the fixed scratch array of sca_compact_no_alloc, the device
 *     counter read by msda_linear_timeouts, and (set once) the GEMM kernel's
 *     shared-memory attribute and the driver's tensor-map encoder.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).
 *     The status covers argument checks and kernel launch errors; errors that
 *     happen while the kernels run surface at the caller's next
 *     synchronisation.  Nothing is launched when the arguments are rejected.
 *     Some kernels are programmatic dependent launches (the SCA compaction's
 *     second pass, the rebatched gather, the camera average): they may begin
 *     while the kernel before them in the stream finishes, and wait for it
 *     before they read what it may write or write anything, so stream order
 *     holds as usual, and the calls can be captured into CUDA graphs.
 *   - Outputs are fully overwritten (including gradients and padded rows).
 *   - Value rows: pixel (y, x) of level l is row level_start_index[l] +
 *     y * W_l + x; a row holds H heads of MSDA_HEAD_DIM channels.
 *     spatial_shapes[2*l] = H_l (rows), spatial_shapes[2*l+1] = W_l.
 *   - Locations are (x, y), normalised to [0, 1] over the level's width and
 *     height; offsets are (dx, dy) in pixels of the level they are read on.
 *   - Alignment: value, out, grad_value and the workspace 16 bytes;
 *     location, offset and reference-point arrays 8 bytes.
 */
#ifndef MSDA_H
#define MSDA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MSDA_HEAD_DIM 32    /* channels per head */
#define MSDA_MAX_LEVELS 8   /* L */
#define MSDA_MAX_POINTS 16  /* P */
#define MSDA_MAX_CAMERAS 32 /* Ncam */
#define MSDA_MAX_BATCH_CAMERAS 1024 /* B * Ncam for the sca_* calls */
#define MSDA_MAX_QUEUES 4   /* T, BEV queues of tsa_forward */

struct CUstream_st;
typedef struct CUstream_st* msda_stream_t; /* the same type as cudaStream_t */

/* Problem sizes.  head_dim is fixed at MSDA_HEAD_DIM. */
typedef struct {
    int32_t B;    /* batch items (BEVFormer TSA: the two queues prev_bev, bev) */
    int32_t Ncam; /* cameras (sca_* calls; ignored by msda_* calls) */
    int32_t Nq;   /* queries per batch item (SCA: BEV queries) */
    int32_t Nv;   /* value rows per batch item (and camera), >= every
                     level_start_index[l] + H_l * W_l */
    int32_t H;    /* heads; a value or output row has H * MSDA_HEAD_DIM channels */
    int32_t L;    /* levels, 1 .. MSDA_MAX_LEVELS */
    int32_t P;    /* points per (head, level), 1 .. MSDA_MAX_POINTS */
    int32_t R;    /* reference anchors per query, divides P (m(k) = k mod R) */
} msda_dims_t;

typedef enum {
    MSDA_F32 = 0, /* value stored as fp32 */
    MSDA_BF16 = 1 /* value stored as bf16; arithmetic and outputs stay fp32 */
} msda_dtype_t;

typedef enum {
    MSDA_OK = 0,
    MSDA_ERR_INVALID_ARG = 1, /* null pointer, bad size, bad alignment, inconsistent levels */
    MSDA_ERR_UNSUPPORTED = 2, /* outside the compiled limits (L, P, Ncam, index range) */
    MSDA_ERR_WORKSPACE = 3,   /* workspace missing or smaller than msda_workspace_size() */
    MSDA_ERR_CUDA = 4         /* a CUDA runtime call or kernel launch failed */
} msda_status_t;

/* MSDA forward from given sampling locations and attention weights
 * ([BQ] 6, 8, 9 and the operator inputs of 18.5).
 *   value              [B, Nv, H, 32]       fp32 or bf16 (vdt)
 *   sampling_locations [B, Nq, H, L, P, 2]  fp32, (x, y) normalised
 *   attention_weights  [B, Nq, H, L, P]     fp32, used as given (normally
 *                                           already softmax-normalised)
 *   out                [B, Nq, H * 32]      fp32, written */
msda_status_t msda_forward(const void* value, msda_dtype_t vdt,
                           const int64_t* spatial_shapes, const int64_t* level_start_index,
                           const float* sampling_locations, const float* attention_weights,
                           msda_dims_t d, float* out, msda_stream_t stream);

/* MSDA forward fused with its producers: softmax of the logits ([BQ] 4.2),
 * location from reference points and pixel offsets ([BQ] 5, 18.4), then the
 * read and weighted sum of msda_forward.  One kernel.
 *   reference_points  [B, Nq, R, 2]        fp32, (x, y) normalised
 *   sampling_offsets  [B, Nq, H, L, P, 2]  fp32, level pixels
 *   attention_logits  [B, Nq, H, L, P]     fp32
 *   out               [B, Nq, H * 32]      fp32, written */
msda_status_t msda_forward_fused(const void* value, msda_dtype_t vdt,
                                 const int64_t* spatial_shapes, const int64_t* level_start_index,
                                 const float* reference_points, const float* sampling_offsets,
                                 const float* attention_logits, msda_dims_t d, float* out,
                                 msda_stream_t stream);

/* TSA reference points ([TS] BEV encoder listing).  The listing takes the
 * ego motion (delta_x, delta_y in metres, the yaw in degrees) from the CAN
 * bus and 0.512 m BEV cells, and stops before it applies them; this call
 * reads "align the BEV of queue t with the current frame" as a rigid motion
 * of the cell centres:
 *   query q = i * bev_w + j has the centre p = ((j + 1/2 - bev_w/2) gx,
 *   (i + 1/2 - bev_h/2) gy) metres about the BEV centre; queue t sees it at
 *   p' = Rot(theta) p + (dx, dy), returned normalised as
 *   (p'_x / (bev_w gx) + 1/2, p'_y / (bev_h gy) + 1/2).
 * A queue with zero motion gets the cell centres ((j + 1/2) / bev_w,
 * (i + 1/2) / bev_h).  Computed in double, rounded once to fp32.
 *   ego_motion        [B, T, 3]             fp32 (dx m, dy m, theta degrees,
 *                                           counter-clockwise from +x to +y)
 *   reference_points  [B, T, bev_h*bev_w, 2] fp32, written; as [B*T, Nq, 1, 2]
 *                                           it is tsa_forward's input (R = 1)
 * grid_length_y, grid_length_x: metres per BEV cell along the height and the
 * width (BEVFormer: 0.512, 0.512), finite and > 0. */
msda_status_t tsa_reference_points(const float* ego_motion, int32_t B, int32_t num_queues,
                                   int32_t bev_h, int32_t bev_w, double grid_length_y,
                                   double grid_length_x, float* reference_points,
                                   msda_stream_t stream);

/* TSA forward ([TS] 二.2): every BEV query attends to T = num_queues BEV
 * queues (BEVFormer: the ego-aligned previous BEV, then the current one),
 * each with its own offsets and logits, through the fused MSDA of
 * msda_forward_fused; the output is the mean over the queues (the pages give
 * TSA only as generic attention: the mean is this library's reading).  One
 * kernel: the per-queue rows stay in registers.
 *   d.B                 BEV samples; the value holds d.B * T batch items,
 *                       item b * T + t being queue t of sample b
 *   value               [B*T, Nv, H, 32]        fp32 or bf16 (vdt)
 *   reference_points    [B*T, Nq, R, 2]         fp32, (x, y) normalised
 *   sampling_offsets    [B*T, Nq, H, L, P, 2]   fp32, level pixels
 *   attention_logits    [B*T, Nq, H, L, P]      fp32
 *   out                 [B, Nq, H * 32]         fp32, written:
 *                       (1/T) sum_t msda_forward_fused(item b*T + t)
 * num_queues: 1 .. MSDA_MAX_QUEUES, else MSDA_ERR_UNSUPPORTED. */
msda_status_t tsa_forward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                          const int64_t* level_start_index, const float* reference_points,
                          const float* sampling_offsets, const float* attention_logits,
                          int32_t num_queues, msda_dims_t d, float* out, msda_stream_t stream);

/* TSA backward: the derivative of tsa_forward (the pages give no backward).
 * Queue t of sample b receives grad_out[b] / T; the fused MSDA backward of
 * every queue row gives its location and weight gradients (workspace), and
 * the chain through the location and the softmax gives:
 *   grad_value             [B*T, Nv, H, 32]       fp32, written (zeroed, then
 *                                                 accumulated with atomics)
 *   grad_sampling_offsets  [B*T, Nq, H, L, P, 2]  = d/d s / (W_l, H_l)
 *   grad_attention_logits  [B*T, Nq, H, L, P]     softmax backward
 *   grad_reference_points  [B*T, Nq, R, 2]        sum over the points k with
 *                                                 k mod R = m
 *   grad_out               [B, Nq, H * 32]
 * Other arguments as tsa_forward; workspace >= tsa_backward_workspace_size(d,
 * num_queues) bytes (256-byte aligned). */
size_t tsa_backward_workspace_size(msda_dims_t d, int32_t num_queues);
msda_status_t tsa_backward(const void* value, msda_dtype_t vdt, const int64_t* spatial_shapes,
                           const int64_t* level_start_index, const float* reference_points,
                           const float* sampling_offsets, const float* attention_logits,
                           int32_t num_queues, const float* grad_out, msda_dims_t d,
                           void* workspace, size_t workspace_bytes, float* grad_value,
                           float* grad_sampling_offsets, float* grad_attention_logits,
                           float* grad_reference_points, msda_stream_t stream);

/* MSDA backward: the derivative of msda_forward (the pages give no backward;
 * this is the analytic derivative of [BQ] 6 and 8).
 *   grad_out                [B, Nq, H * 32]      fp32
 *   grad_value              [B, Nv, H, 32]       fp32, written (zeroed, then
 *                                                accumulated with atomics:
 *                                                the summation order varies)
 *   grad_sampling_locations [B, Nq, H, L, P, 2]  fp32, written
 *   grad_attention_weights  [B, Nq, H, L, P]     fp32, written
 * At an integer pixel coordinate the derivative is that of the cell floor()
 * selects; a location that reads nothing has zero gradients. */
msda_status_t msda_backward(const void* value, msda_dtype_t vdt,
                            const int64_t* spatial_shapes, const int64_t* level_start_index,
                            const float* sampling_locations, const float* attention_weights,
                            const float* grad_out, msda_dims_t d, float* grad_value,
                            float* grad_sampling_locations, float* grad_attention_weights,
                            msda_stream_t stream);

/* Deterministic variants of msda_backward and sca_backward (the pages give no
 * backward; the derivative is the same).  grad_value is accumulated without
 * floating-point atomics: every contribution alpha * w_g * grad_out is scaled
 * by 2^32 (exact), rounded once to a 64-bit integer and added with integer
 * atomics into a fixed-point copy in the workspace, then rounded once to
 * fp32.  Integer addition does not depend on order, so grad_value is bitwise
 * reproducible from run to run, and its error (at most 2^-33 per
 * contribution before the final rounding) is below that of fp32 sums.  The
 * partial sums must stay below 2^31 in magnitude.  The other gradients are
 * deterministic in both variants.  The workspace (caller-owned device
 * memory, 256-byte aligned, contents ignored) holds the fixed-point copy (and,
 * for the SCA call, the compaction lists). */
size_t msda_backward_deterministic_workspace_size(msda_dims_t d);
msda_status_t msda_backward_deterministic(const void* value, msda_dtype_t vdt,
                                          const int64_t* spatial_shapes,
                                          const int64_t* level_start_index,
                                          const float* sampling_locations,
                                          const float* attention_weights, const float* grad_out,
                                          msda_dims_t d, void* workspace, size_t workspace_bytes,
                                          float* grad_value, float* grad_sampling_locations,
                                          float* grad_attention_weights, msda_stream_t stream);
size_t sca_backward_deterministic_workspace_size(msda_dims_t d);
msda_status_t sca_backward_deterministic(const void* value, msda_dtype_t vdt,
                                         const int64_t* spatial_shapes,
                                         const int64_t* level_start_index,
                                         const float* reference_points_cam,
                                         const uint8_t* bev_mask, const float* sampling_offsets,
                                         const float* attention_logits, const float* grad_out,
                                         msda_dims_t d, void* workspace, size_t workspace_bytes,
                                         float* grad_value, float* grad_sampling_locations_rb,
                                         float* grad_attention_weights_rb, msda_stream_t stream);

/* Dense projection on the tensor cores ([BQ] 3 value projection W_v, 4.1
 * offset head W_Delta, 4.2 weight head W_alpha, 11 output projection W_o, 13
 * residual):  y = x w^T (+ bias) (+ residual).
 *   x        [M, K] bf16, row-major
 *   w        [N, K] bf16 (the nn.Linear weight layout, out x in)
 *   bias     [N] fp32 or NULL
 *   residual [M, N] fp32 or NULL, added after the bias (the SCA module's
 *            q_hat = q + output_proj(g) with dropout off, [BQ] 13)
 *   y        [M, N] fp32 (y_dtype MSDA_F32) or bf16 (MSDA_BF16), written
 * Products are exact and accumulate in fp32 (tensor memory).  Limits: N a
 * positive multiple of 256, K one of 64, 128, 192, 256, M >= 0; every pointer
 * 16-byte aligned. */
msda_status_t msda_linear(const void* x, const void* w, const float* bias,
                          const float* residual, int32_t M, int32_t N, int32_t K,
                          msda_dtype_t y_dtype, void* y, msda_stream_t stream);

/* msda_linear with training-time dropout of x w^T + bias before the residual
 * is added ([BQ] 12: m / (1 - p) * o):  y = residual + m (x w^T + bias) / (1 - p).
 * The pages' dropout draws from PyTorch's generator; this mask is element
 * e = row * N + col kept when word (e mod 4) of the counter-based generator
 * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as
 * easy as 1, 2, 3", SC 2011) at counter (e div 4 low, high, 0, 0) and key
 * (seed low, seed high) is >= floor(p * 2^32).  0 <= dropout_p < 1 (else
 * MSDA_ERR_INVALID_ARG); dropout_p = 0 is msda_linear. */
msda_status_t msda_linear_dropout(const void* x, const void* w, const float* bias,
                                  const float* residual, int32_t M, int32_t N, int32_t K,
                                  msda_dtype_t y_dtype, void* y, float dropout_p,
                                  uint64_t dropout_seed, msda_stream_t stream);

/* Number of msda_linear tiles that gave up waiting on their load or MMA
 * pipeline (each wait is bounded, about a second); 0 in normal operation.
 * Reads a device word, so it synchronises with the device. */
uint32_t msda_linear_timeouts(void);

/* Test hook of the bounded-wait path (no counterpart on the pages): the next
 * msda_linear launch holds back the first X-tile load of its first CTA.  That
 * CTA's tensor-core wait then runs out (about two seconds), counts one
 * timeout (msda_linear_timeouts), raises its stop flag, waits for the copies
 * it did issue and frees its tensor memory; the other CTAs finish normally.
 * The output of that one call is incomplete.  Synchronises with the device. */
msda_status_t msda_linear_test_withhold_load(void);

/* Bytes of device workspace sca_forward / sca_backward need for these
 * sizes: the compaction lists and, for the forward, the rebatched rows
 * (B * Ncam * Nq * H * 32 floats, of which only the seeing rows are used). */
size_t msda_workspace_size(msda_dims_t d);

/* Bytes of device workspace sca_compact needs (per-chunk counts and the
 * per-(batch, camera) row offsets, a few KB). */
size_t sca_compact_workspace_size(msda_dims_t d);

/* SCA mask compaction ([SCA] rebatch listing; counts of the average listing).
 * A camera c sees query q of batch item b when any of its R anchors is set.
 *   bev_mask  [Ncam, B, Nq, R] uint8 (0 = not visible)
 *   workspace >= sca_compact_workspace_size(d) bytes of device memory,
 *             caller-owned, contents ignored and overwritten
 *   idx       [B, Ncam, Nq] int32: the seeing queries in ascending order, then -1
 *   count     [B, Ncam]     int32: number of seeing queries
 *   pos       [B, Ncam, Nq] int32: rank of q in idx, -1 when not seen
 *   hits      [B, Nq]       int32: number of cameras seeing q
 * Bit-exact and deterministic; no host synchronisation. */
msda_status_t sca_compact(const uint8_t* bev_mask, msda_dims_t d, void* workspace,
                          size_t workspace_bytes, int32_t* idx, int32_t* count, int32_t* pos,
                          int32_t* hits, msda_stream_t stream);

/* sca_compact for callers that cannot allocate device memory.  (The pages
 * have no counterpart: this is a library convenience.)
 * Some callers cannot call cudaMalloc: the framework around them owns all
 * device memory and hands out no scratch for this step, or the pipeline
 * forbids allocation once it runs, because cudaMalloc can block and cudaFree
 * synchronises the device.  This call takes no workspace: the per-chunk
 * counts of the two compaction passes live in a fixed array inside the
 * library, MSDA_NO_ALLOC_COUNT_SLOTS ints (256 KiB), which every GPU that
 * loads the library holds until the process exits.  It allocates nothing.
 * Arguments and outputs are those of sca_compact (without the workspace).
 *   - Limit: B * Ncam * ceil(Nq / 1024) <= MSDA_NO_ALLOC_COUNT_SLOTS, else
 *     MSDA_ERR_UNSUPPORTED with a message (e.g. B = 1, Ncam = 6 allows
 *     Nq up to about 11 million).
 *   - The first call in a CUDA context looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and remembers it for
 *     that context, keyed by the context's unique id: after cudaDeviceReset,
 *     or in another context, the next call looks it up again.  Make the first
 *     call in each context before any stream capture.
 *   - Every call shares the one array per device and leaves its counts
 *     there; calls whose work overlaps on the GPU (different streams, or
 *     different host threads, without ordering) race on it.  Calls on one
 *     stream are safe.  Nothing in it needs to start at zero. */
#define MSDA_NO_ALLOC_COUNT_SLOTS 65536
msda_status_t sca_compact_no_alloc(const uint8_t* bev_mask, msda_dims_t d, int32_t* idx,
                                   int32_t* count, int32_t* pos, int32_t* hits,
                                   msda_stream_t stream);

/* SCA, stage 2 ([SCA] rebatch listing and MSDA call; [BQ] 10): the fused
 * MSDA of every camera's seeing queries, on the compaction of sca_compact.
 * Row i of camera c of batch item b reads BEV query q = idx[b, c, i]: its
 * offsets and logits (shared by every camera, [BQ] 10) and camera c's
 * reference points of q.  All rows of the batch and all cameras run in one
 * persistent kernel; the row counts are read on the device.
 *   value                [B, Ncam, Nv, H, 32]   fp32 or bf16
 *   reference_points_cam [Ncam, B, Nq, R, 2]    fp32
 *   sampling_offsets     [B, Nq, H, L, P, 2]    fp32, level pixels
 *   attention_logits     [B, Nq, H, L, P]       fp32
 *   idx, count           from sca_compact
 *   out_rb               [B, Ncam, Nq, H * 32]  fp32; rows < count[b, c]
 *                        written, the others left untouched */
msda_status_t sca_rebatched_forward(const void* value, msda_dtype_t vdt,
                                    const int64_t* spatial_shapes,
                                    const int64_t* level_start_index,
                                    const float* reference_points_cam,
                                    const float* sampling_offsets, const float* attention_logits,
                                    const int32_t* idx, const int32_t* count, msda_dims_t d,
                                    float* out_rb, msda_stream_t stream);

/* SCA, stage 3 ([SCA] scatter-add and clamp(count, 1) listing; [BQ] 10):
 *   out[b, q] = (sum over c with pos[b, c, q] >= 0, ascending c, of
 *                out_rb[b, c, pos[b, c, q]]) / max(1, hits[b, q]).
 * A gather (one thread per 16 bytes of output), no atomics: deterministic.
 *   out_rb [B, Ncam, Nq, H * 32]; pos, hits from sca_compact;
 *   out    [B, Nq, H * 32] fp32, written */
msda_status_t sca_camera_average(const float* out_rb, const int32_t* pos, const int32_t* hits,
                                 msda_dims_t d, float* out, msda_stream_t stream);

/* SCA, stage 3 fused into the output projection ([SCA] scatter-add and
 * clamp(count, 1) listing; [BQ] 10 then 11-13):
 *   g[b, q]     = bf16(sca_camera_average(out_rb, pos, hits)[b, q])
 *   y[b * Nq + q] = residual + dropout(g[b, q] W^T + bias)
 * in one kernel: the tensor-core projection of msda_linear_dropout whose X
 * tiles are formed in shared memory from the rebatched rows (the same sum in
 * ascending camera order, the same division and rounding as
 * sca_camera_average followed by a bf16 conversion), so g is never stored.
 *   out_rb  [B, Ncam, Nq, K] fp32, 32-byte aligned, K = H * 32 (64 .. 256)
 *   pos, hits from sca_compact; Ncam <= 8 (else MSDA_ERR_UNSUPPORTED)
 *   w       [N, K] bf16 (nn.Linear layout), N a positive multiple of 256
 *   bias    [N] fp32 or NULL; residual [B * Nq, N] fp32 or NULL
 *   y       [B * Nq, N] fp32 or bf16 (y_dtype), written
 *   dropout_p, dropout_seed as msda_linear_dropout (element e = row * N + col).
 * Pointers 16-byte aligned.  Errors as msda_linear. */
msda_status_t sca_camera_average_linear(const float* out_rb, const int32_t* pos,
                                        const int32_t* hits, msda_dims_t d, const void* w,
                                        const float* bias, const float* residual, int32_t N,
                                        msda_dtype_t y_dtype, void* y, float dropout_p,
                                        uint64_t dropout_seed, msda_stream_t stream);

/* SCA forward ([BQ] 10; [SCA] listings): sca_compact, sca_rebatched_forward
 * and sca_camera_average in one call, with the lists and the rebatched rows
 * in the caller's workspace, bit for bit the result of those three calls.
 * A query no camera sees gets 0. */
/*   value                [B, Ncam, Nv, H, 32]   fp32 or bf16
 *   reference_points_cam [Ncam, B, Nq, R, 2]    fp32
 *   bev_mask             [Ncam, B, Nq, R]       uint8
 *   sampling_offsets     [B, Nq, H, L, P, 2]    fp32, level pixels
 *   attention_logits     [B, Nq, H, L, P]       fp32
 *   workspace            >= msda_workspace_size(d) bytes of device memory,
 *                        caller-owned, contents ignored and overwritten
 *   out                  [B, Nq, H * 32]        fp32, written */
msda_status_t sca_forward(const void* value, msda_dtype_t vdt,
                          const int64_t* spatial_shapes, const int64_t* level_start_index,
                          const float* reference_points_cam, const uint8_t* bev_mask,
                          const float* sampling_offsets, const float* attention_logits,
                          msda_dims_t d, void* workspace, size_t workspace_bytes, float* out,
                          msda_stream_t stream);

/* SCA forward, query-major ([BQ] 10: each BEV query samples the cameras that
 * see it and averages them; [SCA] average listing: the count is clamped at
 * one).  The same result as sca_forward, from one kernel and without
 * workspace: one warp per (query, head) takes the softmax once, walks the
 * seeing cameras in ascending order into the same partial sums and writes
 * the mean once.  Arguments and layouts as sca_forward's; B * Ncam is not
 * limited to MSDA_MAX_BATCH_CAMERAS here.  The camera sum is formed before
 * the four-corner reduction, so results differ from sca_forward's in
 * rounding only. */
msda_status_t sca_forward_query_major(const void* value, msda_dtype_t vdt,
                                      const int64_t* spatial_shapes,
                                      const int64_t* level_start_index,
                                      const float* reference_points_cam, const uint8_t* bev_mask,
                                      const float* sampling_offsets,
                                      const float* attention_logits, msda_dims_t d, float* out,
                                      msda_stream_t stream);


/* SCA backward on a given compaction: derivative of sca_forward with respect
 * to the value and to the per-camera (rebatched) sampling locations and
 * attention weights.  The upstream gradient of row i of camera c is
 * grad_out[b, idx[b, c, i]] / max(1, hits[b, idx[b, c, i]]).
 *   grad_out                   [B, Nq, H * 32]              fp32
 *   idx, count, hits           from sca_compact
 *   grad_value                 [B, Ncam, Nv, H, 32]         fp32, written
 *                                                           (atomics)
 *   grad_sampling_locations_rb [B, Ncam, Nq, H, L, P, 2]    fp32, written;
 *   grad_attention_weights_rb  [B, Ncam, Nq, H, L, P]       fp32, written;
 *                              rows >= count[b, c] are zero */
msda_status_t sca_rebatched_backward(const void* value, msda_dtype_t vdt,
                                     const int64_t* spatial_shapes,
                                     const int64_t* level_start_index,
                                     const float* reference_points_cam,
                                     const float* sampling_offsets,
                                     const float* attention_logits, const float* grad_out,
                                     const int32_t* idx, const int32_t* count,
                                     const int32_t* hits, msda_dims_t d, float* grad_value,
                                     float* grad_sampling_locations_rb,
                                     float* grad_attention_weights_rb, msda_stream_t stream);

/* SCA backward: sca_compact then sca_rebatched_backward, the lists in the
 * caller's workspace (>= msda_workspace_size(d) bytes).  Outputs as above. */
msda_status_t sca_backward(const void* value, msda_dtype_t vdt,
                           const int64_t* spatial_shapes, const int64_t* level_start_index,
                           const float* reference_points_cam, const uint8_t* bev_mask,
                           const float* sampling_offsets, const float* attention_logits,
                           const float* grad_out, msda_dims_t d, void* workspace,
                           size_t workspace_bytes, float* grad_value,
                           float* grad_sampling_locations_rb, float* grad_attention_weights_rb,
                           msda_stream_t stream);

/* The BEVFormer SCA module forward, end to end on the GPU ([BQ] 3, 4, 10-14;
 * [SCA] listings):
 *   q~ = bf16(q + pos);  V = F~ W_v^T + b_v;  Delta = q~ W_Delta^T + b_Delta;
 *   a = q~ W_alpha^T + b_alpha;  g = sca_forward(V, Delta, a, rho, mask);
 *   q_hat = q + dropout(bf16(g) W_o^T + b_o)   (dropout as msda_linear_dropout
 *   with the params' rate and seed, the identity at rate 0, [BQ] 12; the
 *   LayerNorm after it belongs to the outer layer, [BQ] 13).
 * C = H * 32.  The projections run on msda_linear, so C and H*L*P must be
 * multiples of 256 and C one of 64..256 (BEVFormer-base: C = 256, H = 8,
 * L = 4, P = 8).  Weights use the nn.Linear layout (out x in), bf16; biases
 * fp32 (may be NULL). */
typedef struct {
    const float* query;                /* [B, Nq, C] fp32: q, also the residual */
    const float* query_pos;            /* [B, Nq, C] fp32 or NULL: pos */
    const void* features;              /* [B, Ncam, Nv, C] bf16: the FPN features F, level
                                          rows as level_start_index; F~ = F + e_cam +
                                          e_level ([BQ] 3), the embeddings below (NULL
                                          = already in F).  They enter the value
                                          projection as a bias per (camera, level):
                                          (e_cam + e_level) W_v^T + b_v, computed in
                                          double, so F itself is never re-rounded */
    const void* w_value;               /* [C, C] bf16 */
    const float* b_value;              /* [C] */
    const void* w_offsets;             /* [H*L*P*2, C] bf16 (rows h, l, k, xy) */
    const float* b_offsets;            /* [H*L*P*2] */
    const void* w_weights;             /* [H*L*P, C] bf16 */
    const float* b_weights;            /* [H*L*P] */
    const void* w_output;              /* [C, C] bf16 */
    const float* b_output;             /* [C] */
    const float* reference_points_cam; /* [Ncam, B, Nq, R, 2] */
    const uint8_t* bev_mask;           /* [Ncam, B, Nq, R] */
    msda_dtype_t value_dtype;          /* storage of V for the sampling: fp32 or bf16 */
    float dropout_p;                   /* training-time dropout rate in [0, 1); 0 = inference */
    uint64_t dropout_seed;             /* key of the dropout mask (see msda_linear_dropout) */
    const float* camera_embeds;        /* [Ncam, C] fp32 or NULL: e_cam of [BQ] 3 */
    const float* level_embeds;         /* [L, C] fp32 or NULL: e_level of [BQ] 3 */
} sca_module_params_t;

/* Bytes of device workspace sca_module_forward needs (q~, V, Delta, a, the
 * bf16 g and the sca_forward workspace), 256-byte alignment included.  The
 * camera average stores g directly as bf16, the output projection's operand. */
size_t sca_module_workspace_size(msda_dims_t d, msda_dtype_t value_dtype);

/*   q_hat [B, Nq, C] fp32, written.  workspace 256-byte aligned. */
msda_status_t sca_module_forward(const sca_module_params_t* params,
                                 const int64_t* spatial_shapes,
                                 const int64_t* level_start_index, msda_dims_t d,
                                 void* workspace, size_t workspace_bytes, float* q_hat,
                                 msda_stream_t stream);

/* Gradients of the SCA inputs from sca_rebatched_backward's rebatched
 * gradients ([BQ] 4.2 softmax, 5 location, 10: offsets and logits are the
 * BEV query's and every camera shares them, so their gradients sum over the
 * cameras that see the query, in ascending camera order, without atomics):
 *   grad_sampling_offsets     [B, Nq, H, L, P, 2] = sum_c grad_loc / (W_l, H_l)
 *   grad_attention_logits     [B, Nq, H, L, P]    = alpha (G - <alpha, G>),
 *                                                   G = sum_c grad_attn
 *   grad_reference_points_cam [Ncam, B, Nq, R, 2] = sum over the points k with
 *                                 k mod R = m of the camera's grad_loc (zero
 *                                 where the camera does not see the query)
 *   attention_logits          [B, Nq, H, L, P] (alpha is recomputed)
 *   pos                       from sca_compact
 *   grad_*_rb                 from sca_rebatched_backward */
msda_status_t sca_backward_inputs(const int64_t* spatial_shapes, const int64_t* level_start_index,
                                  const float* attention_logits, const int32_t* pos,
                                  const float* grad_sampling_locations_rb,
                                  const float* grad_attention_weights_rb, msda_dims_t d,
                                  float* grad_sampling_offsets, float* grad_attention_logits,
                                  float* grad_reference_points_cam, msda_stream_t stream);

/* The whole SCA backward down to the SCA inputs, in one call ([BQ] 4.2
 * softmax, 5 location, 6 bilinear read, 8 weighted sum, 10 camera average;
 * the pages give no backward, this is the analytic derivative):
 * sca_compact, the rebatched backward and sca_backward_inputs' chain, with
 * the location gradients kept to double accuracy between the two stages
 * (the softmax weight and each location gradient are formed in double and
 * passed on as fp32 value plus fp32 rounding residual, summed in double), so
 * that the chained sums over up to H*L*P terms stay within the fp32 bound of
 * the exact derivative.
 *   inputs as sca_backward; grad_out [B, Nq, H*32] fp32
 *   grad_value                [B, Ncam, Nv, H, 32]  fp32, fully written
 *   grad_sampling_offsets     [B, Nq, H, L, P, 2]   fp32
 *   grad_attention_logits     [B, Nq, H, L, P]      fp32
 *   grad_reference_points_cam [Ncam, B, Nq, R, 2]   fp32 (zero where the
 *                                                   camera does not see q)
 *   workspace: sca_backward_full_workspace_size(d) bytes, 256-byte aligned
 *   (compaction lists and the rebatched gradients with residuals).
 * grad_value is accumulated with fp32 atomics (order-dependent rounding). */
size_t sca_backward_full_workspace_size(msda_dims_t d);
msda_status_t sca_backward_full(const void* value, msda_dtype_t vdt,
                                const int64_t* spatial_shapes, const int64_t* level_start_index,
                                const float* reference_points_cam, const uint8_t* bev_mask,
                                const float* sampling_offsets, const float* attention_logits,
                                const float* grad_out, msda_dims_t d, void* workspace,
                                size_t workspace_bytes, float* grad_value,
                                float* grad_sampling_offsets, float* grad_attention_logits,
                                float* grad_reference_points_cam, msda_stream_t stream);

/* Fixed text for a status code. */
const char* msda_status_string(msda_status_t status);

/* Detail of the last failure on the calling thread ("" after a success). */
const char* msda_last_error(void);

/* Library version, major * 10000 + minor * 100 + patch. */
int32_t msda_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MSDA_H */
