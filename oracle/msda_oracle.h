/*
 * Oracle for multi-scale deformable attention (MSDA) and BEVFormer Spatial
 * Cross-Attention (SCA): plain, slow, double-precision CPU loops.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * Sources (all on the pages this project was written from):
 *   [BQ]  "BEV(三) BEVFormer: how the Query interacts with the 8 Heads of
 *         the Feature" (leheavengame.com repost of a CSDN article),
 *         sections 4.2 (softmax), 5 (anchor index and location),
 *         6 (bilinear read), 7-9 (weighted sum, head concat),
 *         10 (camera average), 15 (worked example), 18.4-18.5 (op inputs).
 *   [SCA] "Spatial Cross-Attention" walkthrough, Tencent Cloud developer
 *         article 2321140: the bev_mask query rebatch listing and the
 *         scatter-add / clamp(count, 1) average listing.
 *   [PX]  Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as
 *         1, 2, 3", SC 2011: the counter-based generator Philox4x32-10,
 *         used for training-time dropout (the pages' dropout draws from
 *         PyTorch's generator, which no second implementation can replay).
 *   [TS]  "【论文阅读】BEVFormer论文解析及Temporal Self-Attention、Spatial
 *         Cross-Attention注意力机制详解及代码示例" (wsisp.com): section 二.2
 *         (TSA between the previous and the current BEV) and the BEV encoder
 *         listing (ego motion delta_x, delta_y, ego_angle in degrees from the
 *         CAN bus; grid_length 0.512 m per BEV cell).  The listing stops
 *         before it applies the motion and the section gives TSA only as
 *         generic attention; the two TSA entry points below state the
 *         reading they take.
 *
 * Conventions shared by every entry point below:
 *   - every array is host memory, contiguous, row-major in the shape given;
 *   - floating-point inputs and outputs are double; the tests pass fp32 (or
 *     bf16-rounded) data widened exactly to double;
 *   - value rows: the pixel (y, x) of level l is row start[l] + y*W_l + x,
 *     and a row holds H heads of Dh channels ("view as [.., H, Dh]", [BQ] 3);
 *   - shapes[2*l] = H_l (rows), shapes[2*l+1] = W_l (columns);
 *   - locations are (x, y) in [0,1]^2 normalised image coordinates;
 *   - coord_f32 = 1 takes the corner decision (x = W*s - 1/2, then floor) in
 *     IEEE binary32 with round-to-nearest and no fused multiply-add, the
 *     precision the CUDA kernels use; coord_f32 = 0 does it in double (used
 *     for finite-difference checks, where inputs are not fp32 values).
 *     With coord_f32 = 1 the fused location rho + dx/W is also formed in
 *     binary32 (one division, one addition, each rounded);
 *   - return value: 0 on success, -1 on an argument error (nothing written).
 */
#ifndef MSDA_ORACLE_H
#define MSDA_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Softmax over each contiguous group of n logits, max-subtracted ([BQ] 4.2). */
int oracle_softmax(const double* logits, int64_t groups, int n, double* alpha);

/* MSDA forward from given locations and weights ([BQ] 6-9, 18.5).
 * value [B, Nv, H, Dh]; loc [B, Nq, H, L, P, 2]; attn [B, Nq, H, L, P];
 * out [B, Nq, H*Dh]. */
int oracle_msda_forward(const double* value, int B, int Nv, int H, int Dh,
                        int L, const int64_t* shapes, const int64_t* starts,
                        int Nq, int P, const double* loc, const double* attn,
                        int coord_f32, double* out);

/* MSDA forward from reference points, pixel offsets and logits
 * ([BQ] 4.2 softmax, 5 location, 6-9 sampling and sum).
 * ref [B, Nq, R, 2]; off [B, Nq, H, L, P, 2] in level pixels;
 * logits [B, Nq, H, L, P]; out [B, Nq, H*Dh].  R must divide P. */
int oracle_msda_forward_fused(const double* value, int B, int Nv, int H, int Dh,
                              int L, const int64_t* shapes, const int64_t* starts,
                              int Nq, int P, int R, const double* ref,
                              const double* off, const double* logits,
                              int coord_f32, double* out);

/* Locations and weights the fused forward uses: loc [B, Nq, H, L, P, 2] and
 * attn [B, Nq, H, L, P] (softmax of logits; rho_{m(k)} + (dx/W_l, dy/H_l)). */
int oracle_fused_locations(int B, int H, int L, const int64_t* shapes,
                           int Nq, int P, int R, const double* ref,
                           const double* off, const double* logits,
                           int coord_f32, double* loc, double* attn);

/* MSDA backward: analytic derivative of the forward above.
 * grad_out [B, Nq, H*Dh] -> grad_value [B, Nv, H, Dh] (overwritten),
 * grad_loc [B, Nq, H, L, P, 2], grad_attn [B, Nq, H, L, P]. */
int oracle_msda_backward(const double* value, int B, int Nv, int H, int Dh,
                         int L, const int64_t* shapes, const int64_t* starts,
                         int Nq, int P, const double* loc, const double* attn,
                         const double* grad_out, int coord_f32,
                         double* grad_value, double* grad_loc, double* grad_attn);

/* SCA mask compaction ([SCA] rebatch listing; counts from the average listing).
 * bev_mask [Ncam, B, Nq, R] (0 / non-zero bytes).
 * idx [B, Ncam, Nq]: ascending hit queries, then -1;  count [B, Ncam];
 * pos [B, Ncam, Nq]: rank of q in idx or -1;  hits [B, Nq]: cameras hit. */
int oracle_sca_compact(const uint8_t* bev_mask, int Ncam, int B, int Nq, int R,
                       int32_t* idx, int32_t* count, int32_t* pos, int32_t* hits);

/* SCA forward: compaction, per-camera rebatched fused MSDA, scatter-add in
 * ascending camera order, division by max(1, hits) ([BQ] 10; [SCA]).
 * value [B, Ncam, Nv, H, Dh]; ref_cam [Ncam, B, Nq, R, 2];
 * bev_mask [Ncam, B, Nq, R]; off [B, Nq, H, L, P, 2]; logits [B, Nq, H, L, P];
 * out [B, Nq, H*Dh].  out_rb (optional, may be NULL) [B, Ncam, Nq, H*Dh]
 * receives the rebatched per-camera rows (rows >= count set to 0). */
int oracle_sca_forward(const double* value, int B, int Ncam, int Nv, int H, int Dh,
                       int L, const int64_t* shapes, const int64_t* starts,
                       int Nq, int P, int R, const double* ref_cam,
                       const uint8_t* bev_mask, const double* off,
                       const double* logits, int coord_f32,
                       double* out, double* out_rb);

/* SCA camera average on its own ([SCA] scatter-add and clamp(count, 1)
 * listing; [BQ] 10): for every (b, q), the rows out_rb[b, c, pos[b, c, q]] of
 * the cameras c with pos >= 0, added in ascending c, divided by
 * max(1, hits[b, q]).  out_rb [B, Ncam, Nq, HD]; pos [B, Ncam, Nq];
 * hits [B, Nq]; out [B, Nq, HD]. */
int oracle_sca_camera_average(const double* out_rb, const int32_t* pos, const int32_t* hits,
                              int B, int Ncam, int Nq, int64_t HD, double* out);

/* SCA backward (derivative of oracle_sca_forward w.r.t. value and the
 * rebatched sampling locations and attention weights).
 * grad_out [B, Nq, H*Dh] -> grad_value [B, Ncam, Nv, H, Dh],
 * grad_loc_rb [B, Ncam, Nq, H, L, P, 2], grad_attn_rb [B, Ncam, Nq, H, L, P];
 * rebatched rows >= count are 0. */
int oracle_sca_backward(const double* value, int B, int Ncam, int Nv, int H, int Dh,
                        int L, const int64_t* shapes, const int64_t* starts,
                        int Nq, int P, int R, const double* ref_cam,
                        const uint8_t* bev_mask, const double* off,
                        const double* logits, const double* grad_out, int coord_f32,
                        double* grad_value, double* grad_loc_rb, double* grad_attn_rb);

/* Gradients of the SCA inputs from the rebatched gradients of
 * oracle_sca_backward.  Offsets and logits belong to the BEV query and are
 * shared by every camera ([BQ] 10), so their gradients sum over the cameras
 * that see the query; s = rho_{k mod R} + (dx / W_l, dy / H_l) ([BQ] 5) gives
 * d/d dx = d/d s_x / W_l and d/d rho_m = sum over the points k with
 * k mod R = m; alpha = softmax(a) ([BQ] 4.2) gives
 * d/d a_j = alpha_j (G_j - sum_i alpha_i G_i).
 *   grad_off [B, Nq, H, L, P, 2], grad_logits [B, Nq, H, L, P],
 *   grad_ref_cam [Ncam, B, Nq, R, 2] (zero for cameras that do not see q). */
int oracle_sca_backward_inputs(int B, int Ncam, int Nq, int H, int L, const int64_t* shapes,
                               int P, int R, const uint8_t* bev_mask, const double* logits,
                               const double* grad_loc_rb, const double* grad_attn_rb,
                               double* grad_off, double* grad_logits, double* grad_ref_cam);

/* Dense projection ([BQ] 3 value projection, 4.1 offset head, 4.2 weight
 * head, 11 output projection, 13 residual):
 *   y[m, n] = sum_k x[m, k] w[n, k] + bias[n] + residual[m, n]
 * x [M, K]; w [N, K] (nn.Linear layout); bias [N] or NULL; residual [M, N]
 * or NULL; y [M, N]. */
int oracle_linear(const double* x, const double* w, const double* bias, const double* residual,
                  int M, int N, int K, double* y);

/* TSA reference points ([TS] BEV encoder listing; the transform is this
 * oracle's reading of "align the previous BEV with the ego motion"):
 * BEV query q = i * bev_w + j has the cell centre ((j + 1/2) / bev_w,
 * (i + 1/2) / bev_h), in metres about the BEV centre
 * p = ((j + 1/2 - bev_w / 2) gx, (i + 1/2 - bev_h / 2) gy).  Queue t sees
 * that point at p' = Rot(theta) p + (dx, dy), returned normalised:
 * (p'_x / (bev_w gx) + 1/2, p'_y / (bev_h gy) + 1/2).
 * ego [B, T, 3] = (dx metres, dy metres, theta degrees, counter-clockwise
 * from +x towards +y); a queue with (0, 0, 0) gets the cell centres.
 * ref [B, T, bev_h * bev_w, 2]. */
int oracle_tsa_reference_points(int B, int T, int bev_h, int bev_w, double gx, double gy,
                                const double* ego, double* ref);

/* TSA forward ([TS] 二.2 read as: every BEV query samples each of the T
 * queues with its own offsets and logits, by the fused MSDA above, and its
 * output is the mean over the queues, summed in ascending t):
 * value [B*T, Nv, H, Dh] (row b*T + t); ref [B*T, Nq, R, 2];
 * off [B*T, Nq, H, L, P, 2]; logits [B*T, Nq, H, L, P]; out [B, Nq, H*Dh]. */
int oracle_tsa_forward(const double* value, int B, int T, int Nv, int H, int Dh,
                       int L, const int64_t* shapes, const int64_t* starts,
                       int Nq, int P, int R, const double* ref,
                       const double* off, const double* logits,
                       int coord_f32, double* out);

/* Philox4x32-10 ([PX]): ten rounds of two multiply-xor S-boxes with
 * multipliers 0xD2511F53, 0xCD9E8D57 and key increments 0x9E3779B9,
 * 0xBB67AE85; out = the four output words for counter ctr and key key. */
void oracle_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* Training-time dropout ([BQ] 12: m / (1 - p) * o): element e of o [n] is
 * kept when word (e mod 4) of Philox4x32-10 at counter (e div 4 as two
 * 32-bit words low first, 0, 0) and key (seed low, seed high) is
 * >= floor(p * 2^32), and then scaled by 1 / (1 - p); otherwise 0.
 * 0 <= p < 1; p = 0 is the identity. */
int oracle_dropout(const double* o, int64_t n, double p, uint64_t seed, double* out);

#ifdef __cplusplus
}
#endif
#endif
