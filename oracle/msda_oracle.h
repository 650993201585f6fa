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

/* Dense projection ([BQ] 3 value projection, 4.1 offset head, 4.2 weight
 * head, 11 output projection, 13 residual):
 *   y[m, n] = sum_k x[m, k] w[n, k] + bias[n] + residual[m, n]
 * x [M, K]; w [N, K] (nn.Linear layout); bias [N] or NULL; residual [M, N]
 * or NULL; y [M, N]. */
int oracle_linear(const double* x, const double* w, const double* bias, const double* residual,
                  int M, int N, int K, double* y);

#ifdef __cplusplus
}
#endif
#endif
