// sca_backward_inputs: gradients of the SCA inputs from the rebatched
// gradients of sca_rebatched_backward ("BEV(三) BEVFormer: how the Query
// interacts with the 8 Heads of the Feature", sections 4.2, 5 and 10):
// offsets and logits belong to the BEV query and every camera shares them, so
// their gradients sum over the cameras that see the query (ascending camera
// order, a gather, no atomics):
//   grad_offsets[q, h, l, k]  = sum_c grad_loc_rb[c, pos_c(q), h, l, k] / (W_l, H_l)
//   grad_logits[q, h, :]      = alpha * (G - <alpha, G>),  G = sum_c grad_attn_rb[...]
//   grad_ref_cam[c, q, m]     = sum over (h, l, k) with k mod R = m of grad_loc_rb
#include <cuda_runtime.h>

#include "msda.h"
#include "msda_launch.h"

namespace msda {
namespace {

constexpr int kIgWarps = 8;

// One warp per (batch, query); heads in turn; lanes over the L*P samples.
template <int NC>
__global__ void __launch_bounds__(kIgWarps * 32)
sca_offset_logit_grads_kernel(const float* __restrict__ logits, const int32_t* __restrict__ pos,
                              const float* __restrict__ grad_loc_rb,
                              const float* __restrict__ grad_attn_rb, int B, int Ncam, int Nq,
                              int H, int L, int P, Levels levels, float* __restrict__ grad_off,
                              float* __restrict__ grad_logits)
{
    __shared__ SmemLevels s_lv;
    stage_levels(s_lv, levels);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t bq = (int64_t)blockIdx.x * kIgWarps + (threadIdx.x >> 5);
    if (bq >= (int64_t)B * Nq) return;  // warp-uniform
    const int b = (int)(bq / Nq), q = (int)(bq - (int64_t)b * Nq);
    const int n = L * P, S = H * n;
    const int p = lane < Ncam ? __ldg(pos + ((int64_t)b * Ncam + lane) * Nq + q) : -1;
    const unsigned seen = __ballot_sync(0xffffffffu, p >= 0);
    float wl[NC], hl[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        const int l = j < n ? j / P : 0;
        wl[c] = (float)s_lv.w[l];
        hl[c] = (float)s_lv.h[l];
    }
    for (int h = 0; h < H; ++h) {
        float G[NC], gx[NC], gy[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) G[c] = gx[c] = gy[c] = 0.f;
        unsigned cams = seen;
        while (cams) {
            const int cam = __ffs(cams) - 1;  // ascending camera order
            cams &= cams - 1;
            const int row = __shfl_sync(0xffffffffu, p, cam);
            const int64_t r = (((int64_t)b * Ncam + cam) * Nq + row) * S + (int64_t)h * n;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int j = c * 32 + lane;
                if (j < n) {
                    G[c] += __ldcs(grad_attn_rb + r + j);
                    const float2 v = __ldcs(reinterpret_cast<const float2*>(grad_loc_rb) + r + j);
                    gx[c] += v.x;
                    gy[c] += v.y;
                }
            }
        }
        const int64_t o = bq * S + (int64_t)h * n;
        float a[NC];
        float m = -INFINITY;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = c * 32 + lane;
            a[c] = j < n ? __ldg(logits + o + j) : -INFINITY;
            m = fmaxf(m, a[c]);
        }
        m = warp_max(m);
        float z = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = c * 32 + lane;
            a[c] = j < n ? expf(a[c] - m) : 0.f;
            z += a[c];
        }
        z = warp_sum(z);
        float dot = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            a[c] = a[c] / z;
            dot += a[c] * G[c];
        }
        dot = warp_sum(dot);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = c * 32 + lane;
            if (j < n) {
                grad_logits[o + j] = a[c] * (G[c] - dot);
                reinterpret_cast<float2*>(grad_off)[o + j] = make_float2(gx[c] / wl[c], gy[c] / hl[c]);
            }
        }
    }
}

// One warp per (camera, batch, query): the row's H*L*P location gradients
// summed per anchor m = k mod R (zero when the camera does not see the query).
__global__ void __launch_bounds__(kIgWarps * 32)
sca_reference_grads_kernel(const int32_t* __restrict__ pos, const float* __restrict__ grad_loc_rb,
                           int B, int Ncam, int Nq, int S, int P, int R,
                           float* __restrict__ grad_ref_cam)
{
    const int lane = threadIdx.x & 31;
    const int64_t cbq = (int64_t)blockIdx.x * kIgWarps + (threadIdx.x >> 5);  // (c * B + b) * Nq + q
    if (cbq >= (int64_t)Ncam * B * Nq) return;  // warp-uniform
    const int q = (int)(cbq % Nq);
    const int64_t cb = cbq / Nq;
    const int b = (int)(cb % B), c = (int)(cb / B);
    const int p = __ldg(pos + ((int64_t)b * Ncam + c) * Nq + q);
    float* out = grad_ref_cam + cbq * R * 2;
    if (p < 0) {
        if (lane < 2 * R) out[lane] = 0.f;
        return;
    }
    const float2* g = reinterpret_cast<const float2*>(grad_loc_rb) +
                      (((int64_t)b * Ncam + c) * Nq + p) * S;
    float sx[MSDA_MAX_POINTS], sy[MSDA_MAX_POINTS];
#pragma unroll
    for (int m = 0; m < MSDA_MAX_POINTS; ++m) sx[m] = sy[m] = 0.f;
    for (int e = lane; e < S; e += 32) {
        const float2 v = __ldcs(g + e);
        const int m = (e % P) % R;
#pragma unroll
        for (int mm = 0; mm < MSDA_MAX_POINTS; ++mm)
            if (mm == m) {
                sx[mm] += v.x;
                sy[mm] += v.y;
            }
    }
#pragma unroll
    for (int m = 0; m < MSDA_MAX_POINTS; ++m) {
        if (m < R) {  // warp-uniform
            const float x = warp_sum(sx[m]), y = warp_sum(sy[m]);
            if (lane == 0) {
                out[2 * m] = x;
                out[2 * m + 1] = y;
            }
        }
    }
}

}  // namespace

cudaError_t launch_sca_input_grads(const float* logits, const int32_t* pos,
                                   const float* grad_loc_rb, const float* grad_attn_rb, int B,
                                   int Ncam, int Nq, int H, int L, int P, int R, const Levels& lv,
                                   float* grad_off, float* grad_logits, float* grad_ref_cam,
                                   cudaStream_t s)
{
    const int64_t rows = (int64_t)B * Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kIgWarps - 1) / kIgWarps);
    const int nc = (L * P + 31) / 32;
#define IG_CASE(NCV)                                                                             \
    case NCV:                                                                                    \
        sca_offset_logit_grads_kernel<NCV><<<grid, kIgWarps * 32, 0, s>>>(                       \
            logits, pos, grad_loc_rb, grad_attn_rb, B, Ncam, Nq, H, L, P, lv, grad_off,          \
            grad_logits);                                                                        \
        break;
    switch (nc) {
        IG_CASE(1)
        IG_CASE(2)
        IG_CASE(3)
        IG_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef IG_CASE
    const int64_t crows = (int64_t)Ncam * B * Nq;
    sca_reference_grads_kernel<<<(unsigned)((crows + kIgWarps - 1) / kIgWarps), kIgWarps * 32, 0,
                                 s>>>(pos, grad_loc_rb, B, Ncam, Nq, H * L * P, P, R, grad_ref_cam);
    return cudaGetLastError();
}

}  // namespace msda
