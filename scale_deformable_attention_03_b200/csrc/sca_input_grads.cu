// sca_backward_inputs: gradients of the SCA inputs from the rebatched
// gradients of sca_rebatched_backward ("BEV(三) BEVFormer: how the Query
// interacts with the 8 Heads of the Feature", sections 4.2, 5 and 10):
// offsets and logits belong to the BEV query and every camera shares them, so
// their gradients sum over the cameras that see the query (ascending camera
// order, a gather, no atomics):
//   grad_offsets[q, h, l, k]  = sum_c grad_loc_rb[c, pos_c(q), h, l, k] / (W_l, H_l)
//   grad_logits[q, h, :]      = alpha * (G - <alpha, G>),  G = sum_c grad_attn_rb[...]
//   grad_ref_cam[c, q, m]     = sum over (h, l, k) with k mod R = m of grad_loc_rb
// The long sums (the reference points' H*L*P/R terms, <alpha, G>) and the
// camera sums of the offsets are formed in double: their terms may cancel.
// When the row kernels provide the fp32 rounding residuals of the location
// gradients (grad_loc_lo_rb), each term enters the sums as hi + lo, so the
// chain keeps the double accuracy of the precise location gradients.
#include <cuda_runtime.h>

#include "msda.h"
#include "msda_launch.h"

namespace msda {
namespace {

constexpr int kIgWarps = 8;

__device__ __forceinline__ double warp_sum_f64(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// One warp per (batch, query); lanes over the L*P samples; heads in chunks
// of kIgHeads whose loads are issued together (they are independent).
// REF (all heads in one chunk, R dividing 32): the same pass also forms the
// reference-point gradients of every camera: sample j of a head has the
// anchor (j mod P) mod R = j mod R, which is lane mod R for every chunk, so a
// lane sums its samples over the heads and a butterfly over the lanes of one
// anchor finishes each camera's sums.
constexpr int kIgHeads = 8;

// The pass is latency-bound (positions, then the rebatched gradients, per
// query): six resident CTAs at 40 registers (with spills) measured faster
// than two at 93 (0.207 vs 0.291 ms on the BEVFormer-base chain).
#ifndef MSDA_IG_MIN_BLOCKS
#define MSDA_IG_MIN_BLOCKS 6  // resident CTAs asked of the register allocation (rows of <= 32 samples)
#endif

template <int NC, bool REF>
__global__ void __launch_bounds__(kIgWarps * 32, NC == 1 ? MSDA_IG_MIN_BLOCKS : 0)
sca_offset_logit_grads_kernel(const float* __restrict__ logits, const int32_t* __restrict__ pos,
                              const float* __restrict__ grad_loc_rb,
                              const float* __restrict__ grad_loc_lo_rb,
                              const float* __restrict__ grad_attn_rb, int B, int Ncam, int Nq,
                              int H, int L, int P, int R, Levels levels,
                              float* __restrict__ grad_off, float* __restrict__ grad_logits,
                              float* __restrict__ grad_ref_cam)
{
    __shared__ SmemLevels s_lv;
    stage_levels(s_lv, levels);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t bq = (int64_t)blockIdx.x * kIgWarps + (threadIdx.x >> 5);
    if (bq >= (int64_t)B * Nq) return;  // warp-uniform
    const int b = (int)(bq / Nq), q = (int)(bq - (int64_t)b * Nq);
    const int n = L * P, S = H * n;
    // pos == null: one camera whose row i is query i (the TSA queues)
    const int p = lane < Ncam ? (pos ? __ldg(pos + ((int64_t)b * Ncam + lane) * Nq + q) : q) : -1;
    const unsigned seen = __ballot_sync(0xffffffffu, p >= 0);
    if (REF) {  // the cameras that do not see the query get zero reference gradients
        for (int i = lane; i < Ncam * R * 2; i += 32) {
            const int c = i / (2 * R);
            if (!((seen >> c) & 1u))
                grad_ref_cam[(((int64_t)c * B + b) * Nq + q) * R * 2 + (i - c * 2 * R)] = 0.f;
        }
    }
    float wl[NC], hl[NC];
    bool in[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        in[c] = j < n;
        const int l = in[c] ? j / P : 0;
        wl[c] = (float)s_lv.w[l];
        hl[c] = (float)s_lv.h[l];
    }
    for (int h0 = 0; h0 < H; h0 += kIgHeads) {
        const int nh = min(kIgHeads, H - h0);
        float G[kIgHeads][NC];
        double gx[kIgHeads][NC], gy[kIgHeads][NC];
#pragma unroll
        for (int hh = 0; hh < kIgHeads; ++hh)
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                G[hh][c] = 0.f;
                gx[hh][c] = gy[hh][c] = 0.0;
            }
        unsigned cams = seen;
        while (cams) {
            const int cam = __ffs(cams) - 1;  // ascending camera order
            cams &= cams - 1;
            const int row = __shfl_sync(0xffffffffu, p, cam);
            const int64_t r = (((int64_t)b * Ncam + cam) * Nq + row) * S + (int64_t)h0 * n;
            double rx = 0.0, ry = 0.0;
#pragma unroll
            for (int hh = 0; hh < kIgHeads; ++hh)
#pragma unroll
                for (int c = 0; c < NC; ++c) {
                    const int j = c * 32 + lane;
                    if (hh < nh && in[c]) {
                        G[hh][c] += __ldcs(grad_attn_rb + r + hh * n + j);
                        const float2 v =
                            __ldcs(reinterpret_cast<const float2*>(grad_loc_rb) + r + hh * n + j);
                        const float2 lo =
                            grad_loc_lo_rb ? __ldcs(reinterpret_cast<const float2*>(grad_loc_lo_rb) +
                                                    r + hh * n + j)
                                           : make_float2(0.f, 0.f);
                        const double vx = (double)v.x + (double)lo.x;
                        const double vy = (double)v.y + (double)lo.y;
                        gx[hh][c] += vx;
                        gy[hh][c] += vy;
                        if (REF) {
                            rx += vx;
                            ry += vy;
                        }
                    }
                }
            if (REF) {
                for (int o = 16; o >= R; o >>= 1) {
                    rx += __shfl_xor_sync(0xffffffffu, rx, o);
                    ry += __shfl_xor_sync(0xffffffffu, ry, o);
                }
                if (lane < R) {
                    float* out = grad_ref_cam + (((int64_t)cam * B + b) * Nq + q) * R * 2;
                    out[2 * lane] = (float)rx;
                    out[2 * lane + 1] = (float)ry;
                }
            }
        }
        float a[kIgHeads][NC];
#pragma unroll
        for (int hh = 0; hh < kIgHeads; ++hh)
#pragma unroll
            for (int c = 0; c < NC; ++c)
                a[hh][c] = (hh < nh && in[c])
                               ? __ldg(logits + bq * S + (int64_t)(h0 + hh) * n + c * 32 + lane)
                               : -INFINITY;
#pragma unroll
        for (int hh = 0; hh < kIgHeads; ++hh) {
            if (hh >= nh) break;  // warp-uniform
            float m = -INFINITY;
#pragma unroll
            for (int c = 0; c < NC; ++c) m = fmaxf(m, a[hh][c]);
            m = warp_max(m);
            float z = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                a[hh][c] = in[c] ? expf(a[hh][c] - m) : 0.f;
                z += a[hh][c];
            }
            z = warp_sum(z);
            double dot = 0.0;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                a[hh][c] = a[hh][c] / z;
                dot += (double)a[hh][c] * (double)G[hh][c];
            }
            dot = warp_sum_f64(dot);
            const int64_t o = bq * S + (int64_t)(h0 + hh) * n;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                const int j = c * 32 + lane;
                if (in[c]) {
                    grad_logits[o + j] = (float)((double)a[hh][c] * ((double)G[hh][c] - dot));
                    reinterpret_cast<float2*>(grad_off)[o + j] =
                        make_float2((float)(gx[hh][c] / (double)wl[c]),
                                    (float)(gy[hh][c] / (double)hl[c]));
                }
            }
        }
    }
}

// Rows of L*P <= 16 samples, in the forward's group layout: lane (s, k)
// takes sample k of head h0 + s (npad = L*P rounded up to a power of two,
// G = 32 / npad heads per pass), so the softmax and <alpha, G> are segmented
// reductions over npad lanes instead of whole-warp ones for a few samples.
// REF (all heads in one pass, R dividing npad): lane mod R is the sample's
// anchor, and a butterfly over the lanes of one anchor gives each camera's
// reference-point sums, as in the per-head kernel.
__device__ __forceinline__ double segment_sum_f64(double v, int npad)
{
    for (int o = npad >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

template <int NPL, bool REF>
__global__ void __launch_bounds__(kIgWarps * 32)
sca_offset_logit_grads_group_kernel(const float* __restrict__ logits,
                                    const int32_t* __restrict__ pos,
                                    const float* __restrict__ grad_loc_rb,
                                    const float* __restrict__ grad_loc_lo_rb,
                                    const float* __restrict__ grad_attn_rb, int B, int Ncam,
                                    int Nq, int H, int L, int P, int R, Levels levels,
                                    float* __restrict__ grad_off, float* __restrict__ grad_logits,
                                    float* __restrict__ grad_ref_cam)
{
    constexpr int npad = 1 << NPL;
    constexpr int G = 32 >> NPL;
    __shared__ SmemLevels s_lv;
    stage_levels(s_lv, levels);
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t bq = (int64_t)blockIdx.x * kIgWarps + (threadIdx.x >> 5);
    if (bq >= (int64_t)B * Nq) return;  // warp-uniform
    const int b = (int)(bq / Nq), q = (int)(bq - (int64_t)b * Nq);
    const int n = L * P, S = H * n;
    const int p = lane < Ncam ? (pos ? __ldg(pos + ((int64_t)b * Ncam + lane) * Nq + q) : q) : -1;
    const unsigned seen = __ballot_sync(0xffffffffu, p >= 0);
    if (REF) {
        for (int i = lane; i < Ncam * R * 2; i += 32) {
            const int c = i / (2 * R);
            if (!((seen >> c) & 1u))
                grad_ref_cam[(((int64_t)c * B + b) * Nq + q) * R * 2 + (i - c * 2 * R)] = 0.f;
        }
    }
    const int s = lane >> NPL, k = lane & (npad - 1);
    const bool kin = k < n;
    const int l = kin ? k / P : 0;
    const float wl = (float)s_lv.w[l], hl = (float)s_lv.h[l];
    for (int h0 = 0; h0 < H; h0 += G) {
        const bool in = kin && h0 + s < H;
        const int64_t e = (int64_t)(h0 + s) * n + k;  // element within the row
        float Gs = 0.f;
        double gx = 0.0, gy = 0.0;
        unsigned cams = seen;
        while (cams) {
            const int cam = __ffs(cams) - 1;  // ascending camera order
            cams &= cams - 1;
            const int row = __shfl_sync(0xffffffffu, p, cam);
            const int64_t r = (((int64_t)b * Ncam + cam) * Nq + row) * S;
            double vx = 0.0, vy = 0.0;
            if (in) {
                Gs += __ldcs(grad_attn_rb + r + e);
                const float2 v = __ldcs(reinterpret_cast<const float2*>(grad_loc_rb) + r + e);
                const float2 lo = grad_loc_lo_rb
                                      ? __ldcs(reinterpret_cast<const float2*>(grad_loc_lo_rb) + r + e)
                                      : make_float2(0.f, 0.f);
                vx = (double)v.x + (double)lo.x;
                vy = (double)v.y + (double)lo.y;
                gx += vx;
                gy += vy;
            }
            if (REF) {
                double rx = vx, ry = vy;
                for (int o = 16; o >= R; o >>= 1) {
                    rx += __shfl_xor_sync(0xffffffffu, rx, o);
                    ry += __shfl_xor_sync(0xffffffffu, ry, o);
                }
                if (lane < R) {
                    float* out = grad_ref_cam + (((int64_t)cam * B + b) * Nq + q) * R * 2;
                    out[2 * lane] = (float)rx;
                    out[2 * lane + 1] = (float)ry;
                }
            }
        }
        const float a = in ? __ldg(logits + bq * S + e) : -INFINITY;
        const float m = segment_max(a, npad);
        const float ex = in ? expf(a - m) : 0.f;
        const float z = segment_sum(ex, npad);
        const float alpha = in ? ex / z : 0.f;
        const double dot = segment_sum_f64((double)alpha * (double)Gs, npad);
        if (in) {
            grad_logits[bq * S + e] = (float)((double)alpha * ((double)Gs - dot));
            reinterpret_cast<float2*>(grad_off)[bq * S + e] =
                make_float2((float)(gx / (double)wl), (float)(gy / (double)hl));
        }
    }
}

// One warp per (camera, batch, query): the row's H*L*P location gradients
// summed per anchor m = k mod R (zero when the camera does not see the query).
__global__ void __launch_bounds__(kIgWarps * 32)
sca_reference_grads_kernel(const int32_t* __restrict__ pos, const float* __restrict__ grad_loc_rb,
                           const float* __restrict__ grad_loc_lo_rb, int B, int Ncam, int Nq,
                           int S, int P, int R, float* __restrict__ grad_ref_cam)
{
    const int lane = threadIdx.x & 31;
    const int64_t cbq = (int64_t)blockIdx.x * kIgWarps + (threadIdx.x >> 5);  // (c * B + b) * Nq + q
    if (cbq >= (int64_t)Ncam * B * Nq) return;  // warp-uniform
    const int q = (int)(cbq % Nq);
    const int64_t cb = cbq / Nq;
    const int b = (int)(cb % B), c = (int)(cb / B);
    const int p = pos ? __ldg(pos + ((int64_t)b * Ncam + c) * Nq + q) : q;
    float* out = grad_ref_cam + cbq * R * 2;
    if (p < 0) {
        if (lane < 2 * R) out[lane] = 0.f;
        return;
    }
    const int64_t row = (((int64_t)b * Ncam + c) * Nq + p) * S;
    const float2* g = reinterpret_cast<const float2*>(grad_loc_rb) + row;
    const float2* glo =
        grad_loc_lo_rb ? reinterpret_cast<const float2*>(grad_loc_lo_rb) + row : nullptr;
    if (32 % R == 0) {
        // sample e has anchor (e mod P) mod R = e mod R (R divides P, which
        // divides L*P): lane + 32 i has the anchor lane mod R for every i
        double ax = 0.0, ay = 0.0;
        for (int e = lane; e < S; e += 32) {
            const float2 v = __ldcs(g + e);
            const float2 lo = glo ? __ldcs(glo + e) : make_float2(0.f, 0.f);
            ax += (double)v.x + (double)lo.x;
            ay += (double)v.y + (double)lo.y;
        }
        for (int o = 16; o >= R; o >>= 1) {
            ax += __shfl_xor_sync(0xffffffffu, ax, o);
            ay += __shfl_xor_sync(0xffffffffu, ay, o);
        }
        if (lane < R) {
            out[2 * lane] = (float)ax;
            out[2 * lane + 1] = (float)ay;
        }
        return;
    }
    double sx[MSDA_MAX_POINTS], sy[MSDA_MAX_POINTS];
#pragma unroll
    for (int m = 0; m < MSDA_MAX_POINTS; ++m) sx[m] = sy[m] = 0.0;
    for (int e = lane; e < S; e += 32) {
        const float2 v = __ldcs(g + e);
        const float2 lo = glo ? __ldcs(glo + e) : make_float2(0.f, 0.f);
        const int m = (e % P) % R;
#pragma unroll
        for (int mm = 0; mm < MSDA_MAX_POINTS; ++mm)
            if (mm == m) {
                sx[mm] += (double)v.x + (double)lo.x;
                sy[mm] += (double)v.y + (double)lo.y;
            }
    }
#pragma unroll
    for (int m = 0; m < MSDA_MAX_POINTS; ++m) {
        if (m < R) {  // warp-uniform
            const double x = warp_sum_f64(sx[m]), y = warp_sum_f64(sy[m]);
            if (lane == 0) {
                out[2 * m] = (float)x;
                out[2 * m + 1] = (float)y;
            }
        }
    }
}

}  // namespace

cudaError_t launch_sca_input_grads(const float* logits, const int32_t* pos,
                                   const float* grad_loc_rb, const float* grad_attn_rb, int B,
                                   int Ncam, int Nq, int H, int L, int P, int R, const Levels& lv,
                                   float* grad_off, float* grad_logits, float* grad_ref_cam,
                                   cudaStream_t s, const float* grad_loc_lo_rb)
{
    const int64_t rows = (int64_t)B * Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kIgWarps - 1) / kIgWarps);
    const int n = L * P;
    const int nc = (n + 31) / 32;
    bool fused = H <= kIgHeads && 32 % R == 0;
    if (n <= 16) {
        int npl = 2;
        while ((1 << npl) < n) ++npl;
        fused = H <= (32 >> npl) && (1 << npl) % R == 0;
#define IG_GROUP_CASE(NPLV)                                                                      \
    case NPLV:                                                                                   \
        if (fused)                                                                               \
            sca_offset_logit_grads_group_kernel<NPLV, true><<<grid, kIgWarps * 32, 0, s>>>(      \
                logits, pos, grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, B, Ncam, Nq, H, L, P, R, \
                lv, grad_off,                                                                    \
                grad_logits, grad_ref_cam);                                                      \
        else                                                                                     \
            sca_offset_logit_grads_group_kernel<NPLV, false><<<grid, kIgWarps * 32, 0, s>>>(     \
                logits, pos, grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, B, Ncam, Nq, H, L, P, R, \
                lv, grad_off,                                                                    \
                grad_logits, grad_ref_cam);                                                      \
        break;
        switch (npl) {
            IG_GROUP_CASE(2)
            IG_GROUP_CASE(3)
            IG_GROUP_CASE(4)
            default: return cudaErrorInvalidValue;
        }
#undef IG_GROUP_CASE
    } else {
#define IG_CASE(NCV)                                                                             \
    case NCV:                                                                                    \
        if (fused)                                                                               \
            sca_offset_logit_grads_kernel<NCV, true><<<grid, kIgWarps * 32, 0, s>>>(             \
                logits, pos, grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, B, Ncam, Nq, H, L, P, R, \
                lv, grad_off,                                                                    \
                grad_logits, grad_ref_cam);                                                      \
        else                                                                                     \
            sca_offset_logit_grads_kernel<NCV, false><<<grid, kIgWarps * 32, 0, s>>>(            \
                logits, pos, grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, B, Ncam, Nq, H, L, P, R, \
                lv, grad_off,                                                                    \
                grad_logits, grad_ref_cam);                                                      \
        break;
        switch (nc) {
            IG_CASE(1)
            IG_CASE(2)
            IG_CASE(3)
            IG_CASE(4)
            default: return cudaErrorInvalidValue;
        }
#undef IG_CASE
    }
    if (fused) return cudaGetLastError();
    const int64_t crows = (int64_t)Ncam * B * Nq;
    sca_reference_grads_kernel<<<(unsigned)((crows + kIgWarps - 1) / kIgWarps), kIgWarps * 32, 0,
                                 s>>>(pos, grad_loc_rb, grad_loc_lo_rb, B, Ncam, Nq, H * L * P, P,
                                      R, grad_ref_cam);
    return cudaGetLastError();
}

}  // namespace msda
