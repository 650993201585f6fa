// K6 for rows of up to 32 samples: the SCA row backward in the four-lane
// layout of sca_gather_quad.cu (the pages give no backward; this is the
// analytic derivative of "BEV(三) BEVFormer: how the Query interacts with the
// 8 Heads of the Feature", sections 4.2-8, on the rebatched rows of the
// Tencent Cloud "Spatial Cross-Attention" walkthrough).
//
// A warp serves eight (row, head) items; lanes 4u .. 4u + 3 own item u and
// channels 8t .. 8t + 7 (t = lane mod 4).  Before the item, the quad forms
// its samples' softmax weights and locations and keeps (alpha, s_x, s_y) in
// shared memory.  Sample by sample, every lane of the quad decides the
// corners itself, reads its eight channels of each corner slice and
//   - adds alpha w_g grad_out to grad_value (fp32 vector reductions, lanes
//     t and t ^ 1 completing each 32-byte sector in one instruction; or, for
//     the deterministic variant, 64-bit fixed-point adds, four lanes per
//     sector),
//   - forms its partial dot products D_g = <grad_out, V_g> over its channels
//     (double: products of two fp32 numbers are exact there) and from them
//     the partial sums sum_g w_g D_g, sum_g dw_g/dlx D_g, sum_g dw_g/dly D_g.
// Every two (or four) samples a butterfly over the quad leaves the totals of
// each sample on one lane, which turns them into the weight and location
// gradients.
#include <algorithm>
#include <type_traits>

#include "msda_launch.h"

namespace msda {

#ifndef MSDA_QBWD_MIN_CTAS
#define MSDA_QBWD_MIN_CTAS 2  // register cap (resident CTAs per SM)
#endif
#ifndef MSDA_QBWD_BATCH
#define MSDA_QBWD_BATCH 2  // samples per butterfly (2 or 4): their loads are in flight together
#endif

namespace {

constexpr int kQbSamples = 32;
constexpr int kQbStride = kQbSamples + 1;  // the eight quads of a warp on distinct banks

struct __align__(16) QbMeta {
    int w, h, start, m;
};
constexpr int kQbMetaSlots = kQbSamples + kQbSamples / 8;
__device__ __forceinline__ int qb_slot(int j) { return j + (j >> 3); }

__device__ __forceinline__ void qb_red_v4(float* addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

constexpr float kQbFixScale = 4294967296.f;  // 2^32: fixed-point grad_value units

__device__ __forceinline__ void qb_red_fix(long long* addr, float v)
{
    const long long q = __float2ll_rn(v * kQbFixScale);
    asm volatile("red.global.add.u64 [%0], %1;" ::"l"(addr), "l"(q) : "memory");
}

// Channels of a lane's grad_value reductions: lanes t and t ^ 1 cover the two
// halves of one 32-byte sector in the same instruction.
__device__ __forceinline__ int qb_red_channel(int t) { return 16 * (t >> 1) + 4 * (t & 1); }

template <typename VT>
struct QbCorner;

template <>
struct QbCorner<float> {
    __device__ __forceinline__ static void load(const float* p, float (&v)[8])
    {
        asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                     : "=f"(v[0]), "=f"(v[1]), "=f"(v[2]), "=f"(v[3]), "=f"(v[4]), "=f"(v[5]),
                       "=f"(v[6]), "=f"(v[7])
                     : "l"(p));
    }
};

template <>
struct QbCorner<__nv_bfloat16> {
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, float (&v)[8])
    {
        const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
        bf16x2_to_f32(u.x, v[0], v[1]);
        bf16x2_to_f32(u.y, v[2], v[3]);
        bf16x2_to_f32(u.z, v[4], v[5]);
        bf16x2_to_f32(u.w, v[6], v[7]);
    }
};

template <typename VT>
struct QbBounds {
    static constexpr int kMin = MSDA_QBWD_MIN_CTAS;
};

// Butterfly over the quad: lane t ends with the totals of sample t of the
// four (three values each).
__device__ __forceinline__ void qb_reduce(const double (&p)[4][3], int t, double (&out)[3])
{
    double h[2][3];
    const bool hi2 = t & 2;
#pragma unroll
    for (int s = 0; s < 2; ++s)
#pragma unroll
        for (int v = 0; v < 3; ++v)
            h[s][v] = (hi2 ? p[2 + s][v] : p[s][v]) +
                      __shfl_xor_sync(0xffffffffu, hi2 ? p[s][v] : p[2 + s][v], 2);
    const bool hi1 = t & 1;
#pragma unroll
    for (int v = 0; v < 3; ++v)
        out[v] = (hi1 ? h[1][v] : h[0][v]) + __shfl_xor_sync(0xffffffffu, hi1 ? h[0][v] : h[1][v], 1);
}

// Two samples: lane t ends with the totals of sample t & 1 (lanes t and t ^ 2
// both hold them).
__device__ __forceinline__ void qb_reduce(const double (&p)[2][3], int t, double (&out)[3])
{
    const bool hi1 = t & 1;
#pragma unroll
    for (int v = 0; v < 3; ++v) {
        out[v] = (hi1 ? p[1][v] : p[0][v]) + __shfl_xor_sync(0xffffffffu, hi1 ? p[0][v] : p[1][v], 1);
        out[v] += __shfl_xor_sync(0xffffffffu, out[v], 2);
    }
}

}  // namespace

// DET: fixed-point grad_value (grad_value_fix, zeroed by the caller).
// PREC: softmax weights and location gradients in double, the fp32 rounding
// residual of each location gradient into grad_loc_lo_rb.
template <typename VT, bool DET, bool PREC>
__global__ void __launch_bounds__(kThreads, QbBounds<VT>::kMin)
sca_backward_quad_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                         const float* __restrict__ logits, const float* __restrict__ ref_cam,
                         const float* __restrict__ grad_out, const int32_t* __restrict__ idx,
                         const int32_t* __restrict__ hits, const int32_t* __restrict__ count,
                         float* __restrict__ grad_value, long long* __restrict__ grad_value_fix,
                         float* __restrict__ grad_loc_rb, float* __restrict__ grad_loc_lo_rb,
                         float* __restrict__ grad_attn_rb, int B, int Ncam, int Nq, int Nv,
                         int H, int L, int P, int R, Levels levels)
{
    __shared__ QbMeta s_meta[kQbMetaSlots];
    __shared__ int s_prefix[kMaxBatchCameras + 1];
    __shared__ float s_in[kWarps][3][8][kQbStride];
    __shared__ double s_ad[PREC ? kWarps : 1][8][kQbStride];
    const int n = L * P;
    if (threadIdx.x < kQbSamples) {
        const int j = threadIdx.x;
        QbMeta mt{1, 1, 0, 0};
        if (j < n) {
            const int l = j / P, k = j - l * P;
#pragma unroll
            for (int i = 0; i < kMaxLevels; ++i)  // constant indices: Levels stays in registers
                if (i == l) mt = QbMeta{levels.w[i], levels.h[i], levels.start[i], k % R};
        }
        s_meta[qb_slot(j)] = mt;
    }
    const int nbc = B * Ncam;
    stage_row_prefix(count, nbc, Nq, s_prefix);  // block barrier: s_meta is visible after it

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = lane >> 2, t = lane & 3;
    const int total_rows = s_prefix[nbc];
    const int64_t n_items = (int64_t)total_rows * H;
    const int64_t n_tiles = (n_items + 7) >> 3;
    const int64_t stride = (int64_t)gridDim.x * kWarps;
    const int pix = H * kHeadDim;  // elements per value pixel
    const int rc = qb_red_channel(t);
    float* sa = s_in[warp][0][u];
    float* sxs = s_in[warp][1][u];
    float* sys = s_in[warp][2][u];
    int bc = 0;  // this quad's (batch, camera): its rows only grow

    for (int64_t tile = (int64_t)blockIdx.x * kWarps + warp; tile < n_tiles; tile += stride) {
        // ---- the quad's item ----
        const int64_t item = tile * 8 + u;
        bool live = false;
        int h = 0, b = 0, c = 0, i = 0, q = 0;
        if (item < n_items) {
            const int row = (int)(item / H);
            h = (int)(item - (int64_t)row * H);
            while (row >= s_prefix[bc + 1]) ++bc;
            i = row - s_prefix[bc];
            b = bc / Ncam;
            c = bc - b * Ncam;
            q = __ldg(idx + (int64_t)bc * Nq + i);
            live = (unsigned)q < (unsigned)Nq;  // inconsistent lists: read and write nothing
        }
        const int64_t bq = (int64_t)b * Nq + (live ? q : 0);
        const int64_t qh = bq * H + h;
        // logits and pixel offsets of samples 8t .. 8t + 7
        float a[8], x[8], y[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int j = 8 * t + r;
            const bool in = live && j < n;
            a[r] = in ? __ldcs(logits + qh * n + j) : -INFINITY;
            const float2 o = in ? __ldcs(reinterpret_cast<const float2*>(off) + qh * n + j)
                                : make_float2(0.f, 0.f);
            x[r] = o.x;
            y[r] = o.y;
        }
        // softmax over the item's n logits (section 4.2)
        float m = -INFINITY;
#pragma unroll
        for (int r = 0; r < 8; ++r) m = fmaxf(m, a[r]);
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        if constexpr (PREC) {
            double e[8], z = 0.0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                e[r] = (live && 8 * t + r < n) ? exp((double)a[r] - (double)m) : 0.0;
                z += e[r];
            }
            z += __shfl_xor_sync(0xffffffffu, z, 1);
            z += __shfl_xor_sync(0xffffffffu, z, 2);
            const double zi = live ? z : 1.0;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const double ad = e[r] / zi;
                s_ad[warp][u][8 * t + r] = ad;
                a[r] = (float)ad;
            }
        } else {
            float z = 0.f;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                a[r] = (live && 8 * t + r < n) ? expf(a[r] - m) : 0.f;
                z += a[r];
            }
            z += __shfl_xor_sync(0xffffffffu, z, 1);
            z += __shfl_xor_sync(0xffffffffu, z, 2);
            const float zi = live ? z : 1.f;
#pragma unroll
            for (int r = 0; r < 8; ++r) a[r] = a[r] / zi;
        }
        // locations rho_m + (dx / W_l, dy / H_l) (section 5)
        const float* rf = ref_cam + (((int64_t)c * B + b) * Nq + (live ? q : 0)) * R * 2;
#pragma unroll
        for (int r = 0; r < 8; ++r) {
            const int j = 8 * t + r;
            float sx = __int_as_float(0x7fffffff), sy = sx;  // NaN: no corner is read
            if (live && j < n) {
                const QbMeta mt = s_meta[qb_slot(j)];
                const float2 rv = __ldg(reinterpret_cast<const float2*>(rf) + mt.m);
                sx = __fadd_rn(rv.x, __fdiv_rn(x[r], (float)mt.w));
                sy = __fadd_rn(rv.y, __fdiv_rn(y[r], (float)mt.h));
            }
            sa[j] = a[r];
            sxs[j] = sx;
            sys[j] = sy;
        }
        // the head's upstream gradient / max(1, hits): dot channels 8t .. 8t + 7,
        // reduction channels rc + 0..3 and rc + 8..11 (DET: channels 4e + t)
        float go[8], gr[8];
        {
            const float scale = live ? (float)max(1, __ldg(hits + bq)) : 1.f;
            const float4* g4 = reinterpret_cast<const float4*>(grad_out + qh * kHeadDim);
            float4 v0 = make_float4(0.f, 0.f, 0.f, 0.f), v1 = v0, w0 = v0, w1 = v0;
            if (live) {
                v0 = __ldg(g4 + 2 * t);
                v1 = __ldg(g4 + 2 * t + 1);
                if (!DET) {
                    w0 = __ldg(g4 + rc / 4);
                    w1 = __ldg(g4 + rc / 4 + 2);
                }
            }
            go[0] = v0.x / scale; go[1] = v0.y / scale; go[2] = v0.z / scale; go[3] = v0.w / scale;
            go[4] = v1.x / scale; go[5] = v1.y / scale; go[6] = v1.z / scale; go[7] = v1.w / scale;
            if (DET) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    gr[e] = live ? __ldg(grad_out + qh * kHeadDim + 4 * e + t) / scale : 0.f;
            } else {
                gr[0] = w0.x / scale; gr[1] = w0.y / scale; gr[2] = w0.z / scale; gr[3] = w0.w / scale;
                gr[4] = w1.x / scale; gr[5] = w1.y / scale; gr[6] = w1.z / scale; gr[7] = w1.w / scale;
            }
        }
        __syncwarp();

        // ---- samples, four at a time ----
        const int64_t bc64 = (int64_t)b * Ncam + c;
        const VT* vb = value + bc64 * Nv * pix;
        float* gvb = grad_value + bc64 * Nv * pix;
        long long* gvi = DET ? grad_value_fix + bc64 * Nv * pix : nullptr;
        const int64_t row_h = ((bc64 * Nq + i) * H + h) * n;
        constexpr int KB = MSDA_QBWD_BATCH;
        for (int jb = 0; jb < n; jb += KB) {
            double part[KB][3];
#pragma unroll
            for (int k = 0; k < KB; ++k) {
                const int j = jb + k;
                part[k][0] = part[k][1] = part[k][2] = 0.0;
                if (j >= n) continue;  // warp-uniform
                const float al = sa[j], sx = sxs[j], sy = sys[j];
                const QbMeta mt = s_meta[qb_slot(j)];
                // corner decision (section 6), as the forward takes it
                const float fW = (float)mt.w, fH = (float)mt.h;
                const float xx = __fsub_rn(__fmul_rn(fW, sx), 0.5f);
                const float yy = __fsub_rn(__fmul_rn(fH, sy), 0.5f);
                const bool valid = (xx > -1.f) && (xx < fW) && (yy > -1.f) && (yy < fH);
                const float x0f = floorf(valid ? xx : 0.f), y0f = floorf(valid ? yy : 0.f);
                const float lx = valid ? __fsub_rn(xx, x0f) : 0.f;
                const float ly = valid ? __fsub_rn(yy, y0f) : 0.f;
                const float hx = __fsub_rn(1.f, lx), hy = __fsub_rn(1.f, ly);
                const int x0 = (int)x0f, y0 = (int)y0f;
                const bool x0in = valid && x0 >= 0, x1in = valid && x0 + 1 < mt.w;
                const bool y0in = valid && y0 >= 0, y1in = valid && y0 + 1 < mt.h;
                const int base = ((mt.start + y0 * mt.w + x0) * H + h) * kHeadDim;
                const int offs[4] = {base, base + pix, base + mt.w * pix, base + (mt.w + 1) * pix};
                const bool ins[4] = {x0in && y0in, x1in && y0in, x0in && y1in, x1in && y1in};
                const float wg[4] = {__fmul_rn(hx, hy), __fmul_rn(lx, hy), __fmul_rn(hx, ly),
                                     __fmul_rn(lx, ly)};
                float v[4][8];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[g][e] = 0.f;
                    if (ins[g]) QbCorner<VT>::load(vb + offs[g] + 8 * t, v[g]);
                }
                // grad_value: alpha w_g grad_out on the corners inside the map
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float wa = wg[g] * al;
                    if (!ins[g] || wa == 0.f) continue;
                    if (DET) {
#pragma unroll
                        for (int e = 0; e < 8; ++e) qb_red_fix(gvi + offs[g] + 4 * e + t, wa * gr[e]);
                    } else {
                        float* dst = gvb + offs[g] + rc;
                        qb_red_v4(dst, wa * gr[0], wa * gr[1], wa * gr[2], wa * gr[3]);
                        qb_red_v4(dst + 8, wa * gr[4], wa * gr[5], wa * gr[6], wa * gr[7]);
                    }
                }
                // partial dot products over the lane's channels, combined per corner
                const double dlx[4] = {-(1.0 - (double)ly), 1.0 - (double)ly, -(double)ly,
                                       (double)ly};
                const double dly[4] = {-(1.0 - (double)lx), -(double)lx, 1.0 - (double)lx,
                                       (double)lx};
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    double d = 0.0;
#pragma unroll
                    for (int e = 0; e < 8; ++e) d += (double)go[e] * (double)v[g][e];
                    part[k][0] += (double)wg[g] * d;
                    part[k][1] += dlx[g] * d;
                    part[k][2] += dly[g] * d;
                }
            }
            double tot[3];
            qb_reduce(part, t, tot);
            // the sample whose totals this lane writes (none: j = n)
            const int j = KB == 4 ? jb + t : (t < 2 ? jb + t : n);
            if (live && j < n) {
                grad_attn_rb[row_h + j] = (float)tot[0];
                const QbMeta mt = s_meta[qb_slot(j)];
                float2* gl = reinterpret_cast<float2*>(grad_loc_rb) + row_h + j;
                if constexpr (PREC) {
                    const double ad = s_ad[warp][u][j];
                    const double gx = ad * (double)mt.w * tot[1];
                    const double gy = ad * (double)mt.h * tot[2];
                    const float hxv = (float)gx, hyv = (float)gy;
                    *gl = make_float2(hxv, hyv);
                    reinterpret_cast<float2*>(grad_loc_lo_rb)[row_h + j] =
                        make_float2((float)(gx - (double)hxv), (float)(gy - (double)hyv));
                } else {
                    const float al = sa[j];
                    *gl = make_float2(al * (float)mt.w * (float)tot[1],
                                      al * (float)mt.h * (float)tot[2]);
                }
            }
        }
        __syncwarp();  // this item's shared entries are read before the next item writes
    }
}

bool sca_backward_quad_fits(const Problem& p) { return p.L * p.P <= kQbSamples; }

template <typename VT, bool DET, bool PREC>
static cudaError_t launch_qb_t(const Problem& p, const float* ref_cam, const float* off,
                               const float* logits, const float* grad_out, const int32_t* idx,
                               const int32_t* hits, const int32_t* count, float* grad_value,
                               long long* grad_value_fix, float* grad_loc_rb,
                               float* grad_loc_lo_rb, float* grad_attn_rb, cudaStream_t s)
{
    const int64_t n_items = (int64_t)p.B * p.Ncam * p.Nq * p.H;
    if (n_items == 0) return cudaSuccess;
    const int64_t max_ctas = ((n_items + 7) / 8 + kWarps - 1) / kWarps;
    static int occ = [] {
        int k = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
                &k, sca_backward_quad_kernel<VT, DET, PREC>, kThreads, 0) != cudaSuccess ||
            k < 1)
            k = 1;
        return k;
    }();
    const int64_t grid = std::min<int64_t>(max_ctas, (int64_t)occ * device_sm_count());
    sca_backward_quad_kernel<VT, DET, PREC><<<(unsigned)grid, kThreads, 0, s>>>(
        static_cast<const VT*>(p.value), off, logits, ref_cam, grad_out, idx, hits, count,
        grad_value, grad_value_fix, grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, p.B, p.Ncam, p.Nq,
        p.Nv, p.H, p.L, p.P, p.R, p.lv);
    return cudaGetLastError();
}

cudaError_t launch_sca_backward_quad(const Problem& p, const float* ref_cam, const float* off,
                                     const float* logits, const float* grad_out,
                                     const int32_t* idx, const int32_t* hits,
                                     const int32_t* count, float* grad_value,
                                     long long* grad_value_fix, float* grad_loc_rb,
                                     float* grad_loc_lo_rb, float* grad_attn_rb, cudaStream_t s)
{
#define QB_ARGS                                                                                  \
    p, ref_cam, off, logits, grad_out, idx, hits, count, grad_value, grad_value_fix, grad_loc_rb, \
        grad_loc_lo_rb, grad_attn_rb, s
    if (grad_value_fix)
        return p.bf16 ? launch_qb_t<__nv_bfloat16, true, false>(QB_ARGS)
                      : launch_qb_t<float, true, false>(QB_ARGS);
    if (grad_loc_lo_rb)
        return p.bf16 ? launch_qb_t<__nv_bfloat16, false, true>(QB_ARGS)
                      : launch_qb_t<float, false, true>(QB_ARGS);
    return p.bf16 ? launch_qb_t<__nv_bfloat16, false, false>(QB_ARGS)
                  : launch_qb_t<float, false, false>(QB_ARGS);
#undef QB_ARGS
}

}  // namespace msda
