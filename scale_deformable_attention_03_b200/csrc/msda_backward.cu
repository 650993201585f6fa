// MSDA / SCA backward: the analytic derivative of the forward read and sum
// (the pages give no backward; it follows from "BEV(三) BEVFormer: how the
// Query interacts with the 8 Heads of the Feature", sections 6 and 8).
//   f = sum_g w_g V_g,  d out / d alpha = f,
//   d f / d x = (1-ly)(V_10 - V_00) + ly (V_11 - V_01),
//   d f / d y = (1-lx)(V_01 - V_00) + lx (V_11 - V_10),
//   x = W s_x - 1/2  =>  d / d s_x = W * d / d x   (same for y with H),
//   d out / d V_g = alpha w_g   (neighbours inside the map only).
// One warp per (row, head) with the forward's lane layout.  For every sample
// each lane forms dot_g = <grad_out, V_g> over its channels and adds
// alpha w_g grad_out to grad_value with 16-byte vector reductions
// (red.global.add.v4.f32, paired across lanes so that every instruction
// covers whole 32-byte L2 sectors); the per-sample scalars are reduced with
// shuffles and land on the lane that owns the sample, which writes them
// coalesced.  Rows of at most 16 samples take the head-group form
// (backward_group_kernel): one warp builds a 32-sample table for several
// heads of a row, as the forward's group kernels do.
// Deterministic variant (DET): instead of fp32 reductions, each contribution
// is scaled by 2^32 (exact), rounded once to a 64-bit integer and added with
// red.global.add.u64 into a fixed-point copy of grad_value; integer addition
// does not depend on order, so the result is bitwise reproducible, and one
// conversion kernel rounds it to fp32 at the end.  The 64-bit adds are
// issued lane per channel (one warp instruction adds a whole 256-byte corner
// slice, eight full L2 sectors), from a per-sample copy of the coefficients.
// The dot products and everything derived from them are formed in double
// (a product of two fp32 numbers is exact in double): the location gradient
// multiplies a difference of dot products by alpha * W_l (up to ~40 at
// W_l = 200), and fp32 sums of the 32 products leave errors near 1e-4 there.
#include <algorithm>
#include <type_traits>

#include "msda_launch.h"

namespace msda {

constexpr int kBwdRowsPerTile = 2;

// The four corners of one sample, for the deterministic adds (read as two
// broadcast 16-byte loads).
struct __align__(16) DetEntry {
    int off[4];
    float wa[4];  // alpha * bilinear weight
};

// Sample table of one (row, head): corner g of sample j as (element offset,
// -1 outside; alpha * w_g as float bits), and the sample's fractions (lx, ly),
// from which w_g and its derivatives are formed again.
struct BwdTable {
    int2 ow[4][kMetaStride];
    float2 l[kMetaStride];
};

__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d)
{
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
                 "f"(c), "f"(d)
                 : "memory");
}

constexpr float kFixScale = 4294967296.f;  // 2^32: fixed-point grad_value units

__device__ __forceinline__ void red_add_fix(long long* addr, float v)
{
    const long long q = __float2ll_rn(v * kFixScale);
    asm volatile("red.global.add.u64 [%0], %1;" ::"l"(addr), "l"(q) : "memory");
}

__device__ __forceinline__ double warp_sum_d(double v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ double segment_sum_d(double v, int npad)
{
    for (int o = npad >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// row_weights with the softmax formed in double ("BEV(三)..." section 4.2):
// ad = exp(x - max) / sum in double, a = ad rounded once to fp32.
template <bool FUSED, int NC>
__device__ __forceinline__ void row_weights_f64(const float* __restrict__ src, int n, int lane,
                                                float (&a)[NC], double (&ad)[NC])
{
    float x[NC];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        x[c] = (j < n) ? ld_stream(src + j) : (FUSED ? -INFINITY : 0.f);
    }
    if (!FUSED) {
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            a[c] = x[c];
            ad[c] = x[c];
        }
        return;
    }
    float m = x[0];
#pragma unroll
    for (int c = 1; c < NC; ++c) m = fmaxf(m, x[c]);
    m = warp_max(m);
    double z = 0.0;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        ad[c] = (c * 32 + lane < n) ? exp((double)x[c] - (double)m) : 0.0;
        z += ad[c];
    }
    z = warp_sum_d(z);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        ad[c] = ad[c] / z;
        a[c] = (float)ad[c];
    }
}

// d w_g / d lx and d w_g / d ly for neighbour g.
__device__ __forceinline__ double dw_dlx(int g, float ly)
{
    const double a = (g >> 1) ? (double)ly : 1.0 - (double)ly;
    return (g & 1) ? a : -a;
}
__device__ __forceinline__ double dw_dly(int g, float lx)
{
    const double a = (g & 1) ? (double)lx : 1.0 - (double)lx;
    return (g >> 1) ? a : -a;
}

// Butterfly reduce-scatter over the lanes that differ only in the low bits
// of t (three bits for eight entries, two for four): lane t ends with the
// full sum of entry t (t mod the entry count).
__device__ __forceinline__ double reduce_scatter8(const double (&part)[8], int t)
{
    double q[4], r[2];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool hi = t & 4;
        q[i] = (hi ? part[i + 4] : part[i]) +
               __shfl_xor_sync(0xffffffffu, hi ? part[i] : part[i + 4], 4);
    }
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool hi = t & 2;
        r[i] = (hi ? q[i + 2] : q[i]) + __shfl_xor_sync(0xffffffffu, hi ? q[i] : q[i + 2], 2);
    }
    const bool hi = t & 1;
    return (hi ? r[1] : r[0]) + __shfl_xor_sync(0xffffffffu, hi ? r[0] : r[1], 1);
}

__device__ __forceinline__ double reduce_scatter4(const double (&part)[4], int t)
{
    double q[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const bool hi = t & 2;
        q[i] = (hi ? part[i + 2] : part[i]) +
               __shfl_xor_sync(0xffffffffu, hi ? part[i] : part[i + 2], 2);
    }
    const bool hi = t & 1;
    return (hi ? q[1] : q[0]) + __shfl_xor_sync(0xffffffffu, hi ? q[0] : q[1], 1);
}

// Sums over the four corner-group lanes, scattered: afterwards the lane of
// group g holds the total of c[g].  `stride` is the lane distance between
// neighbouring groups.  Three double shuffles for three sums (c[3] unused).
__device__ __forceinline__ double reduce_scatter_groups(const double (&c)[4], int g, int stride)
{
    const bool hi2 = g & 2;
    const double a0 =
        (hi2 ? c[2] : c[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? c[0] : c[2], 2 * stride);
    const double a1 =
        (hi2 ? c[3] : c[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? c[1] : c[3], 2 * stride);
    const bool hi1 = g & 1;
    return (hi1 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, hi1 ? a0 : a1, stride);
}

// w_g (as locate() rounds it) and, in double, d w_g / d lx and d w_g / d ly.
__device__ __forceinline__ void corner_weight(int g, float2 l, float& wg, double& dx, double& dy)
{
    const float hx = __fsub_rn(1.f, l.x), hy = __fsub_rn(1.f, l.y);
    wg = __fmul_rn((g & 1) ? l.x : hx, (g >> 1) ? l.y : hy);
    dx = dw_dlx(g, l.y);
    dy = dw_dly(g, l.x);
}

// Samples are processed eight at a time.  Each lane forms its partial dot
// products <grad_out, V_g> for the eight samples (over its own channels), and
// a butterfly reduce-scatter over the lanes that share a corner leaves every
// lane with the full dot product of one sample: 7 (fp32) or 3 (bf16) double
// shuffles per eight samples instead of 3 (or 2) per sample.
template <typename VT>
struct BwdLanes;

// fp32 value: lanes 8g + t hold corner g, channels 4t..4t+3.  After batch(),
// lane (g, t) holds D_g of sample j0 + t.
template <>
struct BwdLanes<float> {
    float4 go;
    __device__ __forceinline__ void load_grad(const float* __restrict__ grow, float scale,
                                              int lane)
    {
        const float4 v = __ldg(reinterpret_cast<const float4*>(grow) + (lane & 7));
        go = make_float4(v.x / scale, v.y / scale, v.z / scale, v.w / scale);
    }
    static constexpr int kStride = 8;  // lanes between corner groups
    __device__ __forceinline__ static int group(int lane) { return lane >> 3; }
    // sample (within the batch) whose dot product the lane holds after batch()
    __device__ __forceinline__ static int held(int lane) { return lane & 7; }
    // a group-0 lane holding sample u of the batch
    __device__ __forceinline__ static int holder(int u) { return u; }
    template <bool DET, bool LF>
    __device__ __forceinline__ double batch(const float* __restrict__ vb,
                                            float* __restrict__ gvb, long long* __restrict__ gvi,
                                            const BwdTable& tab, int j0, int cnt, int lane) const
    {
        const int g = lane >> 3, t = lane & 7;
        double part[8];
        if constexpr (!DET && LF) {  // every load of the batch in flight before its reductions
            int o[8];
            float4 v[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int j = j0 + k;
                o[k] = j < cnt ? tab.ow[g][j].x : -1;
                v[k] = o[k] >= 0 ? __ldg(reinterpret_cast<const float4*>(vb + o[k] + 4 * t))
                                 : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float w = o[k] >= 0 ? __int_as_float(tab.ow[g][j0 + k].y) : 0.f;
                if (w != 0.f)
                    red_add_v4(gvb + o[k] + 4 * t, w * go.x, w * go.y, w * go.z, w * go.w);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k)
                part[k] = (double)go.x * v[k].x + (double)go.y * v[k].y +
                          (double)go.z * v[k].z + (double)go.w * v[k].w;
            return reduce_scatter8(part, t);
        } else {
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const int j = j0 + k;
                const int2 e = j < cnt ? tab.ow[g][j] : make_int2(-1, 0);
                part[k] = 0.0;
                if (e.x >= 0) {
                    const float4 v = __ldg(reinterpret_cast<const float4*>(vb + e.x + 4 * t));
                    part[k] = (double)go.x * v.x + (double)go.y * v.y + (double)go.z * v.z +
                              (double)go.w * v.w;
                    const float w = __int_as_float(e.y);
                    if (!DET && w != 0.f)
                        red_add_v4(gvb + e.x + 4 * t, w * go.x, w * go.y, w * go.z, w * go.w);
                }
            }
            return reduce_scatter8(part, t);
        }
    }
};

// bf16 value: lanes 16s + 4g + t hold corner g, channels 8t..8t+7, of the
// samples j0 + 2k + s.  After batch(), lane (s, g, t) holds D_g of sample
// j0 + 2t + s.  The grad_value reductions use another channel split so that
// every 16-byte vector add has its 32-byte sector's other half in the same
// instruction (one L2 sector operation instead of two): lanes t = 2p + h add
// channels 16p + 4h .. +3 in the first instruction and 16p + 8 + 4h .. +3 in
// the second (red_channel).
__device__ __forceinline__ int red_channel(int t) { return 16 * (t >> 1) + 4 * (t & 1); }

template <>
struct BwdLanes<__nv_bfloat16> {
    float go[8];  // channels 8t .. 8t+7 (dot products)
    float gr[8];  // channels red_channel(t) + 0..3 and + 8..11 (reductions)
    __device__ __forceinline__ void load_grad(const float* __restrict__ grow, float scale,
                                              int lane)
    {
        const int t = lane & 3;
        const float4* g4 = reinterpret_cast<const float4*>(grow);
        const float4 a = __ldg(g4 + 2 * t), b = __ldg(g4 + 2 * t + 1);
        go[0] = a.x / scale; go[1] = a.y / scale; go[2] = a.z / scale; go[3] = a.w / scale;
        go[4] = b.x / scale; go[5] = b.y / scale; go[6] = b.z / scale; go[7] = b.w / scale;
        const int rc = red_channel(t) / 4;
        const float4 c = __ldg(g4 + rc), d = __ldg(g4 + rc + 2);
        gr[0] = c.x / scale; gr[1] = c.y / scale; gr[2] = c.z / scale; gr[3] = c.w / scale;
        gr[4] = d.x / scale; gr[5] = d.y / scale; gr[6] = d.z / scale; gr[7] = d.w / scale;
    }
    static constexpr int kStride = 4;
    __device__ __forceinline__ static int group(int lane) { return (lane >> 2) & 3; }
    __device__ __forceinline__ static int held(int lane) { return 2 * (lane & 3) + (lane >> 4); }
    __device__ __forceinline__ static int holder(int u) { return 16 * (u & 1) + (u >> 1); }
    template <bool DET, bool LF>
    __device__ __forceinline__ double batch(const __nv_bfloat16* __restrict__ vb,
                                            float* __restrict__ gvb, long long* __restrict__ gvi,
                                            const BwdTable& tab, int j0, int cnt, int lane) const
    {
        const int s = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
        double part[4];
        if constexpr (!DET && LF) {  // every load of the batch in flight before its reductions
            int o[4];
            uint4 raw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = j0 + 2 * k + s;
                o[k] = j < cnt ? tab.ow[g][j].x : -1;
                raw[k] = o[k] >= 0 ? __ldg(reinterpret_cast<const uint4*>(vb + o[k] + 8 * t))
                                   : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = j0 + 2 * k + s;
                const float w = o[k] >= 0 ? __int_as_float(tab.ow[g][j].y) : 0.f;
                if (w != 0.f) {
                    float* dst = gvb + o[k] + red_channel(t);
                    red_add_v4(dst, w * gr[0], w * gr[1], w * gr[2], w * gr[3]);
                    red_add_v4(dst + 8, w * gr[4], w * gr[5], w * gr[6], w * gr[7]);
                }
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                float v[8];
                bf16x2_to_f32(raw[k].x, v[0], v[1]);
                bf16x2_to_f32(raw[k].y, v[2], v[3]);
                bf16x2_to_f32(raw[k].z, v[4], v[5]);
                bf16x2_to_f32(raw[k].w, v[6], v[7]);
                double d = 0.0;
#pragma unroll
                for (int i = 0; i < 8; ++i) d += (double)go[i] * v[i];
                part[k] = d;
            }
            return reduce_scatter4(part, t);
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int j = j0 + 2 * k + s;
                const int2 e = j < cnt ? tab.ow[g][j] : make_int2(-1, 0);
                part[k] = 0.0;
                if (e.x >= 0) {
                    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(vb + e.x + 8 * t));
                    float v[8];
                    bf16x2_to_f32(raw.x, v[0], v[1]);
                    bf16x2_to_f32(raw.y, v[2], v[3]);
                    bf16x2_to_f32(raw.z, v[4], v[5]);
                    bf16x2_to_f32(raw.w, v[6], v[7]);
                    double d = 0.0;
#pragma unroll
                    for (int i = 0; i < 8; ++i) d += (double)go[i] * v[i];
                    part[k] = d;
                    const float w = __int_as_float(e.y);
                    if (!DET && w != 0.f) {
                        float* dst = gvb + e.x + red_channel(t);
                        red_add_v4(dst, w * gr[0], w * gr[1], w * gr[2], w * gr[3]);
                        red_add_v4(dst + 8, w * gr[4], w * gr[5], w * gr[6], w * gr[7]);
                    }
                }
            }
            return reduce_scatter4(part, t);
        }
    }
};

// Backward of one (row, head).  grow: grad_out of the row's head (32 floats),
// divided by `scale` (1 for MSDA, max(1, hits) for SCA).  gvb: grad_value of
// the batch item (and camera), or (DET) gvi its fixed-point copy.  gloc_row
// [L, P, 2], gattn_row [L, P].  LF: issue a batch's eight corner loads before
// its grad_value reductions (more registers; faster in the persistent SCA
// kernel, whose grid is sized to the resident CTAs, slower elsewhere).
// PREC (the precise location gradients that the chain to offsets and
// reference points sums): the softmax weight and the location gradient are
// formed in double, and gloc_lo_row receives the residual of the fp32
// rounding (gloc = hi, gloc_lo = fp32(exact - hi)), so that sums over many
// samples keep double accuracy.
template <typename VT, bool FUSED, int NC, bool DET, bool LF = false, bool PREC = false>
__device__ __forceinline__ void row_backward(const VT* __restrict__ vb, int H, int h,
                                             const float* __restrict__ lo,
                                             const float* __restrict__ wl,
                                             const float* __restrict__ ref, int n,
                                             const LaneSamples<NC>& ls, BwdTable& tab,
                                             const float* __restrict__ grow, float scale,
                                             float* __restrict__ gvb, long long* __restrict__ gvi,
                                             DetEntry* __restrict__ det,
                                             float* __restrict__ gloc_row,
                                             float* __restrict__ gattn_row, int lane,
                                             float* __restrict__ gloc_lo_row = nullptr)
{
    // DET: channel `lane` of the row's upstream gradient, as BwdLanes forms it
    const float go_c = DET ? __ldg(grow + lane) / scale : 0.f;
    float a[NC];
    double ad[NC];
    if constexpr (PREC)
        row_weights_f64<FUSED, NC>(wl, n, lane, a, ad);
    else
        row_weights<FUSED, NC>(wl, n, lane, a);
    using Lanes = BwdLanes<VT>;
    Lanes lanes;
    lanes.load_grad(grow, scale, lane);
    const int g = Lanes::group(lane);
    const int held = Lanes::held(lane);
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        Corners cr;
        float Wl = 0.f, Hl = 0.f;
        if (ls.in[c]) {
            float sx, sy;
            sample_location<FUSED>(lo, ref, j, ls.m[c], ls.h[c], ls.w[c], sx, sy);
            locate(sx, sy, ls.h[c], ls.w[c], ls.start[c], H, h, cr);
            Wl = (float)ls.w[c];
            Hl = (float)ls.h[c];
        } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                cr.off[q] = -1;
                cr.w[q] = 0.f;
            }
            cr.lx = cr.ly = 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
            tab.ow[q][lane] = make_int2(cr.off[q], __float_as_int(a[c] * cr.w[q]));
        tab.l[lane] = make_float2(cr.lx, cr.ly);
        if (DET) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                det[lane].off[q] = cr.off[q];
                det[lane].wa[q] = a[c] * cr.w[q];  // the same product as the fp32 path
            }
        }
        __syncwarp();
        float res_w = 0.f;
        typename std::conditional<PREC, double, float>::type res_x = 0, res_y = 0;
        const int cnt = min(32, n - c * 32);
        for (int j0 = 0; j0 < cnt; j0 += 8) {
            const double d = lanes.template batch<DET, LF>(vb, gvb, gvi, tab, j0, cnt, lane);
            if (DET) {  // lane = channel: one 256-byte slice per (sample, corner)
                for (int j = j0; j < min(j0 + 8, cnt); ++j) {
                    const int4 o = *reinterpret_cast<const int4*>(det[j].off);
                    const float4 w = *reinterpret_cast<const float4*>(det[j].wa);
                    if (o.x >= 0 && w.x != 0.f) red_add_fix(gvi + o.x + lane, w.x * go_c);
                    if (o.y >= 0 && w.y != 0.f) red_add_fix(gvi + o.y + lane, w.y * go_c);
                    if (o.z >= 0 && w.z != 0.f) red_add_fix(gvi + o.z + lane, w.z * go_c);
                    if (o.w >= 0 && w.w != 0.f) red_add_fix(gvi + o.w + lane, w.w * go_c);
                }
            }
            const int js = j0 + held;  // the sample whose D_g this lane holds
            double c4[4] = {0.0, 0.0, 0.0, 0.0};
            if (js < cnt) {
                float wg;
                double dx, dy;
                corner_weight(g, tab.l[js], wg, dx, dy);
                c4[0] = (double)wg * d;
                c4[1] = dx * d;
                c4[2] = dy * d;
            }
            // lanes of group 0, 1, 2 now hold the weight, x and y sums
            using R = typename std::conditional<PREC, double, float>::type;
            const R r = (R)reduce_scatter_groups(c4, g, Lanes::kStride);
            // the owner of sample j0 + u is lane j0 + u; fetch from the lanes holding it
            const int src = Lanes::holder(lane & 7);
            const float tw = __shfl_sync(0xffffffffu, (float)r, src);
            const R tx = __shfl_sync(0xffffffffu, r, src + Lanes::kStride);
            const R ty = __shfl_sync(0xffffffffu, r, src + 2 * Lanes::kStride);
            if ((lane & ~7) == j0) {
                res_w = tw;
                res_x = tx;
                res_y = ty;
            }
        }
        if (j < n) {
            gattn_row[j] = res_w;
            if constexpr (PREC) {
                const double gx = cr.valid ? ad[c] * (double)Wl * res_x : 0.0;
                const double gy = cr.valid ? ad[c] * (double)Hl * res_y : 0.0;
                const float hx = (float)gx, hy = (float)gy;
                *reinterpret_cast<float2*>(gloc_row + 2 * j) = make_float2(hx, hy);
                *reinterpret_cast<float2*>(gloc_lo_row + 2 * j) =
                    make_float2((float)(gx - (double)hx), (float)(gy - (double)hy));
            } else {
                const float al = a[c];
                *reinterpret_cast<float2*>(gloc_row + 2 * j) = make_float2(
                    cr.valid ? al * Wl * res_x : 0.f, cr.valid ? al * Hl * res_y : 0.f);
            }
        }
        __syncwarp();
    }
}

// ---------------------------------------------------------------------------
// Grouped backward for rows of L*P <= 16 samples, in the forward's group
// layout (see group_compute): a warp takes G = 32 / npad heads of one row and
// lane (s, k) builds sample k of head h0 + s, so the softmax, the corner
// decision and the table cost one pass per 32 samples instead of one per
// head.  The batches of eight then walk the 32-entry table in order, each
// sample with its own head's upstream gradient (a per-warp copy of grad_out,
// already divided by the scale).

struct __align__(16) GroupBwdTable {
    int2 ow[32][4];        // corner g of sample j: offset (-1 outside), alpha * w_g (bits)
    float2 l[32];          // (lx, ly) of sample j
    float go[32 * 8];      // grad_out / scale of the heads, head s at 32 s
};

template <typename VT>
struct GroupBwdLanes;

// fp32 value: lanes 8g + t hold corner g, channels 4t..4t+3 (as BwdLanes).
template <>
struct GroupBwdLanes<float> {
    __device__ __forceinline__ static int group(int lane) { return lane >> 3; }
    __device__ __forceinline__ static int held(int lane) { return lane & 7; }
    __device__ __forceinline__ static int holder(int u) { return u; }
    template <bool DET>
    __device__ __forceinline__ static double corner(const float* __restrict__ vb,
                                                    float* __restrict__ gvb, int2 e, float4 go,
                                                    int t)
    {
        if (e.x < 0) return 0.0;
        const float4 v = __ldg(reinterpret_cast<const float4*>(vb + e.x + 4 * t));
        if (!DET) {
            const float w = __int_as_float(e.y);
            if (w != 0.f) red_add_v4(gvb + e.x + 4 * t, w * go.x, w * go.y, w * go.z, w * go.w);
        }
        return (double)go.x * v.x + (double)go.y * v.y + (double)go.z * v.z + (double)go.w * v.w;
    }
    // Samples j0 .. j0 + 7; with npad = 4 the second four belong to the next head.
    template <int NPL, bool DET>
    __device__ __forceinline__ static double batch(const float* __restrict__ vb,
                                                   float* __restrict__ gvb,
                                                   const GroupBwdTable& tab, int j0, int lane)
    {
        const int g = lane >> 3, t = lane & 7;
        const float* gs = tab.go + (j0 >> NPL) * kHeadDim + 4 * t;
        const float4 ga = *reinterpret_cast<const float4*>(gs);
        const float4 gb = NPL == 2 ? *reinterpret_cast<const float4*>(gs + kHeadDim) : ga;
        double part[8];
#pragma unroll
        for (int k = 0; k < 8; ++k)
            part[k] = corner<DET>(vb, gvb, tab.ow[j0 + k][g], (NPL == 2 && k >= 4) ? gb : ga, t);
        return reduce_scatter8(part, t);
    }
};

// bf16 value: lanes 16s + 4g + t hold corner g, channels 8t..8t+7, of the
// samples j0 + 2k + s (as BwdLanes).
template <>
struct GroupBwdLanes<__nv_bfloat16> {
    __device__ __forceinline__ static int group(int lane) { return (lane >> 2) & 3; }
    __device__ __forceinline__ static int held(int lane) { return 2 * (lane & 3) + (lane >> 4); }
    __device__ __forceinline__ static int holder(int u) { return 16 * (u & 1) + (u >> 1); }
    // g0, g1: channels 8t .. 8t+7 of the sample's head; rs: the head's
    // channels red_channel(t) + 0..3 and + 8..11 (see BwdLanes), read from
    // the shared copy only when the add happens
    template <bool DET>
    __device__ __forceinline__ static double corner(const __nv_bfloat16* __restrict__ vb,
                                                    float* __restrict__ gvb, int2 e, float4 g0,
                                                    float4 g1, const float4* rs, int t)
    {
        if (e.x < 0) return 0.0;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(vb + e.x + 8 * t));
        float v[8];
        bf16x2_to_f32(raw.x, v[0], v[1]);
        bf16x2_to_f32(raw.y, v[2], v[3]);
        bf16x2_to_f32(raw.z, v[4], v[5]);
        bf16x2_to_f32(raw.w, v[6], v[7]);
        if (!DET) {
            const float w = __int_as_float(e.y);
            if (w != 0.f) {
                const float4 r0 = rs[0], r1 = rs[2];
                float* dst = gvb + e.x + red_channel(t);
                red_add_v4(dst, w * r0.x, w * r0.y, w * r0.z, w * r0.w);
                red_add_v4(dst + 8, w * r1.x, w * r1.y, w * r1.z, w * r1.w);
            }
        }
        return (double)g0.x * v[0] + (double)g0.y * v[1] + (double)g0.z * v[2] +
               (double)g0.w * v[3] + (double)g1.x * v[4] + (double)g1.y * v[5] +
               (double)g1.z * v[6] + (double)g1.w * v[7];
    }
    template <int NPL, bool DET>
    __device__ __forceinline__ static double batch(const __nv_bfloat16* __restrict__ vb,
                                                   float* __restrict__ gvb,
                                                   const GroupBwdTable& tab, int j0, int lane)
    {
        const int s = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
        const float* head = tab.go + (j0 >> NPL) * kHeadDim;
        const float4* gs = reinterpret_cast<const float4*>(head + 8 * t);
        const float4* rs = reinterpret_cast<const float4*>(head + red_channel(t));
        const float4 ga0 = gs[0], ga1 = gs[1];
        const float4 gb0 = NPL == 2 ? gs[kHeadDim / 4] : ga0;
        const float4 gb1 = NPL == 2 ? gs[kHeadDim / 4 + 1] : ga1;
        double part[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const bool second = NPL == 2 && k >= 2;  // samples j0 + 4 .. j0 + 7
            part[k] = corner<DET>(vb, gvb, tab.ow[j0 + 2 * k + s][g], second ? gb0 : ga0,
                                  second ? gb1 : ga1, second ? rs + kHeadDim / 4 : rs, t);
        }
        return reduce_scatter4(part, t);
    }
};

// One row, heads h0 .. h0 + G - 1 (those < H).  The lane's inputs come
// preloaded: a (logit, or the weight when !FUSED), v (offset, or the
// location), r (reference point), `valid` = the lane's sample exists, go =
// the lane's channel of each head's grad_out / scale.  gvb / gvi: grad_value
// of the batch item or its fixed-point copy; gloc0 [G, S, 2] and gattn0
// [G, S]: head h0's gradients (+S per head).
// PREC: as in row_backward (double softmax and location gradients, the fp32
// rounding residual of the location gradients into gloc_lo0).
template <typename VT, bool FUSED, int NPL, bool DET, bool PREC = false>
__device__ __forceinline__ void group_backward(const VT* __restrict__ vb, int H, int h0, int S,
                                               float a, float2 v, float2 r, bool valid,
                                               const float (&go)[32 >> NPL], const GroupLane& gl,
                                               GroupBwdTable& tab, float* __restrict__ gvb,
                                               long long* __restrict__ gvi,
                                               float* __restrict__ gloc0,
                                               float* __restrict__ gattn0, int lane,
                                               float* __restrict__ gloc_lo0 = nullptr)
{
    constexpr int G = 32 >> NPL;
    constexpr int npad = 1 << NPL;
    double ad = 0.0;
    if (FUSED) {
        const float m = segment_max(a, npad);
        if constexpr (PREC) {
            const double e = valid ? exp((double)a - (double)m) : 0.0;
            const double z = segment_sum_d(e, npad);
            ad = valid ? e / z : 0.0;
            a = (float)ad;
        } else {
            const float e = valid ? expf(a - m) : 0.f;
            const float z = segment_sum(e, npad);
            a = valid ? e / z : 0.f;
        }
    } else if (!valid) {
        a = 0.f;
    }
    if (!FUSED) ad = a;
    Corners cr;
    if (valid) {
        float sx = v.x, sy = v.y;
        if (FUSED) {
            sx = __fadd_rn(r.x, __fdiv_rn(v.x, (float)gl.w));
            sy = __fadd_rn(r.y, __fdiv_rn(v.y, (float)gl.h));
        }
        locate(sx, sy, gl.h, gl.w, gl.start, H, h0 + gl.s, cr);
    } else {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            cr.off[g] = -1;
            cr.w[g] = 0.f;
        }
        cr.lx = cr.ly = 0.f;
        cr.valid = false;
    }
    int4* row = reinterpret_cast<int4*>(tab.ow[lane]);
    row[0] = make_int4(cr.off[0], __float_as_int(a * cr.w[0]), cr.off[1],
                       __float_as_int(a * cr.w[1]));
    row[1] = make_int4(cr.off[2], __float_as_int(a * cr.w[2]), cr.off[3],
                       __float_as_int(a * cr.w[3]));
    tab.l[lane] = make_float2(cr.lx, cr.ly);
#pragma unroll
    for (int i = 0; i < G; ++i) tab.go[i * kHeadDim + lane] = go[i];
    __syncwarp();

    using Lanes = GroupBwdLanes<VT>;
    const int g = Lanes::group(lane);
    const int held = Lanes::held(lane);
    const int nheads = min(G, H - h0);
    using R = typename std::conditional<PREC, double, float>::type;
    float res_w = 0.f;
    R res_x = 0, res_y = 0;
#pragma unroll
    for (int j0 = 0; j0 < 32; j0 += 8) {
        if ((j0 >> NPL) >= nheads) break;
        const double d = Lanes::template batch<NPL, DET>(vb, gvb, tab, j0, lane);
        if (DET) {  // lane = channel: one 256-byte slice per (sample, corner)
#pragma unroll
            for (int j = j0; j < j0 + 8; ++j) {
                const int4* e = reinterpret_cast<const int4*>(tab.ow[j]);
                const int4 p = e[0], q = e[1];
                const float go_c = tab.go[(j >> NPL) * kHeadDim + lane];
                if (p.x >= 0 && __int_as_float(p.y) != 0.f)
                    red_add_fix(gvi + p.x + lane, __int_as_float(p.y) * go_c);
                if (p.z >= 0 && __int_as_float(p.w) != 0.f)
                    red_add_fix(gvi + p.z + lane, __int_as_float(p.w) * go_c);
                if (q.x >= 0 && __int_as_float(q.y) != 0.f)
                    red_add_fix(gvi + q.x + lane, __int_as_float(q.y) * go_c);
                if (q.z >= 0 && __int_as_float(q.w) != 0.f)
                    red_add_fix(gvi + q.z + lane, __int_as_float(q.w) * go_c);
            }
        }
        // d = D_g of sample j0 + held; its bilinear weight and the weight's
        // derivatives follow from (lx, ly) as in locate()
        float wg;
        double dx, dy;
        corner_weight(g, tab.l[j0 + held], wg, dx, dy);
        const double c4[4] = {(double)wg * d, dx * d, dy * d, 0.0};
        const R r = (R)reduce_scatter_groups(c4, g, BwdLanes<VT>::kStride);
        // sample j0 + u lands on lane j0 + u
        const int src = Lanes::holder(lane & 7);
        const float tw = __shfl_sync(0xffffffffu, (float)r, src);
        const R tx = __shfl_sync(0xffffffffu, r, src + BwdLanes<VT>::kStride);
        const R ty = __shfl_sync(0xffffffffu, r, src + 2 * BwdLanes<VT>::kStride);
        if ((lane & ~7) == j0) {
            res_w = tw;
            res_x = tx;
            res_y = ty;
        }
    }
    if (valid) {
        const int j = gl.s * S + gl.k;
        gattn0[j] = res_w;
        if constexpr (PREC) {
            const double gx = cr.valid ? ad * (double)gl.w * res_x : 0.0;
            const double gy = cr.valid ? ad * (double)gl.h * res_y : 0.0;
            const float hx = (float)gx, hy = (float)gy;
            *reinterpret_cast<float2*>(gloc0 + 2 * j) = make_float2(hx, hy);
            *reinterpret_cast<float2*>(gloc_lo0 + 2 * j) =
                make_float2((float)(gx - (double)hx), (float)(gy - (double)hy));
        } else {
            *reinterpret_cast<float2*>(gloc0 + 2 * j) =
                make_float2(cr.valid ? a * (float)gl.w * res_x : 0.f,
                            cr.valid ? a * (float)gl.h * res_y : 0.f);
        }
    }
    __syncwarp();
}

// Register caps: four CTAs per SM for fp32 value, three for bf16 rows of up
// to 32 samples, two for longer bf16 rows.
template <typename VT, int NC, bool DET>
__global__ void __launch_bounds__(kThreads, sizeof(VT) == 4 ? 4 : (NC == 1 ? 3 : 2))
msda_backward_kernel(const VT* __restrict__ value, const float* __restrict__ loc,
                     const float* __restrict__ attn, const float* __restrict__ grad_out,
                     float* __restrict__ grad_value, long long* __restrict__ grad_value_fix,
                     float* __restrict__ grad_loc,
                     float* __restrict__ grad_attn, int B, int Nq, int Nv, int H, int L, int P,
                     Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) BwdTable s_tab[kWarps];
    __shared__ DetEntry s_det[DET ? kWarps : 1][kMetaStride];
    stage_levels(s_lv, levels);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, 1, lane, ls);
    const int S = L * P;
    const int64_t rows = (int64_t)B * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kBwdRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    ItemCursor cur(warp, H);
    for (int it = warp; it < kBwdRowsPerTile * H; it += kWarps, cur.next()) {
        const int64_t bq = row0 + cur.rr;
        if (bq >= rows) break;
        int q = q0 + cur.rr, b = b0;
        while (q >= Nq) {
            q -= Nq;
            ++b;
        }
        const int64_t item = bq * H + cur.h;
        const int64_t vofs = (int64_t)b * Nv * H * kHeadDim;
        row_backward<VT, false, NC, DET>(value + vofs, H, cur.h, loc + item * S * 2,
                                         attn + item * S, nullptr, S, ls, s_tab[warp],
                                         grad_out + item * kHeadDim, 1.f, grad_value + vofs,
                                         DET ? grad_value_fix + vofs : nullptr,
                                         s_det[DET ? warp : 0], grad_loc + item * S * 2,
                                         grad_attn + item * S, lane);
    }
}

// PREC: precise location gradients with their rounding residual into
// grad_loc_lo_rb (see row_backward), for the chain to offsets and reference
// points.
template <typename VT, int NC, bool DET, bool PREC>
__global__ void __launch_bounds__(kThreads)
sca_backward_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                    const float* __restrict__ logits, const float* __restrict__ ref_cam,
                    const float* __restrict__ grad_out, const int32_t* __restrict__ idx,
                    const int32_t* __restrict__ hits, const int32_t* __restrict__ count,
                    float* __restrict__ grad_value, long long* __restrict__ grad_value_fix,
                    float* __restrict__ grad_loc_rb, float* __restrict__ grad_loc_lo_rb,
                    float* __restrict__ grad_attn_rb, int B, int Ncam, int Nq, int Nv, int H,
                    int L, int P, int R, Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) BwdTable s_tab[kWarps];
    __shared__ DetEntry s_det[DET ? kWarps : 1][kMetaStride];
    __shared__ int s_prefix[kMaxBatchCameras + 1];
    const int nbc = B * Ncam;
    stage_levels(s_lv, levels);
    stage_row_prefix(count, nbc, Nq, s_prefix);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, R, lane, ls);
    const int S = L * P;
    const int total = s_prefix[nbc];
    int bc = 0, b = 0, c = 0, bc_cached = -1;
    for (int64_t tile = blockIdx.x; tile * kBwdRowsPerTile < total; tile += gridDim.x) {
        const int r0 = (int)(tile * kBwdRowsPerTile);
        ItemCursor cur(warp, H);
        for (int it = warp; it < kBwdRowsPerTile * H; it += kWarps, cur.next()) {
            const int r = r0 + cur.rr;
            if (r >= total) break;
            while (r >= s_prefix[bc + 1]) ++bc;  // rows only grow: bc is monotone
            if (bc != bc_cached) {
                b = bc / Ncam;
                c = bc - b * Ncam;
                bc_cached = bc;
            }
            const int i = r - s_prefix[bc];
            const int q = __ldg(idx + (int64_t)bc * Nq + i);
            if ((unsigned)q >= (unsigned)Nq) continue;  // inconsistent lists: read nothing
            const int h = cur.h;
            const int64_t bq = (int64_t)b * Nq + q;
            const int64_t bqh = bq * H + h;
            const int64_t vofs = (int64_t)bc * Nv * H * kHeadDim;
            const int64_t rowh = ((int64_t)bc * Nq + i) * H + h;
            const float scale = (float)max(1, __ldg(hits + bq));
            row_backward<VT, true, NC, DET, true, PREC>(
                value + vofs, H, h, off + bqh * S * 2, logits + bqh * S,
                ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2, S, ls, s_tab[warp],
                grad_out + bqh * kHeadDim, scale, grad_value + vofs,
                DET ? grad_value_fix + vofs : nullptr, s_det[DET ? warp : 0],
                grad_loc_rb + rowh * S * 2, grad_attn_rb + rowh * S, lane,
                PREC ? grad_loc_lo_rb + rowh * S * 2 : nullptr);
        }
    }
}

// TSA: the fused backward of every queue's MSDA; queue t of sample b (value
// item b * T + t) receives grad_out[b] / T (the queue mean).  Rows are
// (b * T + t, q); location and weight gradients per queue row.
template <typename VT, int NC>
__global__ void __launch_bounds__(kThreads)
tsa_backward_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                    const float* __restrict__ logits, const float* __restrict__ ref,
                    const float* __restrict__ grad_out, float* __restrict__ grad_value,
                    float* __restrict__ grad_loc, float* __restrict__ grad_loc_lo,
                    float* __restrict__ grad_attn, int BT, int T, int Nq, int Nv, int H, int L,
                    int P, int R, Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) BwdTable s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, R, lane, ls);
    const int S = L * P;
    const int64_t rows = (int64_t)BT * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kBwdRowsPerTile;
    const int bt0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)bt0 * Nq);
    ItemCursor cur(warp, H);
    for (int it = warp; it < kBwdRowsPerTile * H; it += kWarps, cur.next()) {
        const int64_t r = row0 + cur.rr;
        if (r >= rows) break;
        int q = q0 + cur.rr, bt = bt0;
        while (q >= Nq) {
            q -= Nq;
            ++bt;
        }
        const int64_t item = r * H + cur.h;
        const int64_t gitem = ((int64_t)(bt / T) * Nq + q) * H + cur.h;
        const int64_t vofs = (int64_t)bt * Nv * H * kHeadDim;
        row_backward<VT, true, NC, false, false, true>(
            value + vofs, H, cur.h, off + item * S * 2, logits + item * S, ref + r * R * 2, S, ls,
            s_tab[warp], grad_out + gitem * kHeadDim, (float)T, grad_value + vofs, nullptr,
            nullptr, grad_loc + item * S * 2, grad_attn + item * S, lane,
            grad_loc_lo + item * S * 2);
    }
}

constexpr int kBwdGroupRowsPerTile = MSDA_GROUP_ROWS_PER_TILE;

// Rows with L*P <= 16: a warp item is (row, head group), see group_backward.
// TSA: rows are (b * T + t, q), each queue receiving grad_out[b] / T.  MSDA
// (T = 1, !FUSED): rows are (b, q) with the locations and weights given.
// Register budget: rows of up to four samples (eight heads per warp) run
// fastest at five CTAs per SM despite spills (TSA backward 0.48 -> 0.43 ms
// at four, 0.425 ms at five; six gained nothing more), longer rows at three.
#ifndef MSDA_BWD_GROUP4_MIN_CTAS
#define MSDA_BWD_GROUP4_MIN_CTAS 5
#endif
#ifndef MSDA_BWD_GROUP_MIN_CTAS
#define MSDA_BWD_GROUP_MIN_CTAS 3
#endif
template <typename VT, int NPL, bool FUSED, bool DET, bool PREC>
__global__ void __launch_bounds__(kThreads,
                                  NPL == 2 ? MSDA_BWD_GROUP4_MIN_CTAS : MSDA_BWD_GROUP_MIN_CTAS)
backward_group_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                      const float* __restrict__ logits, const float* __restrict__ ref,
                      const float* __restrict__ grad_out, float* __restrict__ grad_value,
                      long long* __restrict__ grad_value_fix, float* __restrict__ grad_loc,
                      float* __restrict__ grad_loc_lo, float* __restrict__ grad_attn, int BT,
                      int T, int Nq, int Nv, int H, int L, int P, int R, Levels levels)
{
    constexpr int G = 32 >> NPL;
    __shared__ SmemLevels s_lv;
    __shared__ GroupBwdTable s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    GroupLane gl;
    group_lane(s_lv, L, P, R, NPL, lane, gl);
    const int S = L * P;
    const int HG = (H + G - 1) / G;
    const int64_t rows = (int64_t)BT * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kBwdGroupRowsPerTile;
    const int bt0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)bt0 * Nq);
    const int n_items = kBwdGroupRowsPerTile * HG;
    const int64_t vstride = (int64_t)Nv * H * kHeadDim;
    const float scale = (float)T;

    struct Item {
        bool ok, valid;
        int bt, q, h0;
        int64_t r;
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.r = row0 + cur.rr;
        x.ok = it < n_items && x.r < rows;
        x.h0 = cur.h * G;
        x.valid = gl.in && x.h0 + gl.s < H;
        x.q = q0 + cur.rr;
        x.bt = bt0;
        while (x.q >= Nq) {
            x.q -= Nq;
            ++x.bt;
        }
        return x;
    };
    struct In {
        float a;
        float2 v, r;
        float go[G];
    };
    auto fetch = [&](const Item& x, In& in) {
        const int64_t row_h = (x.r * H + x.h0 + gl.s) * S + gl.k;
        in.a = x.valid ? ld_stream(logits + row_h) : (FUSED ? -INFINITY : 0.f);
        in.v = x.valid ? ld_stream2(off + 2 * row_h) : make_float2(0.f, 0.f);
        in.r = (FUSED && x.valid)
                   ? __ldg(reinterpret_cast<const float2*>(ref + x.r * R * 2) + gl.m)
                   : make_float2(0.f, 0.f);
        const int64_t gitem = ((int64_t)(x.bt / T) * Nq + x.q) * H + x.h0;
#pragma unroll
        for (int i = 0; i < G; ++i)
            in.go[i] = x.h0 + i < H ? __ldg(grad_out + (gitem + i) * kHeadDim + lane) / scale
                                    : 0.f;
    };

    ItemCursor cur(warp, HG);
    int it = warp;
    Item x0 = resolve(it, cur);
    In in0, in1;
    if (x0.ok) fetch(x0, in0);
    while (x0.ok) {
        ItemCursor nx = cur;
        nx.next();
        const Item x1 = resolve(it + kWarps, nx);
        if (x1.ok) fetch(x1, in1);
        const int64_t vofs = (int64_t)x0.bt * vstride;
        const int64_t item0 = x0.r * H + x0.h0;
        group_backward<VT, FUSED, NPL, DET, PREC>(
            value + vofs, H, x0.h0, S, in0.a, in0.v, in0.r, x0.valid, in0.go, gl, s_tab[warp],
            grad_value + vofs, DET ? grad_value_fix + vofs : nullptr, grad_loc + item0 * S * 2,
            grad_attn + item0 * S, lane, PREC ? grad_loc_lo + item0 * S * 2 : nullptr);
        x0 = x1;
        in0 = in1;
        cur = nx;
        it += kWarps;
    }
}

// npad = L*P rounded up to a power of two, at least 4; 0 when the row is
// too long for the group kernels (or H = 1, where a warp would hold one head).
static int group_npl(int S, int H)
{
    if (S > 16 || H < 2) return 0;
    int npl = 2;
    while ((1 << npl) < S) ++npl;
    return npl;
}

template <typename VT, bool FUSED, bool DET, bool PREC = false>
static cudaError_t launch_backward_group(const Problem& p, int npl, int BT, int T,
                                         const float* ref, const float* off, const float* logits,
                                         const float* grad_out, float* grad_value,
                                         long long* grad_value_fix, float* grad_loc,
                                         float* grad_attn, cudaStream_t s,
                                         float* grad_loc_lo = nullptr)
{
    const int64_t rows = (int64_t)BT * p.Nq;
    const unsigned grid = (unsigned)((rows + kBwdGroupRowsPerTile - 1) / kBwdGroupRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    switch (npl) {
#define BWD_GROUP_CASE(NPLV)                                                                     \
    case NPLV:                                                                                   \
        backward_group_kernel<VT, NPLV, FUSED, DET, PREC><<<grid, kThreads, 0, s>>>(             \
            v, off, logits, ref, grad_out, grad_value, grad_value_fix, grad_loc, grad_loc_lo,    \
            grad_attn, BT, T, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                             \
        break;
        BWD_GROUP_CASE(2)
        BWD_GROUP_CASE(3)
        BWD_GROUP_CASE(4)
#undef BWD_GROUP_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename VT>
static cudaError_t launch_tsa_backward_t(const Problem& p, int T, const float* ref,
                                         const float* off, const float* logits,
                                         const float* grad_out, float* grad_value,
                                         float* grad_loc, float* grad_loc_lo, float* grad_attn,
                                         cudaStream_t s)
{
    const int BT = p.B * T;
    const int64_t rows = (int64_t)BT * p.Nq;
    if (rows == 0) return cudaSuccess;
    if (const int npl = group_npl(p.L * p.P, p.H))
        return launch_backward_group<VT, true, false, true>(p, npl, BT, T, ref, off, logits,
                                                            grad_out, grad_value, nullptr,
                                                            grad_loc, grad_attn, s, grad_loc_lo);
    const unsigned grid = (unsigned)((rows + kBwdRowsPerTile - 1) / kBwdRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    switch ((p.L * p.P + 31) / 32) {
#define TSA_BWD_CASE(NCV)                                                                        \
    case NCV:                                                                                    \
        tsa_backward_kernel<VT, NCV><<<grid, kThreads, 0, s>>>(                                  \
            v, off, logits, ref, grad_out, grad_value, grad_loc, grad_loc_lo, grad_attn, BT, T,  \
            p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                                               \
        break;
        TSA_BWD_CASE(1)
        TSA_BWD_CASE(2)
        TSA_BWD_CASE(3)
        TSA_BWD_CASE(4)
#undef TSA_BWD_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_tsa_backward(const Problem& p, int T, const float* ref, const float* off,
                                const float* logits, const float* grad_out, float* grad_value,
                                float* grad_loc, float* grad_loc_lo, float* grad_attn,
                                cudaStream_t s)
{
    return p.bf16 ? launch_tsa_backward_t<__nv_bfloat16>(p, T, ref, off, logits, grad_out,
                                                         grad_value, grad_loc, grad_loc_lo,
                                                         grad_attn, s)
                  : launch_tsa_backward_t<float>(p, T, ref, off, logits, grad_out, grad_value,
                                                 grad_loc, grad_loc_lo, grad_attn, s);
}

// ---------------------------------------------------------------------------

__device__ __forceinline__ void zero_range(float* __restrict__ p, int64_t n, int64_t tid,
                                           int64_t nthreads)
{
    // scalar head up to 16-byte alignment, float4 body, scalar tail
    const int64_t head = std::min<int64_t>(n, (int64_t)((16 - ((uintptr_t)p & 15)) & 15) / 4);
    for (int64_t i = tid; i < head; i += nthreads) p[i] = 0.f;
    float4* body = reinterpret_cast<float4*>(p + head);
    const int64_t n4 = (n - head) / 4;
    for (int64_t i = tid; i < n4; i += nthreads) body[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t i = head + n4 * 4 + tid; i < n; i += nthreads) p[i] = 0.f;
}

__global__ void zero_kernel(float* __restrict__ p, int64_t n)
{
    zero_range(p, n, (int64_t)blockIdx.x * blockDim.x + threadIdx.x,
               (int64_t)gridDim.x * blockDim.x);
}

// Rebatched rows count[bc] .. Nq-1 of every (batch, camera) are contiguous in
// both gradient arrays; zero them.
__global__ void sca_zero_tail_kernel(const int32_t* __restrict__ count, int Nq, int S,
                                     float* __restrict__ grad_loc_rb,
                                     float* __restrict__ grad_attn_rb)
{
    const int bc = blockIdx.y;
    const int n = min(max(__ldg(count + bc), 0), Nq);  // inconsistent counts stay in the block
    const int64_t first = (int64_t)bc * Nq + n, last = (int64_t)bc * Nq + Nq;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t nthreads = (int64_t)gridDim.x * blockDim.x;
    zero_range(grad_loc_rb + first * S * 2, (last - first) * S * 2, tid, nthreads);
    zero_range(grad_attn_rb + first * S, (last - first) * S, tid, nthreads);
}

cudaError_t launch_zero(float* p, int64_t n, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n / 4 + 255) / 256 + 1, (int64_t)device_sm_count() * 16);
    zero_kernel<<<(unsigned)blocks, 256, 0, s>>>(p, n);
    return cudaGetLastError();
}

// grad_value = fixed-point accumulator * 2^-32, rounded once to fp32.
__global__ void fix_to_float_kernel(const long long* __restrict__ acc, float* __restrict__ out,
                                    int64_t n)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x)
        out[i] = (float)((double)__ldcs(acc + i) * (1.0 / 4294967296.0));
}

cudaError_t launch_fix_to_float(const long long* acc, float* out, int64_t n, cudaStream_t s)
{
    if (n <= 0) return cudaSuccess;
    const int64_t blocks = std::min<int64_t>((n + 255) / 256, (int64_t)device_sm_count() * 16);
    fix_to_float_kernel<<<(unsigned)blocks, 256, 0, s>>>(acc, out, n);
    return cudaGetLastError();
}

cudaError_t launch_sca_zero_tail(const int32_t* count, int B, int Ncam, int Nq, int S,
                                 float* grad_loc_rb, float* grad_attn_rb, cudaStream_t s)
{
    if (B == 0 || Nq == 0) return cudaSuccess;
    const int64_t per_bc = (int64_t)Nq * S * 3;
    const int bx = (int)std::min<int64_t>((per_bc / 4 + 255) / 256 + 1, 64);
    sca_zero_tail_kernel<<<dim3(bx, B * Ncam), 256, 0, s>>>(count, Nq, S, grad_loc_rb,
                                                            grad_attn_rb);
    return cudaGetLastError();
}

template <typename VT, bool DET>
static cudaError_t launch_msda_backward_t(const Problem& p, const float* loc, const float* attn,
                                          const float* grad_out, float* grad_value,
                                          long long* grad_value_fix, float* grad_loc,
                                          float* grad_attn, cudaStream_t s)
{
    const int64_t rows = (int64_t)p.B * p.Nq;
    if (rows == 0) return cudaSuccess;
    if (const int npl = group_npl(p.L * p.P, p.H))
        return launch_backward_group<VT, false, DET>(p, npl, p.B, 1, nullptr, loc, attn, grad_out,
                                                     grad_value, grad_value_fix, grad_loc,
                                                     grad_attn, s);
    const unsigned grid = (unsigned)((rows + kBwdRowsPerTile - 1) / kBwdRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define MSDA_BWD_CASE(NCV)                                                                       \
    case NCV:                                                                                    \
        msda_backward_kernel<VT, NCV, DET><<<grid, kThreads, 0, s>>>(                            \
            v, loc, attn, grad_out, grad_value, grad_value_fix, grad_loc, grad_attn, p.B, p.Nq,  \
            p.Nv, p.H, p.L, p.P, p.lv);                                                          \
        break;
    switch (nc) {
        MSDA_BWD_CASE(1)
        MSDA_BWD_CASE(2)
        MSDA_BWD_CASE(3)
        MSDA_BWD_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef MSDA_BWD_CASE
    return cudaGetLastError();
}

cudaError_t launch_msda_backward(const Problem& p, const float* loc, const float* attn,
                                 const float* grad_out, float* grad_value,
                                 long long* grad_value_fix, float* grad_loc, float* grad_attn,
                                 cudaStream_t s)
{
    if (grad_value_fix)
        return p.bf16 ? launch_msda_backward_t<__nv_bfloat16, true>(
                            p, loc, attn, grad_out, grad_value, grad_value_fix, grad_loc,
                            grad_attn, s)
                      : launch_msda_backward_t<float, true>(p, loc, attn, grad_out, grad_value,
                                                            grad_value_fix, grad_loc, grad_attn, s);
    return p.bf16 ? launch_msda_backward_t<__nv_bfloat16, false>(p, loc, attn, grad_out,
                                                                 grad_value, nullptr, grad_loc,
                                                                 grad_attn, s)
                  : launch_msda_backward_t<float, false>(p, loc, attn, grad_out, grad_value,
                                                         nullptr, grad_loc, grad_attn, s);
}

template <typename K>
static int bwd_resident_ctas(K kernel)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, kThreads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

template <typename VT, bool DET, bool PREC>
static cudaError_t launch_sca_backward_t(const Problem& p, const float* ref_cam, const float* off,
                                         const float* logits, const float* grad_out,
                                         const int32_t* idx, const int32_t* hits,
                                         const int32_t* count, float* grad_value,
                                         long long* grad_value_fix, float* grad_loc_rb,
                                         float* grad_loc_lo_rb, float* grad_attn_rb,
                                         cudaStream_t s)
{
    const int64_t max_rows = (int64_t)p.B * p.Ncam * p.Nq;
    if (max_rows == 0) return cudaSuccess;
    const int64_t max_ctas = (max_rows + kBwdRowsPerTile - 1) / kBwdRowsPerTile;
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define SCA_BWD_CASE(NCV)                                                                        \
    case NCV: {                                                                                  \
        static int occ = bwd_resident_ctas(sca_backward_kernel<VT, NCV, DET, PREC>);             \
        const int64_t grid = std::min<int64_t>(max_ctas, (int64_t)occ * device_sm_count());      \
        sca_backward_kernel<VT, NCV, DET, PREC><<<(unsigned)grid, kThreads, 0, s>>>(             \
            v, off, logits, ref_cam, grad_out, idx, hits, count, grad_value, grad_value_fix,     \
            grad_loc_rb, grad_loc_lo_rb, grad_attn_rb, p.B, p.Ncam, p.Nq, p.Nv, p.H, p.L, p.P,   \
            p.R, p.lv);                                                                          \
        break;                                                                                   \
    }
    switch (nc) {
        SCA_BWD_CASE(1)
        SCA_BWD_CASE(2)
        SCA_BWD_CASE(3)
        SCA_BWD_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef SCA_BWD_CASE
    return cudaGetLastError();
}

cudaError_t launch_sca_backward_rows(const Problem& p, const float* ref_cam, const float* off,
                                     const float* logits, const float* grad_out,
                                     const int32_t* idx, const int32_t* hits,
                                     const int32_t* count, float* grad_value,
                                     long long* grad_value_fix, float* grad_loc_rb,
                                     float* grad_attn_rb, cudaStream_t s, float* grad_loc_lo_rb)
{
#define SCA_BWD_ARGS                                                                             \
    p, ref_cam, off, logits, grad_out, idx, hits, count, grad_value, grad_value_fix, grad_loc_rb, \
        grad_loc_lo_rb, grad_attn_rb, s
    if (grad_value_fix)
        return p.bf16 ? launch_sca_backward_t<__nv_bfloat16, true, false>(SCA_BWD_ARGS)
                      : launch_sca_backward_t<float, true, false>(SCA_BWD_ARGS);
    if (grad_loc_lo_rb)
        return p.bf16 ? launch_sca_backward_t<__nv_bfloat16, false, true>(SCA_BWD_ARGS)
                      : launch_sca_backward_t<float, false, true>(SCA_BWD_ARGS);
    return p.bf16 ? launch_sca_backward_t<__nv_bfloat16, false, false>(SCA_BWD_ARGS)
                  : launch_sca_backward_t<float, false, false>(SCA_BWD_ARGS);
#undef SCA_BWD_ARGS
}

}  // namespace msda
