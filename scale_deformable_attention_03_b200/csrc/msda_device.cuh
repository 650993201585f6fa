// Device building blocks of the MSDA / SCA kernels (sm_100a).
//
// One warp computes one output row of one head: the 32 channels of
//   g^(h) = sum_{l,k} alpha_{h,l,k} * bilinear(V_l^(h), s_{h,l,k})
// ("BEV(三) BEVFormer: how the Query interacts with the 8 Heads of the
// Feature", sections 6 and 8).  The warp works in chunks of 32 samples:
//   1. lane j owns sample j of the chunk: it forms the location, the corner
//      decision and the four corner offsets and weights (alpha folded in) and
//      writes them to a per-warp table in shared memory (structure of arrays,
//      rows padded to 36 words so that the quad reads below are free of bank
//      conflicts);
//   2. the warp walks the table four samples at a time.  fp32 value: lanes
//      8g..8g+7 read corner g of one sample, 16 bytes each, so one warp load
//      fetches the four 128-byte corner slices of a sample.  bf16 value: lanes
//      16s + 4g + t read corner g of sample 2p + s (16 bytes = 8 channels), so
//      one warp load fetches two samples.  Each lane accumulates its own
//      corner and channels; the corners (and sample halves) are summed with
//      shuffles once per row, not once per sample.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace msda {

// Programmatic dependent launch (see launch_pdl): let the next kernel in the
// stream begin launching, and wait for the kernel before this one.
__device__ __forceinline__ void pdl_trigger()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

constexpr int kHeadDim = 32;
constexpr int kMaxLevels = 8;
constexpr int kWarps = 8;               // warps per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kMetaStride = 36;         // words per corner row of the sample table
constexpr int kMaxBatchCameras = 1024;  // B * Ncam limit of the SCA kernels

// Build-time tuning of the gather kernels (defaults are the tuned values).
#ifndef MSDA_BF16_FFMA2
#define MSDA_BF16_FFMA2 1  // bf16 corner adds as packed fp32x2 FMAs (0: scalar FMAs)
#endif
#ifndef MSDA_GATHER_UNROLL
#define MSDA_GATHER_UNROLL 4   // table quads unrolled in the gather loop
#endif
#ifndef MSDA_ROWS_PER_TILE
#define MSDA_ROWS_PER_TILE 8   // consecutive rows per CTA tile (<= 32)
#endif
// Minimum resident CTAs per SM of the forward gathers (a register cap).  Rows
// of up to 32 samples (NC = 1) by value type: fp32 rows take the compiler's
// own choice (0: 64 registers, four CTAs; an explicit 4 measured 1.6 %
// slower), bf16 head pairs three CTAs (80 registers, 7 % faster than the
// compiler's choice).  Longer rows hold more per-lane state: two CTAs for
// NC = 2, no cap beyond.
#ifndef MSDA_MIN_CTAS_F32
#define MSDA_MIN_CTAS_F32 0
#endif
#ifndef MSDA_MIN_CTAS_BF16
#define MSDA_MIN_CTAS_BF16 3
#endif
#define MSDA_GATHER_BOUNDS(VT, NC)                                                       \
    __launch_bounds__(kThreads, (NC) == 1 ? (sizeof(VT) == 4 ? MSDA_MIN_CTAS_F32         \
                                                             : MSDA_MIN_CTAS_BF16)       \
                                          : ((NC) == 2 ? 2 : 1))
// Consecutive rows per CTA tile of the small-row group kernels.
#ifndef MSDA_GROUP_ROWS_PER_TILE
#define MSDA_GROUP_ROWS_PER_TILE 16
#endif
// Minimum resident CTAs of the small-row group kernels (a register cap).
#ifndef MSDA_GROUP_MIN_CTAS
#define MSDA_GROUP_MIN_CTAS 3
#endif
#define MSDA_GROUP_BOUNDS __launch_bounds__(kThreads, MSDA_GROUP_MIN_CTAS)
#ifndef MSDA_PAIR_UNROLL
#define MSDA_PAIR_UNROLL 4     // the same for the bf16 head-pair gather
#endif
constexpr int kGatherUnroll = MSDA_GATHER_UNROLL;
constexpr int kPairUnroll = MSDA_PAIR_UNROLL;

// Level geometry, passed by value to every kernel.
struct Levels {
    int h[kMaxLevels];      // rows H_l
    int w[kMaxLevels];      // columns W_l
    int start[kMaxLevels];  // first value row of the level
};

struct SmemLevels {
    int h[kMaxLevels], w[kMaxLevels], start[kMaxLevels];
};

// Per-warp sample table: corner g of sample j is (off[g][j], w[g][j]).
struct WarpTable {
    int off[4][kMetaStride];
    float w[4][kMetaStride];
};

__device__ __forceinline__ void stage_levels(SmemLevels& s, const Levels& lv)
{
    if (threadIdx.x == 0) {
#pragma unroll
        for (int i = 0; i < kMaxLevels; ++i) {
            s.h[i] = lv.h[i];
            s.w[i] = lv.w[i];
            s.start[i] = lv.start[i];
        }
    }
}

// Maximum over the warp in one instruction (sm_100a redux.sync on f32; a NaN
// lane is ignored like fmaxf ignores it).
__device__ __forceinline__ float warp_max(float v)
{
    float r;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(r) : "f"(v));
    return r;
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Streaming loads for data read once per row (evict-first).
__device__ __forceinline__ float ld_stream(const float* p) { return __ldcs(p); }
__device__ __forceinline__ float2 ld_stream2(const float* p)
{
    return __ldcs(reinterpret_cast<const float2*>(p));
}

// Attention weights of one (row, head): lane holds samples lane + 32c.
// FUSED: softmax over the L*P logits, max-subtracted (section 4.2).
template <bool FUSED, int NC>
__device__ __forceinline__ void row_weights(const float* __restrict__ src, int n, int lane,
                                            float (&a)[NC])
{
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        a[c] = (j < n) ? ld_stream(src + j) : (FUSED ? -INFINITY : 0.f);
    }
    if (FUSED) {
        float m = a[0];
#pragma unroll
        for (int c = 1; c < NC; ++c) m = fmaxf(m, a[c]);
        m = warp_max(m);
        float z = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int j = c * 32 + lane;
            a[c] = (j < n) ? expf(a[c] - m) : 0.f;
            z += a[c];
        }
        z = warp_sum(z);
#pragma unroll
        for (int c = 0; c < NC; ++c) a[c] = a[c] / z;
    }
}

// Corner decision of one sample (section 6): x = W s_x - 1/2, y = H s_y - 1/2
// in binary32, round-to-nearest, never contracted; four neighbours with
// bilinear weights; a neighbour outside the map gets offset -1.  A location
// with x <= -1 or x >= W (same for y), or a NaN, reads nothing.
struct Corners {
    int off[4];    // element offset of the head slice, -1 when outside
    float w[4];    // bilinear weight (without alpha)
    float lx, ly;  // fractional parts
    bool valid;
};

__device__ __forceinline__ void locate(float sx, float sy, int Hl, int Wl, int start, int H,
                                       int h, Corners& c)
{
    const float fW = (float)Wl, fH = (float)Hl;
    const float x = __fsub_rn(__fmul_rn(fW, sx), 0.5f);
    const float y = __fsub_rn(__fmul_rn(fH, sy), 0.5f);
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        c.off[g] = -1;
        c.w[g] = 0.f;
    }
    c.lx = c.ly = 0.f;
    c.valid = (x > -1.f) && (x < fW) && (y > -1.f) && (y < fH);
    if (c.valid) {
        const float x0f = floorf(x), y0f = floorf(y);
        const float lx = __fsub_rn(x, x0f), ly = __fsub_rn(y, y0f);
        const int x0 = (int)x0f, y0 = (int)y0f;  // x0 in [-1, W-1], y0 in [-1, H-1]
        const float hx = __fsub_rn(1.f, lx), hy = __fsub_rn(1.f, ly);
        c.lx = lx;
        c.ly = ly;
        c.w[0] = __fmul_rn(hx, hy);
        c.w[1] = __fmul_rn(lx, hy);
        c.w[2] = __fmul_rn(hx, ly);
        c.w[3] = __fmul_rn(lx, ly);
        const bool x0in = x0 >= 0, x1in = x0 + 1 < Wl, y0in = y0 >= 0, y1in = y0 + 1 < Hl;
        const int p = start + y0 * Wl + x0;  // pixel of neighbour 0 (used only when inside)
        if (x0in && y0in) c.off[0] = (p * H + h) * kHeadDim;
        if (x1in && y0in) c.off[1] = ((p + 1) * H + h) * kHeadDim;
        if (x0in && y1in) c.off[2] = ((p + Wl) * H + h) * kHeadDim;
        if (x1in && y1in) c.off[3] = ((p + Wl + 1) * H + h) * kHeadDim;
    }
}

// What lane `lane` needs to know about its samples j = c * 32 + lane of every
// row: the sample's level geometry and its anchor m(k) = k mod R.  The same for
// every row and head, so a warp computes it once, before its row loop.
template <int NC>
struct LaneSamples {
    int w[NC], h[NC], start[NC];  // level of sample j (W_l, H_l, first row)
    int m[NC];                    // anchor of point k: k mod R
    bool in[NC];                  // j < L * P
};

template <int NC>
__device__ __forceinline__ void lane_samples(const SmemLevels& lv, int L, int P, int R, int lane,
                                             LaneSamples<NC>& ls)
{
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
        ls.in[c] = j < L * P;
        const int l = ls.in[c] ? j / P : 0;
        const int k = j - l * P;
        ls.w[c] = lv.w[l];
        ls.h[c] = lv.h[l];
        ls.start[c] = lv.start[l];
        ls.m[c] = ls.in[c] ? k % R : 0;
    }
}

// Sampling location of sample j of one (row, head).
// FUSED: rho_{m} + (dx / W_l, dy / H_l), each step one rounded binary32
// operation (section 5); otherwise the given location.
template <bool FUSED>
__device__ __forceinline__ void sample_location(const float* __restrict__ lo,
                                                const float* __restrict__ ref, int j, int m,
                                                int Hl, int Wl, float& sx, float& sy)
{
    const float2 v = ld_stream2(lo + 2 * j);
    if (FUSED) {
        const float2 r = __ldg(reinterpret_cast<const float2*>(ref) + m);
        sx = __fadd_rn(r.x, __fdiv_rn(v.x, (float)Wl));
        sy = __fadd_rn(r.y, __fdiv_rn(v.y, (float)Hl));
    } else {
        sx = v.x;
        sy = v.y;
    }
}

// bf16 pair (packed in 32 bits) -> two floats, exact.
__device__ __forceinline__ void bf16x2_to_f32(uint32_t u, float& lo, float& hi)
{
    lo = __uint_as_float(u << 16);
    hi = __uint_as_float(u & 0xffff0000u);
}

// Gather over the first `cnt` samples of the table; see the file comment for
// the lane layout.  acc: fp32 value -> 4 channels (4t..4t+3) of corner g;
// bf16 value -> 8 channels (8t..8t+7) of corner g for the lane's half.
template <typename VT>
struct Gather;

template <>
struct Gather<float> {
    static constexpr int kAcc = 4;
    // samples base .. base + cnt - 1 of the table (base a multiple of 4)
    __device__ __forceinline__ static void run(const float* __restrict__ vb,
                                               const WarpTable& tab, int cnt, int lane,
                                               float (&acc)[4], int base = 0)
    {
        const int g = lane >> 3, t = lane & 7;
        const float* v = vb + 4 * t;
        const int quads = (cnt + 3) >> 2;
#pragma unroll kGatherUnroll
        for (int p = 0; p < quads; ++p) {
            const int4 o = *reinterpret_cast<const int4*>(&tab.off[g][base + 4 * p]);
            const float4 w = *reinterpret_cast<const float4*>(&tab.w[g][base + 4 * p]);
            float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, x2 = x0, x3 = x0;
            if (o.x >= 0) x0 = __ldg(reinterpret_cast<const float4*>(v + o.x));
            if (o.y >= 0) x1 = __ldg(reinterpret_cast<const float4*>(v + o.y));
            if (o.z >= 0) x2 = __ldg(reinterpret_cast<const float4*>(v + o.z));
            if (o.w >= 0) x3 = __ldg(reinterpret_cast<const float4*>(v + o.w));
            acc[0] += w.x * x0.x + w.y * x1.x + w.z * x2.x + w.w * x3.x;
            acc[1] += w.x * x0.y + w.y * x1.y + w.z * x2.y + w.w * x3.y;
            acc[2] += w.x * x0.z + w.y * x1.z + w.z * x2.z + w.w * x3.z;
            acc[3] += w.x * x0.w + w.y * x1.w + w.z * x2.w + w.w * x3.w;
        }
    }
    // Q quads of the table from `base`, straight-line (entries past the
    // row's samples hold offset -1 and read nothing).
    template <int Q>
    __device__ __forceinline__ static void run_quads(const float* __restrict__ vb,
                                                     const WarpTable& tab, int lane,
                                                     float (&acc)[4], int base)
    {
        const int g = lane >> 3, t = lane & 7;
        const float* v = vb + 4 * t;
#pragma unroll
        for (int p = 0; p < Q; ++p) {
            const int4 o = *reinterpret_cast<const int4*>(&tab.off[g][base + 4 * p]);
            const float4 w = *reinterpret_cast<const float4*>(&tab.w[g][base + 4 * p]);
            float4 x0 = make_float4(0.f, 0.f, 0.f, 0.f), x1 = x0, x2 = x0, x3 = x0;
            if (o.x >= 0) x0 = __ldg(reinterpret_cast<const float4*>(v + o.x));
            if (o.y >= 0) x1 = __ldg(reinterpret_cast<const float4*>(v + o.y));
            if (o.z >= 0) x2 = __ldg(reinterpret_cast<const float4*>(v + o.z));
            if (o.w >= 0) x3 = __ldg(reinterpret_cast<const float4*>(v + o.w));
            acc[0] += w.x * x0.x + w.y * x1.x + w.z * x2.x + w.w * x3.x;
            acc[1] += w.x * x0.y + w.y * x1.y + w.z * x2.y + w.w * x3.y;
            acc[2] += w.x * x0.z + w.y * x1.z + w.z * x2.z + w.w * x3.z;
            acc[3] += w.x * x0.w + w.y * x1.w + w.z * x2.w + w.w * x3.w;
        }
    }
    // Sum the four corners; lanes 0..7 store channels 4t..4t+3.
    __device__ __forceinline__ static void store(float (&acc)[4], int lane, float* __restrict__ out)
    {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
        }
        if (lane < 8)
            *reinterpret_cast<float4*>(out + 4 * lane) = make_float4(acc[0], acc[1], acc[2], acc[3]);
    }
};

template <>
struct Gather<__nv_bfloat16> {
    static constexpr int kAcc = 8;
    __device__ __forceinline__ static void fma8(float (&acc)[8], float w, uint4 r)
    {
#if MSDA_BF16_FFMA2
        // bf16 pair -> fp32 pair (the low half shifted up, the high half
        // masked), then two fused multiply-adds in one fma.rn.f32x2
        const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
            asm("{\n .reg .b32 lo, hi;\n .reg .b64 a, c, w;\n"
                " shl.b32 lo, %2, 16;\n and.b32 hi, %2, 0xffff0000;\n"
                " mov.b64 a, {lo, hi};\n mov.b64 c, {%0, %1};\n mov.b64 w, {%3, %3};\n"
                " fma.rn.f32x2 c, w, a, c;\n mov.b64 {%0, %1}, c;\n}\n"
                : "+f"(acc[2 * i]), "+f"(acc[2 * i + 1])
                : "r"(u[i]), "f"(w));
#else
        float a, b;
        bf16x2_to_f32(r.x, a, b);
        acc[0] += w * a;
        acc[1] += w * b;
        bf16x2_to_f32(r.y, a, b);
        acc[2] += w * a;
        acc[3] += w * b;
        bf16x2_to_f32(r.z, a, b);
        acc[4] += w * a;
        acc[5] += w * b;
        bf16x2_to_f32(r.w, a, b);
        acc[6] += w * a;
        acc[7] += w * b;
#endif
    }
    // samples base .. base + cnt - 1 of the table (base a multiple of 4)
    __device__ __forceinline__ static void run(const __nv_bfloat16* __restrict__ vb,
                                               const WarpTable& tab, int cnt, int lane,
                                               float (&acc)[8], int base = 0)
    {
        const int half = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
        const __nv_bfloat16* v = vb + 8 * t;
        const int quads = (cnt + 3) >> 2;
#pragma unroll kGatherUnroll
        for (int p = 0; p < quads; ++p) {
            const int4 o = *reinterpret_cast<const int4*>(&tab.off[g][base + 4 * p]);
            const float4 w = *reinterpret_cast<const float4*>(&tab.w[g][base + 4 * p]);
            const int oa = half ? o.y : o.x, ob = half ? o.w : o.z;
            const float wa = half ? w.y : w.x, wb = half ? w.w : w.z;
            uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
            if (oa >= 0) ra = __ldg(reinterpret_cast<const uint4*>(v + oa));
            if (ob >= 0) rb = __ldg(reinterpret_cast<const uint4*>(v + ob));
            fma8(acc, wa, ra);
            fma8(acc, wb, rb);
        }
    }
    template <int Q>
    __device__ __forceinline__ static void run_quads(const __nv_bfloat16* __restrict__ vb,
                                                     const WarpTable& tab, int lane,
                                                     float (&acc)[8], int base)
    {
        const int half = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
        const __nv_bfloat16* v = vb + 8 * t;
#pragma unroll
        for (int p = 0; p < Q; ++p) {
            const int4 o = *reinterpret_cast<const int4*>(&tab.off[g][base + 4 * p]);
            const float4 w = *reinterpret_cast<const float4*>(&tab.w[g][base + 4 * p]);
            const int oa = half ? o.y : o.x, ob = half ? o.w : o.z;
            const float wa = half ? w.y : w.x, wb = half ? w.w : w.z;
            uint4 ra = make_uint4(0u, 0u, 0u, 0u), rb = ra;
            if (oa >= 0) ra = __ldg(reinterpret_cast<const uint4*>(v + oa));
            if (ob >= 0) rb = __ldg(reinterpret_cast<const uint4*>(v + ob));
            fma8(acc, wa, ra);
            fma8(acc, wb, rb);
        }
    }
    // Sum corners and halves; lanes 0..3 store channels 8t..8t+7.
    __device__ __forceinline__ static void store(float (&acc)[8], int lane, float* __restrict__ out)
    {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 4);
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
        }
        if (lane < 4) {
            float4* o = reinterpret_cast<float4*>(out + 8 * lane);
            o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
            o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        }
    }
};

// Inputs of one row for HP heads, per lane (samples j = c * 32 + lane): the
// logits (or weights), the pixel offsets (or locations) and, fused, the
// reference point of the sample's anchor.  Loaded one row ahead of their use
// so that their memory latency overlaps the previous row's gather.
template <bool FUSED, int NC, int HP>
struct RowIn {
    float a[HP][NC];
    float2 lo[HP][NC];
    float2 rf[NC];
};

// lo, wl: the row's first head; head s follows at +2 s n (lo) and +s n (wl).
template <bool FUSED, int NC, int HP>
__device__ __forceinline__ void load_row(const float* __restrict__ lo,
                                         const float* __restrict__ wl,
                                         const float* __restrict__ ref, int n,
                                         const LaneSamples<NC>& ls, int lane,
                                         RowIn<FUSED, NC, HP>& in)
{
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int j = c * 32 + lane;
#pragma unroll
        for (int s = 0; s < HP; ++s) {
            in.a[s][c] = ls.in[c] ? ld_stream(wl + s * n + j) : (FUSED ? -INFINITY : 0.f);
            in.lo[s][c] = ls.in[c] ? ld_stream2(lo + s * 2 * n + 2 * j) : make_float2(0.f, 0.f);
        }
        in.rf[c] = (FUSED && ls.in[c]) ? __ldg(reinterpret_cast<const float2*>(ref) + ls.m[c])
                                       : make_float2(0.f, 0.f);
    }
}

// Softmax over the L*P logits of one head, in place (section 4.2).
template <bool FUSED, int NC>
__device__ __forceinline__ void normalise(float (&a)[NC], const LaneSamples<NC>& ls)
{
    if (!FUSED) return;
    float m = a[0];
#pragma unroll
    for (int c = 1; c < NC; ++c) m = fmaxf(m, a[c]);
    m = warp_max(m);
    float z = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        a[c] = ls.in[c] ? expf(a[c] - m) : 0.f;
        z += a[c];
    }
    z = warp_sum(z);
#pragma unroll
    for (int c = 0; c < NC; ++c) a[c] = a[c] / z;
}

// Corners of the lane's sample of chunk c, head h (section 5 location, section
// 6 corner decision).
template <bool FUSED, int NC>
__device__ __forceinline__ void lane_corners(float2 v, float2 r, const LaneSamples<NC>& ls, int c,
                                             int H, int h, Corners& cr)
{
    if (ls.in[c]) {
        float sx = v.x, sy = v.y;
        if (FUSED) {
            sx = __fadd_rn(r.x, __fdiv_rn(v.x, (float)ls.w[c]));
            sy = __fadd_rn(r.y, __fdiv_rn(v.y, (float)ls.h[c]));
        }
        locate(sx, sy, ls.h[c], ls.w[c], ls.start[c], H, h, cr);
    } else {
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            cr.off[g] = -1;
            cr.w[g] = 0.f;
        }
    }
}

// One head of one row (all n = L*P samples) from its normalised weights a,
// offsets (or locations) lo and reference points rf, added to the lane's
// partial sums acc (corners not yet reduced: Gather::store does that).
// vb: value of this batch item (and camera), [Nv, H, 32].
template <typename VT, bool FUSED, int NC>
__device__ __forceinline__ void head_gather(const VT* __restrict__ vb, int H, int h,
                                            const float (&a)[NC], const float2 (&lo)[NC],
                                            const float2 (&rf)[NC], int n,
                                            const LaneSamples<NC>& ls, WarpTable& tab,
                                            float (&acc)[Gather<VT>::kAcc], int lane)
{
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        Corners cr;
        lane_corners<FUSED, NC>(lo[c], rf[c], ls, c, H, h, cr);
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            tab.off[g][lane] = cr.off[g];
            tab.w[g][lane] = cr.w[g] * a[c];
        }
        __syncwarp();
        Gather<VT>::run(vb, tab, min(32, n - c * 32), lane, acc);
        __syncwarp();
    }
}

// head_gather after the softmax of the row's logits (in place).
template <typename VT, bool FUSED, int NC>
__device__ __forceinline__ void row_accumulate(const VT* __restrict__ vb, int H, int h,
                                               RowIn<FUSED, NC, 1>& in, int n,
                                               const LaneSamples<NC>& ls, WarpTable& tab,
                                               float (&acc)[Gather<VT>::kAcc], int lane)
{
    normalise<FUSED, NC>(in.a[0], ls);
    head_gather<VT, FUSED, NC>(vb, H, h, in.a[0], in.lo[0], in.rf, n, ls, tab, acc, lane);
}

// One output row of one head, written to out_row[0..32).
template <typename VT, bool FUSED, int NC>
__device__ __forceinline__ void row_compute(const VT* __restrict__ vb, int H, int h,
                                            RowIn<FUSED, NC, 1>& in, int n,
                                            const LaneSamples<NC>& ls, WarpTable& tab,
                                            float* __restrict__ out_row, int lane)
{
    float acc[Gather<VT>::kAcc];
#pragma unroll
    for (int i = 0; i < Gather<VT>::kAcc; ++i) acc[i] = 0.f;
    row_accumulate<VT, FUSED, NC>(vb, H, h, in, n, ls, tab, acc, lane);
    Gather<VT>::store(acc, lane, out_row);
}

// bf16 value, two heads per warp.  A bf16 head slice is 64 bytes, and every
// slice of head h sits in the same half of its 128-byte line ((h * 64) mod
// 128), so four corners of one head always collide on the same L1 banks.
// Pairing heads 2m and 2m+1 in one warp puts the two halves of every warp load
// on opposite bank halves: lanes 16s + 4g + t read corner g of a sample of
// head 2m + s, channels 8t..8t+7.
struct PairTable {
    int off[2][4][kMetaStride];
    float w[2][4][kMetaStride];
};

// Heads h0 and h0 + 1 of one row from normalised weights, added to the
// lane's partial sums (see pair_store for the lane layout).
template <bool FUSED, int NC>
__device__ __forceinline__ void pair_gather(const __nv_bfloat16* __restrict__ vb, int H, int h0,
                                            const RowIn<FUSED, NC, 2>& in,
                                            const float2 (&rf)[NC], int n,
                                            const LaneSamples<NC>& ls, PairTable& tab,
                                            float (&acc)[8], int lane)
{
    const int half = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
    const __nv_bfloat16* v = vb + 8 * t;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
#pragma unroll
        for (int sh = 0; sh < 2; ++sh) {
            Corners cr;
            lane_corners<FUSED, NC>(in.lo[sh][c], rf[c], ls, c, H, h0 + sh, cr);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                tab.off[sh][q][lane] = cr.off[q];
                tab.w[sh][q][lane] = cr.w[q] * in.a[sh][c];
            }
        }
        __syncwarp();
        const int quads = (min(32, n - c * 32) + 3) >> 2;
#pragma unroll kPairUnroll
        for (int p = 0; p < quads; ++p) {
            const int4 o = *reinterpret_cast<const int4*>(&tab.off[half][g][4 * p]);
            const float4 w = *reinterpret_cast<const float4*>(&tab.w[half][g][4 * p]);
            uint4 r0 = make_uint4(0u, 0u, 0u, 0u), r1 = r0, r2 = r0, r3 = r0;
            if (o.x >= 0) r0 = __ldg(reinterpret_cast<const uint4*>(v + o.x));
            if (o.y >= 0) r1 = __ldg(reinterpret_cast<const uint4*>(v + o.y));
            if (o.z >= 0) r2 = __ldg(reinterpret_cast<const uint4*>(v + o.z));
            if (o.w >= 0) r3 = __ldg(reinterpret_cast<const uint4*>(v + o.w));
            Gather<__nv_bfloat16>::fma8(acc, w.x, r0);
            Gather<__nv_bfloat16>::fma8(acc, w.y, r1);
            Gather<__nv_bfloat16>::fma8(acc, w.z, r2);
            Gather<__nv_bfloat16>::fma8(acc, w.w, r3);
        }
        __syncwarp();
    }
}

// Sum the four corners; lanes 16s + t (g = 0) store head h0 + s, channels
// 8t..8t+7; out_row0 is head h0's output, head h0 + 1 follows at +32.
__device__ __forceinline__ void pair_store(float (&acc)[8], int lane, float* __restrict__ out_row0)
{
    const int half = lane >> 4, g = (lane >> 2) & 3, t = lane & 3;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 4);
        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
    }
    if (g == 0) {
        float4* o = reinterpret_cast<float4*>(out_row0 + half * kHeadDim + 8 * t);
        o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    }
}

// Heads h0 and h0 + 1 of one row; out_row0 is head h0's output, head h0 + 1
// follows at +32.
template <bool FUSED, int NC>
__device__ __forceinline__ void row_compute_pair(const __nv_bfloat16* __restrict__ vb, int H,
                                                 int h0, RowIn<FUSED, NC, 2>& in, int n,
                                                 const LaneSamples<NC>& ls, PairTable& tab,
                                                 float* __restrict__ out_row0, int lane)
{
    normalise<FUSED, NC>(in.a[0], ls);
    normalise<FUSED, NC>(in.a[1], ls);
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    pair_gather<FUSED, NC>(vb, H, h0, in, in.rf, n, ls, tab, acc, lane);
    pair_store(acc, lane, out_row0);
}

// Rows with few samples (L*P <= 16): one warp serves G heads of a row at
// once.  Lane j handles sample k = j mod npad of head h0 + j / npad, where
// npad is L*P rounded up to a power of two (at least 4, so that every head's
// samples start on a quad of the table) and G = 32 / npad.  The softmax is a
// segmented reduction over each head's npad lanes; the gather then walks the
// heads' table segments one after the other.
struct GroupLane {
    int npad_log2;  // log2(npad)
    int s, k;       // head within the group, sample within the head
    bool in;        // k < L * P
    int w, h, start, m;
};

__device__ __forceinline__ void group_lane(const SmemLevels& lv, int L, int P, int R, int npad_log2,
                                           int lane, GroupLane& gl)
{
    gl.npad_log2 = npad_log2;
    gl.s = lane >> npad_log2;
    gl.k = lane & ((1 << npad_log2) - 1);
    gl.in = gl.k < L * P;
    const int l = gl.in ? gl.k / P : 0;
    const int kk = gl.k - l * P;
    gl.w = lv.w[l];
    gl.h = lv.h[l];
    gl.start = lv.start[l];
    gl.m = gl.in ? kk % R : 0;
}

__device__ __forceinline__ float segment_max(float v, int npad)
{
    for (int o = npad >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float segment_sum(float v, int npad)
{
    for (int o = npad >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// The table of one row for heads h0 .. h0 + G - 1: softmax of each head's
// segment, locations and corners.  The lane's inputs come preloaded in
// (a, v, r); `valid` = the lane's sample exists.  The caller syncs the warp
// before reading the table.
template <bool FUSED>
__device__ __forceinline__ void group_table(int H, int h0, float a, float2 v, float2 r, bool valid,
                                            const GroupLane& gl, WarpTable& tab, int lane)
{
    const int npad = 1 << gl.npad_log2;
    if (FUSED) {
        const float m = segment_max(a, npad);
        const float e = valid ? expf(a - m) : 0.f;
        const float z = segment_sum(e, npad);
        a = valid ? e / z : 0.f;
    } else if (!valid) {
        a = 0.f;
    }
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
    }
#pragma unroll
    for (int g = 0; g < 4; ++g) {
        tab.off[g][lane] = cr.off[g];
        tab.w[g][lane] = cr.w[g] * a;
    }
}

// One row, heads h0 .. h0 + G - 1 (those < H), from the lane's preloaded
// inputs (see group_table); out_row0: head h0's output (+32 per head).
template <typename VT, bool FUSED, int NPL>
__device__ __forceinline__ void group_compute(const VT* __restrict__ vb, int H, int h0, float a,
                                              float2 v, float2 r, bool valid,
                                              const GroupLane& gl, WarpTable& tab,
                                              float* __restrict__ out_row0, int lane)
{
    constexpr int G = 32 >> NPL;
    group_table<FUSED>(H, h0, a, v, r, valid, gl, tab, lane);
    __syncwarp();
    const int nheads = min(G, H - h0);
    for (int s = 0; s < nheads; ++s) {
        float acc[Gather<VT>::kAcc];
#pragma unroll
        for (int i = 0; i < Gather<VT>::kAcc; ++i) acc[i] = 0.f;
        Gather<VT>::template run_quads<(1 << NPL) / 4>(vb, tab, lane, acc, s << NPL);
        Gather<VT>::store(acc, lane, out_row0 + s * kHeadDim);
    }
    __syncwarp();
}

// Walks the (row, head) items of one warp without divisions: items are
// row * H + h, a warp takes every kWarps-th item of its CTA's tile of
// `rows` consecutive rows, so each step adds kWarps / H rows and
// kWarps % H heads (with a carry).
struct ItemCursor {
    int rr, h;        // row within the tile, head
    int drr, dh, H;
    __device__ __forceinline__ ItemCursor(int warp, int H_) : H(H_)
    {
        rr = warp / H;
        h = warp - rr * H;
        drr = kWarps / H;
        dh = kWarps - drr * H;
    }
    __device__ __forceinline__ void next()
    {
        rr += drr;
        h += dh;
        if (h >= H) {
            h -= H;
            ++rr;
        }
    }
};

// Row offsets of the rebatched layout: s_prefix[bc] = sum of count[0..bc),
// s_prefix[n] = total rows.  Each count is clamped to [0, cap] (cap = Nq, the
// capacity of a (batch, camera) block of rows), so inconsistent counts never
// address rows outside their block.  Warp 0 scans; the whole block must call
// this.
__device__ __forceinline__ void stage_row_prefix(const int32_t* __restrict__ count, int n, int cap,
                                                 int* s_prefix)
{
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int run = 0;
        for (int base = 0; base < n; base += 32) {
            const int v = (base + lane < n) ? min(max(__ldg(count + base + lane), 0), cap) : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            if (base + lane < n) s_prefix[base + lane] = run + incl - v;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) s_prefix[n] = run;
    }
    __syncthreads();
}

// Largest bc in [0, n) with prefix[bc] <= r, given prefix[n] > r.
__device__ __forceinline__ int find_segment(const int* prefix, int n, int r)
{
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (prefix[mid] <= r) lo = mid;
        else hi = mid;
    }
    return lo;
}

}  // namespace msda
