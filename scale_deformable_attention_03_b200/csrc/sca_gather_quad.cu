// K3 for rows of up to 32 samples: the rebatched SCA gather with four lanes
// per (row, head) ("BEV(三) BEVFormer: how the Query interacts with the 8
// Heads of the Feature", sections 4.2-9; Tencent Cloud "Spatial
// Cross-Attention" walkthrough, rebatch listing).
//
// Lane layout.  A warp serves eight (row, head) items at once: lanes
// 4u .. 4u + 3 (a "quad") own item u and channels 8t .. 8t + 7 of it
// (t = lane mod 4).  With H = 8 the eight items are the eight heads of one
// row, so the warp reads the row's logits and offsets as one contiguous block
// and writes the row's 256 output channels as one contiguous 1 KiB store.
//   - Before the row, lane t of a quad forms the softmax weight and the
//     sampling location of its samples j = 8t .. 8t + 7 (one IEEE division
//     per coordinate, as the oracle's binary32 steps).
//   - Sample by sample, the quad takes (alpha, s_x, s_y) of sample j from the
//     lane that formed it (three shuffles inside the quad), decides the four
//     corners itself (every lane of the quad the same way, so no table and no
//     warp barrier), and reads each corner's head slice with one load per
//     lane: 32 bytes (fp32, channels 8t .. 8t + 7) or 16 bytes (bf16).  One
//     warp load then covers eight corner slices of eight different heads,
//     whole 128-byte lines for fp32.
//   - Each lane accumulates its own eight channels over all samples; nothing
//     is reduced across lanes at the end of the row.
// Compared with one warp per (row, head) and a shared-memory sample table,
// this removes the table's stores and loads, the warp barriers and the final
// corner reduction: the L1 data path carries the corner reads and little else.
#include <algorithm>

#include "msda_launch.h"

namespace msda {

#ifndef MSDA_QUAD_MIN_CTAS_F32
#define MSDA_QUAD_MIN_CTAS_F32 3
#endif
#ifndef MSDA_QUAD_MIN_CTAS_BF16
#define MSDA_QUAD_MIN_CTAS_BF16 0
#endif
#ifndef MSDA_QUAD_FFMA2
#define MSDA_QUAD_FFMA2 1  // fp32 value: the corner adds as packed fp32x2 FMAs
#endif
#ifndef MSDA_QUAD_PREFETCH
#define MSDA_QUAD_PREFETCH 0  // 1: load the next tile's logits and offsets during this tile
#endif

namespace {

constexpr int kQuadSamples = 32;  // samples per row this kernel serves

// Per value type: one corner slice per lane (8 channels) and its weighted add.
template <typename VT>
struct QuadCorner;

template <>
struct QuadCorner<float> {
    struct Raw {
        float v[8];
    };
    __device__ __forceinline__ static void zero(Raw& r)
    {
#pragma unroll
        for (int e = 0; e < 8; ++e) r.v[e] = 0.f;
    }
    // 32 bytes in one 256-bit load (read-only path); NA: not allocated in L1.
    template <bool NA>
    __device__ __forceinline__ static void load(const float* p, Raw& r)
    {
        if constexpr (NA)
            asm volatile("ld.global.nc.L1::no_allocate.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=f"(r.v[0]), "=f"(r.v[1]), "=f"(r.v[2]), "=f"(r.v[3]), "=f"(r.v[4]),
                           "=f"(r.v[5]), "=f"(r.v[6]), "=f"(r.v[7])
                         : "l"(p));
        else
            asm volatile("ld.global.nc.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=f"(r.v[0]), "=f"(r.v[1]), "=f"(r.v[2]), "=f"(r.v[3]), "=f"(r.v[4]),
                           "=f"(r.v[5]), "=f"(r.v[6]), "=f"(r.v[7])
                         : "l"(p));
    }
    __device__ __forceinline__ static void fma(float (&acc)[8], float w, const Raw& r)
    {
#if MSDA_QUAD_FFMA2
        // two channels per instruction: fma.rn.f32x2 is two IEEE fp32 fused
        // multiply-adds, the same results as fmaf on each
#pragma unroll
        for (int e = 0; e < 8; e += 2)
            asm("{\n .reg .b64 a, c, w;\n"
                " mov.b64 a, {%2, %3};\n mov.b64 c, {%0, %1};\n mov.b64 w, {%4, %4};\n"
                " fma.rn.f32x2 c, w, a, c;\n mov.b64 {%0, %1}, c;\n}\n"
                : "+f"(acc[e]), "+f"(acc[e + 1])
                : "f"(r.v[e]), "f"(r.v[e + 1]), "f"(w));
#else
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = fmaf(w, r.v[e], acc[e]);
#endif
    }
};

template <>
struct QuadCorner<__nv_bfloat16> {
    struct Raw {
        uint4 u;
    };
    __device__ __forceinline__ static void zero(Raw& r) { r.u = make_uint4(0u, 0u, 0u, 0u); }
    template <bool NA>
    __device__ __forceinline__ static void load(const __nv_bfloat16* p, Raw& r)
    {
        if constexpr (NA)
            asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(r.u.x), "=r"(r.u.y), "=r"(r.u.z), "=r"(r.u.w)
                         : "l"(p));
        else
            r.u = __ldg(reinterpret_cast<const uint4*>(p));
    }
    __device__ __forceinline__ static void fma(float (&acc)[8], float w, const Raw& r)
    {
        float a, b;
        bf16x2_to_f32(r.u.x, a, b);
        acc[0] = fmaf(w, a, acc[0]);
        acc[1] = fmaf(w, b, acc[1]);
        bf16x2_to_f32(r.u.y, a, b);
        acc[2] = fmaf(w, a, acc[2]);
        acc[3] = fmaf(w, b, acc[3]);
        bf16x2_to_f32(r.u.z, a, b);
        acc[4] = fmaf(w, a, acc[4]);
        acc[5] = fmaf(w, b, acc[5]);
        bf16x2_to_f32(r.u.w, a, b);
        acc[6] = fmaf(w, a, acc[6]);
        acc[7] = fmaf(w, b, acc[7]);
    }
};

// Level geometry and anchor of sample j, stored at j + j / 8 so that the
// four lanes of a quad (samples 8t + r) read four different bank groups.
struct __align__(16) QuadMeta {
    int w, h, start, m;
};

// The finest MSDA_QUAD_NOALLOC_LEVELS levels read their corners without
// allocating in L1: those slices are rarely met again, and L1 is left to the
// coarse levels, whose slices neighbouring rows read again.
#ifndef MSDA_QUAD_NOALLOC_LEVELS
#define MSDA_QUAD_NOALLOC_LEVELS 3
#endif
constexpr int kQuadMetaSlots = kQuadSamples + kQuadSamples / 8;

__device__ __forceinline__ int quad_meta_slot(int j) { return j + (j >> 3); }

// One sample of a quad: corner decision ("BEV(三)..." section 6: x = W s_x -
// 1/2, binary32, never contracted; a neighbour outside the map reads
// nothing), then the four corner reads weighted by alpha * w_g.
template <typename VT, bool NA>
__device__ __forceinline__ void quad_sample(const VT* __restrict__ vb, int H, int h, int t,
                                            float alpha, float sx, float sy, const QuadMeta& mt,
                                            float (&acc)[8])
{
    using C = QuadCorner<VT>;
    const float fW = (float)mt.w, fH = (float)mt.h;
    const float x = __fsub_rn(__fmul_rn(fW, sx), 0.5f);
    const float y = __fsub_rn(__fmul_rn(fH, sy), 0.5f);
    const bool valid = (x > -1.f) && (x < fW) && (y > -1.f) && (y < fH);
    // outside (or NaN): finite zero fractions, so the zero corners add nothing
    const float x0f = floorf(valid ? x : 0.f), y0f = floorf(valid ? y : 0.f);
    const float lx = valid ? __fsub_rn(x, x0f) : 0.f, ly = valid ? __fsub_rn(y, y0f) : 0.f;
    const float hx = __fsub_rn(1.f, lx), hy = __fsub_rn(1.f, ly);
    const int x0 = (int)x0f, y0 = (int)y0f;
    const bool x0in = valid && x0 >= 0, x1in = valid && x0 + 1 < mt.w;
    const bool y0in = valid && y0 >= 0, y1in = valid && y0 + 1 < mt.h;
    const int pix = H * kHeadDim;  // elements per pixel
    const int base = ((mt.start + y0 * mt.w + x0) * H + h) * kHeadDim + 8 * t;
    typename C::Raw r0, r1, r2, r3;
    C::zero(r0);
    C::zero(r1);
    C::zero(r2);
    C::zero(r3);
    if (x0in && y0in) C::template load<NA>(vb + base, r0);
    if (x1in && y0in) C::template load<NA>(vb + base + pix, r1);
    if (x0in && y1in) C::template load<NA>(vb + base + mt.w * pix, r2);
    if (x1in && y1in) C::template load<NA>(vb + base + (mt.w + 1) * pix, r3);
    C::fma(acc, __fmul_rn(__fmul_rn(hx, hy), alpha), r0);
    C::fma(acc, __fmul_rn(__fmul_rn(lx, hy), alpha), r1);
    C::fma(acc, __fmul_rn(__fmul_rn(hx, ly), alpha), r2);
    C::fma(acc, __fmul_rn(__fmul_rn(lx, ly), alpha), r3);
}

// Inputs of one item for lane t of its quad: samples 8t .. 8t + 7.
struct QuadIn {
    float a[8];   // logits, then softmax weights
    float x[8];   // offsets (dx), then locations s_x
    float y[8];   // offsets (dy), then locations s_y
};

// Loads the logits and pixel offsets of samples 8t .. 8t + 7 of one
// (query, head); n = L * P samples, missing ones get -inf / 0.  vec: rows of
// 32 samples with 16-byte aligned logits and offsets, read as vectors.
__device__ __forceinline__ void quad_load(const float* __restrict__ lg,
                                          const float* __restrict__ of, int n, int t, bool live,
                                          bool vec, QuadIn& in)
{
    const int j0 = 8 * t;
    if (live && vec) {
        const float4 a0 = __ldcs(reinterpret_cast<const float4*>(lg + j0));
        const float4 a1 = __ldcs(reinterpret_cast<const float4*>(lg + j0 + 4));
        in.a[0] = a0.x; in.a[1] = a0.y; in.a[2] = a0.z; in.a[3] = a0.w;
        in.a[4] = a1.x; in.a[5] = a1.y; in.a[6] = a1.z; in.a[7] = a1.w;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float4 o = __ldcs(reinterpret_cast<const float4*>(of + 2 * j0 + 4 * k));
            in.x[2 * k] = o.x;
            in.y[2 * k] = o.y;
            in.x[2 * k + 1] = o.z;
            in.y[2 * k + 1] = o.w;
        }
        return;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int j = j0 + r;
        const bool in_row = live && j < n;
        in.a[r] = in_row ? __ldcs(lg + j) : -INFINITY;
        const float2 o = in_row ? __ldcs(reinterpret_cast<const float2*>(of) + j)
                                : make_float2(0.f, 0.f);
        in.x[r] = o.x;
        in.y[r] = o.y;
    }
}

// Softmax over the item's n logits (section 4.2: max-subtracted, each head
// its own L * P logits), in place; lanes of dead items get alpha = 0.
__device__ __forceinline__ void quad_softmax(float (&a)[8], int n, int t, bool live)
{
    float m = -INFINITY;
#pragma unroll
    for (int r = 0; r < 8; ++r) m = fmaxf(m, a[r]);
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
    float z = 0.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int j = 8 * t + r;
        a[r] = (live && j < n) ? expf(a[r] - m) : 0.f;
        z += a[r];
    }
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    const float zi = live ? z : 1.f;
#pragma unroll
    for (int r = 0; r < 8; ++r) a[r] = a[r] / zi;
}

// Offsets in level pixels -> normalised offsets dx / W_l, dy / H_l (one IEEE
// division each, section 5), in place.
__device__ __forceinline__ void quad_scale_offsets(float (&x)[8], float (&y)[8],
                                                   const QuadMeta* s_meta, int n, int t, bool live)
{
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int j = 8 * t + r;
        if (live && j < n) {
            const QuadMeta mt = s_meta[quad_meta_slot(j)];
            x[r] = __fdiv_rn(x[r], (float)mt.w);
            y[r] = __fdiv_rn(y[r], (float)mt.h);
        }
    }
}

// Sampling locations rho_m + (dx / W_l, dy / H_l) of the lane's samples from
// the normalised offsets and one reference-point row rf [R, 2]; samples that
// do not exist (or dead items) get NaN, which reads nothing.
__device__ __forceinline__ void quad_locations(const float (&nx)[8], const float (&ny)[8],
                                               float (&sx)[8], float (&sy)[8],
                                               const QuadMeta* s_meta,
                                               const float* __restrict__ rf, int n, int t,
                                               bool live)
{
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int j = 8 * t + r;
        if (live && j < n) {
            const QuadMeta mt = s_meta[quad_meta_slot(j)];
            const float2 ref = __ldg(reinterpret_cast<const float2*>(rf) + mt.m);
            sx[r] = __fadd_rn(ref.x, nx[r]);
            sy[r] = __fadd_rn(ref.y, ny[r]);
        } else {
            sx[r] = __int_as_float(0x7fffffff);  // NaN: no corner is read
            sy[r] = sx[r];
        }
    }
}

// Softmax weights and sampling locations of one rebatched row, in place.
__device__ __forceinline__ void quad_prepare(QuadIn& in, const QuadMeta* s_meta,
                                             const float* __restrict__ rf, int n, int t, bool live)
{
    quad_softmax(in.a, n, t, live);
    quad_scale_offsets(in.x, in.y, s_meta, n, t, live);
    quad_locations(in.x, in.y, in.x, in.y, s_meta, rf, n, t, live);
}

// Samples whose corner loads are issued together (a power of two <= 8).
#ifndef MSDA_QUAD_STEP_F32
#define MSDA_QUAD_STEP_F32 1
#endif
#ifndef MSDA_QUAD_STEP_BF16
#define MSDA_QUAD_STEP_BF16 4
#endif
template <typename VT>
struct QuadStep {
    static constexpr int kSamples = sizeof(VT) == 4 ? MSDA_QUAD_STEP_F32 : MSDA_QUAD_STEP_BF16;
};

// 1: the quads keep their samples' (alpha, s_x, s_y) in shared memory and
// read them there in the corner loop (no registers held, no shuffles).
#ifndef MSDA_QUAD_SMEM
#define MSDA_QUAD_SMEM 0
#endif
constexpr int kQuadSmemStride = kQuadSamples + 1;  // quads u of a warp on distinct banks

template <typename VT>
struct QuadBounds {
    static constexpr int kMin = sizeof(VT) == 4 ? MSDA_QUAD_MIN_CTAS_F32 : MSDA_QUAD_MIN_CTAS_BF16;
};

// The corner loop of one item from the warp's shared-memory copy of its
// quads' samples: sa, sx, sy point at this quad's row of 32 (+1) entries.
template <typename VT>
__device__ __forceinline__ void quad_gather_smem(const VT* __restrict__ vb, int H, int h, int t,
                                                 int n, int P, const float* sa, const float* sx,
                                                 const float* sy, const QuadMeta* s_meta,
                                                 float (&acc)[8])
{
    constexpr int kStep = QuadStep<VT>::kSamples;
    const int na_samples = min(n, MSDA_QUAD_NOALLOC_LEVELS * P);
#pragma unroll kStep
    for (int j = 0; j < na_samples; ++j)
        quad_sample<VT, true>(vb, H, h, t, sa[j], sx[j], sy[j], s_meta[quad_meta_slot(j)], acc);
#pragma unroll kStep
    for (int j = na_samples; j < n; ++j)
        quad_sample<VT, false>(vb, H, h, t, sa[j], sx[j], sy[j], s_meta[quad_meta_slot(j)], acc);
}

// The corner loop of one item: every sample j of the quad's item, taken from
// register j mod 8 of quad lane j / 8 (alpha, s_x, s_y), added into acc.
template <typename VT, bool NA>
__device__ __forceinline__ void quad_gather_range(const VT* __restrict__ vb, int H, int h, int t,
                                                  int src0, int src1, const float (&a)[8],
                                                  const float (&x)[8], const float (&y)[8],
                                                  const QuadMeta* s_meta, float (&acc)[8])
{
    // The register index must be a constant, so r is the unrolled outer
    // loop; each pass of the inner loop handles kStep samples (their corner
    // loads in flight together).
    constexpr int kStep = QuadStep<VT>::kSamples;
#pragma unroll
    for (int r0 = 0; r0 < 8; r0 += kStep) {
#pragma unroll 1
        for (int src = src0; src < src1; ++src) {
#pragma unroll
            for (int r = r0; r < r0 + kStep; ++r) {
                const float al = __shfl_sync(0xffffffffu, a[r], src, 4);
                const float sx = __shfl_sync(0xffffffffu, x[r], src, 4);
                const float sy = __shfl_sync(0xffffffffu, y[r], src, 4);
                const QuadMeta mt = s_meta[quad_meta_slot(8 * src + r)];
                quad_sample<VT, NA>(vb, H, h, t, al, sx, sy, mt, acc);
            }
        }
    }
}

// Groups of eight samples wholly inside the finest MSDA_QUAD_NOALLOC_LEVELS
// levels (the row's first NOALLOC * P samples) load without allocating in L1.
template <typename VT>
__device__ __forceinline__ void quad_gather(const VT* __restrict__ vb, int H, int h, int t, int n,
                                            int P, const float (&a)[8], const float (&x)[8],
                                            const float (&y)[8], const QuadMeta* s_meta,
                                            float (&acc)[8])
{
    const int quads_of_8 = (n + 7) >> 3;
    const int na_groups = min(quads_of_8, (MSDA_QUAD_NOALLOC_LEVELS * P) >> 3);
    quad_gather_range<VT, true>(vb, H, h, t, 0, na_groups, a, x, y, s_meta, acc);
    quad_gather_range<VT, false>(vb, H, h, t, na_groups, quads_of_8, a, x, y, s_meta, acc);
}

}  // namespace

// Rows are ordered (b, c, i) as in sca_gather_kernel; warp w of CTA k takes
// the warp tiles (eight consecutive (row, head) items) w + kWarps * (k + j *
// gridDim.x), so at any moment the GPU works on a narrow window of rows of
// one camera.  The next tile's logits and offsets are loaded before the
// current tile's corner loop.
template <typename VT>
__global__ void __launch_bounds__(kThreads, QuadBounds<VT>::kMin)
sca_gather_quad_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                       const float* __restrict__ logits, const float* __restrict__ ref_cam,
                       const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                       float* __restrict__ out_rb, int B, int Ncam, int Nq, int Nv, int H, int L,
                       int P, int R, Levels levels, bool vec)
{
    __shared__ QuadMeta s_meta[kQuadMetaSlots];
    __shared__ int s_prefix[kMaxBatchCameras + 1];
    __shared__ float s_in[MSDA_QUAD_SMEM ? kWarps : 1][3][8][kQuadSmemStride];
    const int n = L * P;
    if (threadIdx.x < kQuadSamples) {
        const int j = threadIdx.x;
        QuadMeta mt{1, 1, 0, 0};
        if (j < n) {
            const int l = j / P, k = j - l * P;
#pragma unroll
            for (int i = 0; i < kMaxLevels; ++i)  // constant indices: Levels stays in registers
                if (i == l) mt = QuadMeta{levels.w[i], levels.h[i], levels.start[i], k % R};
        }
        s_meta[quad_meta_slot(j)] = mt;
    }
    const int nbc = B * Ncam;
    pdl_trigger();  // the average pass reads the rows only after its pdl_wait
    pdl_wait();     // the compaction lists are complete
    stage_row_prefix(count, nbc, Nq, s_prefix);  // block barrier: s_meta is visible after it

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int u = lane >> 2, t = lane & 3;
#ifndef MSDA_QUAD_HEADSPEC
#define MSDA_QUAD_HEADSPEC 0  // 1: a CTA tile is 64 rows of one head (grid a multiple of H)
#endif
    const int total_rows = s_prefix[nbc];
    const int64_t n_items = (int64_t)total_rows * H;
    const int64_t n_tiles = MSDA_QUAD_HEADSPEC
                                ? (((int64_t)total_rows + kWarps * 8 - 1) / (kWarps * 8)) * H * kWarps
                                : (n_items + 7) >> 3;
    const int64_t stride = (int64_t)gridDim.x * kWarps;
    int bc = 0;  // this quad's (batch, camera): its rows only grow

    struct Item {
        bool live;
        int h, bc, out_row, ref_row;
        const float* lg;
        const float* of;
    };
    auto resolve = [&](int64_t tile) {
        Item it{false, 0, 0, 0, 0, logits, off};
#if MSDA_QUAD_HEADSPEC
        const int64_t X = tile / kWarps;
        const int64_t row64 = (X / H) * (kWarps * 8) + (tile - X * kWarps) * 8 + u;
        if (tile < n_tiles && row64 < total_rows) {
            const int row = (int)row64;
            it.h = (int)(X % H);
#else
        const int64_t item = tile * 8 + u;
        if (tile < n_tiles && item < n_items) {
            const int row = (int)(item / H);
            it.h = (int)(item - (int64_t)row * H);
#endif
            while (row >= s_prefix[bc + 1]) ++bc;
            const int i = row - s_prefix[bc];
            const int b = bc / Ncam, c = bc - b * Ncam;
            const int q = __ldg(idx + (int64_t)bc * Nq + i);
            if ((unsigned)q < (unsigned)Nq) {  // inconsistent lists: read and write nothing
                it.live = true;
                it.bc = bc;
                it.out_row = bc * Nq + i;
                it.ref_row = (c * B + b) * Nq + q;
                const int64_t qh = ((int64_t)b * Nq + q) * H + it.h;
                it.lg = logits + qh * n;
                it.of = off + qh * 2 * n;
            }
        }
        return it;
    };

#ifndef MSDA_QUAD_CHUNK
#define MSDA_QUAD_CHUNK 1  // consecutive warp-tile groups per CTA within each window
#endif
    // CTA k takes kChunk consecutive groups of kWarps warp tiles, then skips
    // to its groups in the next window of gridDim.x * kChunk groups
    constexpr int kChunk = MSDA_QUAD_CHUNK;
    auto advance = [&](int64_t t0) {
        const int64_t g = t0 / kWarps;  // the group (kWarps consecutive tiles) of t0
        return ((g + 1) % kChunk) ? t0 + kWarps
                                  : t0 + kWarps + (int64_t)(gridDim.x - 1) * kChunk * kWarps;
    };
    (void)stride;
    // with out_rb on 32 bytes, each lane's eight output channels are too
    const bool out32 = ((uintptr_t)out_rb & 31) == 0;
    int64_t tile = (int64_t)blockIdx.x * kChunk * kWarps + warp;
    if (tile >= n_tiles) return;  // warp-uniform
    Item cur = resolve(tile);
    QuadIn in;
    quad_load(cur.lg, cur.of, n, t, cur.live, vec, in);
    while (true) {
        const int64_t next_tile = advance(tile);
#if MSDA_QUAD_PREFETCH
        const Item nxt = resolve(next_tile);
        QuadIn in_next;
        quad_load(nxt.lg, nxt.of, n, t, nxt.live, vec, in_next);  // in flight during this tile
#endif

        quad_prepare(in, s_meta, ref_cam + (int64_t)cur.ref_row * R * 2, n, t, cur.live);
        const VT* vb = value + (int64_t)cur.bc * Nv * H * kHeadDim;
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#if MSDA_QUAD_SMEM
        {
            float* sa = s_in[warp][0][u];
            float* sx = s_in[warp][1][u];
            float* sy = s_in[warp][2][u];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                sa[8 * t + r] = in.a[r];
                sx[8 * t + r] = in.x[r];
                sy[8 * t + r] = in.y[r];
            }
            __syncwarp();
            quad_gather_smem<VT>(vb, H, cur.h, t, n, P, sa, sx, sy, s_meta, acc);
            __syncwarp();  // read before the next item overwrites
        }
#else
        quad_gather<VT>(vb, H, cur.h, t, n, P, in.a, in.x, in.y, s_meta, acc);
#endif
        if (cur.live) {
            float4* o = reinterpret_cast<float4*>(
                out_rb + ((int64_t)cur.out_row * H + cur.h) * kHeadDim + 8 * t);
            if (out32) {  // the lane's 32 bytes in one store
                asm volatile("st.global.v8.f32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(o),
                             "f"(acc[0]), "f"(acc[1]), "f"(acc[2]), "f"(acc[3]), "f"(acc[4]),
                             "f"(acc[5]), "f"(acc[6]), "f"(acc[7])
                             : "memory");
            } else {
                o[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
                o[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
            }
        }
        if (next_tile >= n_tiles) break;  // warp-uniform
        tile = next_tile;
#if MSDA_QUAD_PREFETCH
        cur = nxt;
        in = in_next;
#else
        cur = resolve(tile);
        quad_load(cur.lg, cur.of, n, t, cur.live, vec, in);
#endif
    }
}

template <typename VT>
static cudaError_t launch_quad_t(const Problem& p, const float* ref_cam, const float* off,
                                 const float* logits, const int32_t* idx, const int32_t* count,
                                 float* out_rb, cudaStream_t s)
{
    const int64_t max_items = (int64_t)p.B * p.Ncam * p.Nq * p.H;
    if (max_items == 0) return cudaSuccess;
    const int64_t max_ctas = ((max_items + 7) / 8 + kWarps - 1) / kWarps;
    static int occ = [] {
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, sca_gather_quad_kernel<VT>, kThreads,
                                                          0) != cudaSuccess ||
            n < 1)
            n = 1;
        return n;
    }();
    int64_t grid = std::min<int64_t>(max_ctas, (int64_t)occ * device_sm_count());
    if (MSDA_QUAD_HEADSPEC && grid > p.H) grid -= grid % p.H;  // a CTA keeps one head
    const bool vec = p.L * p.P == kQuadSamples && ((uintptr_t)off & 15) == 0 &&
                     ((uintptr_t)logits & 15) == 0;
    return launch_pdl(sca_gather_quad_kernel<VT>, dim3((unsigned)grid), dim3(kThreads), 0, s,
                      static_cast<const VT*>(p.value), off, logits, ref_cam, idx, count, out_rb,
                      p.B, p.Ncam, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv, vec);
}

bool sca_gather_quad_fits(const Problem& p) { return p.L * p.P <= kQuadSamples; }

cudaError_t launch_sca_gather_quad(const Problem& p, const float* ref_cam, const float* off,
                                   const float* logits, const int32_t* idx, const int32_t* count,
                                   float* out_rb, cudaStream_t s)
{
    if (p.bf16)
        return launch_quad_t<__nv_bfloat16>(p, ref_cam, off, logits, idx, count, out_rb, s);
    return launch_quad_t<float>(p, ref_cam, off, logits, idx, count, out_rb, s);
}

}  // namespace msda
