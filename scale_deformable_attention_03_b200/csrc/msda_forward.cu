// K1 / K1f: MSDA forward, one warp per (batch, query, head).
//
// Item order is (b, q, h) with h fastest.  A CTA owns a tile of
// kRowsPerTile consecutive queries; with H = 8 each of its eight warps keeps
// one head and walks the tile's queries, so neighbouring queries' reads of the
// same head slices meet in the SM's L1.  No integer division in the loop; each
// warp loads the next query's inputs before gathering the current one.
#include <type_traits>

#include "msda_launch.h"

namespace msda {

constexpr int kRowsPerTile = MSDA_ROWS_PER_TILE;
constexpr int kGroupRowsPerTile = MSDA_GROUP_ROWS_PER_TILE;

template <typename VT, bool FUSED, int NC, int HP>
__global__ void MSDA_GATHER_BOUNDS(VT, NC)
msda_forward_kernel(const VT* __restrict__ value, const float* __restrict__ lo,
                    const float* __restrict__ wl, const float* __restrict__ ref,
                    float* __restrict__ out, int B, int Nq, int Nv, int H, int L, int P, int R,
                    Levels levels)
{
    using Table = typename std::conditional<HP == 2, PairTable, WarpTable>::type;
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) Table s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, R, lane, ls);
    const int S = L * P;
    const int64_t rows = (int64_t)B * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    const int HG = H / HP;  // head groups: one per warp item
    const int n_items = kRowsPerTile * HG;

    struct Item {
        bool ok;
        int b, h;
        int64_t bq;
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.bq = row0 + cur.rr;
        x.ok = it < n_items && x.bq < rows;
        x.h = cur.h * HP;
        int q = q0 + cur.rr;
        x.b = b0;
        while (q >= Nq) {
            q -= Nq;
            ++x.b;
        }
        return x;
    };
    auto fetch = [&](const Item& x, RowIn<FUSED, NC, HP>& in) {
        const int64_t item = x.bq * H + x.h;
        load_row<FUSED, NC, HP>(lo + item * S * 2, wl + item * S, FUSED ? ref + x.bq * R * 2 : nullptr,
                                S, ls, lane, in);
    };

    ItemCursor cur(warp, HG);
    int it = warp;
    Item x0 = resolve(it, cur);
    RowIn<FUSED, NC, HP> in0, in1;
    if (x0.ok) fetch(x0, in0);
    while (x0.ok) {
        ItemCursor nx = cur;
        nx.next();
        const Item x1 = resolve(it + kWarps, nx);
        if (x1.ok) fetch(x1, in1);  // next row's inputs in flight during this gather
        const int64_t item = x0.bq * H + x0.h;
        const VT* vb = value + (int64_t)x0.b * Nv * H * kHeadDim;
        if constexpr (HP == 2)
            row_compute_pair<FUSED, NC>(vb, H, x0.h, in0, S, ls, s_tab[warp],
                                        out + item * kHeadDim, lane);
        else
            row_compute<VT, FUSED, NC>(vb, H, x0.h, in0, S, ls, s_tab[warp],
                                       out + item * kHeadDim, lane);
        x0 = x1;
        in0 = in1;
        cur = nx;
        it += kWarps;
    }
}

// K1g: rows with L*P <= 16, G = 32 / npad heads per warp item (see
// group_compute).  Items are (row, head group), head groups fastest; a CTA
// owns kGroupRowsPerTile consecutive rows (more than K1: a row has fewer
// samples, and neighbouring queries share more of their reads).
// Register budget: rows of up to four samples (eight heads per warp) run
// fastest at four CTAs per SM (TSA queues as a batch of two: 140 -> 119 us),
// longer rows at the group kernels' three.
#ifndef MSDA_GROUP4_MIN_CTAS
#define MSDA_GROUP4_MIN_CTAS 4
#endif
template <typename VT, bool FUSED, int NPL>
__global__ void __launch_bounds__(kThreads, NPL == 2 ? MSDA_GROUP4_MIN_CTAS : MSDA_GROUP_MIN_CTAS)
msda_forward_group_kernel(const VT* __restrict__ value, const float* __restrict__ lo,
                          const float* __restrict__ wl, const float* __restrict__ ref,
                          float* __restrict__ out, int B, int Nq, int Nv, int H, int L, int P,
                          int R, Levels levels)
{
    constexpr int npad_log2 = NPL;
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) WarpTable s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    GroupLane gl;
    group_lane(s_lv, L, P, R, npad_log2, lane, gl);
    const int S = L * P;
    const int G = 32 >> npad_log2;
    const int HG = (H + G - 1) / G;  // head groups per row
    const int64_t rows = (int64_t)B * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kGroupRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    const int n_items = kGroupRowsPerTile * HG;

    struct Item {
        bool ok, valid;
        int b, h0;
        int64_t bq;
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.bq = row0 + cur.rr;
        x.ok = it < n_items && x.bq < rows;
        x.h0 = cur.h * G;
        x.valid = gl.in && x.h0 + gl.s < H;
        int q = q0 + cur.rr;
        x.b = b0;
        while (q >= Nq) {
            q -= Nq;
            ++x.b;
        }
        return x;
    };
    struct In {
        float a;
        float2 v, r;
    };
    auto fetch = [&](const Item& x, In& in) {
        const int64_t row_h = (x.bq * H + x.h0 + gl.s) * S + gl.k;  // this lane's sample
        in.a = x.valid ? ld_stream(wl + row_h) : (FUSED ? -INFINITY : 0.f);
        in.v = x.valid ? ld_stream2(lo + 2 * row_h) : make_float2(0.f, 0.f);
        in.r = (FUSED && x.valid) ? __ldg(reinterpret_cast<const float2*>(ref + x.bq * R * 2) + gl.m)
                                  : make_float2(0.f, 0.f);
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
        const VT* vb = value + (int64_t)x0.b * Nv * H * kHeadDim;
        group_compute<VT, FUSED, NPL>(vb, H, x0.h0, in0.a, in0.v, in0.r, x0.valid, gl,
                                      s_tab[warp], out + (x0.bq * H + x0.h0) * kHeadDim, lane);
        x0 = x1;
        in0 = in1;
        cur = nx;
        it += kWarps;
    }
}

template <typename VT, bool FUSED>
static cudaError_t launch_group(const Problem& p, const float* lo, const float* wl,
                                const float* ref, float* out, cudaStream_t s)
{
    const int64_t rows = (int64_t)p.B * p.Nq;
    if (rows == 0) return cudaSuccess;
    const int S = p.L * p.P;
    int npad_log2 = 2;
    while ((1 << npad_log2) < S) ++npad_log2;
    const unsigned grid = (unsigned)((rows + kGroupRowsPerTile - 1) / kGroupRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    switch (npad_log2) {
#define MSDA_GROUP_CASE(NPLV)                                                                    \
    case NPLV:                                                                                   \
        msda_forward_group_kernel<VT, FUSED, NPLV><<<grid, kThreads, 0, s>>>(                    \
            v, lo, wl, ref, out, p.B, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                     \
        break;
        MSDA_GROUP_CASE(2)
        MSDA_GROUP_CASE(3)
        MSDA_GROUP_CASE(4)
#undef MSDA_GROUP_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

// Warp layout choice: several heads per warp when a row has at most 16
// samples per head and there is more than one head.
static bool use_group(const Problem& p) { return p.L * p.P <= 16 && p.H > 1; }

template <typename VT, bool FUSED, int HP>
static cudaError_t launch_fwd(const Problem& p, const float* lo, const float* wl,
                              const float* ref, float* out, cudaStream_t s)
{
    const int64_t rows = (int64_t)p.B * p.Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kRowsPerTile - 1) / kRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define MSDA_FWD_CASE(NCV)                                                                       \
    case NCV:                                                                                    \
        msda_forward_kernel<VT, FUSED, NCV, HP><<<grid, kThreads, 0, s>>>(                       \
            v, lo, wl, ref, out, p.B, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                     \
        break;
    switch (nc) {
        MSDA_FWD_CASE(1)
        MSDA_FWD_CASE(2)
        MSDA_FWD_CASE(3)
        MSDA_FWD_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef MSDA_FWD_CASE
    return cudaGetLastError();
}

cudaError_t launch_msda_forward(const Problem& p, const float* loc, const float* attn,
                                float* out, cudaStream_t s)
{
    if (use_group(p))
        return p.bf16 ? launch_group<__nv_bfloat16, false>(p, loc, attn, nullptr, out, s)
                      : launch_group<float, false>(p, loc, attn, nullptr, out, s);
    if (!p.bf16) return launch_fwd<float, false, 1>(p, loc, attn, nullptr, out, s);
    if (p.H % 2 == 0) return launch_fwd<__nv_bfloat16, false, 2>(p, loc, attn, nullptr, out, s);
    return launch_fwd<__nv_bfloat16, false, 1>(p, loc, attn, nullptr, out, s);
}

cudaError_t launch_msda_forward_fused(const Problem& p, const float* ref, const float* off,
                                      const float* logits, float* out, cudaStream_t s)
{
    if (use_group(p))
        return p.bf16 ? launch_group<__nv_bfloat16, true>(p, off, logits, ref, out, s)
                      : launch_group<float, true>(p, off, logits, ref, out, s);
    if (!p.bf16) return launch_fwd<float, true, 1>(p, off, logits, ref, out, s);
    if (p.H % 2 == 0) return launch_fwd<__nv_bfloat16, true, 2>(p, off, logits, ref, out, s);
    return launch_fwd<__nv_bfloat16, true, 1>(p, off, logits, ref, out, s);
}

}  // namespace msda
