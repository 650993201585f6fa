// K1 / K1f: MSDA forward, one warp per (batch, query, head).
//
// Item order is (b, q, h) with h fastest, so the eight warps of a CTA take
// the eight heads of one query; a CTA then walks kRowsPerWarp consecutive
// queries, which keeps neighbouring queries' reads of the same head slices in
// the SM's L1.
#include "msda_launch.h"

namespace msda {

constexpr int kRowsPerWarp = 2;

template <typename VT, bool FUSED, int NC>
__global__ void __launch_bounds__(kThreads)
msda_forward_kernel(const VT* __restrict__ value, const float* __restrict__ lo,
                    const float* __restrict__ wl, const float* __restrict__ ref,
                    float* __restrict__ out, int B, int Nq, int Nv, int H, int L, int P, int R,
                    Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) WarpTable s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t items = (int64_t)B * Nq * H;
    const int64_t tile0 = (int64_t)blockIdx.x * kWarps * kRowsPerWarp;
    const int S = L * P;
    for (int t = 0; t < kRowsPerWarp; ++t) {
        const int64_t item = tile0 + (int64_t)t * kWarps + warp;  // (b * Nq + q) * H + h
        if (item >= items) break;
        const int h = (int)(item % H);
        const int64_t bq = item / H;
        const int b = (int)(bq / Nq);
        const VT* vb = value + (int64_t)b * Nv * H * kHeadDim;
        row_forward<VT, FUSED, NC>(vb, H, h, lo + item * S * 2, wl + item * S,
                                   FUSED ? ref + bq * R * 2 : nullptr, L, P, R, s_lv, s_tab[warp],
                                   out + item * kHeadDim, lane);
    }
}

template <typename VT, bool FUSED>
static cudaError_t launch_fwd(const Problem& p, const float* lo, const float* wl,
                              const float* ref, float* out, cudaStream_t s)
{
    const int64_t items = (int64_t)p.B * p.Nq * p.H;
    if (items == 0) return cudaSuccess;
    const int64_t per_cta = (int64_t)kWarps * kRowsPerWarp;
    const unsigned grid = (unsigned)((items + per_cta - 1) / per_cta);
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define MSDA_FWD_CASE(NCV)                                                                       \
    case NCV:                                                                                    \
        msda_forward_kernel<VT, FUSED, NCV><<<grid, kThreads, 0, s>>>(                           \
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
    return p.bf16 ? launch_fwd<__nv_bfloat16, false>(p, loc, attn, nullptr, out, s)
                  : launch_fwd<float, false>(p, loc, attn, nullptr, out, s);
}

cudaError_t launch_msda_forward_fused(const Problem& p, const float* ref, const float* off,
                                      const float* logits, float* out, cudaStream_t s)
{
    return p.bf16 ? launch_fwd<__nv_bfloat16, true>(p, off, logits, ref, out, s)
                  : launch_fwd<float, true>(p, off, logits, ref, out, s);
}

}  // namespace msda
