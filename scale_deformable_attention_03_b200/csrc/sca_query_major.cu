// SCA forward, query-major ("BEV(三) BEVFormer ..." section 10: a BEV query
// samples every camera that sees it and takes the mean over those cameras;
// Tencent Cloud "Spatial Cross-Attention" walkthrough, average listing: the
// count is clamped at one).
//
// One warp per (b, q, head or head pair): a ballot over the camera lanes of
// bev_mask gives the seeing cameras, the softmax of the query's logits is
// taken once, and each seeing camera in ascending order adds its gather to
// the same partial sums, divided by max(1, hits) before the single store.
// There is no compaction, no rebatched row in memory and no second kernel:
// offsets and logits are read once per query instead of once per camera.
// Items are ordered (b, q, h) like msda_forward's, so a CTA's warps keep one
// head each over a tile of neighbouring queries.
#include <type_traits>

#include "msda_launch.h"

namespace msda {

constexpr int kQmRowsPerTile = MSDA_ROWS_PER_TILE;

// Register budget: an explicit four-CTA bound for fp32 rows of up to 32
// samples (2 % faster here than the compiler's own choice), otherwise as the
// other forward gathers.
#define MSDA_QM_BOUNDS(VT, NC)                                                           \
    __launch_bounds__(kThreads, (NC) == 1 ? (sizeof(VT) == 4 ? 4 : MSDA_MIN_CTAS_BF16)   \
                                          : ((NC) == 2 ? 2 : 1))

// Camera lane: does camera `lane` (< Ncam) see query (b, q)?
__device__ __forceinline__ unsigned seeing_cameras(const uint8_t* __restrict__ mask, int B,
                                                   int Ncam, int Nq, int R, int b, int q, int lane)
{
    bool hit = false;
    if (lane < Ncam) {
        const uint8_t* m = mask + (((int64_t)lane * B + b) * Nq + q) * R;
        for (int r = 0; r < R; ++r) hit |= __ldg(m + r) != 0;
    }
    return __ballot_sync(0xffffffffu, hit);
}

template <int NC>
__device__ __forceinline__ void load_ref(const float* __restrict__ ref_row,
                                         const LaneSamples<NC>& ls, float2 (&rf)[NC])
{
#pragma unroll
    for (int c = 0; c < NC; ++c)
        rf[c] = ls.in[c] ? __ldg(reinterpret_cast<const float2*>(ref_row) + ls.m[c])
                         : make_float2(0.f, 0.f);
}

template <int NA>
__device__ __forceinline__ void divide_acc(float (&acc)[NA], unsigned seen)
{
    const float inv = 1.f / (float)max(1, __popc(seen));
#pragma unroll
    for (int i = 0; i < NA; ++i) acc[i] *= inv;
}

// Eight channels rounded to bf16 (to nearest even) in one 16-byte store.
__device__ __forceinline__ void store_bf16x8(__nv_bfloat16* dst, const float (&v)[8])
{
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const __nv_bfloat162 p = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        u[i] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(dst) = make_uint4(u[0], u[1], u[2], u[3]);
}

// The bf16-output form of pair_store (HP = 2) and Gather<bf16>::store (HP = 1)
// for bf16 value: the mean rounded to bf16, the operand type of the output
// projection that follows it in the SCA module.
template <int HP>
__device__ __forceinline__ void store_row_bf16(float (&acc)[8], int lane,
                                               __nv_bfloat16* __restrict__ out_row0)
{
    const int g = (lane >> 2) & 3, t = lane & 3;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 4);
        acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 8);
        if (HP == 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], 16);
    }
    if (HP == 2) {
        if (g == 0) store_bf16x8(out_row0 + (lane >> 4) * kHeadDim + 8 * t, acc);
    } else if (lane < 4) {
        store_bf16x8(out_row0 + 8 * t, acc);
    }
}

// OUT16: the result is stored as bf16 (bf16 value only).
template <typename VT, int NC, int HP, bool OUT16>
__global__ void MSDA_QM_BOUNDS(VT, NC)
sca_query_major_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                       const float* __restrict__ logits, const float* __restrict__ ref_cam,
                       const uint8_t* __restrict__ mask, void* __restrict__ out, int B,
                       int Ncam, int Nq, int Nv, int H, int L, int P, int R, Levels levels)
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
    const int64_t row0 = (int64_t)blockIdx.x * kQmRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    const int HG = H / HP;
    const int n_items = kQmRowsPerTile * HG;
    const int64_t vstride = (int64_t)Nv * H * kHeadDim;
    const int64_t cam_ref_stride = (int64_t)B * Nq * R * 2;

    struct Item {
        bool ok;
        int b, q, h;
        int64_t bq;
        unsigned seen;  // warp-uniform camera set
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.bq = row0 + cur.rr;
        x.ok = it < n_items && x.bq < rows;
        x.h = cur.h * HP;
        x.q = q0 + cur.rr;
        x.b = b0;
        while (x.q >= Nq) {
            x.q -= Nq;
            ++x.b;
        }
        x.seen = x.ok ? seeing_cameras(mask, B, Ncam, Nq, R, x.b, x.q, lane) : 0u;
        return x;
    };
    // The query's offsets and logits, and the first seeing camera's
    // reference points.
    auto fetch = [&](const Item& x, RowIn<true, NC, HP>& in) {
        const int64_t bqh = x.bq * H + x.h;
        const int c0 = x.seen ? __ffs(x.seen) - 1 : 0;
        load_row<true, NC, HP>(off + bqh * S * 2, logits + bqh * S,
                               ref_cam + c0 * cam_ref_stride + x.bq * R * 2, S, ls, lane, in);
    };

    ItemCursor cur(warp, HG);
    int it = warp;
    Item x0 = resolve(it, cur);
    RowIn<true, NC, HP> in0, in1;
    if (x0.ok) fetch(x0, in0);
    while (x0.ok) {
        ItemCursor nx = cur;
        nx.next();
        const Item x1 = resolve(it + kWarps, nx);
        if (x1.ok) fetch(x1, in1);  // next query's inputs in flight during this one's gathers
#pragma unroll
        for (int s = 0; s < HP; ++s) normalise<true, NC>(in0.a[s], ls);
        float acc[HP == 2 ? 8 : Gather<VT>::kAcc];
#pragma unroll
        for (int i = 0; i < (HP == 2 ? 8 : Gather<VT>::kAcc); ++i) acc[i] = 0.f;
        float2 rf[NC];
#pragma unroll
        for (int c = 0; c < NC; ++c) rf[c] = in0.rf[c];
        unsigned cams = x0.seen;
        while (cams) {
            const int cam = __ffs(cams) - 1;
            cams &= cams - 1;
            float2 rf_next[NC];
            if (cams)  // the next camera's reference points, in flight during this gather
                load_ref<NC>(ref_cam + (__ffs(cams) - 1) * cam_ref_stride + x0.bq * R * 2, ls,
                             rf_next);
            const VT* vb = value + ((int64_t)x0.b * Ncam + cam) * vstride;
            if constexpr (HP == 2)
                pair_gather<true, NC>(vb, H, x0.h, in0, rf, S, ls, s_tab[warp], acc, lane);
            else
                head_gather<VT, true, NC>(vb, H, x0.h, in0.a[0], in0.lo[0], rf, S, ls,
                                          s_tab[warp], acc, lane);
            if (cams) {
#pragma unroll
                for (int c = 0; c < NC; ++c) rf[c] = rf_next[c];
            }
        }
        divide_acc(acc, x0.seen);
        const int64_t orow = (x0.bq * H + x0.h) * kHeadDim;
        if constexpr (OUT16) {
            store_row_bf16<HP>(acc, lane, static_cast<__nv_bfloat16*>(out) + orow);
        } else if constexpr (HP == 2) {
            pair_store(acc, lane, static_cast<float*>(out) + orow);
        } else {
            Gather<VT>::store(acc, lane, static_cast<float*>(out) + orow);
        }
        x0 = x1;
        in0 = in1;
        cur = nx;
        it += kWarps;
    }
}

template <typename VT, int HP, bool OUT16 = false>
static cudaError_t launch_qm_t(const Problem& p, const float* ref_cam, const uint8_t* mask,
                               const float* off, const float* logits, void* out, cudaStream_t s)
{
    const int64_t rows = (int64_t)p.B * p.Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kQmRowsPerTile - 1) / kQmRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    switch ((p.L * p.P + 31) / 32) {
#define SCA_QM_CASE(NCV)                                                                         \
    case NCV:                                                                                    \
        sca_query_major_kernel<VT, NCV, HP, OUT16><<<grid, kThreads, 0, s>>>(                    \
            v, off, logits, ref_cam, mask, out, p.B, p.Ncam, p.Nq, p.Nv, p.H, p.L, p.P, p.R,     \
            p.lv);                                                                               \
        break;
        SCA_QM_CASE(1)
        SCA_QM_CASE(2)
        SCA_QM_CASE(3)
        SCA_QM_CASE(4)
#undef SCA_QM_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_sca_query_major(const Problem& p, const float* ref_cam, const uint8_t* mask,
                                   const float* off, const float* logits, void* out,
                                   bool out_bf16, cudaStream_t s)
{
    if (!p.bf16) {
        if (out_bf16) return cudaErrorInvalidValue;  // bf16 output serves bf16 value only
        return launch_qm_t<float, 1>(p, ref_cam, mask, off, logits, out, s);
    }
    if (p.H % 2 == 0)
        return out_bf16 ? launch_qm_t<__nv_bfloat16, 2, true>(p, ref_cam, mask, off, logits, out, s)
                        : launch_qm_t<__nv_bfloat16, 2>(p, ref_cam, mask, off, logits, out, s);
    return out_bf16 ? launch_qm_t<__nv_bfloat16, 1, true>(p, ref_cam, mask, off, logits, out, s)
                    : launch_qm_t<__nv_bfloat16, 1>(p, ref_cam, mask, off, logits, out, s);
}

}  // namespace msda
