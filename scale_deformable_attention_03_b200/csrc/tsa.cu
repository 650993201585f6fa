// Temporal Self-Attention ("【论文阅读】BEVFormer论文解析及Temporal
// Self-Attention、Spatial Cross-Attention注意力机制详解及代码示例", section
// 二.2 and its BEV encoder listing):
//   K5a tsa_reference_kernel  cell centres moved by each queue's ego motion
//   K5b tsa_forward_*_kernel  fused MSDA over the T queues of every BEV query,
//                             averaged in registers and written once
// The queues of BEV sample b are value batch items b*T .. b*T + T - 1 (the
// previous BEV first, the current one last, in BEVFormer's order).  A warp
// keeps one output item (query, head or head group) and reads all T queues
// for it, so the per-queue rows never reach memory.
#include <algorithm>

#include "msda_launch.h"

namespace msda {

constexpr int kTsaRowsPerTile = MSDA_ROWS_PER_TILE;
constexpr int kTsaGroupRowsPerTile = MSDA_GROUP_ROWS_PER_TILE;

// One thread per (b, t, q).  The listing reads delta_x, delta_y (metres) and
// the yaw in degrees from the CAN bus and uses 0.512 m BEV cells, then breaks
// off; the motion is applied here as a rigid transform of the cell centre
// (rotation about the BEV centre, then translation), in double precision.
__global__ void tsa_reference_kernel(const float* __restrict__ ego, int64_t BT, int bev_h,
                                     int bev_w, double gx, double gy, float2* __restrict__ ref)
{
    const int64_t Nq = (int64_t)bev_h * bev_w;
    const int64_t n = BT * Nq;
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < n;
         k += (int64_t)gridDim.x * blockDim.x) {
        const int64_t bt = k / Nq;
        const int64_t qq = k - bt * Nq;
        const int i = (int)(qq / bev_w), j = (int)(qq - (int64_t)i * bev_w);
        const double dx = __ldg(ego + bt * 3 + 0), dy = __ldg(ego + bt * 3 + 1);
        double sn, cs;
        sincospi((double)__ldg(ego + bt * 3 + 2) / 180.0, &sn, &cs);
        const double px = ((double)j + 0.5 - 0.5 * bev_w) * gx;
        const double py = ((double)i + 0.5 - 0.5 * bev_h) * gy;
        const double qx = cs * px - sn * py + dx;
        const double qy = sn * px + cs * py + dy;
        ref[k] = make_float2((float)(qx / (bev_w * gx) + 0.5), (float)(qy / (bev_h * gy) + 0.5));
    }
}

cudaError_t launch_tsa_reference(const float* ego, int B, int T, int bev_h, int bev_w, double gx,
                                 double gy, float* ref, cudaStream_t s)
{
    const int64_t n = (int64_t)B * T * bev_h * bev_w;
    if (n == 0) return cudaSuccess;
    const int threads = 256;
    const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads,
                                             (int64_t)device_sm_count() * 8);
    tsa_reference_kernel<<<(unsigned)blocks, threads, 0, s>>>(
        ego, (int64_t)B * T, bev_h, bev_w, gx, gy, reinterpret_cast<float2*>(ref));
    return cudaGetLastError();
}

template <int NA>
__device__ __forceinline__ void scale_acc(float (&acc)[NA], float f)
{
#pragma unroll
    for (int i = 0; i < NA; ++i) acc[i] *= f;
}

// Rows with L*P <= 16 (see group_compute): a warp item is (b, q, head
// group); the warp builds one table per queue, then each head's output sums
// the T queues' gathers before its single store.
template <typename VT, int T, int NPL>
__global__ void MSDA_GROUP_BOUNDS
tsa_forward_group_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                         const float* __restrict__ logits, const float* __restrict__ ref,
                         float* __restrict__ out, int B, int Nq, int Nv, int H, int L, int P,
                         int R, Levels levels)
{
    constexpr int npad_log2 = NPL;
    constexpr int G = 32 >> NPL;
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) WarpTable s_tab[kWarps][T];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    GroupLane gl;
    group_lane(s_lv, L, P, R, npad_log2, lane, gl);
    const int S = L * P;
    const int HG = (H + G - 1) / G;
    const int64_t rows = (int64_t)B * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kTsaGroupRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    const int n_items = kTsaGroupRowsPerTile * HG;
    const int64_t vstride = (int64_t)Nv * H * kHeadDim;
    const float inv_t = 1.f / (float)T;

    struct Item {
        bool ok, valid;
        int b, q, h0;
        int64_t bq;
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.bq = row0 + cur.rr;
        x.ok = it < n_items && x.bq < rows;
        x.h0 = cur.h * G;
        x.valid = gl.in && x.h0 + gl.s < H;
        x.q = q0 + cur.rr;
        x.b = b0;
        while (x.q >= Nq) {
            x.q -= Nq;
            ++x.b;
        }
        return x;
    };
    struct In {
        float a[T];
        float2 v[T], r[T];
    };
    auto fetch = [&](const Item& x, In& in) {
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const int64_t src = ((int64_t)x.b * T + t) * Nq + x.q;  // queue t's row
            const int64_t row_h = (src * H + x.h0 + gl.s) * S + gl.k;
            in.a[t] = x.valid ? ld_stream(logits + row_h) : -INFINITY;
            in.v[t] = x.valid ? ld_stream2(off + 2 * row_h) : make_float2(0.f, 0.f);
            in.r[t] = x.valid ? __ldg(reinterpret_cast<const float2*>(ref + src * R * 2) + gl.m)
                              : make_float2(0.f, 0.f);
        }
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
#pragma unroll
        for (int t = 0; t < T; ++t)
            group_table<true>(H, x0.h0, in0.a[t], in0.v[t], in0.r[t], x0.valid, gl,
                              s_tab[warp][t], lane);
        __syncwarp();
        const VT* vb = value + (int64_t)x0.b * T * vstride;
        const int nheads = min(G, H - x0.h0);
        float* orow = out + (x0.bq * H + x0.h0) * kHeadDim;
        for (int s = 0; s < nheads; ++s) {
            float acc[Gather<VT>::kAcc];
#pragma unroll
            for (int i = 0; i < Gather<VT>::kAcc; ++i) acc[i] = 0.f;
#pragma unroll
            for (int t = 0; t < T; ++t)
                Gather<VT>::template run_quads<(1 << NPL) / 4>(vb + t * vstride, s_tab[warp][t],
                                                               lane, acc, s << NPL);
            scale_acc(acc, inv_t);
            Gather<VT>::store(acc, lane, orow + s * kHeadDim);
        }
        __syncwarp();
        x0 = x1;
        in0 = in1;
        cur = nx;
        it += kWarps;
    }
}

// Rows with more samples: a warp item is (b, q, h); the T queues' gathers
// accumulate into the same partial sums.
template <typename VT, int NC, int T>
__global__ void MSDA_GATHER_BOUNDS(VT, NC)
tsa_forward_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                   const float* __restrict__ logits, const float* __restrict__ ref,
                   float* __restrict__ out, int B, int Nq, int Nv, int H, int L, int P, int R,
                   Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) WarpTable s_tab[kWarps];
    stage_levels(s_lv, levels);
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, R, lane, ls);
    const int S = L * P;
    const int64_t rows = (int64_t)B * Nq;
    const int64_t row0 = (int64_t)blockIdx.x * kTsaRowsPerTile;
    const int b0 = (int)(row0 / Nq);
    const int q0 = (int)(row0 - (int64_t)b0 * Nq);
    const int n_items = kTsaRowsPerTile * H;
    const int64_t vstride = (int64_t)Nv * H * kHeadDim;
    const float inv_t = 1.f / (float)T;

    struct Item {
        bool ok;
        int b, q, h;
        int64_t bq;
    };
    auto resolve = [&](int it, const ItemCursor& cur) {
        Item x;
        x.bq = row0 + cur.rr;
        x.ok = it < n_items && x.bq < rows;
        x.h = cur.h;
        x.q = q0 + cur.rr;
        x.b = b0;
        while (x.q >= Nq) {
            x.q -= Nq;
            ++x.b;
        }
        return x;
    };
    auto fetch = [&](const Item& x, RowIn<true, NC, 1> (&in)[T]) {
#pragma unroll
        for (int t = 0; t < T; ++t) {
            const int64_t src = ((int64_t)x.b * T + t) * Nq + x.q;
            const int64_t item = src * H + x.h;
            load_row<true, NC, 1>(off + item * S * 2, logits + item * S, ref + src * R * 2, S, ls,
                                  lane, in[t]);
        }
    };

    ItemCursor cur(warp, H);
    int it = warp;
    Item x0 = resolve(it, cur);
    RowIn<true, NC, 1> in0[T], in1[T];
    if (x0.ok) fetch(x0, in0);
    while (x0.ok) {
        ItemCursor nx = cur;
        nx.next();
        const Item x1 = resolve(it + kWarps, nx);
        if (x1.ok) fetch(x1, in1);
        float acc[Gather<VT>::kAcc];
#pragma unroll
        for (int i = 0; i < Gather<VT>::kAcc; ++i) acc[i] = 0.f;
        const VT* vb = value + (int64_t)x0.b * T * vstride;
#pragma unroll
        for (int t = 0; t < T; ++t)
            row_accumulate<VT, true, NC>(vb + t * vstride, H, x0.h, in0[t], S, ls, s_tab[warp],
                                         acc, lane);
        scale_acc(acc, inv_t);
        Gather<VT>::store(acc, lane, out + (x0.bq * H + x0.h) * kHeadDim);
#pragma unroll
        for (int t = 0; t < T; ++t) in0[t] = in1[t];
        x0 = x1;
        cur = nx;
        it += kWarps;
    }
}

template <typename VT, int T>
static cudaError_t launch_tsa_t(const Problem& p, const float* ref, const float* off,
                                const float* logits, float* out, cudaStream_t s)
{
    // p.B counts BEV samples; the value holds p.B * T batch items
    const int64_t rows = (int64_t)p.B * p.Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kTsaRowsPerTile - 1) / kTsaRowsPerTile);
    const unsigned group_grid =
        (unsigned)((rows + kTsaGroupRowsPerTile - 1) / kTsaGroupRowsPerTile);
    const VT* v = static_cast<const VT*>(p.value);
    const int S = p.L * p.P;
    if (S <= 16 && p.H > 1) {
        int npad_log2 = 2;
        while ((1 << npad_log2) < S) ++npad_log2;
        switch (npad_log2) {
#define TSA_GROUP_CASE(NPLV)                                                                     \
    case NPLV:                                                                                   \
        tsa_forward_group_kernel<VT, T, NPLV><<<group_grid, kThreads, 0, s>>>(                   \
            v, off, logits, ref, out, p.B, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                \
        break;
            TSA_GROUP_CASE(2)
            TSA_GROUP_CASE(3)
            TSA_GROUP_CASE(4)
#undef TSA_GROUP_CASE
            default: return cudaErrorInvalidValue;
        }
        return cudaGetLastError();
    }
    switch ((S + 31) / 32) {
#define TSA_CASE(NCV)                                                                            \
    case NCV:                                                                                    \
        tsa_forward_kernel<VT, NCV, T><<<grid, kThreads, 0, s>>>(                                \
            v, off, logits, ref, out, p.B, p.Nq, p.Nv, p.H, p.L, p.P, p.R, p.lv);                \
        break;
        TSA_CASE(1)
        TSA_CASE(2)
        TSA_CASE(3)
        TSA_CASE(4)
#undef TSA_CASE
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

template <typename VT>
static cudaError_t launch_tsa_vt(const Problem& p, int T, const float* ref, const float* off,
                                 const float* logits, float* out, cudaStream_t s)
{
    switch (T) {
        case 1: return launch_tsa_t<VT, 1>(p, ref, off, logits, out, s);
        case 2: return launch_tsa_t<VT, 2>(p, ref, off, logits, out, s);
        case 3: return launch_tsa_t<VT, 3>(p, ref, off, logits, out, s);
        case 4: return launch_tsa_t<VT, 4>(p, ref, off, logits, out, s);
        default: return cudaErrorInvalidValue;
    }
}

cudaError_t launch_tsa_forward(const Problem& p, int T, const float* ref, const float* off,
                               const float* logits, float* out, cudaStream_t s)
{
    return p.bf16 ? launch_tsa_vt<__nv_bfloat16>(p, T, ref, off, logits, out, s)
                  : launch_tsa_vt<float>(p, T, ref, off, logits, out, s);
}

}  // namespace msda
