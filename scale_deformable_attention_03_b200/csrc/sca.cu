// SCA forward pieces (Tencent Cloud "Spatial Cross-Attention" walkthrough,
// rebatch and average listings; "BEV(三) BEVFormer ..." section 10):
//   K2a sca_count_kernel    hits per query, seeing queries per 1024-query chunk
//   K2b sca_scatter_kernel  stable ranks -> idx / pos / count / row prefix
//   K3  sca_gather_kernel   fused MSDA over every camera's seeing queries
//   K4  sca_average_kernel  per-query sum over cameras / max(1, hits)
// Nothing here synchronises with the host: the rebatched row counts live in
// device memory and K3 is a persistent kernel that reads them.
#include <algorithm>

#include "msda_launch.h"

namespace msda {

constexpr int kMaxCameras = 32;
constexpr int kScaRowsPerWarp = 2;

__device__ __forceinline__ int warp_sum_int(int v)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane)
{
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += u;
    }
    return v;
}

// A camera sees query q when any of its R anchor bytes is non-zero.
__device__ __forceinline__ bool seen(const uint8_t* __restrict__ mask, int64_t at, int R)
{
    bool hit = false;
    for (int r = 0; r < R; ++r) hit |= __ldg(mask + at * R + r) != 0;
    return hit;
}

__global__ void __launch_bounds__(kCompactChunk)
sca_count_kernel(const uint8_t* __restrict__ mask, int B, int Ncam, int Nq, int R, int nchunks,
                 int32_t* __restrict__ hits, int32_t* __restrict__ chunk_counts)
{
    __shared__ int s_cnt[kMaxCameras][32];
    const int chunk = blockIdx.x, b = blockIdx.y;
    const int q = chunk * kCompactChunk + threadIdx.x;
    const bool valid = q < Nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int nh = 0;
    for (int c = 0; c < Ncam; ++c) {
        const bool hit = valid && seen(mask, ((int64_t)c * B + b) * Nq + q, R);
        nh += hit;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) s_cnt[c][warp] = __popc(bal);
    }
    if (valid) hits[(int64_t)b * Nq + q] = nh;
    __syncthreads();
    if (warp < Ncam) {
        const int v = warp_sum_int(s_cnt[warp][lane]);
        if (lane == 0) chunk_counts[((int64_t)b * Ncam + warp) * nchunks + chunk] = v;
    }
}

__global__ void __launch_bounds__(kCompactChunk)
sca_scatter_kernel(const uint8_t* __restrict__ mask, int B, int Ncam, int Nq, int R, int nchunks,
                   const int32_t* __restrict__ chunk_counts, int32_t* __restrict__ idx,
                   int32_t* __restrict__ count, int32_t* __restrict__ pos)
{
    __shared__ int s_base[kMaxCameras], s_total[kMaxCameras];
    __shared__ int s_wpre[kMaxCameras][32];
    const int chunk = blockIdx.x, b = blockIdx.y;
    const int q = chunk * kCompactChunk + threadIdx.x;
    const bool valid = q < Nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // seeing queries of camera `warp` in earlier chunks, and in all chunks
    if (warp < Ncam) {
        const int32_t* cc = chunk_counts + ((int64_t)b * Ncam + warp) * nchunks;
        int before = 0, all = 0;
        for (int i = lane; i < nchunks; i += 32) {
            const int v = cc[i];
            all += v;
            if (i < chunk) before += v;
        }
        before = warp_sum_int(before);
        all = warp_sum_int(all);
        if (lane == 0) {
            s_base[warp] = before;
            s_total[warp] = all;
            if (chunk == 0) count[(int64_t)b * Ncam + warp] = all;
        }
    }
    uint32_t hitbits = 0;
    for (int c = 0; c < Ncam; ++c) {
        const bool hit = valid && seen(mask, ((int64_t)c * B + b) * Nq + q, R);
        hitbits |= (uint32_t)hit << c;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        if (lane == 0) s_wpre[c][warp] = __popc(bal);
    }
    __syncthreads();
    if (warp < Ncam) {  // exclusive scan of the per-warp counts of camera `warp`
        const int v = s_wpre[warp][lane];
        s_wpre[warp][lane] = warp_inclusive_scan(v, lane) - v;
    }
    __syncthreads();
    const unsigned below = (1u << lane) - 1u;
    for (int c = 0; c < Ncam; ++c) {
        const bool hit = (hitbits >> c) & 1u;
        const unsigned bal = __ballot_sync(0xffffffffu, hit);
        const int64_t bc = (int64_t)b * Ncam + c;
        if (valid) {
            if (hit) {
                const int r = s_base[c] + s_wpre[c][warp] + __popc(bal & below);
                idx[bc * Nq + r] = q;
                pos[bc * Nq + q] = r;
            } else {
                pos[bc * Nq + q] = -1;
            }
            if (q >= s_total[c]) idx[bc * Nq + q] = -1;
        }
    }
}

cudaError_t launch_sca_compact(const uint8_t* mask, int B, int Ncam, int Nq, int R,
                               int32_t* idx, int32_t* count, int32_t* pos, int32_t* hits,
                               int32_t* chunk_counts, cudaStream_t s)
{
    if (B == 0) return cudaSuccess;
    const int nchunks = Nq > 0 ? (Nq + kCompactChunk - 1) / kCompactChunk : 1;
    const dim3 grid(nchunks, B);
    sca_count_kernel<<<grid, kCompactChunk, 0, s>>>(mask, B, Ncam, Nq, R, nchunks, hits,
                                                    chunk_counts);
    sca_scatter_kernel<<<grid, kCompactChunk, 0, s>>>(mask, B, Ncam, Nq, R, nchunks,
                                                      chunk_counts, idx, count, pos);
    return cudaGetLastError();
}

// Rows are ordered (b, c, i): at any time the whole GPU works on a narrow
// window of rows of one camera, so that camera's value stays in L2.  Offsets
// and logits come from the BEV query and are shared by its cameras; the
// reference points are the camera's own.
template <typename VT, int NC>
__global__ void __launch_bounds__(kThreads)
sca_gather_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                  const float* __restrict__ logits, const float* __restrict__ ref_cam,
                  const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                  float* __restrict__ out_rb, int B, int Ncam, int Nq, int Nv, int H, int L,
                  int P, int R, Levels levels)
{
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) WarpTable s_tab[kWarps];
    __shared__ int s_prefix[kMaxBatchCameras + 1];
    const int nbc = B * Ncam;
    stage_levels(s_lv, levels);
    stage_row_prefix(count, nbc, s_prefix);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t items = (int64_t)s_prefix[nbc] * H;
    const int64_t per_tile = (int64_t)kWarps * kScaRowsPerWarp;
    const int S = L * P;
    for (int64_t tile0 = (int64_t)blockIdx.x * per_tile; tile0 < items;
         tile0 += (int64_t)gridDim.x * per_tile) {
        for (int t = 0; t < kScaRowsPerWarp; ++t) {
            const int64_t item = tile0 + (int64_t)t * kWarps + warp;  // row * H + h
            if (item >= items) break;
            const int r = (int)(item / H), h = (int)(item % H);
            const int bc = find_segment(s_prefix, nbc, r);
            const int i = r - s_prefix[bc];
            const int b = bc / Ncam, c = bc - b * Ncam;
            const int q = __ldg(idx + (int64_t)bc * Nq + i);
            if ((unsigned)q >= (unsigned)Nq) continue;  // inconsistent lists: read nothing
            const int64_t bqh = ((int64_t)b * Nq + q) * H + h;
            const VT* vb = value + (int64_t)bc * Nv * H * kHeadDim;
            const float* rf = ref_cam + (((int64_t)c * B + b) * Nq + q) * R * 2;
            float* orow = out_rb + (((int64_t)bc * Nq + i) * H + h) * kHeadDim;
            row_forward<VT, true, NC>(vb, H, h, off + bqh * S * 2, logits + bqh * S, rf, L, P, R,
                                      s_lv, s_tab[warp], orow, lane);
        }
    }
}

template <typename K>
static int resident_ctas(K kernel, int threads)
{
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, threads, 0) != cudaSuccess || n < 1)
        n = 1;
    return n;
}

template <typename VT>
static cudaError_t launch_gather_t(const Problem& p, const float* ref_cam, const float* off,
                                   const float* logits, const int32_t* idx,
                                   const int32_t* count, float* out_rb, cudaStream_t s)
{
    const int64_t max_items = (int64_t)p.B * p.Ncam * p.Nq * p.H;
    if (max_items == 0) return cudaSuccess;
    const int64_t per_tile = (int64_t)kWarps * kScaRowsPerWarp;
    const int64_t max_tiles = (max_items + per_tile - 1) / per_tile;
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define SCA_GATHER_CASE(NCV)                                                                     \
    case NCV: {                                                                                  \
        static int occ = resident_ctas(sca_gather_kernel<VT, NCV>, kThreads);                    \
        const int64_t grid = std::min<int64_t>(max_tiles, (int64_t)occ * device_sm_count());     \
        sca_gather_kernel<VT, NCV><<<(unsigned)grid, kThreads, 0, s>>>(                          \
            v, off, logits, ref_cam, idx, count, out_rb, p.B, p.Ncam, p.Nq, p.Nv, p.H, p.L,      \
            p.P, p.R, p.lv);                                                                     \
        break;                                                                                   \
    }
    switch (nc) {
        SCA_GATHER_CASE(1)
        SCA_GATHER_CASE(2)
        SCA_GATHER_CASE(3)
        SCA_GATHER_CASE(4)
        default: return cudaErrorInvalidValue;
    }
#undef SCA_GATHER_CASE
    return cudaGetLastError();
}

cudaError_t launch_sca_gather(const Problem& p, const float* ref_cam, const float* off,
                              const float* logits, const int32_t* idx, const int32_t* count,
                              float* out_rb, cudaStream_t s)
{
    return p.bf16 ? launch_gather_t<__nv_bfloat16>(p, ref_cam, off, logits, idx, count, out_rb, s)
                  : launch_gather_t<float>(p, ref_cam, off, logits, idx, count, out_rb, s);
}

// One thread per 16-byte piece of an output row; cameras summed in ascending
// order, then divided by max(1, hits) (the clamp of the average listing).
__global__ void __launch_bounds__(256)
sca_average_kernel(const float4* __restrict__ out_rb, const int32_t* __restrict__ pos,
                   const int32_t* __restrict__ hits, int B, int Ncam, int Nq, int row4,
                   float4* __restrict__ out)
{
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t total = (int64_t)B * Nq * row4;
    if (t >= total) return;
    const int v4 = (int)(t % row4);
    const int64_t bq = t / row4;
    const int b = (int)(bq / Nq), q = (int)(bq - (int64_t)b * Nq);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c = 0; c < Ncam; ++c) {
        const int64_t bc = (int64_t)b * Ncam + c;
        const int p = __ldg(pos + bc * Nq + q);
        if (p >= 0) {
            const float4 x = out_rb[(bc * Nq + p) * row4 + v4];
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
        }
    }
    const float n = (float)max(1, __ldg(hits + bq));
    out[bq * row4 + v4] = make_float4(acc.x / n, acc.y / n, acc.z / n, acc.w / n);
}

cudaError_t launch_sca_average(const float* out_rb, const int32_t* pos, const int32_t* hits,
                               int B, int Ncam, int Nq, int H, float* out, cudaStream_t s)
{
    const int row4 = H * kHeadDim / 4;
    const int64_t total = (int64_t)B * Nq * row4;
    if (total == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((total + 255) / 256);
    sca_average_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(out_rb), pos, hits,
                                            B, Ncam, Nq, row4, reinterpret_cast<float4*>(out));
    return cudaGetLastError();
}

}  // namespace msda
