// SCA forward pieces (Tencent Cloud "Spatial Cross-Attention" walkthrough,
// rebatch and average listings; "BEV(三) BEVFormer ..." section 10):
//   K2a sca_count_kernel    seeing queries per (1024-query chunk, camera)
//   K2s sca_chunk_scan_kernel  per-camera prefix of the chunk counts, count
//                              (only above 64 chunks; below, K2b sums them)
//   K2b sca_scatter_kernel  stable ranks -> idx / pos, hits per query
//   K3  sca_gather_kernel   fused MSDA over every camera's seeing queries
//   K4  sca_average_kernel  per-query sum over cameras / max(1, hits)
// Nothing here synchronises with the host: the rebatched row counts live in
// device memory and K3 is a persistent kernel that reads them.
#include <algorithm>
#include <type_traits>

#include "msda_launch.h"

namespace msda {

constexpr int kScaRowsPerTile = MSDA_ROWS_PER_TILE;  // <= 32: a lane resolves each row

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

// A camera sees query q when any of its R anchor bytes is non-zero.  With
// `word` (R = 1, 2, 4 or 8 and the mask aligned to R bytes) the R bytes are
// read as one word.
__device__ __forceinline__ bool seen(const uint8_t* __restrict__ mask, int64_t at, int R,
                                     bool word)
{
    const uint8_t* p = mask + at * R;
    if (word) {
        switch (R) {
            case 1: return __ldg(p) != 0;
            case 2: return __ldg(reinterpret_cast<const unsigned short*>(p)) != 0;
            case 4: return __ldg(reinterpret_cast<const unsigned int*>(p)) != 0;
            case 8: return __ldg(reinterpret_cast<const unsigned long long*>(p)) != 0;
            default: break;
        }
    }
    bool hit = false;
    for (int r = 0; r < R; ++r) hit |= __ldg(p + r) != 0;
    return hit;
}

// One CTA per (1024-query chunk, batch-camera): the camera's seeing queries
// in the chunk.
__global__ void __launch_bounds__(kCompactChunk)
sca_count_kernel(const uint8_t* __restrict__ mask, int B, int Ncam, int Nq, int R, bool word,
                 int nchunks, int32_t* __restrict__ chunk_counts)
{
    __shared__ int s_cnt[kCompactChunk / 32];
    pdl_trigger();  // the scatter pass reads the counts only after its pdl_wait
    const int chunk = blockIdx.x, bc = blockIdx.y;
    const int b = bc / Ncam, c = bc - b * Ncam;
    const int q = chunk * kCompactChunk + threadIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool hit = q < Nq && seen(mask, ((int64_t)c * B + b) * Nq + q, R, word);
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) s_cnt[warp] = __popc(bal);
    __syncthreads();
    if (warp == 0) {
        const int v = warp_sum_int(lane < kCompactChunk / 32 ? s_cnt[lane] : 0);
        if (lane == 0) chunk_counts[(int64_t)bc * nchunks + chunk] = v;
    }
}

// Exclusive prefix of the per-chunk counts of one (batch, camera), in place,
// and the camera's total into count[bc]: one warp per (batch, camera), so the
// scatter pass reads one base per chunk instead of summing earlier chunks.
__global__ void __launch_bounds__(32)
sca_chunk_scan_kernel(int32_t* __restrict__ chunk_counts, int nchunks, int32_t* __restrict__ count)
{
    const int bc = blockIdx.x, lane = threadIdx.x;
    int32_t* cc = chunk_counts + (int64_t)bc * nchunks;
    int run = 0;
    for (int base = 0; base < nchunks; base += 32) {
        const int i = base + lane;
        const int v = i < nchunks ? cc[i] : 0;
        const int incl = warp_inclusive_scan(v, lane);
        if (i < nchunks) cc[i] = run + incl - v;
        run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) count[bc] = run;
}

// inline_scan (at most kInlineScanChunks chunks): the chunk counts are still
// per chunk, and warp 0 sums the camera's counts of the earlier chunks and of
// all chunks itself (the chunk-0 CTA writes count), so no scan pass runs
// between the count and scatter passes.  Otherwise chunk_base holds the scan
// pass's exclusive prefixes and count its totals.
constexpr int kInlineScanChunks = 64;

// One CTA per (chunk, batch-camera), as the count pass: the stable ranks of
// the camera's seeing queries -> idx / pos; the camera-0 CTAs also write the
// queries' hit counts.
__global__ void __launch_bounds__(kCompactChunk)
sca_scatter_kernel(const uint8_t* __restrict__ mask, int B, int Ncam, int Nq, int R, bool word,
                   int nchunks, const int32_t* __restrict__ chunk_base, int32_t* __restrict__ count,
                   int32_t* __restrict__ idx, int32_t* __restrict__ pos, int32_t* __restrict__ hits,
                   bool inline_scan)
{
    __shared__ int s_base, s_total;
    __shared__ int s_wpre[kCompactChunk / 32];
    const int chunk = blockIdx.x, bc = blockIdx.y;
    const int b = bc / Ncam, c = bc - b * Ncam;
    const int q = chunk * kCompactChunk + threadIdx.x;
    const bool valid = q < Nq;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    pdl_trigger();  // the gather reads the lists only after its pdl_wait
    // the mask part first: it does not depend on the passes before
    const bool hit = valid && seen(mask, ((int64_t)c * B + b) * Nq + q, R, word);
    const unsigned bal = __ballot_sync(0xffffffffu, hit);
    if (lane == 0) s_wpre[warp] = __popc(bal);
    int nh = hit;
    if (c == 0 && valid) {  // the query's seeing cameras, once per (b, q)
#pragma unroll 4
        for (int c2 = 1; c2 < Ncam; ++c2)
            nh += seen(mask, ((int64_t)c2 * B + b) * Nq + q, R, word);
    }
    // a programmatic dependent of the count (or scan) pass: the counts are
    // read, and the outputs written, only after that grid has completed
    pdl_wait();
    if (c == 0 && valid) hits[(int64_t)b * Nq + q] = nh;
    // seeing queries of the camera in earlier chunks, and in all chunks
    if (warp == 0) {
        if (inline_scan) {
            int before = 0, all = 0;
            for (int i = lane; i < nchunks; i += 32) {
                const int v = __ldg(chunk_base + (int64_t)bc * nchunks + i);
                all += v;
                if (i < chunk) before += v;
            }
            before = warp_sum_int(before);
            all = warp_sum_int(all);
            if (lane == 0) {
                s_base = before;
                s_total = all;
                if (chunk == 0) count[bc] = all;
            }
        } else if (lane == 0) {
            s_base = chunk_base[(int64_t)bc * nchunks + chunk];
            s_total = count[bc];
        }
    }
    __syncthreads();
    if (warp == 0) {  // exclusive scan of the per-warp counts
        const int v = s_wpre[lane];
        s_wpre[lane] = warp_inclusive_scan(v, lane) - v;
    }
    __syncthreads();
    if (valid) {
        const int64_t row0 = (int64_t)bc * Nq;
        if (hit) {
            const int r = s_base + s_wpre[warp] + __popc(bal & ((1u << lane) - 1u));
            idx[row0 + r] = q;
            pos[row0 + q] = r;
        } else {
            pos[row0 + q] = -1;
        }
        if (q >= s_total) idx[row0 + q] = -1;
    }
}

cudaError_t launch_sca_compact(const uint8_t* mask, int B, int Ncam, int Nq, int R,
                               int32_t* idx, int32_t* count, int32_t* pos, int32_t* hits,
                               int32_t* chunk_counts, cudaStream_t s)
{
    if (B == 0) return cudaSuccess;
    const int nchunks = Nq > 0 ? (Nq + kCompactChunk - 1) / kCompactChunk : 1;
    const bool word = (R == 1 || R == 2 || R == 4 || R == 8) && (uintptr_t)mask % R == 0;
    const dim3 grid(nchunks, B * Ncam);
    sca_count_kernel<<<grid, kCompactChunk, 0, s>>>(mask, B, Ncam, Nq, R, word, nchunks,
                                                    chunk_counts);
    const bool inline_scan = nchunks <= kInlineScanChunks;
    if (!inline_scan)
        sca_chunk_scan_kernel<<<B * Ncam, 32, 0, s>>>(chunk_counts, nchunks, count);
    // the scatter pass's mask loads overlap the end of the pass before it
    return launch_pdl(sca_scatter_kernel, grid, dim3(kCompactChunk), 0, s, mask, B, Ncam, Nq, R,
                      word, nchunks, chunk_counts, count, idx, pos, hits, inline_scan);
}

// Rows are ordered (b, c, i): at any time the whole GPU works on a narrow
// window of rows of one camera, so that camera's value stays in L2.  A CTA
// takes tiles of kScaRowsPerTile consecutive rows (with H = 8, one head per
// warp), so neighbouring queries' reads of the same head slices meet in L1.
// Offsets and logits come from the BEV query and are shared by its cameras;
// the reference points are the camera's own.
template <typename VT, int NC, int HP>
__global__ void MSDA_GATHER_BOUNDS(VT, NC)
sca_gather_kernel(const VT* __restrict__ value, const float* __restrict__ off,
                  const float* __restrict__ logits, const float* __restrict__ ref_cam,
                  const int32_t* __restrict__ idx, const int32_t* __restrict__ count,
                  float* __restrict__ out_rb, int B, int Ncam, int Nq, int Nv, int H, int L,
                  int P, int R, Levels levels)
{
    using Table = typename std::conditional<HP == 2, PairTable, WarpTable>::type;
    __shared__ SmemLevels s_lv;
    __shared__ __align__(16) Table s_tab[kWarps];
    __shared__ int s_prefix[kMaxBatchCameras + 1];
    const int nbc = B * Ncam;
    pdl_trigger();  // the average pass reads the rows only after its pdl_wait
    stage_levels(s_lv, levels);
    pdl_wait();  // the compaction lists are complete
    stage_row_prefix(count, nbc, Nq, s_prefix);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    LaneSamples<NC> ls;
    lane_samples<NC>(s_lv, L, P, R, lane, ls);
    const int S = L * P;
    const int total = s_prefix[nbc];
    const int HG = H / HP;  // head groups: one per warp item
    const int n_items = kScaRowsPerTile * HG;
    int bc_lane = 0;  // lane's (batch, camera) search start: its rows only grow

    struct Item {
        bool ok, skip;
        int h, bc, in_row, ref_row, out_row;
    };
#ifndef MSDA_GATHER_CHUNK
#define MSDA_GATHER_CHUNK 1  // consecutive tiles per CTA within each window of the row list
#endif
    constexpr int kChunk = MSDA_GATHER_CHUNK;
    for (int64_t tile = (int64_t)blockIdx.x * kChunk; tile * kScaRowsPerTile < total;
         tile = ((tile + 1) % kChunk) ? tile + 1 : tile + 1 + (int64_t)(gridDim.x - 1) * kChunk) {
        const int r0 = (int)(tile * kScaRowsPerTile);
        // lane i < kScaRowsPerTile resolves row r0 + i of the tile: one coalesced index load
        int my_bc = 0, my_in = -1, my_ref = 0, my_out = 0;
        {
            const int r = r0 + lane;
            if (lane < kScaRowsPerTile && r < total) {
                while (r >= s_prefix[bc_lane + 1]) ++bc_lane;
                const int i = r - s_prefix[bc_lane];
                const int b = bc_lane / Ncam, c = bc_lane - b * Ncam;
                const int q = __ldg(idx + (int64_t)bc_lane * Nq + i);
                if ((unsigned)q < (unsigned)Nq) {  // inconsistent lists: read nothing
                    my_bc = bc_lane;
                    my_in = b * Nq + q;
                    my_ref = (c * B + b) * Nq + q;
                    my_out = bc_lane * Nq + i;
                }
            }
        }
        auto resolve = [&](int it, const ItemCursor& cur) {
            Item x;
            const int rr = cur.rr;
            x.ok = it < n_items && r0 + rr < total;  // warp-uniform
            x.h = cur.h * HP;
            x.bc = __shfl_sync(0xffffffffu, my_bc, rr & 31);
            x.in_row = __shfl_sync(0xffffffffu, my_in, rr & 31);
            x.ref_row = __shfl_sync(0xffffffffu, my_ref, rr & 31);
            x.out_row = __shfl_sync(0xffffffffu, my_out, rr & 31);
            x.skip = x.in_row < 0;
            return x;
        };
        auto fetch = [&](const Item& x, RowIn<true, NC, HP>& in) {
            const int64_t bqh = (int64_t)x.in_row * H + x.h;
            load_row<true, NC, HP>(off + bqh * S * 2, logits + bqh * S,
                                   ref_cam + (int64_t)x.ref_row * R * 2, S, ls, lane, in);
        };
        ItemCursor cur(warp, HG);
        int it = warp;
        Item x0 = resolve(it, cur);
        RowIn<true, NC, HP> in0, in1;
        if (x0.ok && !x0.skip) fetch(x0, in0);
        while (x0.ok) {
            ItemCursor nx = cur;
            nx.next();
            const Item x1 = resolve(it + kWarps, nx);
            if (x1.ok && !x1.skip) fetch(x1, in1);  // next row's inputs in flight during this gather
            if (!x0.skip) {
                const VT* vb = value + (int64_t)x0.bc * Nv * H * kHeadDim;
                float* orow = out_rb + ((int64_t)x0.out_row * H + x0.h) * kHeadDim;
                if constexpr (HP == 2)
                    row_compute_pair<true, NC>(vb, H, x0.h, in0, S, ls, s_tab[warp], orow, lane);
                else
                    row_compute<VT, true, NC>(vb, H, x0.h, in0, S, ls, s_tab[warp], orow, lane);
            }
            x0 = x1;
            in0 = in1;
            cur = nx;
            it += kWarps;
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

template <typename VT, int HP>
static cudaError_t launch_gather_t(const Problem& p, const float* ref_cam, const float* off,
                                   const float* logits, const int32_t* idx,
                                   const int32_t* count, float* out_rb, cudaStream_t s)
{
    const int64_t max_items = (int64_t)p.B * p.Ncam * p.Nq * p.H;
    if (max_items == 0) return cudaSuccess;
    const int64_t max_rows = (int64_t)p.B * p.Ncam * p.Nq;
    const int64_t max_tiles = (max_rows + kScaRowsPerTile - 1) / kScaRowsPerTile;
    const VT* v = static_cast<const VT*>(p.value);
    const int nc = (p.L * p.P + 31) / 32;
#define SCA_GATHER_CASE(NCV)                                                                     \
    case NCV: {                                                                                  \
        static int occ = resident_ctas(sca_gather_kernel<VT, NCV, HP>, kThreads);                \
        const int64_t grid = std::min<int64_t>(max_tiles, (int64_t)occ * device_sm_count());     \
        const cudaError_t e = launch_pdl(sca_gather_kernel<VT, NCV, HP>, dim3((unsigned)grid),   \
                                         dim3(kThreads), 0, s, v, off, logits, ref_cam, idx,     \
                                         count, out_rb, p.B, p.Ncam, p.Nq, p.Nv, p.H, p.L, p.P,  \
                                         p.R, p.lv);                                             \
        if (e != cudaSuccess) return e;                                                          \
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

// Which gather serves rows of <= 32 samples: the four-lane kernel
// (sca_gather_quad.cu) measured faster for fp32 value (0.466 vs 0.498 ms on
// the BEVFormer-base step), the head-pair table kernel below for bf16 value
// (0.372 vs 0.417 ms).
#ifndef MSDA_GATHER_QUAD
#define MSDA_GATHER_QUAD 1
#endif
#ifndef MSDA_GATHER_QUAD_BF16
#define MSDA_GATHER_QUAD_BF16 0
#endif

cudaError_t launch_sca_gather(const Problem& p, const float* ref_cam, const float* off,
                              const float* logits, const int32_t* idx, const int32_t* count,
                              float* out_rb, cudaStream_t s)
{
    if ((p.bf16 ? MSDA_GATHER_QUAD_BF16 : MSDA_GATHER_QUAD) && sca_gather_quad_fits(p))
        return launch_sca_gather_quad(p, ref_cam, off, logits, idx, count, out_rb, s);
    if (!p.bf16) return launch_gather_t<float, 1>(p, ref_cam, off, logits, idx, count, out_rb, s);
    if (p.H % 2 == 0)
        return launch_gather_t<__nv_bfloat16, 2>(p, ref_cam, off, logits, idx, count, out_rb, s);
    return launch_gather_t<__nv_bfloat16, 1>(p, ref_cam, off, logits, idx, count, out_rb, s);
}

// One warp per (batch, query): lane c loads the query's position in camera c,
// a ballot gives the seeing cameras, and the warp reads their rows (fully
// coalesced, four cameras' loads in flight at a time), sums them in ascending
// camera order and divides by max(1, hits) (the clamp of the average listing).
constexpr int kAvgWarps = 8;
// Rows of up to 256 channels (PL <= 2): eight resident CTAs (32 registers)
// with one camera row in flight per warp measured faster than four CTAs with
// four rows in flight (0.0205 vs 0.0266 ms after the gather, BEVFormer-base):
// the positions -> rows chain is latency-bound, and more warps hide it.
#ifndef MSDA_AVG_MIN_BLOCKS
#define MSDA_AVG_MIN_BLOCKS 8  // resident CTAs asked of the register allocation (PL <= 2)
#endif
#ifndef MSDA_AVG_INFLIGHT
#define MSDA_AVG_INFLIGHT 2  // float4 per lane loaded together
#endif

// PL: float4 per lane (a power of two >= row4 / 32); rows of up to 16 heads.
// kAvgBatch cameras' rows are loaded together (MSDA_AVG_INFLIGHT float4 per
// lane in flight).  BF16: the mean is stored rounded to bf16 (to nearest
// even), the operand type of the output projection that follows it in the
// SCA module.
template <int PL, bool BF16>
__global__ void __launch_bounds__(kAvgWarps * 32, PL <= 2 ? MSDA_AVG_MIN_BLOCKS : 0)
sca_average_kernel(const float4* __restrict__ out_rb, const int32_t* __restrict__ pos,
                   const int32_t* __restrict__ hits, int B, int Ncam, int Nq, int row4,
                   void* __restrict__ out)
{
    constexpr int kAvgBatch = PL >= MSDA_AVG_INFLIGHT ? 1 : MSDA_AVG_INFLIGHT / PL;
    pdl_wait();  // the rows, positions and hit counts are complete
    const int lane = threadIdx.x & 31;
    const int64_t bq = (int64_t)blockIdx.x * kAvgWarps + (threadIdx.x >> 5);
    if (bq >= (int64_t)B * Nq) return;  // warp-uniform
    const int b = (int)(bq / Nq), q = (int)(bq - (int64_t)b * Nq);
    const int p = lane < Ncam ? __ldg(pos + ((int64_t)b * Ncam + lane) * Nq + q) : -1;
    unsigned seen = __ballot_sync(0xffffffffu, p >= 0);
    float4 acc[PL];
#pragma unroll
    for (int k = 0; k < PL; ++k) acc[k] = make_float4(0.f, 0.f, 0.f, 0.f);
    while (seen) {
        int cams[kAvgBatch], rows[kAvgBatch];
#pragma unroll
        for (int k = 0; k < kAvgBatch; ++k) {
            cams[k] = seen ? __ffs(seen) - 1 : -1;  // ascending camera order
            seen &= seen - 1;
            rows[k] = __shfl_sync(0xffffffffu, p, cams[k] < 0 ? 0 : cams[k]);
        }
        float4 x[kAvgBatch][PL];
#pragma unroll
        for (int k = 0; k < kAvgBatch; ++k)
#pragma unroll
            for (int e = 0; e < PL; ++e) {
                const int v4 = lane + 32 * e;
                x[k][e] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (cams[k] >= 0 && v4 < row4)
                    x[k][e] =
                        __ldcs(out_rb + (((int64_t)b * Ncam + cams[k]) * Nq + rows[k]) * row4 + v4);
            }
#pragma unroll
        for (int k = 0; k < kAvgBatch; ++k)
            if (cams[k] >= 0)
#pragma unroll
                for (int e = 0; e < PL; ++e) {
                    acc[e].x += x[k][e].x;
                    acc[e].y += x[k][e].y;
                    acc[e].z += x[k][e].z;
                    acc[e].w += x[k][e].w;
                }
    }
    const int hn = max(1, __ldg(hits + bq));
    // division by a power of two is the product with its exact reciprocal:
    // the same correctly rounded quotient without the division routine
    const bool pow2 = (hn & (hn - 1)) == 0;  // warp-uniform
    const float n = (float)hn;
    const float rn = __int_as_float((127 - (31 - __clz(hn))) << 23);
    auto quot = [&](float a) { return pow2 ? __fmul_rn(a, rn) : __fdiv_rn(a, n); };
#pragma unroll
    for (int e = 0; e < PL; ++e) {
        const int v4 = lane + 32 * e;
        if (v4 < row4) {
            const float4 m = make_float4(quot(acc[e].x), quot(acc[e].y), quot(acc[e].z),
                                         quot(acc[e].w));
            if constexpr (BF16) {
                const __nv_bfloat162 lo = __floats2bfloat162_rn(m.x, m.y);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(m.z, m.w);
                uint2 u;
                u.x = *reinterpret_cast<const uint32_t*>(&lo);
                u.y = *reinterpret_cast<const uint32_t*>(&hi);
                __stcs(static_cast<uint2*>(out) + bq * row4 + v4, u);
            } else {
                __stcs(static_cast<float4*>(out) + bq * row4 + v4, m);
            }
        }
    }
}

cudaError_t launch_sca_average(const float* out_rb, const int32_t* pos, const int32_t* hits,
                               int B, int Ncam, int Nq, int H, void* out, bool out_bf16,
                               cudaStream_t s)
{
    const int row4 = H * kHeadDim / 4;
    const int64_t rows = (int64_t)B * Nq;
    if (rows == 0) return cudaSuccess;
    const unsigned grid = (unsigned)((rows + kAvgWarps - 1) / kAvgWarps);
    const float4* in = reinterpret_cast<const float4*>(out_rb);
    const int pl = (row4 + 31) / 32;
#define SCA_AVG_CASE(PLV)                                                                        \
    if (pl <= PLV) {                                                                             \
        if (out_bf16)                                                                            \
            return launch_pdl(sca_average_kernel<PLV, true>, dim3(grid), dim3(kAvgWarps * 32), 0, \
                              s, in, pos, hits, B, Ncam, Nq, row4, out);                         \
        return launch_pdl(sca_average_kernel<PLV, false>, dim3(grid), dim3(kAvgWarps * 32), 0,   \
                          s, in, pos, hits, B, Ncam, Nq, row4, out);                             \
    }
    SCA_AVG_CASE(1)
    SCA_AVG_CASE(2)
    SCA_AVG_CASE(4)
    SCA_AVG_CASE(8)
    SCA_AVG_CASE(16)
#undef SCA_AVG_CASE
    return cudaErrorInvalidValue;
}

}  // namespace msda
