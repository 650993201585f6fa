// msda_linear: the dense projections around the MSDA sampling ("BEV(三)
// BEVFormer: how the Query interacts with the 8 Heads of the Feature",
// sections 3 (value projection W_v), 4.1 (offset head W_Delta), 4.2 (weight
// head W_alpha), 11 (output projection W_o) and 13 (residual)):
//   Y = X W^T (+ bias) (+ residual),  X [M, K] bf16, W [N, K] bf16 (the
//   nn.Linear weight layout), fp32 accumulation, Y fp32 or bf16.
//
// A persistent, warp-specialised kernel on the 5th-generation tensor cores,
// one CTA per SM, each walking output tiles of 128 x 256 (N-tile major, so a
// CTA keeps one N-tile for a run of M-tiles):
//   - warp 0 (one elected thread) loads the W tile of the whole K extent
//     (K <= 256) once per run of M-tiles, and streams X in 128 x 64 blocks
//     through a 4-stage shared-memory ring with TMA (128-byte swizzle);
//   - warp 1 (one thread) issues tcgen05.mma (M = 128, N = 256, K = 16, bf16
//     in, fp32 accumulate) into one of two 256-column TMEM accumulators and
//     commits each ring slot back to the loader and each finished tile to the
//     epilogue;
//   - warps 2-5 drain the other accumulator meanwhile: tcgen05.ld of their 32
//     TMEM lanes (tile rows), bias and residual added, the values written to
//     a swizzled shared-memory buffer and stored by TMA.
// So loads, tensor-core work and stores of consecutive tiles overlap.
//
// The SCA output projection can take its X from the camera average instead
// (sca_camera_average_linear; "BEV(三) ..." section 10 then 11-13): two more
// warps (6, 7) form the tile's 128 x K bf16 rows of X in shared memory from
// the rebatched rows, X[b * Nq + q] = bf16(sum over the query's cameras, in
// ascending order, of its rebatched rows / max(1, hits)), in the layout the
// TMA would have written, so the averaged queries never go through HBM.
//
// Every mbarrier wait is bounded: a wait that gives up counts a timeout in a device
// word (msda_linear_timeouts), raises a CTA-wide stop flag that makes the
// other roles leave their loops, and the CTA still waits (bounded) for its
// copies in flight and frees its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "msda.h"
#include "msda_launch.h"

namespace msda {
namespace {

constexpr int kBM = 128;   // tile rows (TMEM lanes)
constexpr int kBN = 256;   // tile columns (TMEM columns, fp32)
constexpr int kBK = 64;    // one 128-byte swizzle row of bf16
constexpr int kMaxK = 256;
constexpr int kMaxKBlocks = kMaxK / kBK;
constexpr int kStages = 4;                          // X ring slots
constexpr int kGemmThreads = 192;                   // 6 warps
constexpr int kAvgThreads = 256;                    // + 2 warps forming X (64 rows each;
                                                    // 8 warps keep 255 registers a thread)
constexpr int kAvgProducers = 64;
constexpr int kMaxAvgCams = 8;                      // cameras of the averaged X
constexpr int kAvgRowsPerBatch = 8;                 // rows whose source loads fly together
constexpr uint32_t kABlockBytes = kBM * kBK * 2;    // 16 KB
constexpr uint32_t kBBlockBytes = kBN * kBK * 2;    // 32 KB
constexpr uint32_t kCBufBytes = 32 * 128;           // 32 rows x 128 bytes
constexpr uint32_t kSpinLimit = 1u << 24;           // mbarrier polls before giving up
constexpr uint64_t kWaitNs = 2000000000ull;         // ... or 2 s of wall time

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16
// = 0), N / 8 in bits 17-22, M / 16 in bits 24-28.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

struct __align__(8) Ctrl {
    uint64_t full[kStages];    // X slot loaded (TMA bytes)
    uint64_t empty[kStages];   // X slot consumed (tcgen05.commit)
    uint64_t b_full;           // W tile loaded
    uint64_t b_free;           // the MMAs of a W tile's run are done
    uint64_t acc_full[2];      // accumulator ready for the epilogue
    uint64_t acc_empty[2];     // accumulator drained (4 epilogue warps)
    uint64_t drain;            // every MMA issued so far has finished (stop path)
    uint32_t tmem_base;
    volatile int stop;
};

// Where the averaged X comes from: out_rb [B, Ncam, Nq, K] fp32, pos
// [B, Ncam, Nq] (row of query q in camera c, or -1), hits [B, Nq].
struct AvgArgs {
    const float* rows;
    const int32_t* pos;
    const int32_t* hits;
    int Ncam, Nq;
};

// Shared memory: W (K/64 blocks of 256 x 64), the X ring, 4 warps x 2
// epilogue buffers, the bias (a plain bias of N = 256), then the control
// block; 1024-byte aligned.
constexpr size_t kSmemB = (size_t)kMaxKBlocks * kBBlockBytes;   // 128 KB
constexpr size_t kSmemA = (size_t)kStages * kABlockBytes;       // 64 KB
constexpr size_t kSmemC = (size_t)4 * 2 * kCBufBytes;           // 32 KB
constexpr size_t kSmemBias = (size_t)kBN * 4;                     // 1 KB: the bias of N = 256
constexpr size_t kSmemBytes = 1024 + kSmemB + kSmemA + kSmemC + kSmemBias + sizeof(Ctrl);
static_assert(kSmemBytes <= 227 * 1024, "shared memory of the projection kernel");
static_assert((kStages & (kStages - 1)) == 0 && kStages >= kMaxKBlocks,
              "a tile's K-blocks fit the ring, whose size is a power of two");

__device__ unsigned int g_gemm_timeouts = 0;
// Test switch of the bounded-wait path (msda_linear_test_withhold_load): when
// set, CTA 0 of the next launch clears it and holds back its first X-tile
// load, so that its tensor-core wait runs out.
__device__ int g_gemm_withhold = 0;

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait for the completion of phase `parity`; false after kSpinLimit polls,
// after kWaitNs of wall time, or once `stop` is raised (when given).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          const volatile int* stop = nullptr)
{
    uint64_t t0 = 0;
    for (uint32_t i = 0; i < kSpinLimit; ++i) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n"
            " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(smem_u32(bar)), "r"(parity)
            : "memory");
        if (done) return true;
        if ((i & 255) == 0) {
            const uint64_t t = global_ns();
            if (i == 0) t0 = t;
            else if (t - t0 > kWaitNs) return false;
            if (stop && *stop) return false;
        }
    }
    return false;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y, const void* src)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(smem_u32(src))
        : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void fence_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major operand in the 128-byte
// swizzle layout: rows of 128 bytes, groups of 8 rows 1024 bytes apart.
// Start address >> 4 in bits 0-13, leading offset (unused here, 16 B) >> 4 in
// bits 16-29, stride offset (1024 B) >> 4 in bits 32-45, descriptor version 1
// in bits 46-47, swizzle mode 2 (128 B) in bits 61-63.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(16u >> 4) << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
        " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kInstrDesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b)
{
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Training-time dropout of the projection ("BEV(三) ..." section 12): element
// e = row * N + col keeps its value when word e mod 4 of Philox4x32-10
// (Salmon et al., SC 2011) at counter (e div 4, 0, 0) and key `seed` is at
// least `thr` (= floor(p * 2^32)), scaled by 1 / (1 - p); else it is 0.
struct Dropout {
    uint32_t thr;
    float scale;
    uint32_t key0, key1;
    int on;
};

// A bias per (camera, level) instead of per column ("BEV(三) ..." section 3:
// F~ = F + e_cam + e_level, and (F + e) W^T = F W^T + e W^T): row r of X is
// pixel v = r mod nv of camera (r div nv) mod ncam, and its level is the last
// l with start[l] <= v; the bias row is table[(camera * L + level) * N].
struct RowBias {
    const float* table;  // [ncam * L, N] or null (then the plain bias)
    int nv, ncam, L;
    int start[8];
};

__device__ __forceinline__ const float* row_bias(const RowBias& rb, int64_t row, int N)
{
    const int64_t v = row % rb.nv;
    const int c = (int)((row / rb.nv) % rb.ncam);
    int l = 0;
#pragma unroll
    for (int i = 1; i < 8; ++i)
        if (i < rb.L && rb.start[i] <= v) l = i;
    return rb.table + ((int64_t)c * rb.L + l) * N;
}

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1)
{
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        const uint32_t hi0 = __umulhi(0xD2511F53u, c.x), lo0 = 0xD2511F53u * c.x;
        const uint32_t hi1 = __umulhi(0xCD9E8D57u, c.z), lo1 = 0xCD9E8D57u * c.z;
        c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
        k0 += 0x9E3779B9u;
        k1 += 0xBB67AE85u;
    }
    return c;
}

// Dropout of the 32 values v of columns col .. col + 31 of `row`.
__device__ __forceinline__ void apply_dropout(float (&v)[32], int64_t row, int col, int N,
                                              const Dropout& d)
{
    const uint64_t blk0 = (uint64_t)(row * N + col) >> 2;  // col is a multiple of 32
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint64_t blk = blk0 + i;
        const uint4 u = philox4x32_10(make_uint4((uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u),
                                      d.key0, d.key1);
        v[4 * i] = u.x >= d.thr ? v[4 * i] * d.scale : 0.f;
        v[4 * i + 1] = u.y >= d.thr ? v[4 * i + 1] * d.scale : 0.f;
        v[4 * i + 2] = u.z >= d.thr ? v[4 * i + 2] * d.scale : 0.f;
        v[4 * i + 3] = u.w >= d.thr ? v[4 * i + 3] * d.scale : 0.f;
    }
}

__device__ __forceinline__ void note_timeout(Ctrl& ctrl)
{
    if (!ctrl.stop) atomicAdd(&g_gemm_timeouts, 1u);
    ctrl.stop = 1;
}

// One 32-row x 128-byte epilogue chunk of thread `lane` (its row) into the
// 128-byte-swizzled buffer the TMA store reads: 16-byte unit c of row r sits
// at unit c ^ (r mod 8).
__device__ __forceinline__ void put_row(uint8_t* buf, int lane, const uint32_t (&u)[32])
{
    uint8_t* row = buf + lane * 128;
#pragma unroll
    for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(row + ((c ^ (lane & 7)) << 4)) =
            make_uint4(u[4 * c], u[4 * c + 1], u[4 * c + 2], u[4 * c + 3]);
}

// Eight fp32 values (32 bytes, read once: no L1 allocation) when `on`; else
// v keeps what it holds.  A predicated load, no branch, so that a batch's
// loads all leave before the first is used.
__device__ __forceinline__ void load8_stream(const float* p, bool on, float (&v)[8])
{
    asm volatile(
        "{\n .reg .pred q;\n setp.ne.b32 q, %9, 0;\n"
        " @q ld.global.nc.L1::no_allocate.v8.f32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];\n}\n"
        : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]),
          "+f"(v[7])
        : "l"(p), "r"((int)on));
}

// One tile row's sources in ascending camera order (global rows of out_rb),
// their number and the divisor max(1, hits).
struct AvgRow {
    int src[kMaxAvgCams];
    int n;
    int div;  // max(1, hits)
};

// The raw lists of tile row bq (its camera positions and hits), loaded ahead
// of their use.
struct AvgRaw {
    int pos[kMaxAvgCams];
    int hits;
};

__device__ __forceinline__ void avg_load_raw(AvgRaw& raw, const AvgArgs& a, int bq, int M)
{
#pragma unroll
    for (int c = 0; c < kMaxAvgCams; ++c) raw.pos[c] = -1;
    raw.hits = 0;
    if (bq < M) {
        const int b = bq / a.Nq, q = bq - b * a.Nq;
#pragma unroll
        for (int c = 0; c < kMaxAvgCams; ++c)
            if (c < a.Ncam) raw.pos[c] = __ldg(a.pos + ((int64_t)b * a.Ncam + c) * a.Nq + q);
        raw.hits = __ldg(a.hits + bq);
    }
}

__device__ __forceinline__ void avg_compact(AvgRow& row, const AvgRaw& raw, const AvgArgs& a,
                                            int bq, int M)
{
    row.n = 0;
#pragma unroll
    for (int c = 0; c < kMaxAvgCams; ++c) row.src[c] = 0;
    if (bq < M) {
        const int b = bq / a.Nq;
#pragma unroll
        for (int c = 0; c < kMaxAvgCams; ++c) {
            if ((unsigned)raw.pos[c] < (unsigned)a.Nq) {
                // row.n <= c: compile-time-indexed selects keep src in registers
#pragma unroll
                for (int k = 0; k <= c; ++k)
                    if (k == row.n) row.src[k] = (b * a.Ncam + c) * a.Nq + raw.pos[c];
                ++row.n;
            }
        }
    }
    row.div = max(1, raw.hits);
}

// 32 tile rows of a producer warp (tile row r0 + i is held by lane i:
// its sources in ascending camera order as global rows of out_rb, their
// number n and the divisor) into the X slots of the tile: lane l forms
// channels 8l .. 8l + 7 of every row (one coalesced K * 4-byte read per
// source row), bf16 unit l mod 8 of the row in K-block l / 8, written where
// the 128-byte-swizzled TMA layout puts it (unit u of row r at u ^ (r mod 8)).
// The sum runs over the sources in order from 0, then one IEEE division by
// max(1, hits), then round to nearest even: the camera average's arithmetic.
__device__ __forceinline__ void avg_rows(uint8_t* sa, int s0, const float* rows,
                                         const AvgRow& t, int K, int rbase, int lane)
{
    const bool active = 8 * lane < K;
    const int u = lane & 7;
    // K-block lane / 8 sits in ring slot (s0 + lane / 8) mod 4
    uint8_t* slot = sa + ((s0 + (lane >> 3)) & (kStages - 1)) * kABlockBytes;
    const float* col = rows + 8 * lane;
#pragma unroll 1
    for (int r0 = 0; r0 < 32; r0 += kAvgRowsPerBatch) {
        float x[kAvgRowsPerBatch][2][8];  // the first two sources of the batch's rows
        int nr[kAvgRowsPerBatch];
#pragma unroll
        for (int a = 0; a < kAvgRowsPerBatch; ++a) {
            nr[a] = __shfl_sync(0xffffffffu, t.n, r0 + a);
#pragma unroll
            for (int s = 0; s < 2; ++s) {
                const int row = __shfl_sync(0xffffffffu, t.src[s], r0 + a);
#pragma unroll
                for (int e = 0; e < 8; ++e) x[a][s][e] = 0.f;
                load8_stream(col + (int64_t)row * K, s < nr[a] && active, x[a][s]);
            }
        }
#pragma unroll
        for (int a = 0; a < kAvgRowsPerBatch; ++a) {
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll
            for (int s = 0; s < 2; ++s)
                if (s < nr[a])
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] += x[a][s][e];
            if (nr[a] > 2) {  // warp-uniform: more than two seeing cameras
                float y[kMaxAvgCams - 2][8];
#pragma unroll
                for (int s = 2; s < kMaxAvgCams; ++s) {
                    const int row = __shfl_sync(0xffffffffu, t.src[s], r0 + a);
#pragma unroll
                    for (int e = 0; e < 8; ++e) y[s - 2][e] = 0.f;
                    load8_stream(col + (int64_t)row * K, s < nr[a] && active, y[s - 2]);
                }
#pragma unroll
                for (int s = 2; s < kMaxAvgCams; ++s)
                    if (s < nr[a])
#pragma unroll
                        for (int e = 0; e < 8; ++e) v[e] += y[s - 2][e];
            }
            const int d = __shfl_sync(0xffffffffu, t.div, r0 + a);
            // v / d, correctly rounded: for d a power of two the product with
            // the exact 1 / d is the same number, without the division routine
            if ((d & (d - 1)) == 0) {  // warp-uniform
                const float rd = __int_as_float((127 - (31 - __clz(d))) << 23);
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], rd);
            } else {
                const float df = (float)d;
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = __fdiv_rn(v[e], df);
            }
            if (active) {
                const int r = rbase + r0 + a;
                const uint4 o = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                           pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
                *reinterpret_cast<uint4*>(slot + r * 128 + ((u ^ (r & 7)) << 4)) = o;
            }
        }
    }
}

template <bool AVG>
__global__ void __launch_bounds__(AVG ? kAvgThreads : kGemmThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                 const __grid_constant__ CUtensorMap map_y, const float* __restrict__ bias,
                 const float* __restrict__ residual, int y_bf16, int M, int N, int K, Dropout drop,
                 RowBias rbias, AvgArgs avg)
{
    constexpr int STAGES = kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sb = smem;
    uint8_t* sa = sb + kSmemB;
    uint8_t* sc = sa + kSmemA;
    float* s_bias = reinterpret_cast<float*>(sc + kSmemC);
    Ctrl& ctrl = *reinterpret_cast<Ctrl*>(sc + kSmemC + kSmemBias);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kblocks = K / kBK;
    const int mt = (M + kBM - 1) / kBM;
    const int ntiles = mt * (N / kBN);

    if (threadIdx.x == 0) {
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(&ctrl.full[i], AVG ? kAvgProducers : 1);
            mbar_init(&ctrl.empty[i], 1);
        }
        mbar_init(&ctrl.b_full, 1);
        mbar_init(&ctrl.b_free, 1);
        mbar_init(&ctrl.drain, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ctrl.acc_full[i], 1);
            mbar_init(&ctrl.acc_empty[i], 4);
        }
        ctrl.stop = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctrl.tmem_base)),
                     "r"(2 * kBN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = ctrl.tmem_base;

    if (warp == 0) {
        // ---- loader ----
        if (lane == 0) {
            int stage = 0, cur_n = -1, b_loads = 0;
            uint32_t phase = 0, free_phase = 0;
            int issued[kStages];  // parity of each slot's last load, -1 = none
            for (int i = 0; i < kStages; ++i) issued[i] = -1;
            // the test switch: withhold the first X-tile load (its slot's
            // barrier is then never completed, and nothing is in flight to it)
            bool withhold = blockIdx.x == 0 && atomicExch(&g_gemm_withhold, 0) != 0;
            for (int tile = blockIdx.x; tile < ntiles && !ctrl.stop; tile += gridDim.x) {
                const int m0 = (tile % mt) * kBM, n_tile = tile / mt;
                if (n_tile != cur_n) {
                    if (cur_n >= 0) {
                        if (!mbar_wait(&ctrl.b_free, free_phase, &ctrl.stop)) {
                            note_timeout(ctrl);
                            break;
                        }
                        free_phase ^= 1;
                    }
                    mbar_expect_tx(&ctrl.b_full, (uint32_t)kblocks * kBBlockBytes);
                    for (int kb = 0; kb < kblocks; ++kb)
                        tma_load_2d(sb + kb * kBBlockBytes, &map_w, kb * kBK, n_tile * kBN,
                                    &ctrl.b_full);
                    ++b_loads;
                    cur_n = n_tile;
                }
                if constexpr (!AVG) {  // else X is formed by the producer warps
                    for (int kb = 0; kb < kblocks; ++kb) {
                        if (!mbar_wait(&ctrl.empty[stage], phase ^ 1, &ctrl.stop)) {
                            note_timeout(ctrl);
                            break;
                        }
                        if (withhold) {
                            withhold = false;
                        } else {
                            mbar_expect_tx(&ctrl.full[stage], kABlockBytes);
                            tma_load_2d(sa + stage * kABlockBytes, &map_x, kb * kBK, m0,
                                        &ctrl.full[stage]);
                            issued[stage] = (int)phase;
                        }
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1;
                        }
                    }
                }
            }
            // On a stop, give the copies still in flight a bounded chance to land.
            if (ctrl.stop) {
                for (int i = 0; i < STAGES; ++i)
                    if (issued[i] >= 0) mbar_wait(&ctrl.full[i], (uint32_t)issued[i]);
                if (b_loads > 0) mbar_wait(&ctrl.b_full, (uint32_t)((b_loads - 1) & 1));
            }
        }
    } else if (warp == 1) {
        // ---- tensor-core issuer ----
        if (lane == 0) {
            int stage = 0, acc = 0, cur_n = -1;
            uint32_t phase = 0, acc_phase = 0, b_phase = 0;
            for (int tile = blockIdx.x; tile < ntiles && !ctrl.stop; tile += gridDim.x) {
                const int n_tile = tile / mt;
                if (n_tile != cur_n) {
                    if (!mbar_wait(&ctrl.b_full, b_phase, &ctrl.stop)) {
                        note_timeout(ctrl);
                        break;
                    }
                    b_phase ^= 1;
                    cur_n = n_tile;
                }
                if (!mbar_wait(&ctrl.acc_empty[acc], acc_phase ^ 1, &ctrl.stop)) {
                    note_timeout(ctrl);
                    break;
                }
                asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
                const uint32_t d = tmem + (uint32_t)(acc * kBN);
                bool ok = true;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(&ctrl.full[stage], phase, &ctrl.stop)) {
                        note_timeout(ctrl);
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
                    for (int ks = 0; ks < kBK / 16; ++ks) {
                        const uint64_t ad = smem_desc_sw128(smem_u32(sa + stage * kABlockBytes) + ks * 32);
                        const uint64_t bd = smem_desc_sw128(smem_u32(sb + kb * kBBlockBytes) + ks * 32);
                        umma_bf16(d, ad, bd, (kb | ks) != 0);
                    }
                    umma_commit(&ctrl.empty[stage]);  // the slot is free once these MMAs finish
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                umma_commit(&ctrl.acc_full[acc]);
                const int next = tile + gridDim.x;
                if (next < ntiles && next / mt != n_tile) umma_commit(&ctrl.b_free);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (ctrl.stop) {  // TMEM is freed below: let issued MMAs finish first
                umma_commit(&ctrl.drain);
                mbar_wait(&ctrl.drain, 0);
            }
        }
    } else if (AVG && warp >= 6) {
        // ---- X producers: warps 6, 7; warp w forms tile rows 64w .. 64w + 63 ----
        // Each warp works on its own: one lane waits for the tile's slots and
        // the warp takes its verdict, so a stop leaves no warp behind.  The
        // lists of the warp's next tile are loaded while it forms this one.
        const int rbase = 64 * (warp - 6);
        int stage = 0;
        uint32_t phase = 0;
        AvgRaw raw[2];
        int tile = blockIdx.x;
        if (tile < ntiles) {
            const int m0 = (tile % mt) * kBM;
            avg_load_raw(raw[0], avg, m0 + rbase + lane, M);
            avg_load_raw(raw[1], avg, m0 + rbase + 32 + lane, M);
        }
        for (; tile < ntiles; tile += gridDim.x) {
            const int m0 = (tile % mt) * kBM;
            AvgRow cur[2];
            avg_compact(cur[0], raw[0], avg, m0 + rbase + lane, M);
            avg_compact(cur[1], raw[1], avg, m0 + rbase + 32 + lane, M);
            const int next = tile + gridDim.x;
            if (next < ntiles) {
                const int mn = (next % mt) * kBM;
                avg_load_raw(raw[0], avg, mn + rbase + lane, M);
                avg_load_raw(raw[1], avg, mn + rbase + 32 + lane, M);
            }
            // the tile's K-blocks go to the next kblocks ring slots (from s0,
            // wrapping), as the tensor-core issuer takes them
            const int s0 = stage;
            bool ok = true;
            for (int kb = 0; kb < kblocks; ++kb) {
                if (lane == 0 && ok) ok = mbar_wait(&ctrl.empty[stage], phase ^ 1, &ctrl.stop);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1;
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) {
                if (lane == 0) note_timeout(ctrl);
                break;
            }
            avg_rows(sa, s0, avg.rows, cur[0], K, rbase, lane);
            avg_rows(sa, s0, avg.rows, cur[1], K, rbase + 32, lane);
            fence_async_smem();  // the generic-proxy writes, seen by the tensor cores
            for (int kb = 0; kb < kblocks; ++kb) mbar_arrive(&ctrl.full[(s0 + kb) & (STAGES - 1)]);
        }
    } else if (warp < 6) {
        // ---- epilogue: warps 2..5, TMEM lane quarter q = warp % 4 ----
        const int q = warp & 3;
        uint8_t* cbuf = sc + (size_t)q * 2 * kCBufBytes;
        // a plain bias of one W tile (N = 256) is read from shared memory:
        // staged once by the four epilogue warps, before any of their waits
        const bool bias_smem = bias != nullptr && rbias.table == nullptr && N == kBN;
        if (bias_smem) {
            for (int i = (warp - 2) * 32 + lane; i < kBN; i += 128) s_bias[i] = __ldg(bias + i);
            asm volatile("bar.sync 1, 128;" ::: "memory");
        }
        int acc = 0, buf = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < ntiles; tile += gridDim.x) {
            const int m0 = (tile % mt) * kBM, n0 = (tile / mt) * kBN;
            if (!mbar_wait(&ctrl.acc_full[acc], acc_phase, &ctrl.stop)) {
                if (lane == 0) note_timeout(ctrl);
                break;
            }
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            const int row = m0 + q * 32 + lane;
            const bool row_ok = row < M;
            const bool block_ok = m0 + q * 32 < M;
            const uint32_t taddr = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kBN);
            const int cols = y_bf16 ? 64 : 32;  // columns per 128-byte store row
            for (int c0 = 0; c0 < kBN; c0 += cols) {
                uint32_t u[32];
                for (int half = 0; half < cols / 32; ++half) {
                    uint32_t r[32];
                    tmem_ld32(taddr + (uint32_t)(c0 + 32 * half), r);
                    float v[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                    const int col = n0 + c0 + 32 * half;
                    const float* brow = bias_smem ? s_bias - n0 : bias;
                    if (rbias.table) brow = row_ok ? row_bias(rbias, row, N) : nullptr;
                    if (bias_smem) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 b4 = *reinterpret_cast<const float4*>(brow + col + j);
                            v[j] += b4.x; v[j + 1] += b4.y; v[j + 2] += b4.z; v[j + 3] += b4.w;
                        }
                    } else if (brow) {
#pragma unroll
                        for (int j = 0; j < 32; j += 4) {
                            const float4 b4 = __ldg(reinterpret_cast<const float4*>(brow + col + j));
                            v[j] += b4.x; v[j + 1] += b4.y; v[j + 2] += b4.z; v[j + 3] += b4.w;
                        }
                    }
                    if (drop.on) apply_dropout(v, row, col, N, drop);
                    if (residual && row_ok) {
                        const float4* rp = reinterpret_cast<const float4*>(residual + (int64_t)row * N + col);
#pragma unroll
                        for (int j = 0; j < 8; ++j) {
                            const float4 t = __ldcs(rp + j);
                            v[4 * j] += t.x; v[4 * j + 1] += t.y; v[4 * j + 2] += t.z; v[4 * j + 3] += t.w;
                        }
                    }
                    if (y_bf16) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) u[16 * half + j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) u[j] = __float_as_uint(v[j]);
                    }
                }
                // the buffer written two chunks ago must have been read by its store
                if (lane == 0) bulk_wait_read<1>();
                __syncwarp();
                uint8_t* b = cbuf + buf * kCBufBytes;
                put_row(b, lane, u);
                fence_async_smem();
                __syncwarp();
                if (lane == 0 && block_ok) {
                    tma_store_2d(&map_y, n0 + c0, m0 + q * 32, b);
                    bulk_commit();
                }
                buf ^= 1;
            }
            asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(&ctrl.acc_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
        }
        if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
        __syncwarp();
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        __syncwarp();
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * kBN)
                     : "memory");
    }
}

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                 const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                 const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                 CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encode_tiled()
{
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

// A [rows, K] bf16 row-major matrix read in boxes of (box_rows x 64).
bool make_map(CUtensorMap* map, const void* base, int rows, int K, int box_rows)
{
    EncodeTiled enc = encode_tiled();
    if (enc == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kBK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

// Y [M, N] (fp32 or bf16) written in boxes of 32 rows x 128 bytes.
bool make_store_map(CUtensorMap* map, void* base, int M, int N, bool bf16)
{
    EncodeTiled enc = encode_tiled();
    if (enc == nullptr) return false;
    const int elem = bf16 ? 2 : 4;
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)N * elem};
    const cuuint32_t box[2] = {(cuuint32_t)(128 / elem), 32};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
               base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace msda

namespace msda {

// Bias table of the embedding prologue: table[c * L + l, n] = b[n] +
// sum_k (e_cam[c, k] + e_level[l, k]) w[n, k] (double accumulation; either
// embedding may be null).  One thread per table entry.
__global__ void embed_bias_kernel(const float* __restrict__ e_cam, const float* __restrict__ e_lvl,
                                  const __nv_bfloat16* __restrict__ w, const float* __restrict__ b,
                                  int ncam, int L, int N, int K, float* __restrict__ table)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (int64_t)ncam * L * N) return;
    const int n = (int)(i % N);
    const int cl = (int)(i / N);
    const int c = cl / L, l = cl - c * L;
    double acc = b ? (double)b[n] : 0.0;
    for (int k = 0; k < K; ++k) {
        const float e = (e_cam ? e_cam[(int64_t)c * K + k] : 0.f) +
                        (e_lvl ? e_lvl[(int64_t)l * K + k] : 0.f);
        acc += (double)e * (double)__bfloat162float(w[(int64_t)n * K + k]);
    }
    table[i] = (float)acc;
}

cudaError_t launch_embed_bias(const float* e_cam, const float* e_lvl, const void* w,
                              const float* b, int ncam, int L, int N, int K, float* table,
                              cudaStream_t s)
{
    const int64_t n = (int64_t)ncam * L * N;
    if (n == 0) return cudaSuccess;
    embed_bias_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(
        e_cam, e_lvl, static_cast<const __nv_bfloat16*>(w), b, ncam, L, N, K, table);
    return cudaGetLastError();
}

msda_status_t linear_impl(const void* x, const void* w, const float* bias, const float* residual,
                          int32_t M, int32_t N, int32_t K, msda_dtype_t y_dtype, void* y,
                          float dropout_p, uint64_t dropout_seed, const RowBiasArgs* rb,
                          cudaStream_t stream);

}  // namespace msda

extern "C" msda_status_t msda_linear_dropout(const void* x, const void* w, const float* bias,
                                             const float* residual, int32_t M, int32_t N,
                                             int32_t K, msda_dtype_t y_dtype, void* y,
                                             float dropout_p, uint64_t dropout_seed,
                                             msda_stream_t stream)
{
    return msda::linear_impl(x, w, bias, residual, M, N, K, y_dtype, y, dropout_p, dropout_seed,
                             nullptr, (cudaStream_t)stream);
}

namespace msda {
namespace {

// Checks shared by both X sources; then the launch.  avg null: X from x by
// TMA; else X is the camera average of avg's rebatched rows (x unused).
msda_status_t launch_projection(const void* x, const AvgArgs* avg, const void* w,
                                const float* bias, const float* residual, int32_t M, int32_t N,
                                int32_t K, msda_dtype_t y_dtype, void* y, float dropout_p,
                                uint64_t dropout_seed, const RowBiasArgs* rb, cudaStream_t stream)
{
    if (!(dropout_p >= 0.f && dropout_p < 1.f))
        return api_fail(MSDA_ERR_INVALID_ARG, "dropout_p must be in [0, 1)");
    if (M < 0) return api_fail(MSDA_ERR_INVALID_ARG, "M must be >= 0");
    if (N < kBN || N % kBN != 0)
        return api_fail(MSDA_ERR_UNSUPPORTED, "N must be a positive multiple of 256");
    if (K < kBK || K > kMaxK || K % kBK != 0)
        return api_fail(MSDA_ERR_UNSUPPORTED, "K must be 64, 128, 192 or 256");
    if (y_dtype != MSDA_F32 && y_dtype != MSDA_BF16)
        return api_fail(MSDA_ERR_INVALID_ARG, "unknown output dtype");
    if (M == 0) return api_ok();
    if (M > INT32_MAX - 2 * kBM) return api_fail(MSDA_ERR_UNSUPPORTED, "M too large");
    auto bad = [](const void* p) { return p == nullptr || ((uintptr_t)p & 15) != 0; };
    if ((avg == nullptr && bad(x)) || bad(w) || bad(y))
        return api_fail(MSDA_ERR_INVALID_ARG, "x, w and y must be non-null and 16-byte aligned");
    if ((bias && ((uintptr_t)bias & 15)) || (residual && ((uintptr_t)residual & 15)))
        return api_fail(MSDA_ERR_INVALID_ARG, "bias and residual must be 16-byte aligned");
    CUtensorMap mx, mw, my;
    if ((avg == nullptr && !make_map(&mx, x, M, K, kBM)) || !make_map(&mw, w, N, K, kBN) ||
        !make_store_map(&my, y, M, N, y_dtype == MSDA_BF16))
        return api_fail(MSDA_ERR_CUDA, "cuTensorMapEncodeTiled failed or is unavailable");
    if (avg) mx = mw;  // not read
    const int64_t ntiles = (int64_t)((M + kBM - 1) / kBM) * (N / kBN);
    const unsigned grid = (unsigned)std::min<int64_t>(ntiles, device_sm_count());
    Dropout drop;
    drop.on = dropout_p > 0.f;
    drop.thr = (uint32_t)((double)dropout_p * 4294967296.0);
    drop.scale = (float)(1.0 / (1.0 - (double)dropout_p));
    drop.key0 = (uint32_t)dropout_seed;
    drop.key1 = (uint32_t)(dropout_seed >> 32);
    RowBias rbias;
    rbias.table = nullptr;
    rbias.nv = rbias.ncam = rbias.L = 1;
    for (int i = 0; i < 8; ++i) rbias.start[i] = 0;
    if (rb) {
        if (rb->table == nullptr || rb->nv < 1 || rb->ncam < 1 || rb->L < 1 || rb->L > 8)
            return api_fail(MSDA_ERR_INVALID_ARG, "bad per-(camera, level) bias");
        rbias.table = rb->table;
        rbias.nv = rb->nv;
        rbias.ncam = rb->ncam;
        rbias.L = rb->L;
        for (int i = 0; i < rb->L; ++i) rbias.start[i] = rb->start[i];
    }
    // the shared-memory attribute belongs to the current device: set on every launch
    cudaError_t e;
    if (avg) {
        e = cudaFuncSetAttribute(proj_gemm_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes);
        if (e != cudaSuccess) return api_cuda(e, "msda_linear: shared memory size");
        proj_gemm_kernel<true><<<grid, kAvgThreads, kSmemBytes, stream>>>(
            mx, mw, my, bias, residual, y_dtype == MSDA_BF16, M, N, K, drop, rbias, *avg);
    } else {
        e = cudaFuncSetAttribute(proj_gemm_kernel<false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes);
        if (e != cudaSuccess) return api_cuda(e, "msda_linear: shared memory size");
        const AvgArgs none{nullptr, nullptr, nullptr, 1, 1};
        proj_gemm_kernel<false><<<grid, kGemmThreads, kSmemBytes, stream>>>(
            mx, mw, my, bias, residual, y_dtype == MSDA_BF16, M, N, K, drop, rbias, none);
    }
    return api_cuda(cudaGetLastError(), "msda_linear");
}

}  // namespace
}  // namespace msda

msda_status_t msda::linear_impl(const void* x, const void* w, const float* bias,
                                const float* residual, int32_t M, int32_t N, int32_t K,
                                msda_dtype_t y_dtype, void* y, float dropout_p,
                                uint64_t dropout_seed, const RowBiasArgs* rb, cudaStream_t stream)
{
    return launch_projection(x, nullptr, w, bias, residual, M, N, K, y_dtype, y, dropout_p,
                             dropout_seed, rb, stream);
}

msda_status_t msda::average_linear_impl(const float* out_rb, const int32_t* pos,
                                        const int32_t* hits, int32_t B, int32_t Ncam, int32_t Nq,
                                        const void* w, const float* bias, const float* residual,
                                        int32_t N, int32_t K, msda_dtype_t y_dtype, void* y,
                                        float dropout_p, uint64_t dropout_seed,
                                        cudaStream_t stream)
{
    if (B < 0 || Nq < 0 || Ncam < 1)
        return api_fail(MSDA_ERR_INVALID_ARG, "bad sizes");
    if (Ncam > kMaxAvgCams)
        return api_fail(MSDA_ERR_UNSUPPORTED, "at most 8 cameras for the averaged projection");
    if ((int64_t)B * Ncam * Nq > INT32_MAX)
        return api_fail(MSDA_ERR_UNSUPPORTED, "too many rebatched rows");
    if ((int64_t)B * Nq == 0) return api_ok();
    if (out_rb == nullptr || ((uintptr_t)out_rb & 31) || pos == nullptr || ((uintptr_t)pos & 3) ||
        hits == nullptr || ((uintptr_t)hits & 3))
        return api_fail(MSDA_ERR_INVALID_ARG,
                        "out_rb (32-byte aligned), pos and hits (4-byte aligned) are required");
    const AvgArgs a{out_rb, pos, hits, Ncam, Nq};
    return launch_projection(nullptr, &a, w, bias, residual, B * Nq, N, K, y_dtype, y, dropout_p,
                             dropout_seed, nullptr, stream);
}

extern "C" msda_status_t msda_linear(const void* x, const void* w, const float* bias,
                                     const float* residual, int32_t M, int32_t N, int32_t K,
                                     msda_dtype_t y_dtype, void* y, msda_stream_t stream)
{
    return msda_linear_dropout(x, w, bias, residual, M, N, K, y_dtype, y, 0.f, 0, stream);
}

extern "C" uint32_t msda_linear_timeouts(void)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, msda::g_gemm_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

extern "C" msda_status_t msda_linear_test_withhold_load(void)
{
    const int one = 1;
    return msda::api_cuda(cudaMemcpyToSymbol(msda::g_gemm_withhold, &one, sizeof(one)),
                          "msda_linear_test_withhold_load");
}
