// msda_linear: the dense projections around the MSDA sampling ("BEV(三)
// BEVFormer: how the Query interacts with the 8 Heads of the Feature",
// sections 3 (value projection W_v), 4.1 (offset head W_Delta), 4.2 (weight
// head W_alpha), 11 (output projection W_o) and 13 (residual)):
//   Y = X W^T (+ bias) (+ residual),  X [M, K] bf16, W [N, K] bf16 (the
//   nn.Linear weight layout), fp32 accumulation, Y fp32 or bf16.
//
// One CTA computes a 128 x 256 tile of Y on the 5th-generation tensor cores:
//   - one thread issues the TMA loads of the whole K extent (K <= 256) of the
//     X tile and the W tile into shared memory, 128-byte swizzled, and waits
//     on an mbarrier for their bytes;
//   - the same thread issues tcgen05.mma (M = 128, N = 256, K = 16, bf16 in,
//     fp32 accumulate) into a 256-column TMEM accumulator, then
//     tcgen05.commit to a second mbarrier;
//   - four warps read the accumulator rows back with tcgen05.ld (warp w owns
//     TMEM lanes 32w..32w+31 = tile rows), add bias and residual and store.
// Every mbarrier wait is bounded: a wait that gives up counts a timeout in a
// device word (msda_linear_timeouts), skips the rest of the tile and still
// frees its TMEM.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

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
constexpr int kGemmThreads = 128;
constexpr uint32_t kABlockBytes = kBM * kBK * 2;  // 16 KB
constexpr uint32_t kBBlockBytes = kBN * kBK * 2;  // 32 KB
constexpr uint32_t kSpinLimit = 1u << 24;         // mbarrier polls before giving up

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator (bits
// 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major (bits 15, 16
// = 0), N / 8 in bits 17-22, M / 16 in bits 24-28.
constexpr uint32_t kInstrDesc = (1u << 4) | (1u << 7) | (1u << 10) |
                                ((uint32_t)(kBN >> 3) << 17) | ((uint32_t)(kBM >> 4) << 24);

struct __align__(8) Ctrl {
    uint64_t load_bar;
    uint64_t mma_bar;
    uint32_t tmem_base;
    int failed;
};

constexpr size_t kSmemBytes = 1024 /* alignment slack */ + kMaxKBlocks * (kABlockBytes + kBBlockBytes) +
                              sizeof(Ctrl);

__device__ unsigned int g_gemm_timeouts = 0;

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

// Wait for the completion of phase `parity`; false after kSpinLimit polls.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity)
{
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
    }
    return false;
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

__global__ void __launch_bounds__(kGemmThreads, 1)
proj_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
                 const float* __restrict__ bias, const float* __restrict__ residual,
                 void* __restrict__ y, int y_bf16, int M, int N, int K)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t* sa = smem;                                 // K/64 blocks of 128 x 64 bf16
    uint8_t* sb = smem + kMaxKBlocks * kABlockBytes;    // K/64 blocks of 256 x 64 bf16
    Ctrl& ctrl = *reinterpret_cast<Ctrl*>(sb + kMaxKBlocks * kBBlockBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kBM, n0 = blockIdx.y * kBN;
    const int kblocks = K / kBK;

    if (threadIdx.x == 0) {
        mbar_init(&ctrl.load_bar, 1);
        mbar_init(&ctrl.mma_bar, 1);
        ctrl.failed = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&ctrl.tmem_base)),
                     "r"(kBN)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = ctrl.tmem_base;

    if (threadIdx.x == 0) {
        mbar_expect_tx(&ctrl.load_bar, (uint32_t)kblocks * (kABlockBytes + kBBlockBytes));
        for (int kb = 0; kb < kblocks; ++kb) {
            tma_load_2d(sa + kb * kABlockBytes, &map_x, kb * kBK, m0, &ctrl.load_bar);
            tma_load_2d(sb + kb * kBBlockBytes, &map_w, kb * kBK, n0, &ctrl.load_bar);
        }
        if (mbar_wait(&ctrl.load_bar, 0)) {
            asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
            for (int kb = 0; kb < kblocks; ++kb)
                for (int ks = 0; ks < kBK / 16; ++ks) {
                    const uint64_t ad = smem_desc_sw128(smem_u32(sa + kb * kABlockBytes) + ks * 32);
                    const uint64_t bd = smem_desc_sw128(smem_u32(sb + kb * kBBlockBytes) + ks * 32);
                    umma_bf16(tmem, ad, bd, (kb | ks) != 0);
                }
            umma_commit(&ctrl.mma_bar);
        } else {
            ctrl.failed = 1;
            atomicAdd(&g_gemm_timeouts, 1u);
            mbar_wait(&ctrl.load_bar, 0);  // give copies still in flight a last chance
        }
    }
    __syncthreads();
    bool ok = !ctrl.failed;
    if (ok) ok = mbar_wait(&ctrl.mma_bar, 0);
    if (!ok && threadIdx.x == 0 && !ctrl.failed) atomicAdd(&g_gemm_timeouts, 1u);
    ok = __all_sync(0xffffffffu, ok);
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");

    if (ok) {
        const int row = m0 + warp * 32 + lane;
        const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
        for (int c0 = 0; c0 < kBN; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(lane_base + (uint32_t)c0, r);
            if (row < M) {
                const int col0 = n0 + c0;
                float v[32];
#pragma unroll
                for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
                if (bias) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + col0 + j));
                        v[j] += b4.x; v[j + 1] += b4.y; v[j + 2] += b4.z; v[j + 3] += b4.w;
                    }
                }
                if (residual) {
                    const float4* rp =
                        reinterpret_cast<const float4*>(residual + (int64_t)row * N + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 q = __ldcs(rp + j);
                        v[4 * j] += q.x; v[4 * j + 1] += q.y; v[4 * j + 2] += q.z; v[4 * j + 3] += q.w;
                    }
                }
                if (y_bf16) {
                    uint4* yp = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(y) +
                                                         (int64_t)row * N + col0);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 u;
                        u.x = pack_bf16x2(v[8 * j], v[8 * j + 1]);
                        u.y = pack_bf16x2(v[8 * j + 2], v[8 * j + 3]);
                        u.z = pack_bf16x2(v[8 * j + 4], v[8 * j + 5]);
                        u.w = pack_bf16x2(v[8 * j + 6], v[8 * j + 7]);
                        __stcs(yp + j, u);
                    }
                } else {
                    float4* yp = reinterpret_cast<float4*>(static_cast<float*>(y) + (int64_t)row * N + col0);
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        __stcs(yp + j, make_float4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]));
                }
            }
        }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kBN)
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

}  // namespace
}  // namespace msda

extern "C" msda_status_t msda_linear(const void* x, const void* w, const float* bias,
                                     const float* residual, int32_t M, int32_t N, int32_t K,
                                     msda_dtype_t y_dtype, void* y, msda_stream_t stream)
{
    using namespace msda;
    if (M < 0) return api_fail(MSDA_ERR_INVALID_ARG, "M must be >= 0");
    if (N < kBN || N % kBN != 0)
        return api_fail(MSDA_ERR_UNSUPPORTED, "N must be a positive multiple of 256");
    if (K < kBK || K > kMaxK || K % kBK != 0)
        return api_fail(MSDA_ERR_UNSUPPORTED, "K must be 64, 128, 192 or 256");
    if (y_dtype != MSDA_F32 && y_dtype != MSDA_BF16)
        return api_fail(MSDA_ERR_INVALID_ARG, "unknown output dtype");
    if (M == 0) return api_ok();
    auto bad = [](const void* p) { return p == nullptr || ((uintptr_t)p & 15) != 0; };
    if (bad(x) || bad(w) || bad(y))
        return api_fail(MSDA_ERR_INVALID_ARG, "x, w and y must be non-null and 16-byte aligned");
    if ((bias && ((uintptr_t)bias & 15)) || (residual && ((uintptr_t)residual & 15)))
        return api_fail(MSDA_ERR_INVALID_ARG, "bias and residual must be 16-byte aligned");
    CUtensorMap mx, mw;
    if (!make_map(&mx, x, M, K, kBM) || !make_map(&mw, w, N, K, kBN))
        return api_fail(MSDA_ERR_CUDA, "cuTensorMapEncodeTiled failed or is unavailable");
    static std::once_flag attr_once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(attr_once, [] {
        attr_err = cudaFuncSetAttribute(proj_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)kSmemBytes);
    });
    if (attr_err != cudaSuccess) return api_cuda(attr_err, "msda_linear: shared memory size");
    const dim3 grid((unsigned)((M + kBM - 1) / kBM), (unsigned)(N / kBN));
    proj_gemm_kernel<<<grid, kGemmThreads, kSmemBytes, (cudaStream_t)stream>>>(
        mx, mw, bias, residual, y, y_dtype == MSDA_BF16, M, N, K);
    return api_cuda(cudaGetLastError(), "msda_linear");
}

extern "C" uint32_t msda_linear_timeouts(void)
{
    unsigned int v = 0;
    if (cudaMemcpyFromSymbol(&v, msda::g_gemm_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}
