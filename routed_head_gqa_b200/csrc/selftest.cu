// selftest.cu -- libgqe_selftest: unit checks of the tensor-core building
// blocks used by the routed prefill kernel, on one 128x128x128 bf16 tile:
//   mode 0: A [M][K] K-major (smem, TMA, 128B swizzle) x B [N][K] K-major
//   mode 1: A K-major x B [K][N] MN-major (the P.V operand layout of V tiles)
//   mode 2: A written into TMEM by tcgen05.st (packed bf16 pairs) x B MN-major
// C [M][N] fp32 = sum_k A[m,k] * B(k,n).  Also the FMA-pipe 2^x of the prefill
// softmax, element by element.  Test-only; not part of the product API.
#include "common.cuh"
#include "exp2_fma.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

using namespace gqe;
using namespace gqe::sm100;

namespace {

constexpr int kTile = 128;
constexpr uint32_t kHalfBytes = kTile * 64 * 2;  // [128 rows][64 bf16] = 16 KB

__global__ void __launch_bounds__(128) umma_tile_kernel(const __grid_constant__ CUtensorMap mapA,
                                                        const __grid_constant__ CUtensorMap mapB, int mode,
                                                        const __nv_bfloat16* __restrict__ A_global,
                                                        float* __restrict__ C, uint32_t* __restrict__ status) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = smem_align1024<uint8_t>(smem_raw);
    uint8_t* sA = smem;                 // 2 x 16 KB
    uint8_t* sB = smem + 2 * kHalfBytes;  // 2 x 16 KB
    __shared__ __align__(8) uint64_t bar_load, bar_mma;
    __shared__ uint32_t tmem_base_sh;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        mbar_init(&bar_load, 1);
        mbar_init(&bar_mma, 1);
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&tmem_base_sh, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_sh;

    if (tid == 0) {
        mbar_arrive_expect_tx(&bar_load, 4 * kHalfBytes);
        tma_load_2d(&mapA, &bar_load, sA, 0, 0);
        tma_load_2d(&mapA, &bar_load, sA + kHalfBytes, 64, 0);
        tma_load_2d(&mapB, &bar_load, sB, 0, 0);
        tma_load_2d(&mapB, &bar_load, sB + kHalfBytes, 64, 0);
    }
    bool ok = mbar_wait(&bar_load, 0);

    const uint32_t a_tmem = tmem + 128;  // columns 128..191 hold A as packed bf16 pairs
    if (mode == 2) {
        // Row m = thread: A[m, 2c], A[m, 2c+1] -> column c (low, high halves).
        const uint32_t* arow = reinterpret_cast<const uint32_t*>(A_global + (size_t)tid * kTile);
        for (int c0 = 0; c0 < 64; c0 += 16) {
            uint32_t r[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) r[i] = arow[c0 + i];
            tmem_st16(tmem_addr(a_tmem, warp * 32, c0), r);
        }
        tmem_st_wait();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (tid == 0 && ok) {
        const bool b_mn = mode != 0;
        const uint32_t idesc = idesc_bf16_f32(128, 128, false, b_mn);
        for (int kk = 0; kk < kTile / 16; ++kk) {
            uint64_t bdesc;
            if (!b_mn) {
                // K-major: 16-element K step = 32 bytes inside a 64-element half
                bdesc = smem_desc(smem_u32(sB) + (kk / 4) * kHalfBytes + (kk % 4) * 32, 16, 1024, kSwizzle128B);
            } else {
                // MN-major: K rows of 128 bytes, 8-row groups 1024 B apart (SBO),
                // the two 64-wide N halves 16 KB apart (LBO); a K step is 2 groups.
                bdesc = smem_desc(smem_u32(sB) + kk * 2048, kHalfBytes, 1024, kSwizzle128B);
            }
            if (mode == 2) {
                umma_ts(tmem, a_tmem + kk * 8, bdesc, idesc, kk > 0);
            } else {
                const uint64_t adesc =
                    smem_desc(smem_u32(sA) + (kk / 4) * kHalfBytes + (kk % 4) * 32, 16, 1024, kSwizzle128B);
                umma_ss(tmem, adesc, bdesc, idesc, kk > 0);
            }
        }
        umma_commit(&bar_mma);
    }
    if (ok) ok = mbar_wait(&bar_mma, 0);
    tc_fence_after();
    if (!ok) {
        if (tid == 0) atomicExch(status, (uint32_t)GQE_ERR_DEVICE_TIMEOUT);
    } else {
        for (int c0 = 0; c0 < kTile; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tmem, warp * 32, c0), r);
            tmem_ld_wait();
            float* crow = C + (size_t)(warp * 32 + lane) * kTile + c0;
#pragma unroll
            for (int i = 0; i < 32; ++i) crow[i] = __uint_as_float(r[i]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tmem, 256);
}

// A bounded wait on an mbarrier that nothing completes: the wait must give up
// and the kernel must record GQE_ERR_DEVICE_TIMEOUT instead of hanging.
__global__ void wait_timeout_kernel(uint32_t* __restrict__ status) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_barrier_init();
    }
    __syncthreads();
    const bool ok = mbar_wait(&bar, 0);
    if (threadIdx.x == 0) atomicExch(status, ok ? (uint32_t)GQE_OK : (uint32_t)GQE_ERR_DEVICE_TIMEOUT);
}

// y[i] = the prefill softmax's FMA-pipe 2^x of x[i] (clamped at -126), pairs
// of consecutive elements per thread as in the kernel.
__global__ void exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i >= n) return;
    const float x0 = x[i], x1 = (i + 1 < n) ? x[i + 1] : 0.f;
    float y0, y1;
    up2(exp2_poly2_clamped(x0, x1), y0, y1);
    y[i] = y0;
    if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace

extern "C" int gqe_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
    if (!x || !y || n < 0) return GQE_ERR_INVALID_ARGUMENT;
    if (n == 0) return GQE_OK;
    const int pairs = (n + 1) / 2;
    exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, (cudaStream_t)stream>>>(x, y, n);
    return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}

extern "C" int gqe_selftest_wait_timeout(uint32_t* status, void* stream) {
    if (!status) return GQE_ERR_INVALID_ARGUMENT;
    wait_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(status);
    return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}

extern "C" int gqe_selftest_umma_tile(int mode, const void* A, const void* B, float* C, uint32_t* status,
                                      void* stream) {
    if (mode < 0 || mode > 2 || !A || !B || !C || !status) return GQE_ERR_INVALID_ARGUMENT;
    CUtensorMap mapA, mapB;
    const uint64_t dims[2] = {128, 128};
    const uint64_t strides[1] = {128 * 2};
    const uint32_t box[2] = {64, 128};
    if (!make_bf16_map(&mapA, A, 2, dims, strides, box)) return GQE_ERR_CUDA;
    if (!make_bf16_map(&mapB, B, 2, dims, strides, box)) return GQE_ERR_CUDA;
    const size_t smem = 4 * kHalfBytes + 1024;
    cudaFuncSetAttribute(umma_tile_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    umma_tile_kernel<<<1, 128, smem, (cudaStream_t)stream>>>(mapA, mapB, mode, (const __nv_bfloat16*)A, C,
                                                             status);
    return cudaGetLastError() == cudaSuccess ? GQE_OK : GQE_ERR_CUDA;
}
