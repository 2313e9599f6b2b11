// qproj.cu -- routed query projection on the sm_100a tensor cores.
//
// "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
// (gist.science summary), "Activation Conditionnelle" and "Chemin KV Dense":
// the routing makes the query-side computation conditional, while K/V stay
// dense.  Here the query row of head j is computed only for the tokens that
// selected j:
//   Q[b,t,j,:] = x[b,t,:] . W_Q[:, j*d_h : (j+1)*d_h]     for (t, j) routed,
// a grouped GEMM over the compaction's per-(b, j) position lists.  Rows of Q
// whose head was not selected are not written.
//
// CTA (m-block, head j, batch b): up to 256 routed tokens of (b, j) form two
// M = 128 tiles that share every W_Q stage; N = d_h = 128; K = d_model in
// 64-wide stages.  Warp 0 loads the tokens' x rows: a tile of 128
// consecutive positions (every token of the range selected j, as in dense GQA)
// as one 128-row TMA box, any other tile with TMA tile::gather4 (four rows per
// lane and stage, 128B-swizzled by address; padding rows name an out-of-range
// row and are zero-filled; gathers run about 4x slower than a box on B200), and
// loads W_Q's [64 k][128 n] block of head j as an MN-major operand; warp 1 issues the tcgen05 MMAs into a TMEM accumulator; all four
// warps then write the bf16 rows back to their routed slots.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kM = 128;                       // routed tokens per tile (UMMA M)
constexpr int kN = 128;                       // d_h (UMMA N)
constexpr int kTK = 64;                       // d_model per stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr int kTiles = 2;                     // 128-row tiles per CTA sharing each W_Q stage
constexpr uint32_t kABytes = kM * kTK * 2;    // 16 KB of gathered x rows
constexpr uint32_t kBBlock = kTK * 64 * 2;    // [64 k][64 n] of W_Q, 8 KB
constexpr uint32_t kWhereQproj = 5;

struct QprojSmem {
    uint8_t a[kStages][kTiles][kABytes];
    uint8_t b[kStages][2][kBBlock];
    int32_t rows[kTiles * kM];  // flattened token row b*T + t of each tile row, -1 for padding
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    int32_t failed;
};

__global__ void __launch_bounds__(128)
qproj_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapXT,
             const __grid_constant__ CUtensorMap mapW,
             const int32_t* __restrict__ head_offsets, const int32_t* __restrict__ head_pos, int T, int h,
             int d_model, int bt_rows, __nv_bfloat16* __restrict__ Q, uint32_t* __restrict__ status) {
    const int mb = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    const int32_t beg = head_offsets[(int64_t)b * h + j];
    const int n = head_offsets[(int64_t)b * h + j + 1] - beg;
    if (mb * kTiles * kM >= n) return;  // the whole CTA leaves before any barrier or TMEM use

    extern __shared__ uint8_t smem_raw[];
    QprojSmem& sm = *reinterpret_cast<QprojSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = (d_model + kTK - 1) / kTK;

    for (int r = tid; r < kTiles * kM; r += 128) {
        const int e = mb * kTiles * kM + r;
        sm.rows[r] = (e < n) ? (int32_t)((int64_t)b * T + head_pos[beg + e]) : -1;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        mbar_init(&sm.acc_full, 1);
        sm.failed = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTiles * kN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // TMA producer: lane l gathers tile rows 4l .. 4l+3; lane 0 also loads W_Q.
        int row[kTiles][4];
#pragma unroll
        for (int t = 0; t < kTiles; ++t)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int rr = sm.rows[t * kM + lane * 4 + e];
                row[t][e] = rr >= 0 ? rr : bt_rows;  // out of range: zero-filled
            }
        // A tile whose 128 positions are consecutive (the list is strictly
        // increasing, so first and last differ by 127) is one 128-row box.
        bool contig[kTiles];
#pragma unroll
        for (int t = 0; t < kTiles; ++t) {
            const int r0 = sm.rows[t * kM], r1 = sm.rows[t * kM + kM - 1];
            contig[t] = r0 >= 0 && r1 >= 0 && r1 - r0 == kM - 1;
        }
        if (lane == 0) {
            tma_prefetch_desc(&mapX);
            tma_prefetch_desc(&mapXT);
            tma_prefetch_desc(&mapW);
        }
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.empty[s], ((kb / kStages) & 1) ^ 1))) {
                if (lane == 0) sm.failed = 1;
                ok = false;
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], kTiles * kABytes + 2 * kBBlock);
            __syncwarp();
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                if (contig[t]) {
                    if (lane == 0) tma_load_2d(&mapXT, &sm.full[s], sm.a[s][t], kb * kTK, sm.rows[t * kM]);
                } else {
                    tma_gather4_2d(&mapX, &sm.full[s], sm.a[s][t] + lane * 4 * 128, kb * kTK, row[t][0], row[t][1],
                                   row[t][2], row[t][3]);
                }
            }
            if (lane == 0) {
                tma_load_2d(&mapW, &sm.full[s], sm.b[s][0], j * kN, kb * kTK);
                tma_load_2d(&mapW, &sm.full[s], sm.b[s][1], j * kN + 64, kb * kTK);
            }
        }
        // every issued load lands before the CTA may exit
        const int issued = ok ? nk : 0;
        if (lane == 0)
            for (int back = 1; back <= kStages && back <= issued; ++back) {
                const int kb = issued - back;
                mbar_wait(&sm.full[kb % kStages], (kb / kStages) & 1);
            }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: D[128 tokens][128] += x_rows . W_Q block
        const uint32_t idesc = idesc_bf16_f32(kM, kN, false, true);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait(&sm.full[s], (kb / kStages) & 1)) { sm.failed = 1; break; }
            tc_fence_after();
            const uint32_t ba = smem_u32(sm.b[s][0]);
            for (int t = 0; t < kTiles; ++t) {
                const uint32_t aa = smem_u32(sm.a[s][t]);
                for (int kk = 0; kk < kTK / 16; ++kk) {
                    const uint64_t adesc = smem_desc(aa + kk * 32, 16, 1024, kSwizzle128B);
                    const uint64_t bdesc = smem_desc(ba + kk * 2048, kBBlock, 1024, kSwizzle128B);
                    umma_ss(tmem + t * kN, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
                }
            }
            umma_commit(&sm.empty[s]);
        }
        umma_commit(&sm.acc_full);
    }
    __syncwarp();

    // Epilogue: thread = tile row; fp32 accumulator -> bf16 row of Q[b, t, j, :].
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full, 0));
    tc_fence_after();
    if (!acc_ok) {
        if (lane == 0) sm.failed = 1;
    } else {
#pragma unroll 1
        for (int t = 0; t < kTiles; ++t) {
            const int32_t rr = sm.rows[t * kM + warp * 32 + lane];
            __nv_bfloat16* dst = Q + ((int64_t)(rr >= 0 ? rr : 0) * h + j) * kN;
#pragma unroll 1
            for (int c = 0; c < kN / 32; ++c) {
                uint32_t v[32];
                tmem_ld32(tmem_addr(tmem, warp * 32, t * kN + c * 32), v);
                tmem_ld_wait();
                if (rr >= 0) {
                    uint4* o = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        o[q] = make_uint4(
                            pack_bf16x2(__uint_as_float(v[8 * q + 0]), __uint_as_float(v[8 * q + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTiles * kN);
    }
    if (tid == 0 && sm.failed && status != nullptr)
        report_error(status, GQE_ERR_DEVICE_TIMEOUT, kWhereQproj, (uint32_t)(blockIdx.x + gridDim.x * blockIdx.y));
}

}  // namespace

cudaError_t launch_qproj(const QprojArgs& a) {
    static std::atomic<uint64_t> configured{0};
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    CUtensorMap mapX, mapXT, mapW;
    {
        const uint64_t dims[2] = {(uint64_t)s.d_model, (uint64_t)BT};
        const uint64_t strides[1] = {(uint64_t)s.d_model * 2};
        const uint32_t box[2] = {kTK, 1};  // one row per box: tile::gather4
        if (!make_bf16_map(&mapX, a.x, 2, dims, strides, box)) return cudaErrorInvalidValue;
        const uint32_t tbox[2] = {kTK, kM};  // 128 consecutive rows
        if (!make_bf16_map(&mapXT, a.x, 2, dims, strides, tbox)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)s.h * kN, (uint64_t)s.d_model};
        const uint64_t strides[1] = {(uint64_t)s.h * kN * 2};
        const uint32_t box[2] = {64, kTK};
        if (!make_bf16_map(&mapW, a.W_Q, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(QprojSmem) + 1024;
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        err = cudaFuncSetAttribute(qproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        if (bit) configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    // every (b, j) list holds at most T positions
    const dim3 grid((unsigned)((s.T + kTiles * kM - 1) / (kTiles * kM)), (unsigned)s.h, (unsigned)s.B);
    qproj_kernel<<<grid, 128, smem, a.stream>>>(mapX, mapXT, mapW, a.head_offsets, a.head_pos, s.T, s.h, s.d_model,
                                                (int)BT, (__nv_bfloat16*)a.Q, (uint32_t*)a.status);
    return cudaGetLastError();
}

}  // namespace gqe
