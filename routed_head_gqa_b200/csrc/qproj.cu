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
// 64-wide stages.  A tile of 128 consecutive positions (every token of the
// range selected j, as in dense GQA) arrives as one 128-row TMA box; any other
// tile is staged by two copy warps with 16-byte cp.async per row chunk into
// the same 128B-swizzled layout (TMA tile::gather4 of the rows measured about
// 4x slower than a box on B200, and the copies 1.4-1.5x faster than the
// gathers).  W_Q's [64 k][128 n] block of head j arrives by TMA as an MN-major
// operand; warp 1 issues the tcgen05 MMAs into two TMEM accumulators; all four
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

constexpr int kCopyThreads = 64;               // warps 2-3 stage sparse rows with cp.async
constexpr int kCopyLag = 2;                    // stages a copy thread keeps in flight (< kStages)
static_assert(kCopyLag < kStages, "a copy thread must release a stage before it needs its next");

// 16-byte global -> shared copy; src_bytes = 0 writes zeros (padding rows).
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__global__ void __launch_bounds__(128)
qproj_kernel(const __grid_constant__ CUtensorMap mapXT, const __grid_constant__ CUtensorMap mapW,
             const int32_t* __restrict__ head_offsets, const int32_t* __restrict__ head_pos, int T, int h,
             int d_model, int32_t total, const __nv_bfloat16* __restrict__ X, __nv_bfloat16* __restrict__ Q,
             uint32_t* __restrict__ status) {
    const int mb = blockIdx.x, j = blockIdx.y, b = blockIdx.z;
    // A list that does not lie inside head_pos ([0, B*T*g*k)) is reported and
    // read as empty; a position outside [0, T) is reported and skipped below.
    int32_t beg = head_offsets[(int64_t)b * h + j];
    int32_t end = head_offsets[(int64_t)b * h + j + 1];
    if (beg < 0 || end < beg || end > total) {
        if (mb == 0 && threadIdx.x == 0) report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereQproj, 1);
        beg = end = 0;
    }
    const int n = end - beg;
    if (mb * kTiles * kM >= n) return;  // the whole CTA leaves before any barrier or TMEM use

    extern __shared__ uint8_t smem_raw[];
    QprojSmem& sm = *smem_align1024<QprojSmem>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = (d_model + kTK - 1) / kTK;

    for (int r = tid; r < kTiles * kM; r += 128) {
        const int e = mb * kTiles * kM + r;
        int32_t row = -1;
        if (e < n) {
            const int32_t t = head_pos[beg + e];
            if (t >= 0 && t < T) {
                row = (int32_t)((int64_t)b * T + t);
            } else {
                report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereQproj, 2);
            }
        }
        sm.rows[r] = row;
    }
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1 + kCopyThreads);  // the TMA arrival + each copy thread
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

    // A tile of 128 consecutive positions (the list is strictly increasing, so
    // first and last differ by 127) is one 128-row TMA box; any other tile is
    // staged row by row by the copy warps.
    bool contig[kTiles];
#pragma unroll
    for (int t = 0; t < kTiles; ++t) {
        const int r0 = sm.rows[t * kM], r1 = sm.rows[t * kM + kM - 1];
        contig[t] = r0 >= 0 && r1 >= 0 && r1 - r0 == kM - 1;
    }
    if (warp == 0) {
        // TMA producer (one thread): W_Q's head block and the contiguous tiles.
        if (lane == 0) {
            tma_prefetch_desc(&mapXT);
            tma_prefetch_desc(&mapW);
            uint32_t tx = 2 * kBBlock;
#pragma unroll
            for (int t = 0; t < kTiles; ++t) tx += contig[t] ? kABytes : 0u;
            bool ok = true;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % kStages;
                if (!mbar_wait(&sm.empty[s], ((kb / kStages) & 1) ^ 1)) { sm.failed = 1; ok = false; break; }
                mbar_arrive_expect_tx(&sm.full[s], tx);
#pragma unroll
                for (int t = 0; t < kTiles; ++t)
                    if (contig[t]) tma_load_2d(&mapXT, &sm.full[s], sm.a[s][t], kb * kTK, sm.rows[t * kM]);
                tma_load_2d(&mapW, &sm.full[s], sm.b[s][0], j * kN, kb * kTK);
                tma_load_2d(&mapW, &sm.full[s], sm.b[s][1], j * kN + 64, kb * kTK);
            }
            // every issued load lands before the CTA may exit
            const int issued = ok ? nk : 0;
            for (int back = 1; back <= kStages && back <= issued; ++back) {
                const int kb = issued - back;
                mbar_wait(&sm.full[kb % kStages], (kb / kStages) & 1);
            }
        }
    } else if (warp >= 2) {
        // Copy warps: each thread stages 2 rows per non-contiguous tile and stage,
        // 16 bytes per cp.async, into the 128B-swizzled layout (chunk c of row r
        // at chunk c ^ (r % 8)).  A stage is released after its copies complete
        // (wait_group) and a proxy fence makes them visible to the tensor core.
        const int p = tid - 64;
        auto release = [&](int kb) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&sm.full[kb % kStages]);
        };
        int issued = 0;
        bool ok = true;
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait(&sm.empty[s], ((kb / kStages) & 1) ^ 1)) { sm.failed = 1; ok = false; break; }
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                if (contig[t]) continue;
                const uint32_t base = smem_u32(sm.a[s][t]);
#pragma unroll
                for (int h2 = 0; h2 < kM / kCopyThreads; ++h2) {
                    const int r = p + h2 * kCopyThreads;
                    const int32_t rr = sm.rows[t * kM + r];
                    const __nv_bfloat16* src = X + (int64_t)(rr >= 0 ? rr : 0) * d_model + kb * kTK;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        const bool in = rr >= 0 && kb * kTK + c * 8 < d_model;  // d_model % 8 == 0
                        cp_async16(base + r * 128 + ((c ^ (r & 7)) << 4), in ? (const void*)(src + c * 8) : (const void*)X,
                                   in ? 16u : 0u);
                    }
                }
            }
            cp_async_commit();
            ++issued;
            if (kb >= kCopyLag) {
                cp_async_wait<kCopyLag>();
                release(kb - kCopyLag);
            }
        }
        // release the stages still in flight (all of them complete here)
        cp_async_wait<0>();
        if (ok)
            for (int kb = (issued > kCopyLag ? issued - kCopyLag : 0); kb < issued; ++kb) release(kb);
    }
    if (warp == 1 && lane == 0) {
        // MMA issuer: D[128 tokens][128] += x_rows . W_Q block
        const uint32_t idesc = idesc_bf16_f32(kM, kN, false, true);
        const uint32_t dhi = smem_desc_hi(1024, kSwizzle128B);
        const uint32_t alo0 = smem_desc_lo(smem_u32(sm.a[0][0]), 16);
        const uint32_t blo0 = smem_desc_lo(smem_u32(sm.b[0][0]), kBBlock);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait(&sm.full[s], (kb / kStages) & 1)) { sm.failed = 1; break; }
            tc_fence_after();
            // stage s, tile t: constant strides from stage 0 (16-byte units in the low word)
            const uint32_t blo = blo0 + (uint32_t)s * ((2 * kBBlock) >> 4);
#pragma unroll
            for (int t = 0; t < kTiles; ++t) {
                const uint32_t alo = alo0 + (uint32_t)(s * kTiles + t) * (kABytes >> 4);
#pragma unroll
                for (int kk = 0; kk < kTK / 16; ++kk)
                    umma_ss(tmem + t * kN, smem_desc_join(alo + kk * 2, dhi), smem_desc_join(blo + kk * 128, dhi),
                            idesc, (kb > 0 || kk > 0) ? 1u : 0u);
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
    // When the routed share g*k/h is 3/10 or more, the dense tiled GEMM (every
    // head of a token tile, routed rows written) beats gathering each head's
    // rows: on B200 the gather path ran at 22 % of the bf16 peak at a share of
    // 1/2, the dense one at about 78 % of its (doubled) work.
    if (a.idx != nullptr && a.scratch != nullptr && s.h <= 64 && 10 * s.g * s.k >= 3 * s.h)
        return launch_qproj_dense(a);
    const int64_t BT = (int64_t)s.B * s.T;
    CUtensorMap mapXT, mapW;
    {
        const uint64_t dims[2] = {(uint64_t)s.d_model, (uint64_t)BT};
        const uint64_t strides[1] = {(uint64_t)s.d_model * 2};
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
    qproj_kernel<<<grid, 128, smem, a.stream>>>(mapXT, mapW, a.head_offsets, a.head_pos, s.T, s.h, s.d_model,
                                                (int32_t)((int64_t)s.B * s.T * s.g * s.k),
                                                (const __nv_bfloat16*)a.x, (__nv_bfloat16*)a.Q,
                                                (uint32_t*)a.status);
    return cudaGetLastError();
}

}  // namespace gqe
