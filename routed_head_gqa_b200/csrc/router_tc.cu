// router_tc.cu -- GQE router on the sm_100a tensor cores (bf16 inputs, fp32
// logits): l = x . W_r (+ bias), then per-group top-k and renormalised gates,
// fused in the epilogue.
//
// Router: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
// (gist.science summary), "Architecture et Routage" (k query-head experts per
// GQA group and token) and "Somme Ponderee Renormalisee" (router probabilities
// renormalised over the selection).  The linear form and the tie rule (lower
// head index first) are this library's reading of an unspecified router.
//
// One CTA per 128-token tile.  x tiles [128 tokens][64] arrive by TMA (K-major,
// 128B swizzle); W_r blocks [64 rows of d_model][64 heads] arrive by TMA straight
// from W_r's [d_model, h] layout as an MN-major operand (heads beyond h are
// zero-filled, so the MMA runs N = 64 * ceil(h/64)).  D = x . W_r accumulates in
// TMEM in fp32 (bf16 products are exact in fp32).  The bound is HBM: x is read
// once.
#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kTM = 128;      // tokens per tile (UMMA M)
constexpr int kTK = 64;       // d_model per stage (one 128-byte swizzle row)
constexpr int kStages = 4;
constexpr uint32_t kXBytes = kTM * kTK * 2;  // 16 KB
constexpr uint32_t kWBlock = kTK * 64 * 2;   // [64 k][64 heads] = 8 KB
constexpr uint32_t kWhereRouter = 3;

template <int NB>  // number of 64-head blocks: N = 64 * NB
struct RouterSmem {
    uint8_t x[kStages][kXBytes];
    uint8_t w[kStages][NB][kWBlock];
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    int32_t failed;
};

template <int NB>
__global__ void __launch_bounds__(128)
router_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                 const float* __restrict__ bias, int64_t BT, int d_model, int h, int g, int k,
                 int32_t* __restrict__ idx, float* __restrict__ gate, uint32_t* __restrict__ status) {
    extern __shared__ uint8_t smem_raw[];
    using Smem = RouterSmem<NB>;
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    constexpr uint32_t kCols = 64 * NB;  // TMEM columns (power of two for NB in {1, 2, 4})
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tok0 = (int64_t)blockIdx.x * kTM;
    const int nk = (d_model + kTK - 1) / kTK;

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
        tmem_alloc(&sm.tmem_base, kCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0 && lane == 0) {
        // TMA producer
        tma_prefetch_desc(&mapX);
        tma_prefetch_desc(&mapW);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait(&sm.empty[s], ((kb / kStages) & 1) ^ 1)) { sm.failed = 1; break; }
            mbar_arrive_expect_tx(&sm.full[s], kXBytes + NB * kWBlock);
            tma_load_2d(&mapX, &sm.full[s], sm.x[s], kb * kTK, (int)tok0);
            for (int nb = 0; nb < NB; ++nb) tma_load_2d(&mapW, &sm.full[s], sm.w[s][nb], nb * 64, kb * kTK);
        }
        // every issued load lands before the CTA may exit
        for (int back = 1; back <= kStages && back <= nk; ++back) {
            const int kb = nk - back;
            mbar_wait(&sm.full[kb % kStages], (kb / kStages) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: D[128 tokens][64*NB heads] += x_tile . W_block
        const uint32_t idesc = idesc_bf16_f32(kTM, 64 * NB, false, true);
        for (int kb = 0; kb < nk; ++kb) {
            const int s = kb % kStages;
            if (!mbar_wait(&sm.full[s], (kb / kStages) & 1)) { sm.failed = 1; break; }
            tc_fence_after();
            const uint32_t xa = smem_u32(sm.x[s]);
            const uint32_t wa = smem_u32(sm.w[s][0]);
            for (int kk = 0; kk < kTK / 16; ++kk) {
                const uint64_t adesc = smem_desc(xa + kk * 32, 16, 1024, kSwizzle128B);
                const uint64_t bdesc = smem_desc(wa + kk * 2048, kWBlock, 1024, kSwizzle128B);
                umma_ss(tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit(&sm.empty[s]);
        }
        umma_commit(&sm.acc_full);
    }
    __syncwarp();

    // Epilogue: thread = token row of the tile.  The stages are free once the
    // accumulator is complete; the logits go through them, one padded row per
    // token ([128][64*NB + 1] floats, conflict-free column access).
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full, 0));
    tc_fence_after();
    if (!acc_ok) {
        if (lane == 0) sm.failed = 1;
    } else {
        constexpr int ld = 64 * NB + 1;
        const int row = warp * 32 + lane;
        float* lg = reinterpret_cast<float*>(&sm.x[0][0]) + row * ld;
#pragma unroll 1
        for (int c = 0; c < 2 * NB; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tmem, warp * 32, c * 32), r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) lg[c * 32 + e] = __uint_as_float(r[e]);
        }
        const int64_t tok = tok0 + row;
        if (tok < BT) {
            const int hpg = h / g;
            if (bias)
                for (int j = 0; j < h; ++j) lg[j] += bias[j];
            for (int q = 0; q < g; ++q) {
                // top-k of the group's logits, equal logits -> lower index
                const float* lq = lg + q * hpg;
                uint64_t taken = 0;  // hpg <= 64 on this path
                float m = 0.f, denom = 0.f;
                int sel[16];
                float sel_l[16];
                for (int s = 0; s < k; ++s) {
                    int best = -1;
                    float bv = 0.f;
                    for (int a = 0; a < hpg; ++a) {
                        if ((taken >> a) & 1ull) continue;
                        const float v = lq[a];
                        if (best < 0 || v > bv) {
                            best = a;
                            bv = v;
                        }
                    }
                    taken |= 1ull << best;
                    sel[s] = best;
                    sel_l[s] = bv;
                    if (s == 0) m = bv;
                    denom += expf(bv - m);
                }
                const int64_t o = (tok * g + q) * k;
                for (int s = 0; s < k; ++s) {
                    idx[o + s] = q * hpg + sel[s];
                    gate[o + s] = expf(sel_l[s] - m) / denom;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
    if (tid == 0 && sm.failed && status != nullptr)
        report_error(status, GQE_ERR_DEVICE_TIMEOUT, kWhereRouter, (uint32_t)blockIdx.x);
}

template <int NB>
cudaError_t launch_nb(const RouteArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    CUtensorMap mapX, mapW;
    {
        const uint64_t dims[2] = {(uint64_t)s.d_model, (uint64_t)BT};
        const uint64_t strides[1] = {(uint64_t)s.d_model * 2};
        const uint32_t box[2] = {kTK, kTM};
        if (!make_bf16_map(&mapX, a.x, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)s.h, (uint64_t)s.d_model};
        const uint64_t strides[1] = {(uint64_t)s.h * 2};
        const uint32_t box[2] = {64, kTK};
        if (!make_bf16_map(&mapW, a.W_r, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(RouterSmem<NB>) + 1024;
    cudaError_t err =
        cudaFuncSetAttribute(router_tc_kernel<NB>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    const unsigned blocks = (unsigned)((BT + kTM - 1) / kTM);
    router_tc_kernel<NB><<<blocks, 128, smem, a.stream>>>(mapX, mapW, a.bias, BT, s.d_model, s.h, s.g, s.k, a.idx,
                                                          a.gate, (uint32_t*)a.status);
    return cudaGetLastError();
}

}  // namespace

bool router_tc_supported(const gqe_shape* s) {
    return s->dtype == GQE_BF16 && s->h % 8 == 0 && s->h <= 256 && s->d_model % 8 == 0 && s->h / s->g <= 64;
}

cudaError_t launch_router_tc(const RouteArgs& a) {
    const int h = a.s->h;
    if (h <= 64) return launch_nb<1>(a);
    if (h <= 128) return launch_nb<2>(a);
    return launch_nb<4>(a);
}

}  // namespace gqe
