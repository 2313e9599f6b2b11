// router_tc.cu -- GQE router on the sm_100a tensor cores (bf16 inputs, fp32
// logits): l = x . W_r (+ bias), then per-group top-k and renormalised gates,
// fused in the epilogue, together with the per-(batch, head, 32-token chunk)
// selection counts that the compaction needs.
//
// Router: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
// (gist.science summary), "Architecture et Routage" (k query-head experts per
// GQA group and token) and "Somme Ponderee Renormalisee" (router probabilities
// renormalised over the selection).  The linear form and the tie rule (lower
// head index first) are this library's reading of an unspecified router.
//
// A 128-token tile is computed by a thread-block cluster of KS CTAs (KS = 1, 2
// or 4, chosen so that the grid fills the SMs): CTA r of the cluster
// accumulates x . W_r over its own contiguous slice of d_model in TMEM.  x
// tiles [128 tokens][64] arrive by TMA (K-major, 128B swizzle); W_r blocks
// [64 rows of d_model][64 heads] arrive by TMA straight from W_r's [d_model, h]
// layout as an MN-major operand (heads beyond h are zero-filled, so the MMA runs
// N = 64 * ceil(h/64)).  After a cluster barrier CTA r sums rows
// [r*128/KS, (r+1)*128/KS) of the KS partial logits, reading its peers' shared
// memory (distributed shared memory loads), and runs top-k on those rows.  The
// bound is HBM: x is read once.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kTM = 128;      // tokens per tile (UMMA M)
constexpr int kTK = 64;       // d_model per stage (one 128-byte swizzle row)
constexpr uint32_t kXBytes = kTM * kTK * 2;  // 16 KB
constexpr uint32_t kWBlock = kTK * 64 * 2;   // [64 k][64 heads] = 8 KB
constexpr uint32_t kWhereRouter = 3;

// Pipeline depth.  With up to 64 heads a CTA keeps 4 stages (96 KB), so two
// CTAs share an SM: all tiles of a launch of up to 2 x 148 tiles stream at
// once, instead of a second, partial wave of one-CTA-per-SM tiles (gqe_prefill
// shapes, 256 tiles: route 0.093 -> 0.083 ms).  Wider W_r blocks keep about
// 192 KB of stages in one CTA.
template <int NB>
constexpr int router_stages() { return NB == 1 ? 4 : (NB == 2 ? 6 : 4); }

template <int NB>  // number of 64-head blocks: N = 64 * NB
struct RouterSmem {
    static constexpr int kStages = router_stages<NB>();
    uint8_t x[kStages][kXBytes];
    uint8_t w[kStages][NB][kWBlock];
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full;
    uint32_t tmem_base;
    int32_t failed;
};

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster arrives; release/acquire orders the
// shared-memory writes before the barrier with the peers' reads after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t peer_addr(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// Not volatile: each load depends on a mapa issued after the cluster barrier,
// which keeps it there, and independent loads may overlap.
__device__ __forceinline__ float ld_peer(uint32_t addr) {
    float v;
    asm("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

template <int NB, int KS, int KMAX>
__global__ void __launch_bounds__(128)
router_tc_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW,
                 const float* __restrict__ bias, int64_t BT, int d_model, int h, int g, int k, int T,
                 int nchunk, int32_t* __restrict__ idx, float* __restrict__ gate, int32_t* __restrict__ counts,
                 uint32_t* __restrict__ status, float* __restrict__ logits) {
    extern __shared__ uint8_t smem_raw[];
    using Smem = RouterSmem<NB>;
    constexpr int S = Smem::kStages;
    Smem& sm = *smem_align1024<Smem>(smem_raw);
    constexpr uint32_t kCols = 64 * NB;  // TMEM columns (power of two for NB in {1, 2, 4})
    constexpr int kRows = kTM / KS;      // rows of the tile whose top-k this CTA computes
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const uint32_t rank = (KS > 1) ? cluster_ctarank() : 0u;
    const int64_t tok0 = (int64_t)(blockIdx.x / KS) * kTM;
    const int nk = (d_model + kTK - 1) / kTK;
    const int kb0 = (int)((int64_t)nk * rank / KS);
    const int nkl = (int)((int64_t)nk * (rank + 1) / KS) - kb0;  // >= 1: the host keeps KS <= nk
    // Each tile starts its walk over the slice at a different block, so that the
    // CTAs in flight read different column ranges of their token rows instead of
    // all hitting the same offset of every 8 KB-strided row at once.
    const int rot = (int)(((blockIdx.x / KS) * 7) % nkl);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
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
        // TMA producer over this CTA's d_model slice
        tma_prefetch_desc(&mapX);
        tma_prefetch_desc(&mapW);
        for (int i = 0; i < nkl; ++i) {
            const int s = i % S;
            if (!mbar_wait(&sm.empty[s], ((i / S) & 1) ^ 1)) { sm.failed = 1; break; }
            const int kb = kb0 + (i + rot) % nkl;
            mbar_arrive_expect_tx(&sm.full[s], kXBytes + NB * kWBlock);
            tma_load_2d(&mapX, &sm.full[s], sm.x[s], kb * kTK, (int)tok0);
            for (int nb = 0; nb < NB; ++nb) tma_load_2d(&mapW, &sm.full[s], sm.w[s][nb], nb * 64, kb * kTK);
        }
        // every issued load lands before the CTA may exit
        for (int back = 1; back <= S && back <= nkl; ++back) {
            const int i = nkl - back;
            mbar_wait(&sm.full[i % S], (i / S) & 1);
        }
    } else if (warp == 1 && lane == 0) {
        // MMA issuer: D[128 tokens][64*NB heads] += x_tile . W_block over the slice
        const uint32_t idesc = idesc_bf16_f32(kTM, 64 * NB, false, true);
        const uint32_t dhi = smem_desc_hi(1024, kSwizzle128B);
        const uint32_t xlo0 = smem_desc_lo(smem_u32(sm.x[0]), 16);
        const uint32_t wlo0 = smem_desc_lo(smem_u32(sm.w[0][0]), kWBlock);
        for (int i = 0; i < nkl; ++i) {
            const int s = i % S;
            if (!mbar_wait(&sm.full[s], (i / S) & 1)) { sm.failed = 1; break; }
            tc_fence_after();
            // stage s starts s * sizeof(stage) bytes after stage 0 (16-byte units in the low word)
            const uint32_t xlo = xlo0 + (uint32_t)s * (kXBytes >> 4);
            const uint32_t wlo = wlo0 + (uint32_t)s * ((NB * kWBlock) >> 4);
#pragma unroll
            for (int kk = 0; kk < kTK / 16; ++kk)
                umma_ss(tmem, smem_desc_join(xlo + kk * 2, dhi), smem_desc_join(wlo + kk * 128, dhi), idesc,
                        (i > 0 || kk > 0) ? 1u : 0u);
            umma_commit(&sm.empty[s]);
        }
        umma_commit(&sm.acc_full);
    }
    __syncwarp();

    // The compaction pass may start launching now; it waits for this grid's
    // completion before reading anything.
    asm volatile("griddepcontrol.launch_dependents;");

    // Epilogue.  The stages are free once the accumulator is complete; the
    // partial logits go through them, one padded row per token
    // ([128][64*NB + 1] floats, conflict-free column access).
    constexpr int ld = 64 * NB + 1;
    float* lg_base = reinterpret_cast<float*>(&sm.x[0][0]);
    const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(&sm.acc_full, 0));
    tc_fence_after();
    if (!acc_ok) {
        if (lane == 0) sm.failed = 1;
    } else {
        float* lg = lg_base + (warp * 32 + lane) * ld;
#pragma unroll 1
        for (int c = 0; c < 2 * NB; ++c) {
            uint32_t r[32];
            tmem_ld32(tmem_addr(tmem, warp * 32, c * 32), r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) lg[c * 32 + e] = __uint_as_float(r[e]);
        }
    }
    if constexpr (KS > 1) {
        // Partial logits of every CTA of the cluster are in shared memory; this
        // CTA adds its peers' partials for its own rows, then a second barrier
        // ends all reads of peer memory before any CTA moves on or exits.
        cluster_sync();
        if (tid < kRows && !sm.failed) {
            const int row = (int)rank * kRows + tid;
            float* lg = lg_base + row * ld;
            const uint32_t mine = smem_u32(lg);
#pragma unroll 1
            for (int c = 1; c < KS; ++c) {
                const uint32_t peer = peer_addr(mine, (rank + c) % KS);
#pragma unroll 1
                for (int j = 0; j < h; j += 8) {  // h % 8 == 0 on this path
                    float v[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) v[e] = ld_peer(peer + 4u * (j + e));
#pragma unroll
                    for (int e = 0; e < 8; ++e) lg[j + e] += v[e];
                }
            }
        }
        cluster_sync();
    } else {
        __syncthreads();
    }
    const bool failed = sm.failed != 0;  // final: every writer is before the barrier above
    if (!failed && logits != nullptr) {
        // fp32 logits of this CTA's rows (bias included), heads fastest: coalesced
        for (int e = tid; e < kRows * h; e += 128) {
            const int rloc = e / h, j = e % h;
            const int row = (int)rank * kRows + rloc;
            const int64_t tok = tok0 + row;
            if (tok < BT) logits[tok * h + j] = lg_base[row * ld + j] + (bias ? bias[j] : 0.f);
        }
    }
    if (!failed) {
        // Top-k over (row, group) items, rows fastest: the 32 lanes of a warp
        // take 32 consecutive tokens of one group, which is also one chunk for
        // the selection counts.
        const int hpg = h / g;
        const int nitems = kRows * g;  // kRows is a multiple of 32: whole warps per group
        for (int it = tid; it < nitems; it += 128) {
            const int q = it / kRows, rloc = it % kRows;
            const int row = (int)rank * kRows + rloc;
            const int64_t tok = tok0 + row;
            const float* lq = lg_base + row * ld + q * hpg;
            const float* bq = bias ? bias + q * hpg : nullptr;
            uint64_t taken = 0;  // hpg <= 64 on this path
            if (tok < BT) {
                // top-k of the group's logits (+ bias), equal logits -> lower index
                int sel[KMAX];
                float sl[KMAX];
#pragma unroll
                for (int s = 0; s < KMAX; ++s) {
                    sel[s] = 0;
                    sl[s] = 0.f;
                    if (s < k) {
                        int best = -1;
                        float bv = 0.f;
                        for (int a = 0; a < hpg; ++a) {
                            if ((taken >> a) & 1ull) continue;
                            const float v = bq ? lq[a] + bq[a] : lq[a];
                            if (best < 0 || v > bv) {
                                best = a;
                                bv = v;
                            }
                        }
                        taken |= 1ull << best;
                        sel[s] = best;
                        sl[s] = bv;
                    }
                }
                const float m = sl[0];
                float denom = 0.f;
#pragma unroll
                for (int s = 0; s < KMAX; ++s)
                    if (s < k) {
                        sl[s] = expf(sl[s] - m);
                        denom += sl[s];
                    }
                const int64_t o = (tok * g + q) * k;
#pragma unroll
                for (int s = 0; s < KMAX; ++s)
                    if (s < k) {
                        idx[o + s] = q * hpg + sel[s];
                        gate[o + s] = sl[s] / denom;
                    }
            }
            const int64_t t_first = tok0 + (int)rank * kRows + (rloc - lane);  // the warp's first token
            if (counts != nullptr && t_first < BT) {
                const int cb = (int)(t_first / T), cc = (int)((t_first % T) / kChunk);
                for (int a = 0; a < hpg; ++a) {
                    const unsigned ball = __ballot_sync(0xffffffffu, (taken >> a) & 1ull);
                    if (lane == 0) counts[((int64_t)cb * h + q * hpg + a) * nchunk + cc] = __popc(ball);
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

// Shared-memory opt-in, once per device and kernel instance.
template <typename K>
cudaError_t set_smem_once(K kern, size_t smem, std::atomic<uint64_t>& done) {
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    const uint64_t bit = (dev < 64) ? (uint64_t(1) << dev) : 0;
    if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
    return err;
}

template <int NB, int KS, int KMAX>
cudaError_t launch_nb(const RouteArgs& a, bool fused_counts) {
    static std::atomic<uint64_t> configured{0};
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
    auto kern = router_tc_kernel<NB, KS, KMAX>;
    cudaError_t err = set_smem_once(kern, smem, configured);
    if (err != cudaSuccess) return err;
    const int64_t tiles = (BT + kTM - 1) / kTM;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(tiles * KS));
    cfg.blockDim = dim3(128);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = KS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = (KS > 1) ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, mapX, mapW, a.bias, BT, s.d_model, s.h, s.g, s.k, s.T,
                              gqe_chunk_count(s.T), a.idx, a.gate, fused_counts ? a.counts : (int32_t*)nullptr,
                              (uint32_t*)a.status, a.logits);
}

template <int NB, int KMAX>
cudaError_t launch_ks(const RouteArgs& a, bool fused_counts) {
    const gqe_shape& s = *a.s;
    const int64_t tiles = ((int64_t)s.B * s.T + kTM - 1) / kTM;
    const int nk = (s.d_model + kTK - 1) / kTK;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    // split d_model over a cluster while the grid would leave SMs idle
    if (tiles * 4 <= sms && nk >= 4) return launch_nb<NB, 4, KMAX>(a, fused_counts);
    if (tiles * 2 <= sms && nk >= 2) return launch_nb<NB, 2, KMAX>(a, fused_counts);
    return launch_nb<NB, 1, KMAX>(a, fused_counts);
}

}  // namespace

bool router_tc_supported(const gqe_shape* s) {
    return s->dtype == GQE_BF16 && s->h % 8 == 0 && s->h <= 256 && s->d_model % 8 == 0 && s->h / s->g <= 64;
}

bool router_tc_fuses_counts(const gqe_shape* s) { return s->T % kChunk == 0; }

cudaError_t launch_router_tc(const RouteArgs& a) {
    const int h = a.s->h;
    const bool fused = router_tc_fuses_counts(a.s);
    // selections held in registers: up to 4 (every configuration here), else 16
    if (a.s->k <= 4) {
        if (h <= 64) return launch_ks<1, 4>(a, fused);
        if (h <= 128) return launch_ks<2, 4>(a, fused);
        return launch_ks<4, 4>(a, fused);
    }
    if (h <= 64) return launch_ks<1, 16>(a, fused);
    if (h <= 128) return launch_ks<2, 16>(a, fused);
    return launch_ks<4, 16>(a, fused);
}

}  // namespace gqe
