// proj_tc.cu -- the routed projections around the attention on the sm_100a
// tensor cores, as tiled GEMMs that skip the work no token of a tile routed.
//
// Output projection.  The heads' outputs pass through one more linear layer
// with weight matrix W_Z (IBM GQA page, multi-head attention mechanics); under
// GQE only the selected experts are computed ("Grouped Query Experts:
// Mixture-of-Experts on GQA Self-Attention", gist.science summary,
// "Activation Conditionnelle"), so a token's layer output is the sum over the
// heads it selected:
//   Y[b,t,:] = sum_{q, r} O[b,t,j,:] . W_Z[j*d_h : (j+1)*d_h, :],  j = idx[b,t,q,r].
// O is the gated routed output with zeros in the unselected slots (as the
// routed prefill and decode write it), so this is the product of the
// concatenated head slots with W_Z in which every head that no token of a
// 128-token tile selected drops out of that tile's K loop.
//
// Query projection, dense path.  Q[b,t,j,:] = x[b,t,:] . W_Q[:, j-block] for the
// routed (t, j) (same page, "Activation Conditionnelle").  Here a tile is 128
// tokens x 256 columns of the h*d_h query columns (two heads); a tile none of
// whose heads any of its tokens selected is skipped, and only the routed
// (t, j) rows are written.  Under per-token routing nearly every tile has a
// routed head, so this does the dense product's work; it beats gathering each
// head's routed rows when the routed share g*k/h is not small (qproj.cu
// chooses).
//
// Both: persistent CTA per SM, output tiles of 128 tokens x 256 columns,
// token-tile major (the CTAs in flight share each token tile's A rows and all
// of the weight through L2), dealt in snake order.  Warp 0 streams the stages
// by TMA: A's [128 tokens][64] box (K-major) and the weight's four [64 k][64 n]
// blocks (MN-major), 48 KB per stage, 4 stages.  Warp 1 issues M128 N256 K16
// MMAs into one of two TMEM accumulators (256 columns each), so the epilogue of
// a tile overlaps the next tile's MMAs.  Warps 2-5 read the accumulator
// (thread = token row), round to bf16 and store.  The active-head set of a
// token tile (the OR of its tokens' selections) comes from a first small
// kernel, one warp per tile, into the workspace; every role of the main
// kernel loads the next tile's set while it works on the current one.  Every
// sum runs in a fixed order: the results are reproducible.
#include <atomic>

#include "common.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kM = 128;                     // tokens per tile (UMMA M)
constexpr int kN = 256;                     // output columns per tile (UMMA N)
constexpr int kTK = 64;                     // K per stage (one 128-byte swizzle row of bf16)
constexpr int kStages = 4;
constexpr uint32_t kABytes = kM * kTK * 2;  // 16 KB
constexpr uint32_t kBBlock = kTK * 64 * 2;  // [64 k][64 n], 8 KB
constexpr uint32_t kBBytes = 4 * kBBlock;   // 32 KB
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kWhereOproj = 10;

struct OprojSmem {
    uint8_t a[kStages][kABytes];
    uint8_t b[kStages][kBBytes];
    uint64_t full[kStages], empty[kStages];
    uint64_t acc_full[2], acc_empty[2], drain;
    uint32_t tmem_base;
    int32_t failed;
};

struct ProjParams {
    int64_t BT;             // tokens
    int h, per, d_h;        // heads, selections per token (g*k), head size
    int N;                  // output row length (d_model, or h*d_h for Q)
    int ksteps;             // K steps of 64: per head (output projection) or in all (Q)
    int64_t m_tiles, n_tiles;
    const uint64_t* masks;  // [m_tiles] active heads of each token tile
    const int32_t* idx;     // [B*T, g*k] (Q: which rows to write)
    __nv_bfloat16* out;     // [B*T, N]
    uint32_t* status;
};

__device__ __forceinline__ int64_t snake_tile(int64_t v) {
    const int64_t G = gridDim.x, c = blockIdx.x;
    return v * G + ((v & 1) ? (G - 1 - c) : c);
}

// Heads selected by at least one token of each 128-token tile (bit j), one
// warp per tile: 16-byte loads of the tile's selections (the tile's slice of
// idx starts 16-byte aligned: 128 tokens x g*k x 4 bytes), all in flight at
// once.  An index outside [0, h) is reported and ignored.
__global__ void __launch_bounds__(256)
oproj_masks_kernel(const int32_t* __restrict__ idx, int64_t BT, int per, int h, int64_t m_tiles,
                   uint64_t* __restrict__ masks, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int64_t mt = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (mt >= m_tiles) return;
    const int64_t t0 = mt * kM;
    const int64_t n = (min(t0 + kM, BT) - t0) * per;
    const int32_t* base = idx + t0 * per;
    uint64_t m = 0;
    bool bad = false;
    auto add = [&](int j) {
        if (j >= 0 && j < h) {
            m |= 1ull << j;
        } else {
            bad = true;
        }
    };
    const int64_t n4 = n >> 2;
    const int4* base4 = reinterpret_cast<const int4*>(base);
    for (int64_t e = lane; e < n4; e += 4 * 32) {
        int4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) v[u] = (e + u * 32 < n4) ? base4[e + u * 32] : make_int4(0, 0, 0, 0);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            if (e + u * 32 >= n4) continue;
            add(v[u].x);
            add(v[u].y);
            add(v[u].z);
            add(v[u].w);
        }
    }
    for (int64_t e = 4 * n4 + lane; e < n; e += 32) add(base[e]);
    if (bad) report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereOproj, 1);
    const uint32_t lo = __reduce_or_sync(0xffffffffu, (uint32_t)m);
    const uint32_t hi = __reduce_or_sync(0xffffffffu, (uint32_t)(m >> 32));
    if (lane == 0) masks[mt] = ((uint64_t)hi << 32) | lo;
}

// Heads covered by output column tile nt of the Q projection.
__device__ __forceinline__ uint64_t ntile_heads(const ProjParams& p, int64_t nt) {
    const int hpt = kN / p.d_h;
    const int j0 = (int)nt * hpt;
    return (hpt >= 64 ? ~0ull : ((1ull << hpt) - 1)) << j0;
}

// K steps of one tile: the output projection runs ksteps per active head, the
// Q projection all of K for a tile with a routed head and nothing otherwise.
template <bool kQ>
__device__ __forceinline__ int tile_steps(const ProjParams& p, uint64_t mask, int64_t nt) {
    if (kQ) return (mask & ntile_heads(p, nt)) ? p.ksteps : 0;
    return __popcll(mask) * p.ksteps;
}

template <bool kQ>
__global__ void __launch_bounds__(kThreads, 1)
proj_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapW, const ProjParams p) {
    extern __shared__ uint8_t smem_raw[];
    OprojSmem& sm = *smem_align1024<OprojSmem>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t n_tiles = p.m_tiles * p.n_tiles;
    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.acc_full[i], 1);
            mbar_init(&sm.acc_empty[i], 32 * kEpiWarps);
        }
        mbar_init(&sm.drain, 1);
        sm.failed = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 2 * kN);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // warp-uniform: whether any role has given up
    auto failed = [&]() { return __any_sync(0xffffffffu, *((volatile int32_t*)&sm.failed) != 0); };

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        uint32_t ks = 0;  // stages issued
        bool ok = true;
        if (lane == 0) {
            tma_prefetch_desc(&mapA);
            tma_prefetch_desc(&mapW);
        }
        uint64_t next = n_tiles > 0 ? p.masks[snake_tile(0) / p.n_tiles] : 0;
        for (int64_t v = 0, it = snake_tile(0); it < n_tiles && ok && !failed(); it = snake_tile(++v)) {
            const int64_t mt = it / p.n_tiles, nt = it % p.n_tiles;
            uint64_t heads = next;
            const int64_t it1 = snake_tile(v + 1);
            next = it1 < n_tiles ? p.masks[it1 / p.n_tiles] : 0;
            const int nsteps = tile_steps<kQ>(p, heads, nt);
            int j = -1;  // output projection: the head of the current K steps
            for (int st = 0; st < nsteps; ++st, ++ks) {
                int kcol;
                if (kQ) {
                    kcol = st * kTK;
                } else {
                    const int s2 = st % p.ksteps;
                    if (s2 == 0) {
                        j = __ffsll((long long)heads) - 1;
                        heads &= heads - 1;
                    }
                    kcol = j * p.d_h + s2 * kTK;
                }
                const int s = ks % kStages;
                if (lane == 0) {
                    if (!mbar_wait(&sm.empty[s], ((ks / kStages) & 1) ^ 1)) {
                        sm.failed = 1;
                        ok = false;
                    } else {
                        mbar_arrive_expect_tx(&sm.full[s], kABytes + kBBytes);
                        tma_load_2d(&mapA, &sm.full[s], sm.a[s], kcol, (int)(mt * kM));
#pragma unroll
                        for (int nb = 0; nb < 4; ++nb)
                            tma_load_2d(&mapW, &sm.full[s], sm.b[s] + nb * kBBlock, (int)(nt * kN + nb * 64), kcol);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                if (!ok) break;
            }
        }
        // every issued load lands before the CTA may exit
        if (lane == 0)
            for (uint32_t back = 1; back <= kStages && back <= ks; ++back) {
                const uint32_t x = ks - back;
                mbar_wait(&sm.full[x % kStages], (x / kStages) & 1);
            }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = idesc_bf16_f32(kM, kN, false, true);
        const uint32_t dhi = smem_desc_hi(1024, kSwizzle128B);
        const uint32_t alo0 = smem_desc_lo(smem_u32(sm.a[0]), 16);
        const uint32_t blo0 = smem_desc_lo(smem_u32(sm.b[0]), kBBlock);
        uint32_t ks = 0, tn = 0;  // stages consumed, tiles
        bool ok = true;
        uint64_t next = n_tiles > 0 ? p.masks[snake_tile(0) / p.n_tiles] : 0;
        for (int64_t v = 0, it = snake_tile(0); it < n_tiles && ok && !failed(); it = snake_tile(++v), ++tn) {
            const int nsteps = tile_steps<kQ>(p, next, it % p.n_tiles);
            const int64_t it1 = snake_tile(v + 1);
            next = it1 < n_tiles ? p.masks[it1 / p.n_tiles] : 0;
            const uint32_t buf = tn & 1;
            if (lane == 0) {
                // the epilogue has read this accumulator's previous tile
                if (!mbar_wait(&sm.acc_empty[buf], ((tn >> 1) & 1) ^ 1)) {
                    sm.failed = 1;
                    ok = false;
                }
                tc_fence_after();
                for (int st = 0; st < nsteps && ok; ++st, ++ks) {
                    const int s = ks % kStages;
                    if (!mbar_wait(&sm.full[s], (ks / kStages) & 1)) {
                        sm.failed = 1;
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t alo = alo0 + (uint32_t)s * (kABytes >> 4);
                    const uint32_t blo = blo0 + (uint32_t)s * (kBBytes >> 4);
#pragma unroll
                    for (int kk = 0; kk < kTK / 16; ++kk)
                        umma_ss(tmem + buf * kN, smem_desc_join(alo + kk * 2, dhi), smem_desc_join(blo + kk * 128, dhi),
                                idesc, (st > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&sm.empty[s]);
                }
                if (ok) {
                    if (nsteps > 0) {
                        umma_commit(&sm.acc_full[buf]);
                    } else {
                        mbar_arrive(&sm.acc_full[buf]);  // nothing to accumulate (see the epilogue)
                    }
                }
            }
            ok = __shfl_sync(0xffffffffu, ok, 0);
        }
        if (lane == 0) {
            // every MMA has completed before TMEM is released
            umma_commit(&sm.drain);
            mbar_wait(&sm.drain, 0);
        }
    } else {
        // ------------------------------------------------------------ epilogue (thread = token row)
        const int quarter = warp & 3;  // the TMEM lane quarter this warp may read
        const int r = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        uint32_t tn = 0;
        for (int64_t v = 0, it = snake_tile(0); it < n_tiles && !failed(); it = snake_tile(++v), ++tn) {
            const int64_t mt = it / p.n_tiles, nt = it % p.n_tiles;
            const bool any = tile_steps<kQ>(p, p.masks[mt], nt) > 0;
            const uint32_t buf = tn & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full[buf], (tn >> 1) & 1))) {
                if (lane == 0) sm.failed = 1;
                break;
            }
            tc_fence_after();
            const int64_t tok = mt * kM + r;
            __nv_bfloat16* dst = p.out + (tok < p.BT ? tok : 0) * p.N + nt * kN;
            // Q: the heads this token selected; the output projection writes every column
            uint64_t wsel = ~0ull;
            if (kQ) {
                wsel = 0;
                if (tok < p.BT)
                    for (int e = 0; e < p.per; ++e) {
                        const int j = p.idx[tok * p.per + e];
                        if (j >= 0 && j < p.h) wsel |= 1ull << j;
                    }
            }
#pragma unroll 1
            for (int c = 0; c < kN / 32; ++c) {
                if (kQ && !any) break;  // a skipped Q tile writes nothing
                uint32_t o[32];
                if (any) {
                    tmem_ld32(tmem + lane_off + buf * kN + c * 32, o);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = 0u;
                }
                const int col = (int)nt * kN + c * 32;
                if (tok < p.BT && col < p.N && ((wsel >> (col / p.d_h)) & 1)) {
                    uint4* y = reinterpret_cast<uint4*>(dst + c * 32);
#pragma unroll
                    for (int q = 0; q < 4; ++q)
                        y[q] = make_uint4(pack_bf16x2(__uint_as_float(o[8 * q + 0]), __uint_as_float(o[8 * q + 1])),
                                          pack_bf16x2(__uint_as_float(o[8 * q + 2]), __uint_as_float(o[8 * q + 3])),
                                          pack_bf16x2(__uint_as_float(o[8 * q + 4]), __uint_as_float(o[8 * q + 5])),
                                          pack_bf16x2(__uint_as_float(o[8 * q + 6]), __uint_as_float(o[8 * q + 7])));
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.acc_empty[buf]);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kN);
    }
    if (tid == 0 && sm.failed && p.status != nullptr)
        report_error(p.status, GQE_ERR_DEVICE_TIMEOUT, kWhereOproj, blockIdx.x);
}

// Masks pre-pass, then the tiled GEMM; A as [B*T, K] (K-major boxes), the
// weight as [K, N] (MN-major blocks).
template <bool kQ>
cudaError_t launch_proj(ProjParams p, const void* A, const void* Wt, uint64_t K, const int32_t* idx, int g, int k,
                        void* scratch, cudaStream_t stream) {
    static std::atomic<uint64_t> configured{0};
    p.m_tiles = (p.BT + kM - 1) / kM;
    p.n_tiles = (p.N + kN - 1) / kN;
    p.masks = reinterpret_cast<const uint64_t*>(scratch);
    CUtensorMap mapA, mapW;
    {
        const uint64_t dims[2] = {K, (uint64_t)p.BT};
        const uint64_t strides[1] = {K * 2};
        const uint32_t box[2] = {kTK, kM};
        if (!make_bf16_map(&mapA, A, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)p.N, K};
        const uint64_t strides[1] = {(uint64_t)p.N * 2};
        const uint32_t box[2] = {64, kTK};
        if (!make_bf16_map(&mapW, Wt, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }
    const size_t smem = sizeof(OprojSmem) + 1024;
    int dev = 0, sms = 148;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const uint64_t bit = dev < 64 ? (uint64_t(1) << dev) : 0;
    if (!bit || !(configured.load(std::memory_order_acquire) & bit)) {
        err = cudaFuncSetAttribute(proj_kernel<kQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (err != cudaSuccess) return err;
        if (bit) configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    oproj_masks_kernel<<<(unsigned)((p.m_tiles * 32 + 255) / 256), 256, 0, stream>>>(
        idx, p.BT, g * k, p.h, p.m_tiles, reinterpret_cast<uint64_t*>(scratch), p.status);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    const int64_t tiles = p.m_tiles * p.n_tiles;
    const int grid = (int)(tiles < sms ? tiles : sms);
    proj_kernel<kQ><<<grid, kThreads, smem, stream>>>(mapA, mapW, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_oproj(const OprojArgs& a) {
    const gqe_shape& s = *a.s;
    ProjParams p;
    p.BT = (int64_t)s.B * s.T;
    p.h = s.h;
    p.per = s.g * s.k;
    p.d_h = s.d_h;
    p.N = s.d_model;
    p.ksteps = s.d_h / kTK;
    p.idx = a.idx;
    p.out = (__nv_bfloat16*)a.Y;
    p.status = (uint32_t*)a.status;
    return launch_proj<false>(p, a.O, a.W_Z, (uint64_t)s.h * s.d_h, a.idx, s.g, s.k, a.scratch, a.stream);
}

cudaError_t launch_qproj_dense(const QprojArgs& a) {
    const gqe_shape& s = *a.s;
    ProjParams p;
    p.BT = (int64_t)s.B * s.T;
    p.h = s.h;
    p.per = s.g * s.k;
    p.d_h = s.d_h;
    p.N = s.h * s.d_h;
    p.ksteps = (s.d_model + kTK - 1) / kTK;
    p.idx = a.idx;
    p.out = (__nv_bfloat16*)a.Q;
    p.status = (uint32_t*)a.status;
    return launch_proj<true>(p, a.x, a.W_Q, (uint64_t)s.d_model, a.idx, s.g, s.k, a.scratch, a.stream);
}

size_t oproj_scratch_bytes(const gqe_shape* s) {
    const int64_t m_tiles = ((int64_t)s->B * s->T + kM - 1) / kM;
    return (size_t)(m_tiles * 8 + 255) & ~size_t(255);
}

}  // namespace gqe
