// router.cu -- GQE router (fp32 logits, per-group top-k, renormalised gates)
// on CUDA cores for the inputs the tensor-core router (router_tc.cu) does not
// take (fp32, or h not a multiple of 8), and token compaction (warp ballot +
// prefix sum).
//
// Router: "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
// (gist.science summary), "Architecture et Routage": per token, k query-head
// experts are selected in every GQA group; "Somme Ponderee Renormalisee": the
// router probabilities are renormalised over the selected experts.  The linear
// router x . W_r (+ bias) and the tie rule (lower head index first) are this
// library's reading of an unspecified router.
#include "common.cuh"

namespace gqe {
namespace {

constexpr int kRouterThreads = 256;
constexpr int kRouterTokPerThread = 4;
constexpr int kRouterKC = 32;  // d_model chunk staged in shared memory
constexpr uint32_t kWhereScan = 7;  // status "where" id of the compaction scan

// One block: kRouterTokPerThread * tokgroups tokens, all h heads.
// Thread (tg, j): head j, tokens tg*4 .. tg*4+3 of the block.
template <typename T>
__global__ void __launch_bounds__(kRouterThreads)
router_kernel(const T* __restrict__ x, const T* __restrict__ W, const float* __restrict__ bias,
              int64_t BT, int d_model, int h, int g, int k, int32_t* __restrict__ idx,
              float* __restrict__ gate, float* __restrict__ logits) {
    extern __shared__ float smem[];
    const int tokgroups = blockDim.x / h;
    const int tok_per_block = tokgroups * kRouterTokPerThread;
    float* xs = smem;                                   // [tok_per_block][kRouterKC + 1]
    float* ws = xs + tok_per_block * (kRouterKC + 1);   // [kRouterKC][h]
    float* lg = ws + kRouterKC * h;                     // [tok_per_block][h]

    const int64_t tok0 = (int64_t)blockIdx.x * tok_per_block;
    const int tid = threadIdx.x;
    const int j = tid % h;
    const int tg = tid / h;
    const bool active = tg < tokgroups;

    float acc[kRouterTokPerThread];
#pragma unroll
    for (int r = 0; r < kRouterTokPerThread; ++r) acc[r] = 0.f;

    for (int c0 = 0; c0 < d_model; c0 += kRouterKC) {
        const int kc = min(kRouterKC, d_model - c0);
        for (int e = tid; e < tok_per_block * kRouterKC; e += blockDim.x) {
            const int tt = e / kRouterKC, cc = e % kRouterKC;
            const int64_t tok = tok0 + tt;
            float v = 0.f;
            if (tok < BT && cc < kc) v = Elem<T>::to_f(x[tok * d_model + c0 + cc]);
            xs[tt * (kRouterKC + 1) + cc] = v;
        }
        for (int e = tid; e < kRouterKC * h; e += blockDim.x) {
            const int cc = e / h, jj = e % h;
            ws[e] = (cc < kc) ? Elem<T>::to_f(W[(int64_t)(c0 + cc) * h + jj]) : 0.f;
        }
        __syncthreads();
        if (active) {
            for (int cc = 0; cc < kc; ++cc) {
                const float w = ws[cc * h + j];
#pragma unroll
                for (int r = 0; r < kRouterTokPerThread; ++r)
                    acc[r] = fmaf(xs[(tg * kRouterTokPerThread + r) * (kRouterKC + 1) + cc], w, acc[r]);
            }
        }
        __syncthreads();
    }
    if (active) {
        const float bj = bias ? bias[j] : 0.f;
#pragma unroll
        for (int r = 0; r < kRouterTokPerThread; ++r) {
            const int64_t tok = tok0 + tg * kRouterTokPerThread + r;
            lg[(tg * kRouterTokPerThread + r) * h + j] = acc[r] + bj;
            if (logits != nullptr && tok < BT) logits[tok * h + j] = acc[r] + bj;
        }
    }
    __syncthreads();

    // Per (token, group): top-k by logit, ties to the lower head index; gates.
    const int hpg = h / g;
    for (int e = tid; e < tok_per_block * g; e += blockDim.x) {
        const int tt = e / g, q = e % g;
        const int64_t tok = tok0 + tt;
        if (tok >= BT) continue;
        const float* l = lg + tt * h + q * hpg;
        int sel[16];
        float sel_l[16];
        float m = 0.f, denom = 0.f;
        for (int s = 0; s < k; ++s) {
            int best = -1;
            float bv = 0.f;
            for (int a = 0; a < hpg; ++a) {
                bool taken = false;
                for (int u = 0; u < s; ++u) taken |= (sel[u] == a);
                if (taken) continue;
                if (best < 0 || l[a] > bv) {  // strict: equal logits keep the lower index
                    best = a;
                    bv = l[a];
                }
            }
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

// Compaction pass 1: per (b, chunk of 32 tokens, head) the number of tokens
// routed to the head.  One warp per (b, chunk, group); lane = token.  The
// tensor-core router computes the same counts in its epilogue when T is a
// multiple of the chunk; this pass serves the other inputs.
__global__ void compact_count_kernel(const int32_t* __restrict__ idx, int T, int h, int g, int k,
                                     int nchunk, int32_t* __restrict__ counts) {
    const int c = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int hpg = h / g;
    const int t = c * kChunk + lane;
    for (int q = warp; q < g; q += nwarps) {
        int sel[16];
        for (int s = 0; s < k; ++s) sel[s] = (t < T) ? idx[(((int64_t)b * T + t) * g + q) * k + s] : -1;
        for (int jj = 0; jj < hpg; ++jj) {
            const int j = q * hpg + jj;
            bool hit = false;
            for (int s = 0; s < k; ++s) hit |= (sel[s] == j);
            const unsigned ball = __ballot_sync(0xffffffffu, hit);
            if (lane == 0) counts[((int64_t)b * h + j) * nchunk + c] = __popc(ball);
        }
    }
}

// Compaction pass 2: write positions, with the offsets each block needs.
// Block (chunk c, batch b) first derives, from the batch's counts, the
// head-major exclusive prefix of every (head, c): the sum of all earlier
// heads' totals plus head j's counts in chunks before c (one warp per head,
// lanes striding over chunks; then one warp scans the head totals).  The
// counts of a batch are a few KB, so every block re-reading them costs less
// than a separate scan launch.  Then it scatters as pass 1 counted: a lane's
// rank within its head's chunk is the popcount of the ballot below it.
__global__ void compact_scan_scatter_kernel(const int32_t* __restrict__ idx, int B, int T, int h, int g, int k,
                                            int nchunk, const int32_t* __restrict__ counts,
                                            int32_t* __restrict__ head_offsets,
                                            int32_t* __restrict__ head_chunk_offsets,
                                            int32_t* __restrict__ head_pos, uint32_t* __restrict__ status) {
    extern __shared__ int32_t sh[];  // [h] head totals -> head bases, [h] prefix within head
    int32_t* total = sh;
    int32_t* before = sh + h;
    // Launched as a programmatic dependent of the router: wait for its grid,
    // then let the prefill that follows start its set-up.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    const int c = blockIdx.x, b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int32_t* cnt = counts + (int64_t)b * h * nchunk;
    // Counts that do not match a complete routing (a router that gave up on a
    // bounded wait leaves idx and counts unwritten) must not steer a write out
    // of the batch's T*g*k entries: sums are clamped to that range here and
    // every scatter index is checked below.
    const long long per_batch = (long long)T * g * k;
    // Sums in 32 bits: each clamped count is at most 32, so a head's total is
    // at most 32 * nchunk < T + 32.  Lanes stride over the chunks (coalesced).
    for (int j = warp; j < h; j += nwarps) {
        const int32_t* row = cnt + (int64_t)j * nchunk;
        int tot = 0, pre = 0;
        for (int cc = lane; cc < nchunk; cc += 32) {
            const int v = min(max(row[cc], 0), kChunk);
            tot += v;
            pre += (cc < c) ? v : 0;
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
            tot += __shfl_xor_sync(0xffffffffu, tot, d);
            pre += __shfl_xor_sync(0xffffffffu, pre, d);
        }
        if (lane == 0) {
            total[j] = (int32_t)min((long long)tot, per_batch);
            before[j] = (int32_t)min((long long)pre, per_batch);
        }
    }
    __syncthreads();
    if (warp == 0) {
        long long carry = 0;
        for (int j0 = 0; j0 < h; j0 += 32) {
            const int j = j0 + lane;
            const long long v = (j < h) ? total[j] : 0;
            long long incl = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, d);
                if (lane >= d) incl += y;
            }
            if (j < h) total[j] = (int32_t)min(carry + incl - v, (long long)per_batch);  // head j's base
            carry = min(carry + __shfl_sync(0xffffffffu, incl, 31), (long long)per_batch);
        }
    }
    __syncthreads();
    const int64_t base = (int64_t)b * per_batch;  // every batch holds exactly T*g*k entries
    for (int j = threadIdx.x; j < h; j += blockDim.x) {
        const int32_t off = (int32_t)(base + min((long long)total[j] + before[j], per_batch));
        head_chunk_offsets[((int64_t)b * h + j) * nchunk + c] = off;
        if (c == 0) head_offsets[(int64_t)b * h + j] = off;
    }
    if (b == B - 1 && c == 0 && threadIdx.x == 0) head_offsets[(int64_t)B * h] = (int32_t)((int64_t)B * T * g * k);

    const int hpg = h / g;
    const int t = c * kChunk + lane;
    const unsigned below = (1u << lane) - 1u;
    for (int q = warp; q < g; q += nwarps) {
        // the token's selections in group q as a bit mask of heads within the
        // group (groups of more than 64 heads compare against idx directly)
        const int32_t* sel = idx + (((int64_t)b * T + (t < T ? t : 0)) * g + q) * k;
        uint64_t chosen = 0;
        if (t < T && hpg <= 64) {
            for (int s = 0; s < k; ++s) {
                const int a = sel[s] - q * hpg;
                if (a >= 0 && a < hpg) chosen |= 1ull << a;
            }
        }
        for (int jj = 0; jj < hpg; ++jj) {
            const int j = q * hpg + jj;
            bool hit = false;
            if (hpg <= 64) {
                hit = (chosen >> jj) & 1ull;
            } else if (t < T) {
                for (int s = 0; s < k; ++s) hit |= (sel[s] == j);
            }
            const unsigned ball = __ballot_sync(0xffffffffu, hit);
            if (hit) {
                const long long e = (long long)total[j] + before[j] + __popc(ball & below);
                if (e < per_batch) {
                    head_pos[base + e] = t;
                } else if (status != nullptr) {  // counts and selections disagree: report, skip
                    report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereScan, (uint32_t)b);
                }
            }
        }
    }
}

}  // namespace

cudaError_t launch_route(const RouteArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const int tokgroups = kRouterThreads / s.h;
    const int tok_per_block = tokgroups * kRouterTokPerThread;
    const int threads = tokgroups * s.h;
    const size_t smem = sizeof(float) * ((size_t)tok_per_block * (kRouterKC + 1) +
                                         (size_t)kRouterKC * s.h + (size_t)tok_per_block * s.h);
    const unsigned blocks = (unsigned)((BT + tok_per_block - 1) / tok_per_block);
    if (router_tc_supported(a.s)) {
        cudaError_t e = launch_router_tc(a);
        if (e != cudaSuccess) return e;
    } else if (s.dtype == GQE_BF16) {
        auto kern = router_kernel<__nv_bfloat16>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<blocks, threads, smem, a.stream>>>((const __nv_bfloat16*)a.x, (const __nv_bfloat16*)a.W_r,
                                                  a.bias, BT, s.d_model, s.h, s.g, s.k, a.idx, a.gate, a.logits);
    } else {
        auto kern = router_kernel<float>;
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        kern<<<blocks, threads, smem, a.stream>>>((const float*)a.x, (const float*)a.W_r, a.bias, BT,
                                                  s.d_model, s.h, s.g, s.k, a.idx, a.gate, a.logits);
    }
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;

    const int nchunk = gqe_chunk_count(s.T);
    const int cwarps = s.g < 8 ? s.g : 8;
    dim3 cgrid(nchunk, s.B);
    if (!(router_tc_supported(a.s) && router_tc_fuses_counts(a.s)))
        compact_count_kernel<<<cgrid, 32 * cwarps, 0, a.stream>>>(a.idx, s.T, s.h, s.g, s.k, nchunk, a.counts);
    const int swarps = 8;  // warps of the scan: one head per warp and round
    // Programmatic dependent launch: this grid is scheduled while the router
    // finishes and waits (griddepcontrol.wait) for it before reading.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = cgrid;
    cfg.blockDim = dim3(32 * swarps);
    cfg.dynamicSmemBytes = 2 * s.h * sizeof(int32_t);
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e2 = cudaLaunchKernelEx(&cfg, compact_scan_scatter_kernel, (const int32_t*)a.idx, s.B, s.T, s.h,
                                        s.g, s.k, nchunk, (const int32_t*)a.counts, a.head_offsets,
                                        a.head_chunk_offsets, a.head_pos, (uint32_t*)a.status);
    if (e2 != cudaSuccess) return e2;
    return cudaGetLastError();
}

}  // namespace gqe

// ---------------------------------------------------------------------------
// Scratch owned by the library, for callers that cannot allocate device memory
// (gqe_route_static): the status word of those calls, then their per-chunk
// counts.  Every device that loads this library holds one copy of the array
// until the process exits; the loader zero-fills it, so the status word starts
// clear.  In host code the array's name is only a
// host-side stand-in: the device address of this device's copy comes from
// cudaGetSymbolAddress, looked up once per device with that device current.
// ---------------------------------------------------------------------------
#include <mutex>

static __device__ __align__(256) uint8_t g_route_static_scratch[gqe::kStatusBytes + gqe::kRouteStaticScratchBytes];

namespace gqe {

cudaError_t route_static_scratch(uint8_t** out) {
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static uint8_t* addr[kMaxDevices] = {};
    int dev = -1;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(mu);
    if (addr[dev] == nullptr) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_route_static_scratch);
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<uint8_t*>(p);
    }
    *out = addr[dev];
    return cudaSuccess;
}

}  // namespace gqe
