// aux_loss.cu -- load-balancing auxiliary loss of the GQE router and its
// gradient with respect to the router logits.
//
// The GQE summary (gist.science, "Entrainement et Perte") adds to the language
// modelling loss an auxiliary load-balancing loss that makes the router spread
// the tokens evenly over the experts (query heads) of each group; it gives no
// formula.  This library's reading is the fraction-times-probability form of
// mixture-of-experts routers, per group and averaged over the groups.  With N
// tokens, hpg = h/g heads per group and p[t,j] the softmax of token t's logits
// over all heads of j's group:
//   f_j = (number of tokens whose selection holds j) / (N k)
//   P_j = (1/N) sum_t p[t,j]
//   L   = (1/g) sum_q hpg sum_{j in q} f_j P_j          (1 when both are uniform)
//   dL/dl[t,j] = hpg/(g N) * p[t,j] * (f_j - sum_{i in q} p[t,i] f_i)
// (the counts f are piecewise constant and pass no gradient).
//
// Three launches, all HBM-bound on the logits (N*h*4 bytes read, as many
// written for the gradient): (1) selection counts per head, integer atomics;
// (2) one warp per (32 tokens, group): the group softmax of each token, the
// gradient, and the warp's per-head probability sums (butterfly reduction, a
// fixed order); (3) one block adds the warps' sums in a fixed order (fp64) and
// forms the loss.  The result is bit-reproducible.
#include "common.cuh"

namespace gqe {
namespace {

constexpr uint32_t kWhereAux = 8;
constexpr int kAuxMaxHpg = 64;

__global__ void aux_counts_kernel(const int32_t* __restrict__ idx, int64_t N, int h, int g, int k,
                                  int32_t* __restrict__ counts, uint32_t* __restrict__ status) {
    extern __shared__ int32_t cnt_s[];  // [h]
    for (int j = threadIdx.x; j < h; j += blockDim.x) cnt_s[j] = 0;
    __syncthreads();
    const int hpg = h / g;
    const int64_t items = N * g;
    for (int64_t it = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; it < items;
         it += (int64_t)gridDim.x * blockDim.x) {
        const int q = (int)(it % g);
        for (int s = 0; s < k; ++s) {
            const int j = idx[it * k + s];
            if (j < q * hpg || j >= (q + 1) * hpg) {  // not a head of this group: report, skip
                report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereAux, (uint32_t)q);
                continue;
            }
            atomicAdd(&cnt_s[j], 1);
        }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < h; j += blockDim.x)
        if (cnt_s[j]) atomicAdd(&counts[j], cnt_s[j]);
}

// Warp w: tokens [32*(w / g), +32), group w % g; lane = token.
__global__ void aux_probs_kernel(const float* __restrict__ logits, const int32_t* __restrict__ counts, int64_t N,
                                 int h, int g, int k, float* __restrict__ dlogits, float* __restrict__ partial) {
    const int64_t wglob = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nblk = (N + 31) / 32;
    if (wglob >= nblk * g) return;  // whole warps leave together
    const int hpg = h / g;
    const int q = (int)(wglob % g);
    const int64_t tb = wglob / g;
    const int64_t t = tb * 32 + lane;
    const bool live = t < N;
    const double inv_nk = 1.0 / ((double)N * k);
    float p[kAuxMaxHpg];
    float m = -INFINITY;
    const float* lt = logits + t * h + q * hpg;
#pragma unroll 4
    for (int a = 0; a < hpg; ++a) {
        p[a] = live ? lt[a] : 0.f;
        m = fmaxf(m, p[a]);
    }
    float den = 0.f;
#pragma unroll 4
    for (int a = 0; a < hpg; ++a) {
        p[a] = live ? expf(p[a] - m) : 0.f;
        den += p[a];
    }
    const float inv = live ? 1.0f / den : 0.f;
    float pf = 0.f;
#pragma unroll 4
    for (int a = 0; a < hpg; ++a) {
        p[a] *= inv;
        pf += p[a] * (float)(counts[q * hpg + a] * inv_nk);
    }
    if (dlogits != nullptr && live) {
        const float c = (float)((double)hpg / ((double)g * (double)N));
        float* dt = dlogits + t * h + q * hpg;
#pragma unroll 4
        for (int a = 0; a < hpg; ++a) dt[a] = c * p[a] * ((float)(counts[q * hpg + a] * inv_nk) - pf);
    }
    // per-head sums over the warp's 32 tokens (butterfly: a fixed order)
    for (int a = 0; a < hpg; ++a) {
        float v = p[a];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) v += __shfl_xor_sync(0xffffffffu, v, d);
        if (lane == 0) partial[tb * h + q * hpg + a] = v;
    }
}

__global__ void aux_loss_kernel(const float* __restrict__ partial, const int32_t* __restrict__ counts, int64_t N,
                                int h, int g, int k, float* __restrict__ loss) {
    extern __shared__ double terms[];  // [h]: hpg/g * f_j * P_j
    const int64_t nblk = (N + 31) / 32;
    const int hpg = h / g;
    // one warp per head: lanes stride over the token blocks, then a butterfly
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int j = warp; j < h; j += nw) {
        double acc = 0.0;
        for (int64_t b = lane; b < nblk; b += 32) acc += (double)partial[b * h + j];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);
        if (lane == 0) {
            const double P = acc / (double)N;
            const double f = (double)counts[j] / ((double)N * k);
            terms[j] = (double)hpg / (double)g * f * P;
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double L = 0.0;
        for (int j = 0; j < h; ++j) L += terms[j];
        *loss = (float)L;
    }
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

size_t aux_loss_scratch_bytes(const gqe_shape* s) {
    const int64_t N = (int64_t)s->B * s->T;
    return align256((size_t)s->h * sizeof(int32_t)) + align256((size_t)((N + 31) / 32) * s->h * sizeof(float));
}

cudaError_t launch_aux_loss(const AuxLossArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t N = (int64_t)s.B * s.T;
    int32_t* counts = static_cast<int32_t*>(a.scratch);
    float* partial = reinterpret_cast<float*>(static_cast<char*>(a.scratch) + align256((size_t)s.h * sizeof(int32_t)));
    cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)s.h * sizeof(int32_t), a.stream);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t items = N * s.g;
    const int cblocks = (int)std::min<int64_t>((items + 255) / 256, (int64_t)sms * 4);
    aux_counts_kernel<<<cblocks, 256, s.h * sizeof(int32_t), a.stream>>>(a.idx, N, s.h, s.g, s.k, counts,
                                                                        (uint32_t*)a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t warps = (N + 31) / 32 * s.g;
    const unsigned pblocks = (unsigned)((warps + 7) / 8);
    aux_probs_kernel<<<pblocks, 256, 0, a.stream>>>(a.logits, counts, N, s.h, s.g, s.k, a.dlogits, partial);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    aux_loss_kernel<<<1, 1024, s.h * sizeof(double), a.stream>>>(partial, counts, N, s.h, s.g, s.k, a.loss);
    return cudaGetLastError();
}

}  // namespace gqe
