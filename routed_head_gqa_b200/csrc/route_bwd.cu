// route_bwd.cu -- backward of the linear router, from the logit gradients.
//
// The router is the linear map l = x . W_r + bias ("Grouped Query Experts:
// Mixture-of-Experts on GQA Self-Attention", gist.science summary,
// "Architecture et Routage", with the reading of a linear router), so with
// dl = dL/dl [B*T, h]:
//   dx = dl . W_r^T     [B*T, d_model]
//   dW_r = x^T . dl     [d_model, h]
//   dbias = sum_t dl    [h]
// Each is a contraction with an inner dimension of h (small) or B*T, and all
// three are bound by HBM (dx written, x read once per 32 heads), so they run
// on CUDA cores in fp32 with coalesced rows rather than on the tensor cores.
// dW_r is summed over token ranges into scratch, then the ranges are added in
// a fixed order, so the result does not depend on scheduling.
#include "backward.cuh"

namespace gqe {
namespace {

constexpr int kCols = 256;   // d_model columns per block (one per thread)
constexpr int kTok = 16;     // tokens per dx block
constexpr int kHc = 32;      // heads per pass
constexpr int kStage = 64;   // tokens of dl staged per dW pass

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// dx[bt, i] for kTok tokens and kCols columns i.
template <typename T>
__global__ void __launch_bounds__(kCols)
route_bwd_dx_kernel(int64_t BT, int d_model, int h, const T* __restrict__ W, const float* __restrict__ dl,
                    float* __restrict__ dx) {
    __shared__ float dls[kTok][kHc];
    const int i = blockIdx.x * kCols + threadIdx.x;
    const int64_t t0 = (int64_t)blockIdx.y * kTok;
    float acc[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
    for (int j0 = 0; j0 < h; j0 += kHc) {
        __syncthreads();
        for (int c = threadIdx.x; c < kTok * kHc; c += kCols) {
            const int t = c / kHc, jj = c % kHc;
            dls[t][jj] = (t0 + t < BT && j0 + jj < h) ? dl[(t0 + t) * h + j0 + jj] : 0.f;
        }
        __syncthreads();
        if (i < d_model) {
            float w[kHc];
#pragma unroll
            for (int jj = 0; jj < kHc; ++jj) w[jj] = j0 + jj < h ? ld<T>(W + (int64_t)i * h + j0 + jj) : 0.f;
#pragma unroll
            for (int t = 0; t < kTok; ++t)
#pragma unroll
                for (int jj = 0; jj < kHc; ++jj) acc[t] = fmaf(dls[t][jj], w[jj], acc[t]);
        }
    }
    if (i >= d_model) return;
#pragma unroll
    for (int t = 0; t < kTok; ++t)
        if (t0 + t < BT) dx[(t0 + t) * d_model + i] = acc[t];
}

// partial[split, i, j] = sum over the split's tokens of x[bt, i] * dl[bt, j].
template <typename T>
__global__ void __launch_bounds__(kCols)
route_bwd_dw_kernel(int64_t BT, int d_model, int h, int64_t per_split, const T* __restrict__ x,
                    const float* __restrict__ dl, float* __restrict__ partial) {
    __shared__ float dls[kStage][kHc];
    const int i = blockIdx.x * kCols + threadIdx.x;
    const int64_t b0 = (int64_t)blockIdx.y * per_split;
    const int64_t b1 = min(BT, b0 + per_split);
    for (int j0 = 0; j0 < h; j0 += kHc) {
        float acc[kHc];
#pragma unroll
        for (int jj = 0; jj < kHc; ++jj) acc[jj] = 0.f;
        for (int64_t s0 = b0; s0 < b1; s0 += kStage) {
            __syncthreads();
            for (int c = threadIdx.x; c < kStage * kHc; c += kCols) {
                const int t = c / kHc, jj = c % kHc;
                dls[t][jj] = (s0 + t < b1 && j0 + jj < h) ? dl[(s0 + t) * h + j0 + jj] : 0.f;
            }
            __syncthreads();
            if (i < d_model) {
                const int n = (int)min((int64_t)kStage, b1 - s0);
                for (int t = 0; t < n; ++t) {
                    const float xv = ld<T>(x + (s0 + t) * d_model + i);
#pragma unroll
                    for (int jj = 0; jj < kHc; ++jj) acc[jj] = fmaf(xv, dls[t][jj], acc[jj]);
                }
            }
        }
        if (i < d_model)
            for (int jj = 0; jj < kHc && j0 + jj < h; ++jj)
                partial[((int64_t)blockIdx.y * d_model + i) * h + j0 + jj] = acc[jj];
    }
}

// dW[i, j] = sum over splits, in split order.
__global__ void route_bwd_dw_reduce_kernel(int64_t n, int nsplit, const float* __restrict__ partial,
                                           float* __restrict__ dW) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (int64_t)gridDim.x * blockDim.x) {
        float acc = 0.f;
        for (int sp = 0; sp < nsplit; ++sp) acc += partial[sp * n + e];
        dW[e] = acc;
    }
}

// dbias[j]: one block per head, a fixed-order tree sum over the tokens.
__global__ void __launch_bounds__(256)
route_bwd_dbias_kernel(int64_t BT, int h, const float* __restrict__ dl, float* __restrict__ dbias) {
    __shared__ float red[256];
    const int j = blockIdx.x;
    float acc = 0.f;
    for (int64_t t = threadIdx.x; t < BT; t += 256) acc += dl[t * h + j];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) dbias[j] = red[0];
}

int route_splits(const gqe_shape* s) {
    const int64_t BT = (int64_t)s->B * s->T;
    const int col_blocks = (s->d_model + kCols - 1) / kCols;
    int n = (2 * 148 + col_blocks - 1) / col_blocks;
    n = n < 1 ? 1 : (n > 64 ? 64 : n);
    if (n > BT) n = (int)BT;
    return n;
}

template <typename T>
cudaError_t launch_typed(const RouteBwdArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const unsigned col_blocks = (unsigned)((s.d_model + kCols - 1) / kCols);
    const dim3 gx(col_blocks, (unsigned)((BT + kTok - 1) / kTok));
    route_bwd_dx_kernel<T><<<gx, kCols, 0, a.stream>>>(BT, s.d_model, s.h, (const T*)a.W_r, a.dlogits, a.dx);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nsplit = route_splits(a.s);
    const int64_t per = (BT + nsplit - 1) / nsplit;
    float* partial = static_cast<float*>(a.scratch);
    route_bwd_dw_kernel<T><<<dim3(col_blocks, (unsigned)nsplit), kCols, 0, a.stream>>>(
        BT, s.d_model, s.h, per, (const T*)a.x, a.dlogits, partial);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t n = (int64_t)s.d_model * s.h;
    route_bwd_dw_reduce_kernel<<<(unsigned)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184), 256, 0, a.stream>>>(
        n, nsplit, partial, a.dW);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.dbias == nullptr) return e;
    route_bwd_dbias_kernel<<<(unsigned)s.h, 256, 0, a.stream>>>(BT, s.h, a.dlogits, a.dbias);
    return cudaGetLastError();
}

}  // namespace

size_t route_backward_scratch_bytes(const gqe_shape* s) {
    return ((size_t)route_splits(s) * s->d_model * s->h * sizeof(float) + 255) & ~size_t(255);
}

cudaError_t launch_route_backward(const RouteBwdArgs& a) {
    return a.s->dtype == GQE_BF16 ? launch_typed<__nv_bfloat16>(a) : launch_typed<float>(a);
}

}  // namespace gqe
