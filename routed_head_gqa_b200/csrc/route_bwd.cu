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
// on CUDA cores in fp32 rather than on the tensor cores.  dx and dW_r are
// register-blocked (32 outputs per thread from shared-memory tiles), so each
// shared-memory read feeds 8 or 4 FMAs.  dW_r is summed over token ranges
// into scratch, then the ranges are added in a fixed order, so the result
// does not depend on scheduling.
#include "backward.cuh"

namespace gqe {
namespace {

constexpr int kHc = 32;      // heads per pass
// dx tiles: 64 tokens x 128 columns per block, 8 tokens x 4 columns per thread
constexpr int kXTok = 64, kXCol = 128, kXThreads = 256;
// dW tiles: 128 columns x 32 heads per block, 4 columns x 8 heads per thread,
// tokens staged 32 at a time
constexpr int kWCol = 128, kWThreads = 128, kWStage = 32;

template <typename T>
__device__ __forceinline__ float ld(const T* p);
template <>
__device__ __forceinline__ float ld<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ void fma4(float a, const float4& b, float4& c) {
    c.x = fmaf(a, b.x, c.x);
    c.y = fmaf(a, b.y, c.y);
    c.z = fmaf(a, b.z, c.z);
    c.w = fmaf(a, b.w, c.w);
}

// dx[t, i] for a 64-token x 128-column tile; the heads are summed 32 at a time
// from shared-memory copies of dl (transposed to [head][token]) and W_r
// (transposed to [head][column]).
template <typename T>
__global__ void __launch_bounds__(kXThreads)
route_bwd_dx_kernel(int64_t BT, int d_model, int h, const T* __restrict__ W, const float* __restrict__ dl,
                    float* __restrict__ dx) {
    // rows padded by 4 floats: the transposing stores hit 8 banks instead of 1,
    // and every row still starts on a 16-byte boundary
    __shared__ __align__(16) float dlT[kHc][kXTok + 4];
    __shared__ __align__(16) float WT[kHc][kXCol + 4];
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
    const int i0 = blockIdx.x * kXCol, c0 = tx * 4;
    const int64_t t0 = (int64_t)blockIdx.y * kXTok;
    float4 acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int j0 = 0; j0 < h; j0 += kHc) {
        __syncthreads();
        for (int c = threadIdx.x; c < kXTok * kHc; c += kXThreads) {
            const int t = c / kHc, jj = c % kHc;
            dlT[jj][t] = (t0 + t < BT && j0 + jj < h) ? dl[(t0 + t) * h + j0 + jj] : 0.f;
        }
        for (int c = threadIdx.x; c < kXCol * kHc; c += kXThreads) {
            const int col = c / kHc, jj = c % kHc;
            WT[jj][col] = (i0 + col < d_model && j0 + jj < h) ? ld<T>(W + (int64_t)(i0 + col) * h + j0 + jj) : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int jj = 0; jj < kHc; ++jj) {
            const float4 w = *reinterpret_cast<const float4*>(&WT[jj][c0]);
            const float4 a = *reinterpret_cast<const float4*>(&dlT[jj][ty * 8]);
            const float4 b = *reinterpret_cast<const float4*>(&dlT[jj][ty * 8 + 4]);
            fma4(a.x, w, acc[0]);
            fma4(a.y, w, acc[1]);
            fma4(a.z, w, acc[2]);
            fma4(a.w, w, acc[3]);
            fma4(b.x, w, acc[4]);
            fma4(b.y, w, acc[5]);
            fma4(b.z, w, acc[6]);
            fma4(b.w, w, acc[7]);
        }
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int64_t t = t0 + ty * 8 + r;
        if (t >= BT) break;
        float* out = dx + t * d_model + i0 + c0;
        if (i0 + c0 + 3 < d_model && (d_model & 3) == 0) {
            *reinterpret_cast<float4*>(out) = acc[r];
        } else {
            const float v[4] = {acc[r].x, acc[r].y, acc[r].z, acc[r].w};
            for (int e = 0; e < 4 && i0 + c0 + e < d_model; ++e) out[e] = v[e];
        }
    }
}

// partial[split, i, j] = sum over the split's tokens of x[t, i] * dl[t, j], for
// a 128-column x 32-head tile (blockIdx.z picks the 32 heads).
template <typename T>
__global__ void __launch_bounds__(kWThreads)
route_bwd_dw_kernel(int64_t BT, int d_model, int h, int64_t per_split, const T* __restrict__ x,
                    const float* __restrict__ dl, float* __restrict__ partial) {
    __shared__ __align__(16) float xs[kWStage][kWCol];
    __shared__ __align__(16) float dls[kWStage][kHc];
    const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;  // columns tx*4.., heads ty*8..
    const int i0 = blockIdx.x * kWCol, j0 = blockIdx.z * kHc;
    const int64_t b0 = (int64_t)blockIdx.y * per_split;
    const int64_t b1 = min(BT, b0 + per_split);
    float4 acc[8];  // acc[jj] holds heads j0 + ty*8 + jj for columns tx*4 .. tx*4+3
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) acc[jj] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int64_t s0 = b0; s0 < b1; s0 += kWStage) {
        __syncthreads();
        for (int c = threadIdx.x; c < kWStage * kWCol; c += kWThreads) {
            const int t = c / kWCol, col = c % kWCol;
            xs[t][col] = (s0 + t < b1 && i0 + col < d_model) ? ld<T>(x + (s0 + t) * d_model + i0 + col) : 0.f;
        }
        for (int c = threadIdx.x; c < kWStage * kHc; c += kWThreads) {
            const int t = c / kHc, jj = c % kHc;
            dls[t][jj] = (s0 + t < b1 && j0 + jj < h) ? dl[(s0 + t) * h + j0 + jj] : 0.f;
        }
        __syncthreads();
#pragma unroll 4
        for (int t = 0; t < kWStage; ++t) {
            const float4 xv = *reinterpret_cast<const float4*>(&xs[t][tx * 4]);
            const float4 a = *reinterpret_cast<const float4*>(&dls[t][ty * 8]);
            const float4 b = *reinterpret_cast<const float4*>(&dls[t][ty * 8 + 4]);
            fma4(a.x, xv, acc[0]);
            fma4(a.y, xv, acc[1]);
            fma4(a.z, xv, acc[2]);
            fma4(a.w, xv, acc[3]);
            fma4(b.x, xv, acc[4]);
            fma4(b.y, xv, acc[5]);
            fma4(b.z, xv, acc[6]);
            fma4(b.w, xv, acc[7]);
        }
    }
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
        const int j = j0 + ty * 8 + jj;
        if (j >= h) break;
        const float v[4] = {acc[jj].x, acc[jj].y, acc[jj].z, acc[jj].w};
        for (int e = 0; e < 4; ++e) {
            const int i = i0 + tx * 4 + e;
            if (i < d_model) partial[((int64_t)blockIdx.y * d_model + i) * h + j] = v[e];
        }
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
    // about eight 4-warp blocks per SM, so that the staging loads of some blocks
    // overlap the FMAs of others
    const int tiles = ((s->d_model + kWCol - 1) / kWCol) * ((s->h + kHc - 1) / kHc);
    int n = (8 * 148 + tiles - 1) / tiles;
    n = n < 1 ? 1 : (n > 64 ? 64 : n);
    if (n > BT) n = (int)BT;
    return n;
}

template <typename T>
cudaError_t launch_typed(const RouteBwdArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const dim3 gx((unsigned)((s.d_model + kXCol - 1) / kXCol), (unsigned)((BT + kXTok - 1) / kXTok));
    route_bwd_dx_kernel<T><<<gx, kXThreads, 0, a.stream>>>(BT, s.d_model, s.h, (const T*)a.W_r, a.dlogits, a.dx);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nsplit = route_splits(a.s);
    const int64_t per = (BT + nsplit - 1) / nsplit;
    float* partial = static_cast<float*>(a.scratch);
    const dim3 gw((unsigned)((s.d_model + kWCol - 1) / kWCol), (unsigned)nsplit, (unsigned)((s.h + kHc - 1) / kHc));
    route_bwd_dw_kernel<T><<<gw, kWThreads, 0, a.stream>>>(BT, s.d_model, s.h, per, (const T*)a.x, a.dlogits,
                                                           partial);
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
