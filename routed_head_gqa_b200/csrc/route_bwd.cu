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

// dx[t, i] for 128-column blocks: a block keeps its columns of W_r (transposed
// to [head][column]) in shared memory and walks a range of 64-token tiles,
// loading the next tile's dl (16-byte loads, transposed to [head][token]) into
// registers while the current tile's FMAs and stores run.
constexpr int kXTilesPerBlock = 8;
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
    const int64_t n_tiles = (BT + kXTok - 1) / kXTok;
    const int64_t tile_lo = (int64_t)blockIdx.y * kXTilesPerBlock;
    const int64_t tile_hi = min(n_tiles, tile_lo + kXTilesPerBlock);
    constexpr int kDV = kXTok * kHc / 4 / kXThreads;  // float4 of dl per thread per tile
    const bool vec_dl = (h % 4) == 0;
    for (int j0 = 0; j0 < h; j0 += kHc) {
        __syncthreads();
        for (int c = threadIdx.x; c < kXCol * kHc; c += kXThreads) {
            const int col = c / kHc, jj = c % kHc;
            WT[jj][col] = (i0 + col < d_model && j0 + jj < h) ? ld<T>(W + (int64_t)(i0 + col) * h + j0 + jj) : 0.f;
        }
        float4 dr[kDV];
        auto fetch = [&](int64_t tile) {
            const int64_t t0 = tile * kXTok;
#pragma unroll
            for (int v = 0; v < kDV; ++v) {
                const int c = threadIdx.x + v * kXThreads;  // (token, 4 heads)
                const int t = c / (kHc / 4), jq = (c % (kHc / 4)) * 4;
                const int64_t row = t0 + t;
                if (row < BT && vec_dl && j0 + jq + 3 < h) {
                    dr[v] = *reinterpret_cast<const float4*>(dl + row * h + j0 + jq);
                } else {
                    float e[4];
                    for (int q = 0; q < 4; ++q) e[q] = (row < BT && j0 + jq + q < h) ? dl[row * h + j0 + jq + q] : 0.f;
                    dr[v] = make_float4(e[0], e[1], e[2], e[3]);
                }
            }
        };
        if (tile_lo < tile_hi) fetch(tile_lo);
        for (int64_t tile = tile_lo; tile < tile_hi; ++tile) {
            __syncthreads();
#pragma unroll
            for (int v = 0; v < kDV; ++v) {
                const int c = threadIdx.x + v * kXThreads, t = c / (kHc / 4), jq = (c % (kHc / 4)) * 4;
                dlT[jq][t] = dr[v].x;
                dlT[jq + 1][t] = dr[v].y;
                dlT[jq + 2][t] = dr[v].z;
                dlT[jq + 3][t] = dr[v].w;
            }
            __syncthreads();
            if (tile + 1 < tile_hi) fetch(tile + 1);
            float4 acc[8];
#pragma unroll
            for (int r = 0; r < 8; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
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
            const int64_t t0 = tile * kXTok;
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                const int64_t t = t0 + ty * 8 + r;
                if (t >= BT) break;
                float* out = dx + t * d_model + i0 + c0;
                if (i0 + c0 + 3 < d_model && (d_model & 3) == 0) {
                    if (j0 > 0) {  // heads past the first 32: add to the earlier passes' sums
                        const float4 o = *reinterpret_cast<const float4*>(out);
                        acc[r].x += o.x;
                        acc[r].y += o.y;
                        acc[r].z += o.z;
                        acc[r].w += o.w;
                    }
                    *reinterpret_cast<float4*>(out) = acc[r];
                } else {
                    const float v[4] = {acc[r].x, acc[r].y, acc[r].z, acc[r].w};
                    for (int e = 0; e < 4 && i0 + c0 + e < d_model; ++e) out[e] = (j0 > 0 ? out[e] : 0.f) + v[e];
                }
            }
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
    // The next stage's x and dl are loaded into registers while the current
    // stage's FMAs run (16-byte loads of 8 bf16 or 4 fp32 where the row allows).
    constexpr int kEV = 16 / sizeof(T);                             // elements per 16-byte vector
    constexpr int kXV = kWStage * kWCol / kEV / kWThreads;          // x vectors per thread per stage
    constexpr int kDV = kWStage * kHc / kWThreads;                  // dl values per thread per stage
    const bool vec_ok = (d_model % kEV) == 0 && i0 + kWCol <= d_model;
    float xr[kXV][kEV], dr[kDV];
    auto fetch = [&](int64_t s0) {
#pragma unroll
        for (int v = 0; v < kXV; ++v) {
            const int c = (threadIdx.x + v * kWThreads) * kEV;  // element index in the [kWStage][kWCol] stage
            const int t = c / kWCol, col = c % kWCol;
            const int64_t row = s0 + t;
            if (row < b1 && vec_ok) {
                const uint4 q = *reinterpret_cast<const uint4*>(x + row * d_model + i0 + col);
                if constexpr (sizeof(T) == 2) {
                    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        xr[v][2 * e] = __uint_as_float(w[e] << 16);
                        xr[v][2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
                    }
                } else {
                    xr[v][0] = __uint_as_float(q.x);
                    xr[v][1] = __uint_as_float(q.y);
                    xr[v][2] = __uint_as_float(q.z);
                    xr[v][3] = __uint_as_float(q.w);
                }
            } else {
#pragma unroll
                for (int e = 0; e < kEV; ++e)
                    xr[v][e] = (row < b1 && i0 + col + e < d_model) ? ld<T>(x + row * d_model + i0 + col + e) : 0.f;
            }
        }
#pragma unroll
        for (int v = 0; v < kDV; ++v) {
            const int c = threadIdx.x + v * kWThreads, t = c / kHc, jj = c % kHc;
            dr[v] = (s0 + t < b1 && j0 + jj < h) ? dl[(s0 + t) * h + j0 + jj] : 0.f;
        }
    };
    fetch(b0);
    for (int64_t s0 = b0; s0 < b1; s0 += kWStage) {
        __syncthreads();
#pragma unroll
        for (int v = 0; v < kXV; ++v) {
            const int c = (threadIdx.x + v * kWThreads) * kEV, t = c / kWCol, col = c % kWCol;
#pragma unroll
            for (int e = 0; e < kEV; ++e) xs[t][col + e] = xr[v][e];
        }
#pragma unroll
        for (int v = 0; v < kDV; ++v) {
            const int c = threadIdx.x + v * kWThreads;
            dls[c / kHc][c % kHc] = dr[v];
        }
        __syncthreads();
        if (s0 + kWStage < b1) fetch(s0 + kWStage);
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
    const int64_t x_tiles = (BT + kXTok - 1) / kXTok;
    const dim3 gx((unsigned)((s.d_model + kXCol - 1) / kXCol), (unsigned)((x_tiles + kXTilesPerBlock - 1) / kXTilesPerBlock));
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
