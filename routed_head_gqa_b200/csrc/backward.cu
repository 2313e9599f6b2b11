// backward.cu -- backward pass of the routed attention and of the gates.
//
// The pages give no backward for GQE; this is the chain rule through the
// forward ("Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
// gist.science summary, "Architecture et Routage" and "Somme Ponderee
// Renormalisee"; IBM "Que es la atencion de consultas agrupadas" for the
// scaled dot-product attention).  For a routed (b, t, j) with gate gm,
// attention output o (O = gm * o) and incoming gradient dO:
//   p_s    = exp(q . k_s / sqrt(d_h) - lse),   s <= t
//   D      = gm * dO . o                        (= dO . O)
//   dlogit = D_j - gm_j * sum_{i in S} D_i      (renormalised gates; 0 if j not in S)
//   ds_s   = p_s * (gm * dO . v_s - D)
//   dQ     = sum_s ds_s k_s / sqrt(d_h)
//   dK_s  += ds_s q / sqrt(d_h),   dV_s += p_s * gm * dO
// D is summed in fp32 from p_s and gm dO . v_s rather than read back from the
// forward's output, so it carries no rounding of O to the input dtype.
//
// Three launches, all on CUDA cores in fp32 (a first, correct path: the
// contractions are not yet on the tensor cores):
//  1. bwd_dq_kernel, one block per 32 consecutive entries of a (b, j) list:
//     a first sweep over the visible keys gives each row's log-sum-exp; a
//     second accumulates D, sum_s p_s dp_s k_s and sum_s p_s k_s, hence dQ.
//     The gate, D and the log-sum-exp of every routed row go to scratch.
//  2. bwd_rows_kernel, one warp per (b, t, group): the group's logit
//     gradients, and zero dQ rows for the unselected heads.
//  3. bwd_dkdv_kernel, one block per (b, group, 32-key tile): every routed row
//     of the group's heads at or after the tile's first key adds its share to
//     the tile's dK and dV, which stay in registers.
// Eight lanes share a row (or a key): lane `seg` owns dims 32*m + 4*seg + e,
// so a warp's 16-byte shared-memory reads of one row cover 128 contiguous bytes.
#include "backward.cuh"

namespace gqe {
namespace {

constexpr uint32_t kWhereBwd = 6;  // status "where" id of the backward kernels
constexpr int kRows = 32;          // rows (or keys) per block
constexpr int kSeg = 8;            // lanes per row
constexpr int kThreads = kRows * kSeg;

template <typename T>
__device__ __forceinline__ float4 load4(const T* p);
template <>
__device__ __forceinline__ float4 load4<float>(const float* p) {
    return *reinterpret_cast<const float4*>(p);
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xffff0000u));
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b, float acc) {
    acc = fmaf(a.x, b.x, acc);
    acc = fmaf(a.y, b.y, acc);
    acc = fmaf(a.z, b.z, acc);
    return fmaf(a.w, b.w, acc);
}

__device__ __forceinline__ void axpy4(float a, const float4& x, float4& y) {
    y.x = fmaf(a, x.x, y.x);
    y.y = fmaf(a, x.y, y.y);
    y.z = fmaf(a, x.z, y.z);
    y.w = fmaf(a, x.w, y.w);
}

// Sum of NM independent partial dot products (short dependency chains).
template <int NM>
__device__ __forceinline__ float dot_rows(const float4 (&a)[NM], const float4 (&b)[NM]) {
    float p[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) p[m] = dot4(a[m], b[m], 0.f);
#pragma unroll
    for (int w = 1; w < NM; w *= 2)
#pragma unroll
        for (int m = 0; m + w < NM; m += 2 * w) p[m] += p[m + w];
    return p[0];
}

// Sum over the 8 lanes of a row.
__device__ __forceinline__ float seg_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    return v;
}

// ---------------------------------------------------------------------------
// 1. dQ (with the log-sum-exp and D) per 32 entries of a (b, j) list.
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads)
bwd_dq_kernel(int T_, int h, int g, int k, float scale, float scale_log2, const T* __restrict__ Q,
              const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ dO,
              const int32_t* __restrict__ idx, const float* __restrict__ gate,
              const int32_t* __restrict__ head_offsets, const int32_t* __restrict__ head_pos,
              float* __restrict__ gamma_out, float* __restrict__ delta_out, float* __restrict__ lse_out,
              float* __restrict__ dQ, void* status) {
    constexpr int NM = D / 32;  // float4 groups per lane
    __shared__ __align__(16) float Ks[kRows][D];
    __shared__ __align__(16) float Vs[kRows][D];
    const int bj = blockIdx.y;
    const int b = bj / h, j = bj % h, q = j / (h / g);
    const int e_end = head_offsets[bj + 1];
    const int e0 = head_offsets[bj] + blockIdx.x * kRows;
    if (e0 >= e_end) return;
    const int r = threadIdx.x / kSeg, seg = threadIdx.x % kSeg;
    const int e = e0 + r;
    int t_r = e < e_end ? head_pos[e] : -1;
    if (t_r >= T_) {
        report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwd, (uint32_t)e);
        t_r = -1;
    }
    int t_max = head_pos[min(e0 + kRows, e_end) - 1];  // lists ascend
    t_max = t_max < 0 ? 0 : (t_max >= T_ ? T_ - 1 : t_max);
    const int64_t bt = (int64_t)b * T_ + (t_r < 0 ? 0 : t_r);
    const int64_t row = bt * h + j;
    // the row's gate: the selection slot of (b, t, q) that names head j
    float gm = 0.f;
    if (t_r >= 0)
        for (int s = 0; s < k; ++s)
            if (idx[(bt * g + q) * k + s] == j) gm = gate[(bt * g + q) * k + s];
    float4 qv[NM], dov[NM], acc[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        const int d0 = 32 * m + 4 * seg;
        qv[m] = load4<T>(Q + row * D + d0);
        const float4 o = load4<T>(dO + row * D + d0);
        dov[m] = make_float4(gm * o.x, gm * o.y, gm * o.z, gm * o.w);
        acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const int64_t kv_row0 = (int64_t)b * T_ * g + q;  // row index of (b, s=0, q) in [B,T,g]
    auto load_tile = [&](float (*dst)[D], const T* src, int kt) {
        for (int i = threadIdx.x; i < kRows * (D / 4); i += kThreads) {
            const int key = i / (D / 4), c = (i % (D / 4)) * 4;
            const int s = kt + key;
            const float4 v =
                s < T_ ? load4<T>(src + (kv_row0 + (int64_t)s * g) * D + c) : make_float4(0.f, 0.f, 0.f, 0.f);
            *reinterpret_cast<float4*>(&dst[key][c]) = v;
        }
    };
    // sweep 1: the row's log2-sum-exp over keys s <= t_r
    float mx = -INFINITY, l = 0.f;
    for (int kt = 0; kt <= t_max; kt += kRows) {
        __syncthreads();
        load_tile(Ks, K, kt);
        __syncthreads();
        float sv[kRows];
        float tmx = -INFINITY;
#pragma unroll
        for (int i = 0; i < kRows; ++i) {
            float4 kk[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) kk[m] = *reinterpret_cast<const float4*>(&Ks[i][32 * m + 4 * seg]);
            const float part = seg_sum(dot_rows<NM>(qv, kk));
            sv[i] = (kt + i <= t_r) ? part * scale_log2 : -INFINITY;
            tmx = fmaxf(tmx, sv[i]);
        }
        const float mnew = fmaxf(mx, tmx);
        if (mnew != -INFINITY) {
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < kRows; ++i) sum += exp2f(sv[i] - mnew);
            l = l * exp2f(mx - mnew) + sum;
            mx = mnew;
        }
    }
    const float lse2 = l > 0.f ? mx + log2f(l) : 0.f;
    // sweep 2: with dp_s = gm dO . v_s, D = sum_s p_s dp_s and
    // dQ = scale * sum_s p_s (dp_s - D) k_s = scale * (sum_s p_s dp_s k_s - D sum_s p_s k_s),
    // so D is found in the same sweep and o is never formed.
    float4 ck[NM];  // sum_s p_s k_s; acc holds sum_s p_s dp_s k_s
#pragma unroll
    for (int m = 0; m < NM; ++m) ck[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    float Dr = 0.f;
    for (int kt = 0; kt <= t_max; kt += kRows) {
        __syncthreads();
        load_tile(Ks, K, kt);
        load_tile(Vs, V, kt);
        __syncthreads();
#pragma unroll 4
        for (int i = 0; i < kRows; ++i) {
            float4 kk[NM], vk[NM];
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                kk[m] = *reinterpret_cast<const float4*>(&Ks[i][32 * m + 4 * seg]);
                vk[m] = *reinterpret_cast<const float4*>(&Vs[i][32 * m + 4 * seg]);
            }
            const float pqk = seg_sum(dot_rows<NM>(qv, kk));
            const float pdv = seg_sum(dot_rows<NM>(dov, vk));
            const float p = (kt + i <= t_r) ? exp2f(pqk * scale_log2 - lse2) : 0.f;
            const float pd = p * pdv;
            Dr += pd;
#pragma unroll
            for (int m = 0; m < NM; ++m) {
                axpy4(pd, kk[m], acc[m]);
                axpy4(p, kk[m], ck[m]);
            }
        }
    }
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        acc[m].x = fmaf(-Dr, ck[m].x, acc[m].x);
        acc[m].y = fmaf(-Dr, ck[m].y, acc[m].y);
        acc[m].z = fmaf(-Dr, ck[m].z, acc[m].z);
        acc[m].w = fmaf(-Dr, ck[m].w, acc[m].w);
    }
    if (t_r < 0) return;
#pragma unroll
    for (int m = 0; m < NM; ++m)
        *reinterpret_cast<float4*>(dQ + row * D + 32 * m + 4 * seg) =
            make_float4(acc[m].x * scale, acc[m].y * scale, acc[m].z * scale, acc[m].w * scale);
    if (seg == 0) {
        lse_out[row] = lse2;
        delta_out[row] = Dr;
        gamma_out[row] = gm;
    }
}

// ---------------------------------------------------------------------------
// 2. Per (b, t, group): logit gradients, dQ zero rows.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256)
bwd_rows_kernel(int64_t BT, int h, int g, int k, const int32_t* __restrict__ idx, const float* __restrict__ gate,
                const float* __restrict__ delta, float* __restrict__ dlogits, float* __restrict__ dQ, void* status) {
    const int lane = threadIdx.x & 31;
    const int64_t item = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // bt * g + q
    if (item >= BT * g) return;
    const int64_t bt = item / g;
    const int q = (int)(item % g), hpg = h / g;
    float dsel[16], gsel[16];
    int jsel[16];
    float dsum = 0.f;
#pragma unroll
    for (int s = 0; s < 16; ++s) {
        dsel[s] = 0.f;
        gsel[s] = 0.f;
        jsel[s] = -1;
        if (s < k) {
            const int j = idx[item * k + s];
            if (j < q * hpg || j >= (q + 1) * hpg) {
                if (lane == 0) report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwd, (uint32_t)item);
                continue;
            }
            jsel[s] = j;
            gsel[s] = gate[item * k + s];
            dsel[s] = delta[bt * h + j];
            dsum += dsel[s];
        }
    }
    for (int jj = lane; jj < hpg; jj += 32) {
        const int j = q * hpg + jj;
        float dl = 0.f;
#pragma unroll
        for (int s = 0; s < 16; ++s)
            if (s < k && jsel[s] == j) dl = dsel[s] - gsel[s] * dsum;
        dlogits[bt * h + j] = dl;
    }
    // dQ of an unselected head is 0
    for (int jj = 0; jj < hpg; ++jj) {
        const int j = q * hpg + jj;
        bool sel = false;
#pragma unroll
        for (int s = 0; s < 16; ++s) sel |= (s < k && jsel[s] == j);
        if (sel) continue;
        for (int d0 = lane * 4; d0 < D; d0 += 128)
            *reinterpret_cast<float4*>(dQ + (bt * h + j) * D + d0) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ---------------------------------------------------------------------------
// 3. dK, dV per (b, group, 32-key tile).
// ---------------------------------------------------------------------------
template <typename T, int D>
__global__ void __launch_bounds__(kThreads, 2)
bwd_dkdv_kernel(int T_, int h, int g, int nchunk, float scale, float scale_log2, const T* __restrict__ Q,
                const T* __restrict__ K, const T* __restrict__ V, const T* __restrict__ dO,
                const int32_t* __restrict__ head_offsets, const int32_t* __restrict__ head_pos,
                const int32_t* __restrict__ head_chunk_offsets, const float* __restrict__ gamma,
                const float* __restrict__ delta, const float* __restrict__ lse, float* __restrict__ dK,
                float* __restrict__ dV, void* status) {
    constexpr int NM = D / 32;
    __shared__ __align__(16) float Qs[kRows][D];
    __shared__ __align__(16) float dOs[kRows][D];
    __shared__ int row_t[kRows];
    __shared__ float row_g[kRows], row_lse[kRows], row_d[kRows];
    const int s0 = blockIdx.x * kRows, q = blockIdx.y, b = blockIdx.z;
    const int hpg = h / g;
    const int i = threadIdx.x / kSeg, seg = threadIdx.x % kSeg;
    const int s = s0 + i;
    const bool key_ok = s < T_;
    const int64_t kv_row = ((int64_t)b * T_ + (key_ok ? s : 0)) * g + q;
    float4 kv[NM], vv[NM], dk[NM], dv[NM];
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        const int d0 = 32 * m + 4 * seg;
        kv[m] = key_ok ? load4<T>(K + kv_row * D + d0) : make_float4(0.f, 0.f, 0.f, 0.f);
        vv[m] = key_ok ? load4<T>(V + kv_row * D + d0) : make_float4(0.f, 0.f, 0.f, 0.f);
        dk[m] = make_float4(0.f, 0.f, 0.f, 0.f);
        dv[m] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int jj = 0; jj < hpg; ++jj) {
        const int j = q * hpg + jj;
        const int64_t bj = (int64_t)b * h + j;
        const int e_beg = head_chunk_offsets[bj * nchunk + blockIdx.x];
        const int e_end = head_offsets[bj + 1];
        for (int e0 = e_beg; e0 < e_end; e0 += kRows) {
            const int n = min(kRows, e_end - e0);
            __syncthreads();  // the previous batch is consumed
            if (threadIdx.x < kRows) {
                const int r = threadIdx.x;
                int t = r < n ? head_pos[e0 + r] : -1;
                if (t >= T_) {
                    report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwd, (uint32_t)(e0 + r));
                    t = -1;
                }
                const int64_t row = ((int64_t)b * T_ + (t < 0 ? 0 : t)) * h + j;
                row_t[r] = t;
                row_g[r] = t >= 0 ? gamma[row] : 0.f;
                row_lse[r] = t >= 0 ? lse[row] : 0.f;
                row_d[r] = t >= 0 ? delta[row] : 0.f;
            }
            __syncthreads();
            for (int c = threadIdx.x; c < kRows * (D / 4); c += kThreads) {
                const int r = c / (D / 4), d0 = (c % (D / 4)) * 4;
                const int t = row_t[r];
                float4 qq = make_float4(0.f, 0.f, 0.f, 0.f), oo = qq;
                if (t >= 0) {
                    const int64_t row = ((int64_t)b * T_ + t) * h + j;
                    const float gm = row_g[r];
                    qq = load4<T>(Q + row * D + d0);
                    const float4 o = load4<T>(dO + row * D + d0);
                    oo = make_float4(gm * o.x, gm * o.y, gm * o.z, gm * o.w);
                }
                *reinterpret_cast<float4*>(&Qs[r][d0]) = qq;
                *reinterpret_cast<float4*>(&dOs[r][d0]) = oo;
            }
            __syncthreads();
#pragma unroll 4
            for (int r = 0; r < n; ++r) {
                float4 qr[NM], dr[NM];
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    qr[m] = *reinterpret_cast<const float4*>(&Qs[r][32 * m + 4 * seg]);
                    dr[m] = *reinterpret_cast<const float4*>(&dOs[r][32 * m + 4 * seg]);
                }
                const float pqk = seg_sum(dot_rows<NM>(qr, kv));
                const float pdv = seg_sum(dot_rows<NM>(dr, vv));
                const int t = row_t[r];
                const float p = (key_ok && s <= t) ? exp2f(pqk * scale_log2 - row_lse[r]) : 0.f;
                const float ds = p * (pdv - row_d[r]);
#pragma unroll
                for (int m = 0; m < NM; ++m) {
                    axpy4(p, dr[m], dv[m]);
                    axpy4(ds, qr[m], dk[m]);
                }
            }
        }
    }
    if (!key_ok) return;
#pragma unroll
    for (int m = 0; m < NM; ++m) {
        const int d0 = 32 * m + 4 * seg;
        *reinterpret_cast<float4*>(dK + kv_row * D + d0) =
            make_float4(dk[m].x * scale, dk[m].y * scale, dk[m].z * scale, dk[m].w * scale);
        *reinterpret_cast<float4*>(dV + kv_row * D + d0) = dv[m];
    }
}

size_t a256(size_t n) { return (n + 255) & ~size_t(255); }

template <typename T, int D>
cudaError_t launch_typed(const AttnBwdArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const size_t plane = a256((size_t)BT * s.h * sizeof(float));
    float* gamma = static_cast<float*>(a.scratch);
    float* delta = reinterpret_cast<float*>(static_cast<char*>(a.scratch) + plane);
    float* lse = reinterpret_cast<float*>(static_cast<char*>(a.scratch) + 2 * plane);
    const float scale = (float)(1.0 / sqrt((double)D));
    const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
    const int nchunk = (s.T + kChunk - 1) / kChunk;
    const dim3 gq((unsigned)((s.T + kRows - 1) / kRows), (unsigned)(s.B * s.h));
    bwd_dq_kernel<T, D><<<gq, kThreads, 0, a.stream>>>(s.T, s.h, s.g, s.k, scale, scale_log2, (const T*)a.Q,
                                                       (const T*)a.K, (const T*)a.V, (const T*)a.dO, a.idx, a.gate,
                                                       a.head_offsets, a.head_pos, gamma, delta, lse, a.dQ, a.status);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int64_t warps = BT * s.g;
    bwd_rows_kernel<D><<<(unsigned)((warps * 32 + 255) / 256), 256, 0, a.stream>>>(
        BT, s.h, s.g, s.k, a.idx, a.gate, delta, a.dlogits, a.dQ, a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const dim3 gk((unsigned)((s.T + kRows - 1) / kRows), (unsigned)s.g, (unsigned)s.B);
    bwd_dkdv_kernel<T, D><<<gk, kThreads, 0, a.stream>>>(
        s.T, s.h, s.g, nchunk, scale, scale_log2, (const T*)a.Q, (const T*)a.K, (const T*)a.V, (const T*)a.dO,
        a.head_offsets, a.head_pos, a.head_chunk_offsets, gamma, delta, lse, a.dK, a.dV, a.status);
    return cudaGetLastError();
}

}  // namespace

size_t attn_backward_scratch_bytes(const gqe_shape* s) {
    if (attn_backward_tc_supported(s)) return attn_backward_tc_scratch_bytes(s);
    return 3 * a256((size_t)s->B * s->T * s->h * sizeof(float));
}

cudaError_t launch_attn_backward(const AttnBwdArgs& a) {
    if (attn_backward_tc_supported(a.s)) return launch_attn_backward_tc(a);
    const bool bf16 = a.s->dtype == GQE_BF16;
    switch (a.s->d_h) {
        case 32: return bf16 ? launch_typed<__nv_bfloat16, 32>(a) : launch_typed<float, 32>(a);
        case 64: return bf16 ? launch_typed<__nv_bfloat16, 64>(a) : launch_typed<float, 64>(a);
        case 128: return bf16 ? launch_typed<__nv_bfloat16, 128>(a) : launch_typed<float, 128>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gqe
