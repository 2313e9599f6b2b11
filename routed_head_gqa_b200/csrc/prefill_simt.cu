// prefill_simt.cu -- routed causal attention with the gated scatter, fp32, on
// CUDA cores (one warp per routed row).  This is the fp32 path: fp32 inputs
// need fp32 products, which the bf16 tensor-core path does not give.
//
// Per routed (b, t, j): o = sum_{s<=t} softmax_s(q . k_s / sqrt(d_h)) v_s with K/V
// of group j / hpg (IBM GQA page, scaled dot-product attention; ml-canon
// "56 GQA / MQA", shared KV heads), O[b,t,j] = gate * o, zero for unselected heads
// (gist.science GQE summary, "Construction de la Sortie").
#include "units.cuh"

namespace gqe {
namespace {

constexpr int kSimtW = 32;        // window width (positions per unit)
constexpr int kSimtThreads = 128;
constexpr int kMaxRowsSimt = 16 * kSimtW;  // k <= 16

template <int DPL>  // head dims per lane: d_h / 32
__global__ void __launch_bounds__(kSimtThreads)
prefill_simt_kernel(UnitGeom u, const float* __restrict__ Q, const float* __restrict__ K,
                    const float* __restrict__ V, const int32_t* __restrict__ idx,
                    const float* __restrict__ gate, const int32_t* __restrict__ head_offsets,
                    const int32_t* __restrict__ head_pos, const int32_t* __restrict__ head_chunk_offsets,
                    float* __restrict__ O, void* status, int kv_g, int kv_q0) {
    constexpr int d_h = DPL * 32;
    __shared__ int32_t s_start[64], s_prefix[65];
    __shared__ int32_t rows_t[kMaxRowsSimt];
    __shared__ int16_t rows_j[kMaxRowsSimt];
    __shared__ float rows_gate[kMaxRowsSimt];

    int b, q, w;
    unit_coords(u, blockIdx.x, b, q, w);
    const int w0 = w * kSimtW;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;

    // Row table: each head's slice of its position list inside the window.
    if (threadIdx.x == 0) {
        int acc = 0;
        const int32_t total = (int32_t)((int64_t)u.B * u.T * u.g * u.k);
        for (int jj = 0; jj < u.hpg; ++jj) {
            const int j = q * u.hpg + jj;
            int32_t a0 = list_cut(u, head_offsets, head_chunk_offsets, b, j, w0);
            int32_t a1 = list_cut(u, head_offsets, head_chunk_offsets, b, j, w0 + kSimtW);
            if (a0 < 0 || a1 < a0 || a1 > total) {  // malformed lists: report, use none
                report_error(status, GQE_ERR_INVALID_ARGUMENT, 1, 41);
                a0 = a1 = 0;
            }
            s_start[jj] = a0;
            s_prefix[jj] = acc;
            acc += a1 - a0;
        }
        s_prefix[u.hpg] = min(acc, kMaxRowsSimt);
    }
    __syncthreads();
    const int nrows = s_prefix[u.hpg];
    for (int r = threadIdx.x; r < nrows; r += blockDim.x) {
        int jj = 0;
        while (s_prefix[jj + 1] <= r) ++jj;
        const int j = q * u.hpg + jj;
        int t = head_pos[s_start[jj] + (r - s_prefix[jj])];
        float gv = 0.f;
        if (t < w0 || t >= min(w0 + kSimtW, u.T)) {  // outside the window: report, drop the row
            report_error(status, GQE_ERR_INVALID_ARGUMENT, 1, 40);
            t = -1;
        } else {
            const int64_t sel = (((int64_t)b * u.T + t) * u.g + q) * u.k;
            for (int s = 0; s < u.k; ++s)
                if (idx[sel + s] == j) gv = gate[sel + s];
        }
        rows_t[r] = t;
        rows_j[r] = (int16_t)j;
        rows_gate[r] = gv;
    }
    __syncthreads();

    // Zero-fill the window's unselected head slots.
    const int wend = min(w0 + kSimtW, u.T);
    for (int t = w0 + warp; t < wend; t += nwarps) {
        const int64_t sel = (((int64_t)b * u.T + t) * u.g + q) * u.k;
        for (int jj = 0; jj < u.hpg; ++jj) {
            const int j = q * u.hpg + jj;
            bool hit = false;
            for (int s = 0; s < u.k; ++s) hit |= (idx[sel + s] == j);
            if (!hit) {
                float* o = O + (((int64_t)b * u.T + t) * u.h + j) * d_h;
#pragma unroll
                for (int e = 0; e < DPL; ++e) o[e * 32 + lane] = 0.f;
            }
        }
    }

    // Attention: one warp per routed row.
    const float scale_log2 = rsqrtf((float)d_h) * 1.4426950408889634f;
    for (int r = warp; r < nrows; r += nwarps) {
        const int t = rows_t[r], j = rows_j[r];
        if (t < 0) continue;
        const float* qp = Q + (((int64_t)b * u.T + t) * u.h + j) * d_h;
        float qv[DPL], acc[DPL];
#pragma unroll
        for (int e = 0; e < DPL; ++e) {
            qv[e] = qp[e * 32 + lane] * scale_log2;
            acc[e] = 0.f;
        }
        float m = -INFINITY, l = 0.f;
        const float* kb = K + ((int64_t)b * u.T * kv_g + kv_q0 + q) * d_h;
        const float* vb = V + ((int64_t)b * u.T * kv_g + kv_q0 + q) * d_h;
        for (int s = 0; s <= t; ++s) {
            const float* kr = kb + (int64_t)s * kv_g * d_h;
            float p = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) p = fmaf(qv[e], kr[e * 32 + lane], p);
#pragma unroll
            for (int d = 16; d > 0; d >>= 1) p += __shfl_xor_sync(0xffffffffu, p, d);
            const float m_new = fmaxf(m, p);
            const float corr = exp2f(m - m_new);
            const float e_p = exp2f(p - m_new);
            l = l * corr + e_p;
            const float* vr = vb + (int64_t)s * kv_g * d_h;
#pragma unroll
            for (int e = 0; e < DPL; ++e) acc[e] = fmaf(e_p, vr[e * 32 + lane], acc[e] * corr);
            m = m_new;
        }
        const float f = rows_gate[r] / l;
        float* o = O + (((int64_t)b * u.T + t) * u.h + j) * d_h;
#pragma unroll
        for (int e = 0; e < DPL; ++e) o[e * 32 + lane] = acc[e] * f;
    }
}

}  // namespace

cudaError_t launch_prefill_simt(const PrefillArgs& a) {
    const gqe_shape& s = *a.s;
    UnitGeom u;
    u.B = s.B; u.T = s.T; u.h = s.h; u.g = s.g; u.k = s.k; u.hpg = s.h / s.g;
    u.W = kSimtW;
    u.nwin = (s.T + kSimtW - 1) / kSimtW;
    u.nchunk = gqe_chunk_count(s.T);
    const unsigned blocks = (unsigned)u.count();
#define GQE_SIMT_LAUNCH(DPL)                                                                        \
    prefill_simt_kernel<DPL><<<blocks, kSimtThreads, 0, a.stream>>>(                              \
        u, (const float*)a.Q, (const float*)a.K, (const float*)a.V, a.idx, a.gate, a.head_offsets, \
        a.head_pos, a.head_chunk_offsets, (float*)a.O, a.status, a.kv_g, a.kv_q0)
    switch (s.d_h) {
        case 32: GQE_SIMT_LAUNCH(1); break;
        case 64: GQE_SIMT_LAUNCH(2); break;
        case 128: GQE_SIMT_LAUNCH(4); break;
        default: return cudaErrorInvalidValue;
    }
#undef GQE_SIMT_LAUNCH
    return cudaGetLastError();
}

}  // namespace gqe
