// decode.cu -- GQE decode: one new query token per sequence against a dense
// KV cache [B, Lmax, g, d_h].
//
// The KV path stays dense under GQE (gist.science GQE summary, "Chemin KV
// Dense"), so decode is bound by reading the cache: 2 * n_kv * d_h * L elements
// per sequence and layer (ml-canon "56 GQA / MQA", KV-cache formula).  Each
// block streams one chunk of one sequence's cache rows for all g groups (whole
// contiguous token rows of g*d_h elements) with 16-byte loads; within a warp
// each group's rows are shared by the k routed query rows of that group.
// Partial softmax states (max, sum, accumulator) per chunk are merged by a
// second kernel, which also applies the gate and zero-fills unselected heads.
#include "common.cuh"

namespace gqe {
namespace {

constexpr int kDecodeChunk = 512;   // cache rows per block
constexpr int kDecodeThreads = 256; // 8 warps; warp w serves groups w, w+8, ...
constexpr int kDecodeUnroll = 8;    // token steps in flight per lane
constexpr uint32_t kWhereDecode = 4; // status "where" id of the decode kernels

template <int D>
struct PartRec {
    static constexpr int kFloats = D + 4;  // acc[D], m, l, pad, pad
};

template <typename T, int D, int KR, bool PAGED>
__global__ void __launch_bounds__(kDecodeThreads)
decode_partial_kernel(const T* __restrict__ q, const T* __restrict__ Kc, const T* __restrict__ Vc,
                      const int32_t* __restrict__ lengths, const int32_t* __restrict__ idx, int Lmax,
                      int h, int g, int k, int nchunk_max, float* __restrict__ part,
                      const int32_t* __restrict__ block_table, int max_blocks, int page_shift, int num_pages,
                      void* status) {
    constexpr int EPL = 16 / sizeof(T);  // elements per 16-byte vector
    constexpr int LPR = D / EPL;         // lanes per cache row
    constexpr int TPS = 32 / LPR;        // cache rows per warp step
    static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "unsupported head width");

    const int c = blockIdx.x, b = blockIdx.y;
    const int L = min(max(lengths[b], 1), Lmax);
    const int s0 = c * kDecodeChunk;
    if (s0 >= L) return;
    const int s1 = min(L, s0 + kDecodeChunk);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
    const int slot = lane / LPR, sub = lane % LPR;
    const float scale_log2 = rsqrtf((float)D) * 1.4426950408889634f;
    const int64_t row_stride = (int64_t)g * D;

    for (int grp = warp; grp < g; grp += nwarps) {
        float qv[KR][EPL];
#pragma unroll
        for (int r = 0; r < KR; ++r) {
            if (r < k) {
                int j = idx[((int64_t)b * g + grp) * k + r];
                if (j < grp * (h / g) || j >= (grp + 1) * (h / g)) j = grp * (h / g);  // out of group: clamp
                float f[EPL];
                unpack16(*reinterpret_cast<const uint4*>(q + ((int64_t)b * h + j) * D + sub * EPL), f,
                         (const T*)nullptr);
#pragma unroll
                for (int e = 0; e < EPL; ++e) qv[r][e] = f[e] * scale_log2;
            } else {
#pragma unroll
                for (int e = 0; e < EPL; ++e) qv[r][e] = 0.f;
            }
        }
        float m[KR], l[KR], acc[KR][EPL];
#pragma unroll
        for (int r = 0; r < KR; ++r) {
            m[r] = -INFINITY;
            l[r] = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[r][e] = 0.f;
        }
        // Cache row of logical position s: contiguous [B, Lmax] rows, or a row
        // of a page named by the block table (an entry outside the page pool is
        // reported and read as page 0, never out of bounds).
        const int64_t seq_base = PAGED ? 0 : (int64_t)b * Lmax * row_stride;
        const T* kbase = Kc + seq_base + (int64_t)grp * D + sub * EPL;
        const T* vbase = Vc + seq_base + (int64_t)grp * D + sub * EPL;
        const int32_t* bt = PAGED ? block_table + (int64_t)b * max_blocks : nullptr;
        auto cache_row = [&](int s) -> int64_t {
            if constexpr (PAGED) {
                int pg = bt[s >> page_shift];
                if ((unsigned)pg >= (unsigned)num_pages) {
                    report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereDecode, (uint32_t)b);
                    pg = 0;
                }
                return ((int64_t)pg << page_shift) + (s & ((1 << page_shift) - 1));
            } else {
                return s;  // the sequence's base is in kbase / vbase
            }
        };

        for (int sb = s0; sb < s1; sb += TPS * kDecodeUnroll) {
            uint4 kv[kDecodeUnroll], vv[kDecodeUnroll];
            bool valid[kDecodeUnroll];
#pragma unroll
            for (int u = 0; u < kDecodeUnroll; ++u) {
                const int s = sb + u * TPS + slot;
                valid[u] = s < s1;
                const int sc = valid[u] ? s : s1 - 1;
                const int64_t row = cache_row(sc);
                kv[u] = ld_stream16(kbase + row * row_stride);
                vv[u] = ld_stream16(vbase + row * row_stride);
            }
            float sc_[kDecodeUnroll][KR];
#pragma unroll
            for (int u = 0; u < kDecodeUnroll; ++u) {
                float kf[EPL];
                unpack16(kv[u], kf, (const T*)nullptr);
#pragma unroll
                for (int r = 0; r < KR; ++r) {
                    float p = 0.f;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) p = fmaf(qv[r][e], kf[e], p);
#pragma unroll
                    for (int d = LPR / 2; d > 0; d >>= 1) p += __shfl_xor_sync(0xffffffffu, p, d);
                    sc_[u][r] = valid[u] ? p : -INFINITY;
                }
            }
#pragma unroll
            for (int r = 0; r < KR; ++r) {
                float mx = m[r];
#pragma unroll
                for (int u = 0; u < kDecodeUnroll; ++u) mx = fmaxf(mx, sc_[u][r]);
                if (mx == -INFINITY) continue;  // no valid row for this slot yet
                const float corr = fast_exp2(m[r] - mx);
                l[r] *= corr;
#pragma unroll
                for (int e = 0; e < EPL; ++e) acc[r][e] *= corr;
                m[r] = mx;
            }
#pragma unroll
            for (int u = 0; u < kDecodeUnroll; ++u) {
                float vf[EPL];
                unpack16(vv[u], vf, (const T*)nullptr);
#pragma unroll
                for (int r = 0; r < KR; ++r) {
                    const float p = valid[u] ? fast_exp2(sc_[u][r] - m[r]) : 0.f;
                    l[r] += p;
#pragma unroll
                    for (int e = 0; e < EPL; ++e) acc[r][e] = fmaf(p, vf[e], acc[r][e]);
                }
            }
        }
        // Merge the TPS token slots of the warp.
#pragma unroll
        for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
            for (int r = 0; r < KR; ++r) {
                const float mo = __shfl_xor_sync(0xffffffffu, m[r], off);
                const float lo = __shfl_xor_sync(0xffffffffu, l[r], off);
                const float M = fmaxf(m[r], mo);
                const float fa = (m[r] == -INFINITY) ? 0.f : fast_exp2(m[r] - M);
                const float fb = (mo == -INFINITY) ? 0.f : fast_exp2(mo - M);
                l[r] = l[r] * fa + lo * fb;
#pragma unroll
                for (int e = 0; e < EPL; ++e) {
                    const float ao = __shfl_xor_sync(0xffffffffu, acc[r][e], off);
                    acc[r][e] = acc[r][e] * fa + ao * fb;
                }
                m[r] = M;
            }
        }
        if (slot == 0) {
#pragma unroll
            for (int r = 0; r < KR; ++r) {
                if (r >= k) break;
                float* rec = part + ((((int64_t)b * nchunk_max + c) * g + grp) * k + r) * PartRec<D>::kFloats;
#pragma unroll
                for (int e = 0; e < EPL; e += 4)
                    *reinterpret_cast<float4*>(rec + sub * EPL + e) =
                        make_float4(acc[r][e], acc[r][e + 1], acc[r][e + 2], acc[r][e + 3]);
                if (sub == 0) {
                    rec[D] = m[r];
                    rec[D + 1] = l[r];
                }
            }
        }
    }
}

// Merge the chunk partials of each (b, group, routed row), apply the gate,
// write O[b, j, :]; zero the unselected heads.  One warp per (b, head j):
// lanes hold the chunks' (max, sum) pairs, so the merged max and row sum are
// warp reductions, and the weighted rows of the chunks are read with
// independent loads.
constexpr int kCombineWarps = 8;
template <typename T, int D>
__global__ void __launch_bounds__(32 * kCombineWarps)
decode_combine_kernel(const float* __restrict__ part, const int32_t* __restrict__ lengths,
                      const int32_t* __restrict__ idx, const float* __restrict__ gate, int Lmax, int h, int g,
                      int k, int nchunk_max, T* __restrict__ O) {
    constexpr int DPL = (D + 31) / 32;
    constexpr int kRec = PartRec<D>::kFloats;
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31;
    const int j = blockIdx.y * kCombineWarps + (threadIdx.x >> 5);
    if (j >= h) return;
    const int hpg = h / g, grp = j / hpg;
    T* o = O + ((int64_t)b * h + j) * D;
    // the routed row of head j in this sequence, if any (first match, as the router never repeats a head)
    int r = -1;
    for (int rr = k - 1; rr >= 0; --rr)
        if (idx[((int64_t)b * g + grp) * k + rr] == j) r = rr;
    if (r < 0) {
#pragma unroll
        for (int e = 0; e < DPL; ++e)
            if (e * 32 + lane < D) o[e * 32 + lane] = Elem<T>::from_f(0.f);
        return;
    }
    const int L = min(max(lengths[b], 1), Lmax);
    const int nc = (L + kDecodeChunk - 1) / kDecodeChunk;
    const int64_t stride = (int64_t)g * k * kRec;  // from chunk c to chunk c+1
    const float* rec0 = part + (((int64_t)b * nchunk_max * g + grp) * k + r) * kRec;
    float M = -INFINITY;
    for (int c = lane; c < nc; c += 32) M = fmaxf(M, rec0[c * stride + D]);
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, d));
    float Ls = 0.f, acc[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[e] = 0.f;
    for (int c0 = 0; c0 < nc; c0 += 32) {
        const int c = c0 + lane;
        const float wl = (c < nc) ? fast_exp2(rec0[c * stride + D] - M) : 0.f;
        Ls = (c < nc) ? fmaf(rec0[c * stride + D + 1], wl, Ls) : Ls;
        const int n = min(32, nc - c0);
#pragma unroll 4
        for (int i = 0; i < n; ++i) {
            const float w = __shfl_sync(0xffffffffu, wl, i);
            const float* rec = rec0 + (c0 + i) * stride;
#pragma unroll
            for (int e = 0; e < DPL; ++e)
                if (e * 32 + lane < D) acc[e] = fmaf(rec[e * 32 + lane], w, acc[e]);
        }
    }
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) Ls += __shfl_xor_sync(0xffffffffu, Ls, d);
    const float f = gate[((int64_t)b * g + grp) * k + r] / Ls;
#pragma unroll
    for (int e = 0; e < DPL; ++e)
        if (e * 32 + lane < D) o[e * 32 + lane] = Elem<T>::from_f(acc[e] * f);
}

template <typename T, int D, int KR>
cudaError_t launch_typed(const DecodeArgs& a) {
    const gqe_shape& s = *a.s;
    const int nchunk_max = (a.Lmax + kDecodeChunk - 1) / kDecodeChunk;
    dim3 grid(nchunk_max, s.B);
    if (a.block_table != nullptr)
        decode_partial_kernel<T, D, KR, true><<<grid, kDecodeThreads, 0, a.stream>>>(
            (const T*)a.q, (const T*)a.K_cache, (const T*)a.V_cache, a.lengths, a.idx, a.Lmax, s.h, s.g, s.k,
            nchunk_max, a.partials, a.block_table, a.max_blocks, a.page_shift, a.num_pages, a.status);
    else
        decode_partial_kernel<T, D, KR, false><<<grid, kDecodeThreads, 0, a.stream>>>(
            (const T*)a.q, (const T*)a.K_cache, (const T*)a.V_cache, a.lengths, a.idx, a.Lmax, s.h, s.g, s.k,
            nchunk_max, a.partials, nullptr, 0, 0, 0, a.status);
    cudaError_t err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    dim3 cgrid(s.B, (s.h + kCombineWarps - 1) / kCombineWarps);
    decode_combine_kernel<T, D><<<cgrid, 32 * kCombineWarps, 0, a.stream>>>(
        a.partials, a.lengths, a.idx, a.gate, a.Lmax, s.h, s.g, s.k, nchunk_max, (T*)a.O);
    return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_kr(const DecodeArgs& a) {
    const int k = a.s->k;
    if (k <= 1) return launch_typed<T, D, 1>(a);
    if (k <= 2) return launch_typed<T, D, 2>(a);
    if (k <= 4) return launch_typed<T, D, 4>(a);
    return launch_typed<T, D, 8>(a);
}

}  // namespace

int decode_chunk_tokens(const gqe_shape*) { return kDecodeChunk; }

size_t decode_partials_bytes(const gqe_shape* s, int Lmax) {
    const size_t nchunk_max = (size_t)(Lmax + kDecodeChunk - 1) / kDecodeChunk;
    return nchunk_max * (size_t)s->B * s->g * s->k * (size_t)(s->d_h + 4) * sizeof(float);
}

cudaError_t launch_decode(const DecodeArgs& a) {
    const bool bf = a.s->dtype == GQE_BF16;
    switch (a.s->d_h) {
        case 32: return bf ? launch_kr<__nv_bfloat16, 32>(a) : launch_kr<float, 32>(a);
        case 64: return bf ? launch_kr<__nv_bfloat16, 64>(a) : launch_kr<float, 64>(a);
        case 128: return bf ? launch_kr<__nv_bfloat16, 128>(a) : launch_kr<float, 128>(a);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace gqe
