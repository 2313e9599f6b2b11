// output.cu -- the GQE layer's output construction around the routed heads.
//
// "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention"
// (gist.science summary), "Construction de la Sortie": per GQA group the
// outputs of the k selected experts are concatenated, a weighted sum of those
// outputs with the renormalised router probabilities forms one more slot, and
// one extra attention head is computed for every token whatever the routing
// (the shared head).
//
//  - group_slots_kernel builds the concatenated slots and the weighted sum from
//    the routed prefill's gated output O = gate * o: slot r of group q holds
//    o = O[b,t,idx[r]] / gate[r] (ungated, in selection order) and the sum is
//    sum_r O[b,t,idx[r]].  HBM-bound: one read of the selected rows, one write
//    of each slot.
//  - The shared head runs through the routed prefill itself, as one group of one
//    head that every token selects with gate 1 (identity tables written by
//    identity_tables_kernel), over one KV group of the caller's K/V.
#include "common.cuh"

namespace gqe {
namespace {

// Identity routing of one head: idx = 0, gate = 1, every position listed.
__global__ void identity_tables_kernel(int B, int T, int nchunk, int32_t* __restrict__ idx,
                                       float* __restrict__ gate, int32_t* __restrict__ head_offsets,
                                       int32_t* __restrict__ head_pos, int32_t* __restrict__ head_chunk_offsets) {
    const int64_t n = (int64_t)B * T;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        idx[i] = 0;
        gate[i] = 1.0f;
        head_pos[i] = (int32_t)(i % T);
        if (i % T % kChunk == 0)
            head_chunk_offsets[(i / T) * nchunk + (i % T) / kChunk] = (int32_t)i;
        if (i % T == 0) head_offsets[i / T] = (int32_t)i;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) head_offsets[B] = (int32_t)n;
}

// A group of L lanes per (b, t, group q), L = row bytes / 16: each lane moves 16
// bytes of a row, and the k selected rows are loaded four at a time before any
// is used, so each lane keeps up to 64 bytes in flight.
template <typename T, int D>
struct SlotsCfg {
    static constexpr int kVec = 16 / sizeof(T);     // elements per 16-byte vector
    static constexpr int kLanes = D / kVec;         // lanes per item
    static_assert(32 % kLanes == 0, "row of 64..512 bytes");
};

template <typename T>
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ void unpack16<__nv_bfloat16>(const uint4& v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
template <>
__device__ __forceinline__ void unpack16<float>(const uint4& v, float (&f)[4]) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}
template <typename T>
__device__ __forceinline__ uint4 pack16(const float (&f)[16 / sizeof(T)]);
template <>
__device__ __forceinline__ uint4 pack16<__nv_bfloat16>(const float (&f)[8]) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}
template <>
__device__ __forceinline__ uint4 pack16<float>(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]), __float_as_uint(f[3]));
}

template <typename T, int D>
__global__ void __launch_bounds__(256)
group_slots_kernel(int64_t BT, int h, int g, int k, const T* __restrict__ O, const int32_t* __restrict__ idx,
                   const float* __restrict__ gate, T* __restrict__ cat, T* __restrict__ wsum) {
    using Cfg = SlotsCfg<T, D>;
    constexpr int V = Cfg::kVec, L = Cfg::kLanes;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t item = tid / L;  // (b*T + t) * g + q
    const int sub = (int)(tid % L);
    if (item >= BT * g) return;
    const int64_t bt = item / g;
    const int q = (int)(item % g), hpg = h / g;
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
    for (int r0 = 0; r0 < k; r0 += 4) {
        uint4 raw[4];
        float gv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            raw[i] = make_uint4(0, 0, 0, 0);
            gv[i] = 0.f;
            if (r0 + i < k) {
                const int64_t sel = item * k + r0 + i;
                const int j = idx[sel];
                gv[i] = gate[sel];
                // a selection outside the group (not produced by the router) contributes nothing
                if (j >= q * hpg && j < (q + 1) * hpg)
                    raw[i] = *reinterpret_cast<const uint4*>(O + (bt * h + j) * D + sub * V);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            if (r0 + i >= k) break;
            float v[V];
            unpack16<T>(raw[i], v);
#pragma unroll
            for (int e = 0; e < V; ++e) acc[e] += v[e];
            if (cat != nullptr) {
                // a gate that underflowed to zero leaves nothing to recover: the slot is 0
                const float inv = gv[i] > 0.f ? 1.0f / gv[i] : 0.f;
#pragma unroll
                for (int e = 0; e < V; ++e) v[e] *= inv;
                *reinterpret_cast<uint4*>(cat + (item * k + r0 + i) * D + sub * V) = pack16<T>(v);
            }
        }
    }
    if (wsum != nullptr) *reinterpret_cast<uint4*>(wsum + item * D + sub * V) = pack16<T>(acc);
}

template <typename T>
cudaError_t launch_slots_typed(const GroupSlotsArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const int64_t threads = BT * s.g * (s.d_h * (int64_t)sizeof(T) / 16);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
#define GQE_SLOTS(D)                                                                                      \
    group_slots_kernel<T, D><<<blocks, 256, 0, a.stream>>>(BT, s.h, s.g, s.k, (const T*)a.O, a.idx, a.gate, \
                                                           (T*)a.cat, (T*)a.wsum)
    switch (s.d_h) {
        case 32: GQE_SLOTS(32); break;
        case 64: GQE_SLOTS(64); break;
        case 128: GQE_SLOTS(128); break;
        default: return cudaErrorInvalidValue;
    }
#undef GQE_SLOTS
    return cudaGetLastError();
}

}  // namespace

size_t shared_tables_bytes(int B, int T) {
    auto a256 = [](size_t n) { return (n + 255) & ~size_t(255); };
    const size_t bt = (size_t)B * T * sizeof(int32_t);
    return 3 * a256(bt) + a256((size_t)(B + 1) * sizeof(int32_t)) +
           a256((size_t)B * gqe_chunk_count(T) * sizeof(int32_t));
}

cudaError_t launch_identity_tables(int B, int T, void* tables, IdentityTables* out, cudaStream_t stream) {
    auto a256 = [](size_t n) { return (n + 255) & ~size_t(255); };
    char* p = static_cast<char*>(tables);
    const size_t bt = (size_t)B * T * sizeof(int32_t);
    out->idx = reinterpret_cast<int32_t*>(p);
    p += a256(bt);
    out->gate = reinterpret_cast<float*>(p);
    p += a256(bt);
    out->head_pos = reinterpret_cast<int32_t*>(p);
    p += a256(bt);
    out->head_offsets = reinterpret_cast<int32_t*>(p);
    p += a256((size_t)(B + 1) * sizeof(int32_t));
    out->head_chunk_offsets = reinterpret_cast<int32_t*>(p);
    const int64_t n = (int64_t)B * T;
    const unsigned blocks = (unsigned)((n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024);
    identity_tables_kernel<<<blocks, 256, 0, stream>>>(B, T, gqe_chunk_count(T), out->idx, out->gate,
                                                       out->head_offsets, out->head_pos, out->head_chunk_offsets);
    return cudaGetLastError();
}

cudaError_t launch_group_slots(const GroupSlotsArgs& a) {
    return a.s->dtype == GQE_BF16 ? launch_slots_typed<__nv_bfloat16>(a) : launch_slots_typed<float>(a);
}

}  // namespace gqe
