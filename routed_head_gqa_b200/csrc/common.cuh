// common.cuh -- shared device helpers and internal launch declarations of libgqe.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/gqe.h"

namespace gqe {

constexpr int kChunk = 32;             // compaction chunk (one warp ballot)
constexpr size_t kStatusBytes = 256;   // status word region at the start of the workspace

// Status word layout (uint32 each): [0] error code, [1] kernel id, [2] detail.
struct DeviceStatus {
    uint32_t code;
    uint32_t where;
    uint32_t detail;
};

__device__ __forceinline__ void report_error(void* status, uint32_t code, uint32_t where,
                                             uint32_t detail) {
    DeviceStatus* st = reinterpret_cast<DeviceStatus*>(status);
    if (atomicCAS(&st->code, 0u, code) == 0u) {
        st->where = where;
        st->detail = detail;
    }
}

template <typename T>
struct Elem;
template <>
struct Elem<float> {
    static __device__ __forceinline__ float to_f(float v) { return v; }
    static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <>
struct Elem<__nv_bfloat16> {
    static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
    static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte vector <-> fp32 lanes.  For bf16, 8 elements; for fp32, 4.
template <typename T>
struct Vec16 {
    static constexpr int N = 16 / sizeof(T);
};

__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[8], const __nv_bfloat16*) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ void unpack16(const uint4& v, float (&f)[4], const float*) {
    f[0] = __uint_as_float(v.x);
    f[1] = __uint_as_float(v.y);
    f[2] = __uint_as_float(v.z);
    f[3] = __uint_as_float(v.w);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

__device__ __forceinline__ float fast_exp2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Streaming (read-once) 16-byte global load.
__device__ __forceinline__ uint4 ld_stream16(const void* p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// ------------------------------------------------------------------------
// Internal launchers (host).  Each returns cudaSuccess or the launch error.
// ------------------------------------------------------------------------
struct RouteArgs {
    const gqe_shape* s;
    const void* x;
    const void* W_r;
    const float* bias;
    int32_t* idx;
    float* gate;
    int32_t* head_offsets;
    int32_t* head_pos;
    int32_t* head_chunk_offsets;
    int32_t* counts;  // workspace: [B*h*nchunk]
    void* status;
    cudaStream_t stream;
    float* logits = nullptr;  // optional out: fp32 router logits (bias included) [B*T, h]
};
cudaError_t launch_route(const RouteArgs& a);
bool router_tc_supported(const gqe_shape* s);
cudaError_t launch_router_tc(const RouteArgs& a);  // a1+a2 on tensor cores (bf16)
// True when launch_router_tc also writes RouteArgs::counts (T a multiple of
// the 32-token chunk), so the separate count pass is skipped.
bool router_tc_fuses_counts(const gqe_shape* s);

// Library-held scratch for gqe_route_static: a kStatusBytes status region
// (the device status word of these calls), then the per-(b, head, chunk)
// counts, at most kRouteStaticScratchBytes of them.  Resolves the calling
// thread's current device's copy of the array (once per device) into *out.
constexpr size_t kRouteStaticScratchBytes = size_t(4) << 20;  // 4 MiB of counts
cudaError_t route_static_scratch(uint8_t** out);

struct PrefillArgs {
    const gqe_shape* s;
    const void* Q;
    const void* K;
    const void* V;
    const int32_t* idx;
    const float* gate;
    const int32_t* head_offsets;
    const int32_t* head_pos;
    const int32_t* head_chunk_offsets;
    void* O;
    void* status;
    cudaStream_t stream;
    // K/V layout [B, T, kv_g, d_h]; the shape's group q reads KV group kv_q0 + q.
    // A routed prefill has kv_g = g, kv_q0 = 0; the shared head runs as one
    // group of one head over a chosen KV group of the caller's K/V.
    int kv_g;
    int kv_q0;
    // Training outputs (tensor-core prefill only): when o32 is set, the kernel
    // also writes each routed row's ungated fp32 output o32[b,t,j,:] and its
    // log2-sum-exp lse[b,t,j]; O may then be null (a recompute for the
    // backward: O and its zero fill are skipped).
    float* o32 = nullptr;
    float* lse = nullptr;
    // Scratch for split-KV partials (tensor-core prefill): used when the units
    // would leave SMs idle and split_bytes >= prefill_split_bytes(s); null: no split.
    void* split_scratch = nullptr;
    size_t split_bytes = 0;
};
// Routed query projection (qproj.cu).
struct QprojArgs {
    const gqe_shape* s;
    const void* x;               // [B, T, d_model] bf16
    const void* W_Q;             // [d_model, h * 128] bf16
    const int32_t* idx;          // [B, T, g, k] as written by gqe_route
    const int32_t* head_offsets; // as written by gqe_route
    const int32_t* head_pos;
    void* Q;                     // [B, T, h, 128] bf16, routed rows written
    void* status;
    void* scratch;               // oproj_scratch_bytes(s) bytes (the dense path's tile sets), or null
    cudaStream_t stream;
};
cudaError_t launch_qproj(const QprojArgs& a);
// The dense path (proj_tc.cu): every head of a token tile with a routed head.
cudaError_t launch_qproj_dense(const QprojArgs& a);

// Routed output projection (oproj.cu).
struct OprojArgs {
    const gqe_shape* s;
    const void* O;               // [B, T, h, d_h] bf16, zeros in the unselected slots
    const int32_t* idx;          // [B, T, g, k]
    const void* W_Z;             // [h * d_h, d_model] bf16
    void* Y;                     // [B, T, d_model] bf16, out
    void* status;
    void* scratch;               // oproj_scratch_bytes(s): the token tiles' active-head sets
    cudaStream_t stream;
};
cudaError_t launch_oproj(const OprojArgs& a);
size_t oproj_scratch_bytes(const gqe_shape* s);

// Output construction (output.cu).
struct GroupSlotsArgs {
    const gqe_shape* s;
    const void* O;       // [B, T, h, d_h] gated routed output
    const int32_t* idx;  // [B, T, g, k]
    const float* gate;   // [B, T, g, k]
    void* cat;           // [B, T, g, k, d_h] or null
    void* wsum;          // [B, T, g, d_h] or null
    cudaStream_t stream;
};
cudaError_t launch_group_slots(const GroupSlotsArgs& a);
// Identity routing of one head (every position, gate 1) for the shared head.
struct IdentityTables {
    int32_t* idx;
    float* gate;
    int32_t* head_offsets;
    int32_t* head_pos;
    int32_t* head_chunk_offsets;
};
size_t shared_tables_bytes(int B, int T);
cudaError_t launch_identity_tables(int B, int T, void* tables, IdentityTables* out, cudaStream_t stream);

// Load-balancing auxiliary loss (aux_loss.cu).
struct AuxLossArgs {
    const gqe_shape* s;
    const float* logits;   // [B*T, h]
    const int32_t* idx;    // [B*T, g, k]
    float* loss;           // [1]
    float* dlogits;        // [B*T, h] or null
    void* scratch;         // aux_loss_scratch_bytes(s)
    void* status;
    cudaStream_t stream;
};
size_t aux_loss_scratch_bytes(const gqe_shape* s);
cudaError_t launch_aux_loss(const AuxLossArgs& a);

cudaError_t launch_prefill_simt(const PrefillArgs& a);
cudaError_t launch_prefill_tc(const PrefillArgs& a);
// Scratch the tensor-core prefill uses for split-KV partials on this device (0: no split).
size_t prefill_split_bytes(const gqe_shape* s);

struct DecodeArgs {
    const gqe_shape* s;
    const void* q;
    const void* K_cache;
    const void* V_cache;
    int Lmax;
    const int32_t* lengths;
    const int32_t* idx;
    const float* gate;
    void* O;
    float* partials;  // workspace
    void* status;
    cudaStream_t stream;
    // Paged caches (block_table != null): K_cache/V_cache are [num_pages,
    // page_size, g, d_h]; logical row s of sequence b is row s % page_size of
    // page block_table[b * max_blocks + s / page_size]; Lmax = page_size * max_blocks.
    const int32_t* block_table = nullptr;
    int max_blocks = 0;
    int page_shift = 0;  // log2(page_size)
    int num_pages = 0;
};
int decode_chunk_tokens(const gqe_shape* s);
size_t decode_partials_bytes(const gqe_shape* s, int Lmax);
cudaError_t launch_decode(const DecodeArgs& a);

}  // namespace gqe
