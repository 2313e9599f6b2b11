// backward.cuh -- launcher of the routed attention's backward pass.
#pragma once

#include "common.cuh"

namespace gqe {

struct AttnBwdArgs {
    const gqe_shape* s;
    const void* Q;  // [B,T,h,d_h]
    const void* K;  // [B,T,g,d_h]
    const void* V;
    const void* dO;  // gradient of the loss with respect to the output O [B,T,h,d_h]
    const int32_t* idx;
    const float* gate;
    const int32_t* head_offsets;
    const int32_t* head_pos;
    const int32_t* head_chunk_offsets;
    float* dQ;       // [B,T,h,d_h]
    float* dK;       // [B,T,g,d_h]
    float* dV;       // [B,T,g,d_h]
    float* dlogits;  // [B,T,h]
    void* scratch;   // attn_backward_scratch_bytes(s) bytes, 256-byte aligned
    void* status;
    cudaStream_t stream;
    // Saved by the training forward (tensor-core path): each routed row's
    // ungated fp32 output and log2-sum-exp.  Null: the backward recomputes them.
    const float* o32 = nullptr;
    const float* lse = nullptr;
};

// Per-(b,t,j) scratch of the backward: gate, D = dO.O and the row's log2-sum-exp
// (plus, on the tensor-core path, each routed row's ungated fp32 output).
size_t attn_backward_scratch_bytes(const gqe_shape* s);
cudaError_t launch_attn_backward(const AttnBwdArgs& a);

// Tensor-core backward (backward_tc.cu): bf16, d_h = 128, k <= 4, h/g <= 32.
bool attn_backward_tc_supported(const gqe_shape* s);
size_t attn_backward_tc_scratch_bytes(const gqe_shape* s);
cudaError_t launch_attn_backward_tc(const AttnBwdArgs& a);

struct RouteBwdArgs {
    const gqe_shape* s;
    const void* x;          // [B*T, d_model]
    const void* W_r;        // [d_model, h]
    const float* dlogits;   // [B*T, h]
    float* dx;              // [B*T, d_model]
    float* dW;              // [d_model, h]
    float* dbias;           // [h] or null
    void* scratch;          // route_backward_scratch_bytes(s) bytes
    cudaStream_t stream;
};

// Partial sums of dW_r over token ranges (reduced in a fixed order).
size_t route_backward_scratch_bytes(const gqe_shape* s);
cudaError_t launch_route_backward(const RouteBwdArgs& a);

}  // namespace gqe
