// gqe_api.cu -- extern "C" entry points of libgqe: argument validation on the
// host, then kernel launches on the caller's stream.  See include/gqe.h.
#include <cstring>

#include "backward.cuh"
#include "common.cuh"

using namespace gqe;

namespace {

constexpr int kMaxK = 16;
constexpr int kMaxH = 256;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

gqe_status check_shape(const gqe_shape* s) {
    if (!s) return GQE_ERR_INVALID_ARGUMENT;
    if (s->B < 1 || s->T < 1 || s->h < 1 || s->g < 1 || s->d_h < 1 || s->k < 1 || s->d_model < 1)
        return GQE_ERR_INVALID_ARGUMENT;
    if (s->h % s->g != 0) return GQE_ERR_INVALID_ARGUMENT;
    if (s->k > s->h / s->g) return GQE_ERR_INVALID_ARGUMENT;
    if (s->dtype != GQE_F32 && s->dtype != GQE_BF16) return GQE_ERR_INVALID_ARGUMENT;
    const int64_t rows = (int64_t)s->B * s->T * s->g * s->k;
    if (rows >= ((int64_t)1 << 31)) return GQE_ERR_UNSUPPORTED;
    if (s->k > kMaxK || s->h > kMaxH) return GQE_ERR_UNSUPPORTED;
    return GQE_OK;
}

gqe_status check_workspace(void* ws, size_t bytes, size_t need) {
    if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return GQE_ERR_INVALID_ARGUMENT;
    if (bytes < need) return GQE_ERR_INVALID_ARGUMENT;
    return GQE_OK;
}

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

size_t route_scratch_bytes(const gqe_shape* s) {
    return align256((size_t)s->B * s->h * gqe_chunk_count(s->T) * sizeof(int32_t));
}

gqe_status from_cuda(cudaError_t e) { return e == cudaSuccess ? GQE_OK : GQE_ERR_CUDA; }

}  // namespace

extern "C" {

int gqe_chunk_count(int T) { return T <= 0 ? 0 : (T + kChunk - 1) / kChunk; }

size_t gqe_workspace_bytes(const gqe_shape* s, int Lmax) {
    if (check_shape(s) == GQE_ERR_INVALID_ARGUMENT || Lmax < 0) return 0;
    size_t need = kStatusBytes + route_scratch_bytes(s);
    const size_t shared = kStatusBytes + shared_tables_bytes(s->B, s->T);
    if (shared > need) need = shared;
    const size_t oproj = kStatusBytes + oproj_scratch_bytes(s);
    if (oproj > need) need = oproj;
    const size_t split = kStatusBytes + prefill_split_bytes(s);
    if (split > need) need = split;
    gqe_shape one = *s;  // the shared head: identity tables, then its split-KV partials
    one.h = 1;
    one.g = 1;
    one.k = 1;
    const size_t shared_split = kStatusBytes + shared_tables_bytes(s->B, s->T) + prefill_split_bytes(&one);
    if (shared_split > need) need = shared_split;
    if (Lmax > 0) {
        const size_t dec = kStatusBytes + align256(decode_partials_bytes(s, Lmax));
        if (dec > need) need = dec;
    }
    return need;
}

gqe_status gqe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != GQE_OK) return st;
    return from_cuda(cudaMemsetAsync(workspace, 0, kStatusBytes, (cudaStream_t)stream));
}

gqe_status gqe_route(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                     int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                     int32_t* head_chunk_offsets, void* workspace, size_t workspace_bytes,
                     void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!x || !W_r || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(W_r)) return GQE_ERR_INVALID_ARGUMENT;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + route_scratch_bytes(s));
    if (st != GQE_OK) return st;
    RouteArgs a;
    a.s = s;
    a.x = x;
    a.W_r = W_r;
    a.bias = bias;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes);
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_route(a));
}

gqe_status gqe_route_train(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                           int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                           int32_t* head_chunk_offsets, float* logits, void* workspace, size_t workspace_bytes,
                           void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!x || !W_r || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets || !logits)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(W_r)) return GQE_ERR_INVALID_ARGUMENT;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + route_scratch_bytes(s));
    if (st != GQE_OK) return st;
    RouteArgs a;
    a.s = s;
    a.x = x;
    a.W_r = W_r;
    a.bias = bias;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.counts = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + kStatusBytes);
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.logits = logits;
    return from_cuda(launch_route(a));
}

size_t gqe_aux_loss_workspace_bytes(const gqe_shape* s) {
    if (check_shape(s) == GQE_ERR_INVALID_ARGUMENT) return 0;
    return kStatusBytes + aux_loss_scratch_bytes(s);
}

gqe_status gqe_aux_loss(const gqe_shape* s, const float* logits, const int32_t* idx, float* loss, float* dlogits,
                        void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!logits || !idx || !loss) return GQE_ERR_INVALID_ARGUMENT;
    if (s->h / s->g > 64) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + aux_loss_scratch_bytes(s));
    if (st != GQE_OK) return st;
    AuxLossArgs a;
    a.s = s;
    a.logits = logits;
    a.idx = idx;
    a.loss = loss;
    a.dlogits = dlogits;
    a.scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_aux_loss(a));
}

gqe_status gqe_route_static(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                            int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                            int32_t* head_chunk_offsets, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!x || !W_r || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(W_r)) return GQE_ERR_INVALID_ARGUMENT;
    const size_t need = (size_t)s->B * s->h * gqe_chunk_count(s->T) * sizeof(int32_t);
    if (need > kRouteStaticScratchBytes) return GQE_ERR_SCRATCH_LIMIT;
    uint8_t* scratch = nullptr;
    if (route_static_scratch(&scratch) != cudaSuccess) return GQE_ERR_CUDA;
    RouteArgs a;
    a.s = s;
    a.x = x;
    a.W_r = W_r;
    a.bias = bias;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    // Every count is written before it is read: nothing to clear.  A bounded
    // wait that expires in the router, or counts the compaction cannot trust,
    // are recorded in the status word at the head of the array (read and
    // cleared by gqe_route_static_status).
    a.counts = reinterpret_cast<int32_t*>(scratch + kStatusBytes);
    a.status = scratch;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_route(a));
}

gqe_status gqe_route_static_status(void* stream) {
    uint8_t* scratch = nullptr;
    if (route_static_scratch(&scratch) != cudaSuccess) return GQE_ERR_CUDA;
    return gqe_get_device_status(scratch, stream);
}

gqe_status gqe_attn_prefill(const gqe_shape* s, const void* Q, const void* K, const void* V,
                            const int32_t* idx, const float* gate, const int32_t* head_offsets,
                            const int32_t* head_pos, const int32_t* head_chunk_offsets, void* O,
                            void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!Q || !K || !V || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets || !O)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return GQE_ERR_INVALID_ARGUMENT;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != GQE_OK) return st;
    PrefillArgs a;
    a.s = s;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.O = O;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.kv_g = s->g;
    a.kv_q0 = 0;
    a.split_scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.split_bytes = workspace_bytes - kStatusBytes;
    if (s->dtype == GQE_BF16) {
        if (s->d_h != 128) return GQE_ERR_UNSUPPORTED;
        return from_cuda(launch_prefill_tc(a));
    }
    if (s->d_h != 32 && s->d_h != 64 && s->d_h != 128) return GQE_ERR_UNSUPPORTED;
    if (s->h / s->g > 64) return GQE_ERR_UNSUPPORTED;
    return from_cuda(launch_prefill_simt(a));
}

gqe_status gqe_attn_shared_head(const gqe_shape* s, const void* Qs, const void* K, const void* V, int kv_group,
                                void* Os, void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!Qs || !K || !V || !Os) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(Qs) || !aligned16(K) || !aligned16(V) || !aligned16(Os)) return GQE_ERR_INVALID_ARGUMENT;
    if (kv_group < 0 || kv_group >= s->g) return GQE_ERR_INVALID_ARGUMENT;
    if (s->dtype == GQE_BF16 ? s->d_h != 128 : (s->d_h != 32 && s->d_h != 64 && s->d_h != 128))
        return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + shared_tables_bytes(s->B, s->T));
    if (st != GQE_OK) return st;
    // One group of one head, selected by every token with gate 1.
    gqe_shape one = *s;
    one.h = 1;
    one.g = 1;
    one.k = 1;
    IdentityTables tab;
    cudaError_t err = launch_identity_tables(s->B, s->T, static_cast<char*>(workspace) + kStatusBytes, &tab,
                                             (cudaStream_t)stream);
    if (err != cudaSuccess) return GQE_ERR_CUDA;
    PrefillArgs a;
    a.s = &one;
    a.Q = Qs;
    a.K = K;
    a.V = V;
    a.idx = tab.idx;
    a.gate = tab.gate;
    a.head_offsets = tab.head_offsets;
    a.head_pos = tab.head_pos;
    a.head_chunk_offsets = tab.head_chunk_offsets;
    a.O = Os;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.kv_g = s->g;
    a.kv_q0 = kv_group;
    const size_t used = kStatusBytes + shared_tables_bytes(s->B, s->T);
    a.split_scratch = static_cast<char*>(workspace) + used;
    a.split_bytes = workspace_bytes - used;
    return from_cuda(s->dtype == GQE_BF16 ? launch_prefill_tc(a) : launch_prefill_simt(a));
}

gqe_status gqe_routed_qproj(const gqe_shape* s, const void* x, const void* W_Q, const int32_t* idx,
                            const int32_t* head_offsets, const int32_t* head_pos, void* Q, void* workspace,
                            size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!x || !W_Q || !idx || !head_offsets || !head_pos || !Q) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(x) || !aligned16(W_Q) || !aligned16(idx) || !aligned16(Q)) return GQE_ERR_INVALID_ARGUMENT;
    if (s->dtype != GQE_BF16 || s->d_h != 128 || s->d_model % 8 != 0) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != GQE_OK) return st;
    QprojArgs a;
    a.s = s;
    a.x = x;
    a.W_Q = W_Q;
    a.idx = idx;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.Q = Q;
    a.status = workspace;
    // the dense path's per-tile head sets, when the workspace has room for them
    a.scratch = workspace_bytes >= kStatusBytes + oproj_scratch_bytes(s)
                    ? static_cast<void*>(static_cast<char*>(workspace) + kStatusBytes)
                    : nullptr;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_qproj(a));
}

gqe_status gqe_routed_oproj(const gqe_shape* s, const void* O, const int32_t* idx, const void* W_Z, void* Y,
                            void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!O || !idx || !W_Z || !Y) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(O) || !aligned16(idx) || !aligned16(W_Z) || !aligned16(Y)) return GQE_ERR_INVALID_ARGUMENT;
    if (s->dtype != GQE_BF16 || s->d_h % 64 != 0 || s->h > 64 || s->d_model % 32 != 0) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + oproj_scratch_bytes(s));
    if (st != GQE_OK) return st;
    OprojArgs a;
    a.s = s;
    a.O = O;
    a.idx = idx;
    a.W_Z = W_Z;
    a.Y = Y;
    a.status = workspace;
    a.scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_oproj(a));
}

gqe_status gqe_group_slots(const gqe_shape* s, const void* O, const int32_t* idx, const float* gate, void* O_cat,
                           void* O_wsum, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!O || !idx || !gate || (!O_cat && !O_wsum)) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(O) || (O_cat && !aligned16(O_cat)) || (O_wsum && !aligned16(O_wsum)))
        return GQE_ERR_INVALID_ARGUMENT;
    if (s->d_h != 32 && s->d_h != 64 && s->d_h != 128) return GQE_ERR_UNSUPPORTED;
    GroupSlotsArgs a;
    a.s = s;
    a.O = O;
    a.idx = idx;
    a.gate = gate;
    a.cat = O_cat;
    a.wsum = O_wsum;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_group_slots(a));
}

gqe_status gqe_attn_decode(const gqe_shape* s, const void* q, const void* K_cache,
                           const void* V_cache, int Lmax, const int32_t* lengths,
                           const int32_t* idx, const float* gate, void* O, void* workspace,
                           size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (s->T != 1 || Lmax < 1) return GQE_ERR_INVALID_ARGUMENT;
    if (!q || !K_cache || !V_cache || !lengths || !idx || !gate || !O) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(K_cache) || !aligned16(V_cache) || !aligned16(O))
        return GQE_ERR_INVALID_ARGUMENT;
    if (s->d_h != 32 && s->d_h != 64 && s->d_h != 128) return GQE_ERR_UNSUPPORTED;
    if (s->k > 8) return GQE_ERR_UNSUPPORTED;
    if ((int64_t)s->B * Lmax * s->g * s->d_h >= ((int64_t)1 << 40)) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + align256(decode_partials_bytes(s, Lmax)));
    if (st != GQE_OK) return st;
    DecodeArgs a;
    a.s = s;
    a.q = q;
    a.K_cache = K_cache;
    a.V_cache = V_cache;
    a.Lmax = Lmax;
    a.lengths = lengths;
    a.idx = idx;
    a.gate = gate;
    a.O = O;
    a.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_decode(a));
}

gqe_status gqe_attn_decode_paged(const gqe_shape* s, const void* q, const void* K_pages, const void* V_pages,
                                 int num_pages, int page_size, const int32_t* block_table, int max_blocks,
                                 const int32_t* lengths, const int32_t* idx, const float* gate, void* O,
                                 void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (s->T != 1 || num_pages < 1 || max_blocks < 1) return GQE_ERR_INVALID_ARGUMENT;
    if (page_size < 1 || page_size > (1 << 16) || (page_size & (page_size - 1)) != 0) return GQE_ERR_INVALID_ARGUMENT;
    const int64_t cap = (int64_t)page_size * max_blocks;
    if (cap >= ((int64_t)1 << 31)) return GQE_ERR_UNSUPPORTED;
    if (!q || !K_pages || !V_pages || !block_table || !lengths || !idx || !gate || !O) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(K_pages) || !aligned16(V_pages) || !aligned16(O)) return GQE_ERR_INVALID_ARGUMENT;
    if (s->d_h != 32 && s->d_h != 64 && s->d_h != 128) return GQE_ERR_UNSUPPORTED;
    if (s->k > 8) return GQE_ERR_UNSUPPORTED;
    if ((int64_t)num_pages * page_size * s->g * s->d_h >= ((int64_t)1 << 40)) return GQE_ERR_UNSUPPORTED;
    const int Lmax = (int)cap;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + align256(decode_partials_bytes(s, Lmax)));
    if (st != GQE_OK) return st;
    DecodeArgs a;
    a.s = s;
    a.q = q;
    a.K_cache = K_pages;
    a.V_cache = V_pages;
    a.Lmax = Lmax;
    a.lengths = lengths;
    a.idx = idx;
    a.gate = gate;
    a.O = O;
    a.partials = reinterpret_cast<float*>(static_cast<char*>(workspace) + kStatusBytes);
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.block_table = block_table;
    a.max_blocks = max_blocks;
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    a.page_shift = shift;
    a.num_pages = num_pages;
    return from_cuda(launch_decode(a));
}

size_t gqe_backward_workspace_bytes(const gqe_shape* s) {
    if (check_shape(s) == GQE_ERR_INVALID_ARGUMENT) return 0;
    const size_t a = attn_backward_scratch_bytes(s), r = route_backward_scratch_bytes(s);
    return kStatusBytes + (a > r ? a : r);
}

gqe_status gqe_route_backward(const gqe_shape* s, const void* x, const void* W_r, const float* dlogits, float* dx,
                              float* dW_r, float* dbias, void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!x || !W_r || !dlogits || !dx || !dW_r) return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(dx)) return GQE_ERR_INVALID_ARGUMENT;
    if ((int64_t)s->B * s->T > (int64_t)65535 * 64) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + route_backward_scratch_bytes(s));
    if (st != GQE_OK) return st;
    RouteBwdArgs a;
    a.s = s;
    a.x = x;
    a.W_r = W_r;
    a.dlogits = dlogits;
    a.dx = dx;
    a.dW = dW_r;
    a.dbias = dbias;
    a.scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_route_backward(a));
}

gqe_status gqe_attn_prefill_backward(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                     const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                     const int32_t* head_pos, const int32_t* head_chunk_offsets, const void* dO,
                                     float* dQ, float* dK, float* dV, float* dlogits, void* workspace,
                                     size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!Q || !K || !V || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets || !dO || !dQ || !dK ||
        !dV || !dlogits)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(dQ) || !aligned16(dK) ||
        !aligned16(dV))
        return GQE_ERR_INVALID_ARGUMENT;
    if (s->d_h != 32 && s->d_h != 64 && s->d_h != 128) return GQE_ERR_UNSUPPORTED;
    if ((int64_t)s->B * s->h > 65535 || s->B > 65535 || s->g > 65535) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + attn_backward_scratch_bytes(s));
    if (st != GQE_OK) return st;
    AttnBwdArgs a;
    a.s = s;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.dO = dO;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.dlogits = dlogits;
    a.scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    return from_cuda(launch_attn_backward(a));
}

gqe_status gqe_attn_prefill_train(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                  const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                  const int32_t* head_pos, const int32_t* head_chunk_offsets, void* O, float* O32,
                                  float* lse, void* workspace, size_t workspace_bytes, void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!Q || !K || !V || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets || !O32 || !lse)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || (O && !aligned16(O)) || !aligned16(O32))
        return GQE_ERR_INVALID_ARGUMENT;
    if (!attn_backward_tc_supported(s)) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes);
    if (st != GQE_OK) return st;
    PrefillArgs a;
    a.s = s;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.O = O;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.kv_g = s->g;
    a.kv_q0 = 0;
    a.o32 = O32;
    a.lse = lse;
    return from_cuda(launch_prefill_tc(a));
}

gqe_status gqe_attn_prefill_backward_saved(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                           const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                           const int32_t* head_pos, const int32_t* head_chunk_offsets,
                                           const void* dO, const float* O32, const float* lse, float* dQ, float* dK,
                                           float* dV, float* dlogits, void* workspace, size_t workspace_bytes,
                                           void* stream) {
    gqe_status st = check_shape(s);
    if (st != GQE_OK) return st;
    if (!Q || !K || !V || !idx || !gate || !head_offsets || !head_pos || !head_chunk_offsets || !dO || !O32 || !lse ||
        !dQ || !dK || !dV || !dlogits)
        return GQE_ERR_INVALID_ARGUMENT;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(dO) || !aligned16(O32) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV))
        return GQE_ERR_INVALID_ARGUMENT;
    if (!attn_backward_tc_supported(s)) return GQE_ERR_UNSUPPORTED;
    st = check_workspace(workspace, workspace_bytes, kStatusBytes + attn_backward_scratch_bytes(s));
    if (st != GQE_OK) return st;
    AttnBwdArgs a;
    a.s = s;
    a.Q = Q;
    a.K = K;
    a.V = V;
    a.dO = dO;
    a.idx = idx;
    a.gate = gate;
    a.head_offsets = head_offsets;
    a.head_pos = head_pos;
    a.head_chunk_offsets = head_chunk_offsets;
    a.dQ = dQ;
    a.dK = dK;
    a.dV = dV;
    a.dlogits = dlogits;
    a.scratch = static_cast<char*>(workspace) + kStatusBytes;
    a.status = workspace;
    a.stream = (cudaStream_t)stream;
    a.o32 = O32;
    a.lse = lse;
    return from_cuda(launch_attn_backward(a));
}

gqe_status gqe_get_device_status(void* workspace, void* stream) {
    if (!workspace) return GQE_ERR_INVALID_ARGUMENT;
    DeviceStatus host{};
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&host, workspace, sizeof host, cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return GQE_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return GQE_ERR_CUDA;
    if (host.code != 0) {
        if (cudaMemsetAsync(workspace, 0, sizeof host, st) != cudaSuccess) return GQE_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return GQE_ERR_CUDA;
        return (gqe_status)host.code;
    }
    return GQE_OK;
}

const char* gqe_status_string(gqe_status s) {
    switch (s) {
        case GQE_OK: return "GQE_OK";
        case GQE_ERR_INVALID_ARGUMENT: return "GQE_ERR_INVALID_ARGUMENT";
        case GQE_ERR_UNSUPPORTED: return "GQE_ERR_UNSUPPORTED";
        case GQE_ERR_CUDA: return "GQE_ERR_CUDA";
        case GQE_ERR_DEVICE_TIMEOUT: return "GQE_ERR_DEVICE_TIMEOUT";
        case GQE_ERR_SCRATCH_LIMIT: return "GQE_ERR_SCRATCH_LIMIT";
    }
    return "GQE_UNKNOWN_STATUS";
}

}  // extern "C"
