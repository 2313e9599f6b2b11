/*
 * gqe.h -- C ABI of libgqe: the forward pass of a Grouped Query Experts (GQE)
 * attention layer on NVIDIA B200 (sm_100a).
 *
 * The method ("Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
 * gist.science summary, section "Architecture et Routage"): the KV heads of
 * grouped-query attention stay dense; inside each KV group a per-token router
 * picks k of the group's query heads ("experts"); those heads run causal
 * attention against the group's shared K/V; each selected head's output is
 * scaled by its router probability renormalised over the k selected heads
 * ("Somme Ponderee Renormalisee"); unselected heads output zero.
 *
 * Notation.  B batch, T sequence length, d_model router input width, h query
 * heads, g KV heads (groups), d_h head width, k heads selected per group,
 * hpg = h / g.  Query head j belongs to group j / hpg (contiguous blocks, as in
 * the 8-heads / 2-groups example of the freenetmedia.pl GQA page, section
 * "Jak dzialaja...").
 *
 * Conventions shared by every entry point:
 *  - Pointers named as device pointers must point to device memory of the
 *    current CUDA device; the caller owns every buffer (this library never
 *    allocates or frees memory, and never synchronises except in
 *    gqe_get_device_status).
 *  - Tensors are dense, row-major, last index fastest.  Activation tensors
 *    (x, W_r, Q, K, V, caches, O) must be 16-byte aligned.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Work is
 *    enqueued asynchronously; a call returns once its kernels are launched.
 *  - Arguments are validated on the host before anything is enqueued.  An
 *    invalid argument returns GQE_ERR_INVALID_ARGUMENT and enqueues nothing; a
 *    valid request outside the implemented cases returns GQE_ERR_UNSUPPORTED and
 *    enqueues nothing; a failed launch returns GQE_ERR_CUDA.
 *  - `workspace` is caller-owned device scratch of at least
 *    gqe_workspace_bytes() bytes, 256-byte aligned.  Its first 256 bytes hold a
 *    device status word: zero it once with gqe_workspace_init() after
 *    allocation.  A kernel whose bounded wait expires records
 *    GQE_ERR_DEVICE_TIMEOUT there and returns early; read it with
 *    gqe_get_device_status().  Calls that share a workspace must be ordered on
 *    one stream.
 *  - Outputs must not alias inputs.
 */
#ifndef GQE_H
#define GQE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    GQE_OK = 0,
    GQE_ERR_INVALID_ARGUMENT = 1,
    GQE_ERR_UNSUPPORTED = 2,
    GQE_ERR_CUDA = 3,
    GQE_ERR_DEVICE_TIMEOUT = 4,
    GQE_ERR_SCRATCH_LIMIT = 5
} gqe_status;

typedef enum { GQE_F32 = 0, GQE_BF16 = 1 } gqe_dtype;

typedef struct {
    int B, T, d_model, h, g, d_h, k;
    int dtype; /* gqe_dtype: element type of x, W_r, Q, K, V, caches and O */
} gqe_shape;

/* Number of 32-token chunks per sequence: ceil(T / 32).  Sizes the
 * head_chunk_offsets array of gqe_route. */
int gqe_chunk_count(int T);

/* Bytes of device workspace needed by the calls on shape *s.  Lmax is the
 * cache capacity for gqe_attn_decode (0 for prefill-only use).  Returns 0 for
 * an invalid shape. */
size_t gqe_workspace_bytes(const gqe_shape* s, int Lmax);

/* Zero the status word of a workspace (asynchronous, on `stream`). */
gqe_status gqe_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_route -- router, per-group top-k and token compaction.
 *
 * Router (gist.science GQE summary, "Architecture et Routage"; the linear form
 * is this library's reading, the page gives no formula):
 *   l[b,t,j] = sum_i x[b,t,i] * W_r[i,j] + bias[j], accumulated in fp32.
 * Per token and group q, the k heads of q with the largest fp32 logits are
 * selected; equal logits go to the lower head index.  gate = the softmax of
 * the selected logits (the group softmax renormalised over the selection,
 * "Somme Ponderee Renormalisee").
 * Compaction: for every (b, j), the ascending list of positions t whose
 * selection contains j, built by warp ballots and prefix sums.
 *
 *   x        [B, T, d_model]   device, dtype
 *   W_r      [d_model, h]      device, dtype
 *   bias     [h]               device fp32, or NULL for no bias
 *   idx      [B, T, g, k]      device int32 out: selected global head indices
 *                              per (token, group), by logit descending (ties:
 *                              lower index first)
 *   gate     [B, T, g, k]      device fp32 out: renormalised gates, same order
 *   head_offsets [B*h + 1]     device int32 out: head_pos index of the first
 *                              entry of (b, j) at [b*h + j]; [B*h] = B*T*g*k
 *   head_pos [B*T*g*k]         device int32 out: positions t, ascending within
 *                              each (b, j) list
 *   head_chunk_offsets [B*h*gqe_chunk_count(T)]
 *                              device int32 out: at [(b*h + j)*nchunk + c] the
 *                              head_pos index of the first entry of (b, j) with
 *                              t >= 32*c
 * Requires B >= 1, T >= 1, h % g == 0, 1 <= k <= h/g, B*T*g*k < 2^31 (any
 * other shape returns GQE_ERR_INVALID_ARGUMENT, for every entry point).
 */
gqe_status gqe_route(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                     int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                     int32_t* head_chunk_offsets, void* workspace, size_t workspace_bytes,
                     void* stream);

/*
 * gqe_route_static -- gqe_route without a workspace argument: it allocates
 * nothing and takes no scratch from the caller.  The paper has no counterpart
 * for this entry point; it exists for callers that cannot allocate device
 * memory, such as a serving runtime whose memory is planned up front and
 * handed out by its own arena, code that may not call cudaMalloc or an
 * allocating library (PyTorch's caching allocator included) at the point of
 * the call, or a host that only passes pointers it already owns.
 *
 * Inputs, outputs and results are exactly those of gqe_route.  The per-chunk
 * counts that gqe_route keeps in its workspace live instead in one 4 MiB
 * array of device memory owned by this library (every GPU that loads the
 * library holds its own copy until the process exits), so
 * B * h * gqe_chunk_count(T) must not exceed 1,048,576; larger shapes return
 * GQE_ERR_SCRATCH_LIMIT and enqueue nothing.
 * The first call on a device looks up that device's copy of the array
 * (cudaGetSymbolAddress, with the device current); make that first call before
 * any stream capture.  Every call shares the array and it keeps the last
 * call's contents (each call writes every count before reading it, so nothing
 * needs clearing): calls whose kernels may overlap on the GPU (different
 * streams, or concurrent host threads on one device) race on it and must be
 * serialised by the caller.
 * Device-side failures (a bounded wait in the router that expired, which
 * leaves idx, gate and the lists incomplete, or counts the compaction found
 * inconsistent, whose writes it skips) are recorded in a status word at the
 * head of the same array, not in a caller workspace: read them with
 * gqe_route_static_status.
 */
gqe_status gqe_route_static(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                            int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                            int32_t* head_chunk_offsets, void* stream);

/*
 * gqe_route_static_status -- the device status word of gqe_route_static on
 * the calling thread's current device (no counterpart in the paper; it goes
 * with gqe_route_static).  Synchronises `stream`, returns the first error that
 * any gqe_route_static call recorded since the last read (GQE_OK if none:
 * GQE_ERR_DEVICE_TIMEOUT for an expired wait, GQE_ERR_INVALID_ARGUMENT for
 * inconsistent counts) and clears it.  Allocates nothing; GQE_ERR_CUDA if the
 * copy or the synchronisation fails.
 */
gqe_status gqe_route_static_status(void* stream);

/*
 * gqe_attn_prefill -- routed causal attention with the gated scatter.
 *
 * For every routed (b, t, j), with q = Q[b,t,j,:] and group q_ = j / hpg:
 *   o = sum_{s <= t} softmax_s(q . K[b,s,q_,:] / sqrt(d_h)) V[b,s,q_,:]
 * (scaled dot-product attention, IBM GQA page; KV heads shared per group,
 * ml-canon "56 GQA / MQA", "PyTorch GQA"; causal on the original positions),
 * and O[b,t,j,:] = gate * o.  O[b,t,j,:] = 0 for every unselected (t, j).
 * O is written in full.
 *
 *   Q [B, T, h, d_h], K/V [B, T, g, d_h]   device, dtype
 *   idx, gate, head_offsets, head_pos, head_chunk_offsets
 *                                          device, exactly as written by gqe_route
 *   O [B, T, h, d_h]                       device, dtype, out
 * Implemented cases: bf16 with d_h = 128 (tensor cores); fp32 with
 * d_h in {32, 64, 128} (CUDA cores).
 */
gqe_status gqe_attn_prefill(const gqe_shape* s, const void* Q, const void* K, const void* V,
                            const int32_t* idx, const float* gate, const int32_t* head_offsets,
                            const int32_t* head_pos, const int32_t* head_chunk_offsets, void* O,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_attn_decode -- one new query token per sequence against a KV cache.
 *
 * The cache of sequence b holds rows 0 .. lengths[b]-1 (the new token's own
 * K/V included); the query sits at position lengths[b]-1 and sees all of them.
 * The KV cache stays dense under GQE (gist.science summary, "Chemin KV
 * Dense"), so every group's cache rows are read once and shared by the k
 * routed heads of that group.  Output as for prefill with T = 1.
 *
 *   s->T must be 1.  q [B, 1, h, d_h] device, dtype.
 *   K_cache, V_cache [B, Lmax, g, d_h]   device, dtype
 *   lengths [B]     device int32, each in [1, Lmax] (device-side contract: the
 *                   kernels clamp out-of-range lengths into [1, Lmax])
 *   idx, gate       [B, 1, g, k] as written by gqe_route for the new tokens
 *   O [B, 1, h, d_h] device, dtype, out
 * Implemented cases: bf16 or fp32, d_h in {32, 64, 128}, k <= 8.
 */
gqe_status gqe_attn_decode(const gqe_shape* s, const void* q, const void* K_cache,
                           const void* V_cache, int Lmax, const int32_t* lengths,
                           const int32_t* idx, const float* gate, void* O, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * gqe_routed_qproj -- query projection for the routed heads only.
 *
 * The routing makes the query side conditional while K/V stay dense
 * (gist.science summary, "Activation Conditionnelle", "Chemin KV Dense"), so
 * a head's query row is computed only for the tokens that selected it:
 *   Q[b,t,j,:] = sum_i x[b,t,i] * W_Q[i, j*d_h + c]      for every routed (b, t, j),
 * accumulated in fp32 on the tensor cores and rounded to bf16.  Rows of Q
 * whose head was not selected are not written (gqe_attn_prefill never reads
 * them).
 *
 *   x [B, T, d_model]                  device bf16
 *   W_Q [d_model, h * d_h]             device bf16 (head j's block: columns j*d_h ..)
 *   idx [B, T, g, k]                   device, 16-byte aligned, as written by gqe_route
 *   head_offsets, head_pos             device, exactly as written by gqe_route
 *   Q [B, T, h, d_h]                   device bf16, out (routed rows)
 *   workspace                          the status word; with gqe_workspace_bytes of
 *                                      room, also 8 bytes per 128-token tile for the
 *                                      dense path
 * Two paths, same result.  When the routed share g*k/h is at least 3/10 (and
 * h <= 64, and the workspace has the tile sets' room) a tiled GEMM over every
 * token computes the heads of each 128-token x 2-head tile that holds a routed
 * (t, j) and writes the routed rows only; otherwise a grouped GEMM runs over
 * each head's routed rows, gathered.
 * Implemented cases: bf16, d_h = 128, d_model % 8 == 0; others return
 * GQE_ERR_UNSUPPORTED.
 */
gqe_status gqe_routed_qproj(const gqe_shape* s, const void* x, const void* W_Q, const int32_t* idx,
                            const int32_t* head_offsets, const int32_t* head_pos, void* Q, void* workspace,
                            size_t workspace_bytes, void* stream);

/*
 * gqe_routed_oproj -- output projection over the routed heads.
 *
 * The heads' outputs pass through one more linear layer, the output weight
 * matrix W_Z (IBM GQA page, multi-head attention mechanics); under GQE only
 * the selected experts are computed (gist.science summary, "Activation
 * Conditionnelle"), so a token's output is the sum over the heads it selected:
 *   Y[b,t,n] = sum_{q, r} sum_c O[b,t,j,c] * W_Z[j*d_h + c, n],   j = idx[b,t,q,r],
 * accumulated in fp32 on the tensor cores in a fixed order (reproducible) and
 * rounded to bf16.
 *
 *   O [B, T, h, d_h]       device bf16: the gated routed output as
 *                          gqe_attn_prefill / gqe_attn_decode write it.  The
 *                          unselected slots must hold zeros: a head that some
 *                          token of a 128-token tile selected is multiplied in
 *                          for the whole tile.
 *   idx [B, T, g, k]       device, 16-byte aligned, as written by gqe_route (an
 *                          index outside [0, h) is reported in the status word
 *                          and ignored)
 *   W_Z [h * d_h, d_model] device bf16 (head j's block: rows j*d_h ..)
 *   Y [B, T, d_model]      device bf16, out
 *   workspace              the status word and 8 bytes per 128-token tile
 *                          (gqe_workspace_bytes covers it)
 * Implemented cases: bf16, d_h % 64 == 0, h <= 64, d_model % 32 == 0; others
 * return GQE_ERR_UNSUPPORTED.
 */
gqe_status gqe_routed_oproj(const gqe_shape* s, const void* O, const int32_t* idx, const void* W_Z, void* Y,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_attn_shared_head -- the always-active shared head of the GQE layer.
 *
 * One extra attention head computed for every token whatever the routing
 * (gist.science summary, "Construction de la Sortie", "Tete Partagee
 * Toujours Active").  The page does not say which KV head it attends to; this
 * library's reading: its own query rows attend causally to KV group kv_group
 * of the layer's dense K/V:
 *   Os[b,t,:] = sum_{s <= t} softmax_s(Qs[b,t,:] . K[b,s,kv_group,:] / sqrt(d_h)) V[b,s,kv_group,:]
 *
 *   s            the layer's shape (B, T, g, d_h, dtype are used; h and k
 *                only in the shape checks)
 *   Qs [B, T, d_h]                     device, dtype
 *   K/V [B, T, g, d_h]                 device, dtype (the routed prefill's K/V)
 *   kv_group     0 <= kv_group < g, else GQE_ERR_INVALID_ARGUMENT
 *   Os [B, T, d_h]                     device, dtype, out
 *   workspace    at least gqe_workspace_bytes(s, 0) bytes; the call writes
 *                identity routing tables of the one head into it, so calls
 *                sharing a workspace must be ordered on one stream
 * Implemented cases: as gqe_attn_prefill (bf16 with d_h = 128 on the tensor
 * cores, the same kernel as the routed heads; fp32 with d_h in {32, 64, 128}).
 */
gqe_status gqe_attn_shared_head(const gqe_shape* s, const void* Qs, const void* K, const void* V, int kv_group,
                                void* Os, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_group_slots -- the per-group output slots of the GQE layer.
 *
 * Per group, the outputs of the k selected experts are concatenated and a
 * weighted sum of them with the renormalised router probabilities forms one
 * more slot (gist.science summary, "Construction de la Sortie": "Concatenation
 * Forte", "Somme Ponderee Renormalisee").  Both are built from the gated
 * output of gqe_attn_prefill (or gqe_attn_decode with T = 1):
 *   O_cat[b,t,q,r,:] = O[b,t,idx[b,t,q,r],:] / gate[b,t,q,r]   (the expert's
 *                      ungated output, in selection order; 0 if the gate
 *                      underflowed to 0)
 *   O_wsum[b,t,q,:]  = sum_r O[b,t,idx[b,t,q,r],:] = sum_r gate * o
 * A selection outside its group (not produced by gqe_route) contributes 0.
 *
 *   O [B, T, h, d_h]                   device, dtype (gated routed output)
 *   idx, gate [B, T, g, k]             device, as written by gqe_route
 *   O_cat [B, T, g, k, d_h]            device, dtype, out, or NULL
 *   O_wsum [B, T, g, d_h]              device, dtype, out, or NULL
 * At least one output must be non-NULL; O, O_cat and O_wsum 16-byte aligned
 * (else GQE_ERR_INVALID_ARGUMENT).  d_h in {32, 64, 128}; bf16 or fp32.
 * In bf16, O_cat carries the rounding of O and of the division (relative
 * error about 2^-8).
 */
gqe_status gqe_group_slots(const gqe_shape* s, const void* O, const int32_t* idx, const float* gate, void* O_cat,
                           void* O_wsum, void* stream);

/*
 * gqe_attn_decode_paged -- gqe_attn_decode with the KV cache in pages.
 *
 * The cache stays dense under GQE (gist.science summary, "Chemin KV Dense");
 * only where its rows sit changes: logical row s of sequence b is row
 * s % page_size of page block_table[b * max_blocks + s / page_size].  The
 * result is exactly that of gqe_attn_decode on the gathered cache.
 *
 *   K_pages, V_pages [num_pages, page_size, g, d_h]   device, dtype
 *   page_size        a power of two, 1 .. 65536
 *   block_table [B, max_blocks]   device int32; entries for rows < lengths[b]
 *                    must name pages in [0, num_pages) (device-side contract: an
 *                    entry outside is reported as GQE_ERR_INVALID_ARGUMENT in
 *                    the status word and read as page 0)
 *   lengths [B]      device int32, each in [1, page_size * max_blocks]
 *   q, idx, gate, O  as for gqe_attn_decode
 *   workspace        at least gqe_workspace_bytes(s, page_size * max_blocks)
 * Implemented cases: as gqe_attn_decode.
 */
gqe_status gqe_attn_decode_paged(const gqe_shape* s, const void* q, const void* K_pages, const void* V_pages,
                                 int num_pages, int page_size, const int32_t* block_table, int max_blocks,
                                 const int32_t* lengths, const int32_t* idx, const float* gate, void* O,
                                 void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_attn_prefill_backward -- gradients of the routed attention and of the
 * gates, for training.
 *
 * The pages state no backward; this is the chain rule through
 * gqe_attn_prefill and the renormalised gates of gqe_route (gist.science
 * summary, "Architecture et Routage", "Somme Ponderee Renormalisee"; IBM "Que
 * es la atencion de consultas agrupadas" for the attention).  For a routed
 * (b,t,j) with gate gm, attention output o (O = gm * o), incoming gradient
 * dO, D = dO . O and p_s the attention weights over keys s <= t:
 *   dQ[b,t,j]    = sum_s p_s (gm dO . v_s - D) k_s / sqrt(d_h)
 *   dK[b,s,q]   += p_s (gm dO . v_s - D) q / sqrt(d_h),  dV[b,s,q] += p_s gm dO
 *   dlogits[b,t,j] = D_j - gm_j sum_{i in S(b,t,q)} D_i   (0 when j is not in S)
 * dlogits is the gradient with respect to the router logits through the
 * renormalised gates (the top-k choice itself has no gradient).
 *
 *   Q, K, V, idx, gate, head_offsets, head_pos, head_chunk_offsets
 *                        as passed to gqe_attn_prefill (device)
 *   dO [B,T,h,d_h]       device, dtype: gradient of the loss with respect to O
 *                        (o is recomputed in fp32, so the forward's output is
 *                        not an input)
 *   dQ [B,T,h,d_h]       device float32 out (0 in unselected slots)
 *   dK, dV [B,T,g,d_h]   device float32 out
 *   dlogits [B,T,h]      device float32 out
 *   workspace            at least gqe_backward_workspace_bytes(s) bytes,
 *                        256-byte aligned; its first 256 bytes are the status word
 * Implemented cases: bf16 or fp32, d_h in {32, 64, 128}, k <= 16, h <= 256,
 * B*h <= 65535; others return GQE_ERR_UNSUPPORTED.  All of Q, K, V, dO, dQ,
 * dK, dV must be 16-byte aligned.  An index outside its group, or a
 * position outside [0, T), is reported in the status word and skipped.
 */
/* Bytes of device workspace for gqe_attn_prefill_backward and
 * gqe_route_backward on shape *s (0 for an invalid shape). */
size_t gqe_backward_workspace_bytes(const gqe_shape* s);
gqe_status gqe_attn_prefill_backward(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                     const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                     const int32_t* head_pos, const int32_t* head_chunk_offsets, const void* dO,
                                     float* dQ, float* dK, float* dV, float* dlogits, void* workspace,
                                     size_t workspace_bytes, void* stream);

/*
 * gqe_route_backward -- gradients of the linear router from the logit
 * gradients (for training; the chain rule through the router of gqe_route,
 * l = x . W_r + bias, gist.science summary, "Architecture et Routage"):
 *   dx = dlogits . W_r^T,   dW_r = x^T . dlogits,   dbias = sum over tokens of dlogits
 *
 *   x [B*T, d_model], W_r [d_model, h]   device, dtype (as passed to gqe_route)
 *   dlogits [B*T, h]     device float32 (from gqe_attn_prefill_backward)
 *   dx [B*T, d_model]    device float32 out, 16-byte aligned
 *   dW_r [d_model, h]    device float32 out (summed over token ranges in a
 *                        fixed order: the result is reproducible)
 *   dbias [h]            device float32 out, or NULL to skip it
 *   workspace            at least gqe_backward_workspace_bytes(s) bytes
 * Implemented cases: bf16 or fp32, B*T <= 4194240; others return
 * GQE_ERR_UNSUPPORTED.
 */
gqe_status gqe_route_backward(const gqe_shape* s, const void* x, const void* W_r, const float* dlogits, float* dx,
                              float* dW_r, float* dbias, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_attn_prefill_train -- gqe_attn_prefill for training: besides the gated
 * output O it saves, for every routed row (b, t, j), what the backward needs
 * (the chain rule through the forward; the pages give no backward):
 *   O32 [B, T, h, 128]   device fp32 out: the ungated attention output o of the
 *                        row (O = gate * o), computed so that the rounding of
 *                        the bf16 softmax weights does not reach it (P.V also
 *                        runs over p - bf16(p)); unselected slots untouched
 *   lse [B, T, h]        device fp32 out: log2 of the row's softmax
 *                        denominator in units of the scaled scores, so that the
 *                        weight of key s is 2^(q.k_s log2(e)/sqrt(128) - lse);
 *                        unselected slots untouched
 *   O                    as for gqe_attn_prefill, or NULL to skip it
 * Other arguments as gqe_attn_prefill.  Implemented for bf16 with d_h = 128,
 * k <= 4 and h/g <= 32 (the tensor-core path); other shapes return
 * GQE_ERR_UNSUPPORTED.
 */
gqe_status gqe_attn_prefill_train(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                  const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                  const int32_t* head_pos, const int32_t* head_chunk_offsets, void* O, float* O32,
                                  float* lse, void* workspace, size_t workspace_bytes, void* stream);

/*
 * gqe_attn_prefill_backward_saved -- gqe_attn_prefill_backward from the
 * statistics gqe_attn_prefill_train saved (O32, lse, as written there) instead
 * of running the forward again.  Same results, arguments, workspace and
 * errors as gqe_attn_prefill_backward, plus O32 and lse (device, read only);
 * the same shape limits as gqe_attn_prefill_train.
 */
gqe_status gqe_attn_prefill_backward_saved(const gqe_shape* s, const void* Q, const void* K, const void* V,
                                           const int32_t* idx, const float* gate, const int32_t* head_offsets,
                                           const int32_t* head_pos, const int32_t* head_chunk_offsets,
                                           const void* dO, const float* O32, const float* lse, float* dQ, float* dK,
                                           float* dV, float* dlogits, void* workspace, size_t workspace_bytes,
                                           void* stream);

/*
 * gqe_route_train -- gqe_route that also writes the router's fp32 logits, for
 * training: the load-balancing loss (gqe_aux_loss) and the router's own
 * gradient path read them.  Arguments and results are those of gqe_route, plus
 *   logits [B*T, h]      device float32 out: x . W_r + bias, the values the
 *                        top-k selected on
 */
gqe_status gqe_route_train(const gqe_shape* s, const void* x, const void* W_r, const float* bias,
                           int32_t* idx, float* gate, int32_t* head_offsets, int32_t* head_pos,
                           int32_t* head_chunk_offsets, float* logits, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * gqe_aux_loss -- the router's load-balancing auxiliary loss and its gradient
 * with respect to the logits.  The GQE summary (gist.science, "Entrainement et
 * Perte") adds such a loss so that the router spreads the tokens evenly over
 * the experts of each group, without a formula; this library's reading is the
 * fraction-times-probability form of mixture-of-experts routers, per group,
 * averaged over groups.  With N = B*T tokens and p[t,j] the softmax of token
 * t's logits over ALL heads of j's group:
 *   f_j = #{t : j selected for t} / (N k),  P_j = mean_t p[t,j],
 *   loss = (1/g) sum_q (h/g) sum_{j in q} f_j P_j       (1 when balanced)
 *   dlogits[t,j] = (h/g)/(g N) * p[t,j] * (f_j - sum_{i in j's group} p[t,i] f_i)
 * (f is a count: no gradient flows through it).
 *
 *   logits [B*T, h]      device float32 (gqe_route_train)
 *   idx [B*T, g, k]      device int32 (the selection); a head outside its
 *                        group is reported in the status word and skipped
 *   loss [1]             device float32 out
 *   dlogits [B*T, h]     device float32 out, or NULL for the loss only
 *   workspace            at least gqe_aux_loss_workspace_bytes(s) bytes
 * The sums run in a fixed order: the result is reproducible.  h/g <= 64;
 * larger groups return GQE_ERR_UNSUPPORTED.
 */
size_t gqe_aux_loss_workspace_bytes(const gqe_shape* s);
gqe_status gqe_aux_loss(const gqe_shape* s, const float* logits, const int32_t* idx, float* loss, float* dlogits,
                        void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, read the workspace status word, reset it to zero and
 * return it (GQE_OK when no kernel reported a failure). */
gqe_status gqe_get_device_status(void* workspace, void* stream);

/* Static, human-readable name of a status code. */
const char* gqe_status_string(gqe_status s);

#ifdef __cplusplus
}
#endif

#endif /* GQE_H */
