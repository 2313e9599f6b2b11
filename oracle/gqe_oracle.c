/*
 * gqe_oracle.c -- CPU oracle for the forward pass of a Grouped Query Experts
 * (GQE) attention layer.  TEST INFRASTRUCTURE ONLY: the tests, the smoke check
 * and the CPU-baseline leg of the benchmark are the only callers.  Nothing in
 * the product library links or loads this file, and this file uses nothing from
 * the product library.
 *
 * Plain, slow and direct: every floating-point sum is accumulated in double,
 * one element at a time, in index order.  Inputs are fp32 or bf16 (bf16 is
 * widened exactly to float, then to double).
 *
 * What it computes, with its sources:
 *  - Router.  "Grouped Query Experts: Mixture-of-Experts on GQA
 *    Self-Attention" (gist.science summary, section "Architecture et
 *    Routage"): for each token a router picks a sparse subset of k query-head
 *    experts in every GQA group, and the K/V path stays dense.  The page gives
 *    no router formula; the reading used here is a linear router
 *    l = x . W_r (+ an optional per-head bias), its logits rounded to fp32,
 *    top-k per group on those fp32 logits with equal logits going to the
 *    lower head index.
 *  - Gates.  Same page, "Somme Ponderee Renormalisee": the router
 *    probabilities are renormalised over the selected experts:
 *    gate_j = exp(l_j - m) / sum_{i in S} exp(l_i - m), m = max_{i in S} l_i.
 *  - Head -> group mapping.  "Grouped-Query Attention" (freenetmedia.pl),
 *    section "Jak dzialaja...": with 8 query heads and 2 groups the first 4
 *    heads share KV head 0 and the next 4 share KV head 1, i.e. head j uses
 *    KV head j / (h/g).  The ml-canon page "56 GQA / MQA", section "PyTorch
 *    GQA", expands KV heads the same way (repeat each KV head h/g times).
 *  - Attention.  IBM "Que es la atencion de consultas agrupadas": scores are
 *    q . k scaled by 1/sqrt(d_k), normalised by a softmax, and used to weight
 *    the value vectors.  Causal: key s is visible to query t iff s <= t (the
 *    pages' autoregressive setting; the positions are the original ones).
 *  - Output.  Each selected head's attention output is multiplied by its gate
 *    and written to that head's slot; every unselected head's slot is zero.
 *  - Decode.  One new query per sequence at position L_b - 1 against a cache
 *    holding keys 0 .. L_b - 1 of that sequence (the KV cache of the GQA
 *    pages, which stays dense under GQE).
 *  - Output construction (same GQE page, "Construction de la Sortie"): per
 *    group, the outputs of the k selected experts are concatenated (here in
 *    selection order, ungated), a weighted sum of those outputs with the
 *    renormalised router probabilities forms one more slot, and one extra
 *    attention head is computed for every token whatever the routing (the
 *    shared head).  The page names no KV head for the shared head; the reading
 *    used here: its own query rows attend, causally, to one KV group chosen by
 *    the caller.
 *  - Paged decode.  The same decode with the cache kept in fixed-size pages:
 *    logical row s of sequence b lives in page block_table[b][s / page_size]
 *    at row s % page_size (the KV cache stays dense under GQE; only where its
 *    rows sit in memory changes).
 *  - Routed query projection (same page, "Activation Conditionnelle": the
 *    query-side computation is conditional on the routing): the query row of
 *    head j is x . W_Q[:, j*d_h : (j+1)*d_h], computed only for the heads a
 *    token selected.
 *  - Output projection (IBM GQA page: the heads' outputs, concatenated, pass
 *    through one more linear layer with weight matrix W_Z; GQE page,
 *    "Activation Conditionnelle": only the selected experts are computed): the
 *    layer output of a token is the sum, over the heads it selected, of the
 *    head's (gated) output row times that head's d_h-row block of W_Z.
 *  - Backward (training; the pages state no formula for it): the gradients of
 *    the routed attention, of the gates and of the router's logits, x, W_r and
 *    bias, by the chain rule through the steps above in reverse order.
 *  - Load-balancing auxiliary loss (same page, "Entrainement et Perte": it
 *    makes the router spread tokens evenly over each group's experts; no
 *    formula given): the fraction-times-probability form, per group.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

static double load_elem(const void* p, size_t i, int dtype) {
    if (dtype == ORACLE_F32) return (double)((const float*)p)[i];
    uint32_t bits = ((uint32_t)((const uint16_t*)p)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------ */
/* Router: logits, per-group top-k with ties to the lower head index, gates. */
/* ------------------------------------------------------------------------ */

/*
 * x      [B*T, d_model]  (dtype)
 * W_r    [d_model, h]    (dtype)
 * bias   [h] float or NULL
 * logits [B*T, h]   out: fp32-rounded logits
 * idx    [B*T, g, k] out: selected global head indices, ordered by
 *                         (logit descending, head index ascending)
 * gate   [B*T, g, k] out: renormalised gates (double)
 * margin [B*T, g]    out: l_(k) - l_(k+1) within the group, +inf when k == h/g
 */
int oracle_route(int64_t BT, int d_model, int h, int g, int k, int dtype,
                 const void* x, const void* W_r, const float* bias,
                 float* logits, int32_t* idx, double* gate, double* margin) {
    if (BT < 0 || d_model < 1 || h < 1 || g < 1 || h % g != 0) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    int err = 0;
#pragma omp parallel
    {
        int* order = (int*)malloc(sizeof(int) * (size_t)hpg);
        if (!order) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(static)
            for (int64_t r = 0; r < BT; ++r) {
                for (int j = 0; j < h; ++j) {
                    double acc = 0.0;
                    for (int i = 0; i < d_model; ++i)
                        acc += load_elem(x, (size_t)r * d_model + i, dtype) *
                               load_elem(W_r, (size_t)i * h + j, dtype);
                    if (bias) acc += (double)bias[j];
                    logits[(size_t)r * h + j] = (float)acc;
                }
                for (int q = 0; q < g; ++q) {
                    const float* lg = logits + (size_t)r * h + (size_t)q * hpg;
                    /* insertion sort of the group's heads by (logit desc, index asc) */
                    for (int a = 0; a < hpg; ++a) {
                        int pos = a;
                        while (pos > 0) {
                            int prev = order[pos - 1];
                            if (lg[prev] < lg[a]) {
                                order[pos] = prev;
                                --pos;
                            } else {
                                break;
                            }
                        }
                        order[pos] = a;
                    }
                    const double m = (double)lg[order[0]];
                    double denom = 0.0;
                    for (int s = 0; s < k; ++s) denom += exp((double)lg[order[s]] - m);
                    for (int s = 0; s < k; ++s) {
                        size_t o = ((size_t)r * g + q) * k + s;
                        idx[o] = q * hpg + order[s];
                        gate[o] = exp((double)lg[order[s]] - m) / denom;
                    }
                    margin[(size_t)r * g + q] =
                        (k == hpg) ? INFINITY : (double)lg[order[k - 1]] - (double)lg[order[k]];
                }
            }
        }
        free(order);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Compaction: per (batch, head) the ascending list of routed positions.     */
/* ------------------------------------------------------------------------ */

/*
 * idx          [B, T, g, k]
 * head_offsets [B*h + 1] out: start of the list of (b, j) in head_pos
 * head_pos     [B*T*g*k] out: positions t, ascending within each list
 */
int oracle_compact(int B, int T, int h, int g, int k, const int32_t* idx,
                   int32_t* head_offsets, int32_t* head_pos) {
    if (B < 0 || T < 0 || h < 1 || g < 1 || h % g != 0) return 1;
    const int hpg = h / g;
    int64_t n = 0;
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j < h; ++j) {
            const int q = j / hpg;
            head_offsets[(size_t)b * h + j] = (int32_t)n;
            for (int t = 0; t < T; ++t) {
                const int32_t* sel = idx + (((size_t)b * T + t) * g + q) * k;
                int hit = 0;
                for (int s = 0; s < k; ++s) hit |= (sel[s] == j);
                if (hit) head_pos[n++] = t;
            }
        }
    }
    head_offsets[(size_t)B * h] = (int32_t)n;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Attention for one routed (b, t, j): causal scaled dot-product attention.  */
/* ------------------------------------------------------------------------ */

/* One query vector against keys 0..n_keys-1 taken with a row stride.  The
 * result o[d_h] is the softmax-weighted mean of the value rows. */
static void attend_one(const void* qv, size_t q_off, const void* K, const void* V,
                       size_t kv_base, size_t kv_row_stride, int64_t n_keys, int d_h,
                       int dtype, double* scores, double* o) {
    const double scale = 1.0 / sqrt((double)d_h);
    double mx = -INFINITY;
    for (int64_t s = 0; s < n_keys; ++s) {
        double dot = 0.0;
        const size_t kr = kv_base + (size_t)s * kv_row_stride;
        for (int d = 0; d < d_h; ++d)
            dot += load_elem(qv, q_off + d, dtype) * load_elem(K, kr + d, dtype);
        scores[s] = dot * scale;
        if (scores[s] > mx) mx = scores[s];
    }
    double denom = 0.0;
    for (int64_t s = 0; s < n_keys; ++s) {
        scores[s] = exp(scores[s] - mx);
        denom += scores[s];
    }
    for (int d = 0; d < d_h; ++d) o[d] = 0.0;
    for (int64_t s = 0; s < n_keys; ++s) {
        const size_t vr = kv_base + (size_t)s * kv_row_stride;
        const double w = scores[s] / denom;
        for (int d = 0; d < d_h; ++d) o[d] += w * load_elem(V, vr + d, dtype);
    }
}

/*
 * Full GQE output for a list of token rows.
 * Q [B, T, h, d_h], K/V [B, T, g, d_h] (dtype); idx/gate [B, T, g, k]
 * rows [n_rows]: flattened token index b*T + t
 * O_rows [n_rows, h, d_h] out (double): gate * attention for selected heads,
 *                                        0 for unselected heads
 */
int oracle_attn_rows(int B, int T, int h, int g, int d_h, int k, int dtype,
                     const void* Q, const void* K, const void* V,
                     const int32_t* idx, const double* gate,
                     int64_t n_rows, const int64_t* rows, double* O_rows, int n_threads) {
    if (B < 0 || T < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * T) return 1;
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)T);
        double* o = (double*)malloc(sizeof(double) * (size_t)d_h);
        if (!scores || !o) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n_rows; ++r) {
                const int64_t bt = rows[r];
                const int64_t b = bt / T, t = bt % T;
                double* out = O_rows + (size_t)r * h * d_h;
                for (int i = 0; i < h * d_h; ++i) out[i] = 0.0;
                for (int q = 0; q < g; ++q) {
                    for (int s = 0; s < k; ++s) {
                        const size_t sel = ((size_t)bt * g + q) * k + s;
                        const int j = idx[sel];
                        const size_t q_off = ((size_t)bt * h + j) * d_h;
                        const size_t kv_base = ((size_t)b * T * g + q) * d_h;
                        attend_one(Q, q_off, K, V, kv_base, (size_t)g * d_h, t + 1, d_h, dtype,
                                   scores, o);
                        for (int d = 0; d < d_h; ++d) out[(size_t)j * d_h + d] = gate[sel] * o[d];
                    }
                }
            }
        }
        free(scores);
        free(o);
    }
    return err;
}

/*
 * Decode: one query token per sequence.
 * query [B, h, d_h]; K_cache/V_cache [B, Lmax, g, d_h] (dtype); lengths [B]
 * idx/gate [B, g, k]; O [B, h, d_h] out (double).
 * The query sits at position lengths[b] - 1 and sees cache rows 0 .. lengths[b]-1.
 */
int oracle_decode(int B, int Lmax, int h, int g, int d_h, int k, int dtype,
                  const void* query, const void* K_cache, const void* V_cache,
                  const int32_t* lengths, const int32_t* idx, const double* gate,
                  double* O, int n_threads) {
    if (B < 0 || Lmax < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    for (int b = 0; b < B; ++b)
        if (lengths[b] < 1 || lengths[b] > Lmax) return 1;
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)Lmax);
        double* o = (double*)malloc(sizeof(double) * (size_t)d_h);
        if (!scores || !o) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1) collapse(2)
            for (int b = 0; b < B; ++b) {
                for (int q = 0; q < g; ++q) {
                    for (int jj = 0; jj < hpg; ++jj)
                        for (int d = 0; d < d_h; ++d)
                            O[((size_t)b * h + q * hpg + jj) * d_h + d] = 0.0;
                    for (int s = 0; s < k; ++s) {
                        const size_t sel = ((size_t)b * g + q) * k + s;
                        const int j = idx[sel];
                        const size_t q_off = ((size_t)b * h + j) * d_h;
                        const size_t kv_base = ((size_t)b * Lmax * g + q) * d_h;
                        attend_one(query, q_off, K_cache, V_cache, kv_base, (size_t)g * d_h,
                                   lengths[b], d_h, dtype, scores, o);
                        for (int d = 0; d < d_h; ++d)
                            O[((size_t)b * h + j) * d_h + d] = gate[sel] * o[d];
                    }
                }
            }
        }
        free(scores);
        free(o);
    }
    return err;
}

/*
 * Shared head: one query head computed for every token, attending causally to
 * KV group kv_group.
 * Qs [B, T, d_h], K/V [B, T, g, d_h] (dtype); rows [n_rows]: b*T + t
 * Os_rows [n_rows, d_h] out (double)
 */
int oracle_shared_rows(int B, int T, int g, int d_h, int dtype, int kv_group,
                       const void* Qs, const void* K, const void* V,
                       int64_t n_rows, const int64_t* rows, double* Os_rows, int n_threads) {
    if (B < 0 || T < 1 || g < 1 || d_h < 1 || kv_group < 0 || kv_group >= g) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * T) return 1;
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)T);
        if (!scores) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n_rows; ++r) {
                const int64_t bt = rows[r];
                const int64_t b = bt / T, t = bt % T;
                const size_t kv_base = ((size_t)b * T * g + kv_group) * d_h;
                attend_one(Qs, (size_t)bt * d_h, K, V, kv_base, (size_t)g * d_h, t + 1, d_h, dtype,
                           scores, Os_rows + (size_t)r * d_h);
            }
        }
        free(scores);
    }
    return err;
}

/*
 * Group slots of the layer output for a list of token rows.
 * Q [B, T, h, d_h], K/V [B, T, g, d_h] (dtype); idx/gate [B, T, g, k]
 * cat_rows  [n_rows, g, k, d_h] out (double): the attention output of the
 *           selected head idx[b,t,q,r] in slot (q, r), not gated
 * wsum_rows [n_rows, g, d_h] out (double): sum_r gate[b,t,q,r] * cat(q, r)
 */
int oracle_group_slots_rows(int B, int T, int h, int g, int d_h, int k, int dtype,
                            const void* Q, const void* K, const void* V,
                            const int32_t* idx, const double* gate,
                            int64_t n_rows, const int64_t* rows, double* cat_rows,
                            double* wsum_rows, int n_threads) {
    if (B < 0 || T < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * T) return 1;
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)T);
        if (!scores) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t r = 0; r < n_rows; ++r) {
                const int64_t bt = rows[r];
                const int64_t b = bt / T, t = bt % T;
                for (int q = 0; q < g; ++q) {
                    double* ws = wsum_rows + ((size_t)r * g + q) * d_h;
                    for (int d = 0; d < d_h; ++d) ws[d] = 0.0;
                    for (int s = 0; s < k; ++s) {
                        const size_t sel = ((size_t)bt * g + q) * k + s;
                        const int j = idx[sel];
                        double* slot = cat_rows + (((size_t)r * g + q) * k + s) * d_h;
                        const size_t kv_base = ((size_t)b * T * g + q) * d_h;
                        attend_one(Q, ((size_t)bt * h + j) * d_h, K, V, kv_base, (size_t)g * d_h, t + 1,
                                   d_h, dtype, scores, slot);
                        for (int d = 0; d < d_h; ++d) ws[d] += gate[sel] * slot[d];
                    }
                }
            }
        }
        free(scores);
    }
    return err;
}

/*
 * Routed query projection for a list of token rows.
 * x [B, T, d_model], W_Q [d_model, h*d_h] (dtype); idx [B, T, g, k]
 * Qsel_rows [n_rows, g, k, d_h] out (double): for each selected head
 *           j = idx[b,t,q,r], sum_i x[b,t,i] * W_Q[i, j*d_h + c]
 */
int oracle_qproj_rows(int B, int T, int d_model, int h, int g, int d_h, int k, int dtype,
                      const void* x, const void* W_Q, const int32_t* idx,
                      int64_t n_rows, const int64_t* rows, double* Qsel_rows, int n_threads) {
    if (B < 0 || T < 1 || d_model < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    if (k < 1 || k > h / g) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * T) return 1;
    const size_t ldw = (size_t)h * d_h;
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t bt = rows[r];
        for (int q = 0; q < g; ++q) {
            for (int s = 0; s < k; ++s) {
                const int j = idx[((size_t)bt * g + q) * k + s];
                double* out = Qsel_rows + (((size_t)r * g + q) * k + s) * d_h;
                for (int c = 0; c < d_h; ++c) {
                    double acc = 0.0;
                    for (int i = 0; i < d_model; ++i)
                        acc += load_elem(x, (size_t)bt * d_model + i, dtype) *
                               load_elem(W_Q, (size_t)i * ldw + (size_t)j * d_h + c, dtype);
                    out[c] = acc;
                }
            }
        }
    }
    return 0;
}

/*
 * Routed output projection for a list of token rows.
 * O [B, T, h, d_h] (dtype): the gated routed output; W_Z [h*d_h, d_model]
 * (dtype), head j's block is rows j*d_h .. j*d_h + d_h - 1; idx [B, T, g, k].
 * Y_rows [n_rows, d_model] out (double):
 *   Y[bt, n] = sum_q sum_r sum_c O[bt, j, c] * W_Z[j*d_h + c, n],  j = idx[bt, q, r],
 * the selected heads only (an unselected head's slot does not enter).
 */
int oracle_oproj_rows(int B, int T, int d_model, int h, int g, int d_h, int k, int dtype,
                      const void* O, const void* W_Z, const int32_t* idx,
                      int64_t n_rows, const int64_t* rows, double* Y_rows, int n_threads) {
    if (B < 0 || T < 1 || d_model < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    if (k < 1 || k > h / g) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= (int64_t)B * T) return 1;
    for (int64_t r = 0; r < n_rows; ++r)
        for (int e = 0; e < g * k; ++e) {
            const int j = idx[(size_t)rows[r] * g * k + e];
            if (j < 0 || j >= h) return 1;
        }
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads > 0 ? n_threads : 1)
    for (int64_t r = 0; r < n_rows; ++r) {
        const int64_t bt = rows[r];
        double* out = Y_rows + (size_t)r * d_model;
        for (int n = 0; n < d_model; ++n) {
            double acc = 0.0;
            for (int q = 0; q < g; ++q)
                for (int s = 0; s < k; ++s) {
                    const int jh = idx[((size_t)bt * g + q) * k + s];
                    for (int c = 0; c < d_h; ++c)
                        acc += load_elem(O, ((size_t)bt * h + jh) * d_h + c, dtype) *
                               load_elem(W_Z, ((size_t)jh * d_h + c) * d_model + n, dtype);
                }
            out[n] = acc;
        }
    }
    return 0;
}

/*
 * Paged decode: as oracle_decode, with the caches as pages.
 * K_pages/V_pages [num_pages, page_size, g, d_h] (dtype); block_table
 * [B, max_blocks]: page of logical rows [i*page_size, (i+1)*page_size) of
 * sequence b at [b*max_blocks + i]; lengths[b] <= page_size * max_blocks.
 * query [B, h, d_h]; idx/gate [B, g, k]; O [B, h, d_h] out (double).
 */
int oracle_decode_paged(int B, int page_size, int max_blocks, int num_pages, int h, int g, int d_h, int k,
                        int dtype, const void* query, const void* K_pages, const void* V_pages,
                        const int32_t* block_table, const int32_t* lengths, const int32_t* idx,
                        const double* gate, double* O, int n_threads) {
    if (B < 0 || page_size < 1 || max_blocks < 1 || num_pages < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1)
        return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    const int64_t cap = (int64_t)page_size * max_blocks;
    for (int b = 0; b < B; ++b) {
        if (lengths[b] < 1 || lengths[b] > cap) return 1;
        for (int i = 0; i < (lengths[b] + page_size - 1) / page_size; ++i)
            if (block_table[(size_t)b * max_blocks + i] < 0 || block_table[(size_t)b * max_blocks + i] >= num_pages)
                return 1;
    }
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* scores = (double*)malloc(sizeof(double) * (size_t)cap);
        if (!scores) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1) collapse(2)
            for (int b = 0; b < B; ++b) {
                for (int q = 0; q < g; ++q) {
                    for (int jj = 0; jj < hpg; ++jj)
                        for (int d = 0; d < d_h; ++d) O[((size_t)b * h + q * hpg + jj) * d_h + d] = 0.0;
                    const int L = lengths[b];
                    const double scale = 1.0 / sqrt((double)d_h);
                    for (int r = 0; r < k; ++r) {
                        const size_t sel = ((size_t)b * g + q) * k + r;
                        const int j = idx[sel];
                        const size_t q_off = ((size_t)b * h + j) * d_h;
                        /* scores over the logical rows, each read through the block table */
                        double mx = -INFINITY;
                        for (int s = 0; s < L; ++s) {
                            const size_t pg = (size_t)block_table[(size_t)b * max_blocks + s / page_size];
                            const size_t row = ((pg * page_size + (size_t)(s % page_size)) * g + q) * d_h;
                            double dot = 0.0;
                            for (int d = 0; d < d_h; ++d)
                                dot += load_elem(query, q_off + d, dtype) * load_elem(K_pages, row + d, dtype);
                            scores[s] = dot * scale;
                            if (scores[s] > mx) mx = scores[s];
                        }
                        double denom = 0.0;
                        for (int s = 0; s < L; ++s) {
                            scores[s] = exp(scores[s] - mx);
                            denom += scores[s];
                        }
                        double* out = O + ((size_t)b * h + j) * d_h;
                        for (int s = 0; s < L; ++s) {
                            const size_t pg = (size_t)block_table[(size_t)b * max_blocks + s / page_size];
                            const size_t row = ((pg * page_size + (size_t)(s % page_size)) * g + q) * d_h;
                            const double w = gate[sel] * scores[s] / denom;
                            for (int d = 0; d < d_h; ++d) out[d] += w * load_elem(V_pages, row + d, dtype);
                        }
                    }
                }
            }
        }
        free(scores);
    }
    return err;
}

/* ------------------------------------------------------------------------ */
/* Backward pass (training): the chain rule through the forward above.      */
/* ------------------------------------------------------------------------ */

/*
 * Gradients of a loss whose gradient with respect to the layer output O is dO,
 * taken term by term through the forward's own steps for one routed (b, t, j)
 * with gate gm, softmax weights p_s over keys s <= t and attention output o:
 *   O = gm * o                 ->  dgm = dO . o,   do = gm * dO
 *   o = sum_s p_s v_s          ->  dV[b,s,q] += p_s * do,   dp_s = do . v_s
 *   p = softmax(z),  z_s = q . k_s / sqrt(d_h)
 *                              ->  dz_s = p_s * (dp_s - sum_r p_r dp_r)
 *                              ->  dQ[b,t,j] = sum_s dz_s k_s / sqrt(d_h)
 *                                  dK[b,s,q] += dz_s q / sqrt(d_h)
 * An unselected slot of O is the constant 0, so it passes no gradient.
 *
 * Q [B,T,h,d_h], K/V [B,T,g,d_h] (dtype); idx/gate [B,T,g,k]; dO [B,T,h,d_h]
 * Out, double: dQ [B,T,h,d_h] (0 in unselected slots), dK/dV [B,T,g,d_h],
 *              dgate [B,T,g,k].
 * t_min: only query rows t >= t_min contribute (0: all).  Key rows s >= t_min
 * of dK/dV and query rows t >= t_min of dQ/dgate are then the full result's,
 * since no earlier query row sees a later key; earlier key rows hold only the
 * later query rows' share, and earlier rows of dQ/dgate are 0.
 */
int oracle_attn_backward(int B, int T, int h, int g, int d_h, int k, int dtype, int t_min,
                         const void* Q, const void* K, const void* V,
                         const int32_t* idx, const double* gate, const double* dO,
                         double* dQ, double* dK, double* dV, double* dgate, int n_threads) {
    if (B < 0 || T < 1 || h < 1 || g < 1 || h % g != 0 || d_h < 1) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg || t_min < 0) return 1;
    const double scale = 1.0 / sqrt((double)d_h);
    const size_t kv_stride = (size_t)g * d_h;
    int err = 0;
#pragma omp parallel num_threads(n_threads > 0 ? n_threads : 1)
    {
        double* p = (double*)malloc(sizeof(double) * (size_t)T);
        double* dp = (double*)malloc(sizeof(double) * (size_t)T);
        double* o = (double*)malloc(sizeof(double) * (size_t)d_h);
        double* dov = (double*)malloc(sizeof(double) * (size_t)d_h);
        if (!p || !dp || !o || !dov) {
#pragma omp atomic write
            err = 2;
        } else {
            /* one (b, group) per iteration: it alone writes dK/dV of that group */
#pragma omp for schedule(dynamic, 1) collapse(2)
            for (int b = 0; b < B; ++b) {
                for (int q = 0; q < g; ++q) {
                    const size_t kv_base = ((size_t)b * T * g + q) * d_h;
                    for (int t = 0; t < T; ++t) {
                        for (int d = 0; d < d_h; ++d) {
                            dK[kv_base + (size_t)t * kv_stride + d] = 0.0;
                            dV[kv_base + (size_t)t * kv_stride + d] = 0.0;
                        }
                        for (int jj = 0; jj < hpg; ++jj)
                            for (int d = 0; d < d_h; ++d)
                                dQ[(((size_t)b * T + t) * h + q * hpg + jj) * d_h + d] = 0.0;
                    }
                    for (int t = 0; t < T; ++t) {
                        for (int s_ = 0; s_ < k; ++s_) {
                            const size_t sel = (((size_t)b * T + t) * g + q) * k + s_;
                            if (t < t_min) {
                                dgate[sel] = 0.0;
                                continue;
                            }
                            const int j = idx[sel];
                            const size_t q_off = (((size_t)b * T + t) * h + j) * d_h;
                            /* forward: softmax weights and output */
                            double mx = -INFINITY;
                            for (int s = 0; s <= t; ++s) {
                                double dot = 0.0;
                                for (int d = 0; d < d_h; ++d)
                                    dot += load_elem(Q, q_off + d, dtype) *
                                           load_elem(K, kv_base + (size_t)s * kv_stride + d, dtype);
                                p[s] = dot * scale;
                                if (p[s] > mx) mx = p[s];
                            }
                            double denom = 0.0;
                            for (int s = 0; s <= t; ++s) {
                                p[s] = exp(p[s] - mx);
                                denom += p[s];
                            }
                            for (int s = 0; s <= t; ++s) p[s] /= denom;
                            for (int d = 0; d < d_h; ++d) o[d] = 0.0;
                            for (int s = 0; s <= t; ++s)
                                for (int d = 0; d < d_h; ++d)
                                    o[d] += p[s] * load_elem(V, kv_base + (size_t)s * kv_stride + d, dtype);
                            /* O = gate * o */
                            double dg = 0.0;
                            for (int d = 0; d < d_h; ++d) dg += dO[q_off + d] * o[d];
                            dgate[sel] = dg;
                            for (int d = 0; d < d_h; ++d) dov[d] = gate[sel] * dO[q_off + d];
                            /* o = sum_s p_s v_s */
                            double pdp = 0.0;
                            for (int s = 0; s <= t; ++s) {
                                const size_t kr = kv_base + (size_t)s * kv_stride;
                                double acc = 0.0;
                                for (int d = 0; d < d_h; ++d) {
                                    dV[kr + d] += p[s] * dov[d];
                                    acc += dov[d] * load_elem(V, kr + d, dtype);
                                }
                                dp[s] = acc;
                                pdp += p[s] * acc;
                            }
                            /* p = softmax(z), z = q . k / sqrt(d_h) */
                            for (int s = 0; s <= t; ++s) {
                                const size_t kr = kv_base + (size_t)s * kv_stride;
                                const double dz = p[s] * (dp[s] - pdp);
                                for (int d = 0; d < d_h; ++d) {
                                    dQ[q_off + d] += scale * dz * load_elem(K, kr + d, dtype);
                                    dK[kr + d] += scale * dz * load_elem(Q, q_off + d, dtype);
                                }
                            }
                        }
                    }
                }
            }
        }
        free(p);
        free(dp);
        free(o);
        free(dov);
    }
    return err;
}

/*
 * Router backward.  The gates are a softmax over the selected logits
 * (gate_j = exp(l_j) / sum_{i in S} exp(l_i)), so for j in S
 *   dl_j = gate_j * (dgate_j - sum_{i in S} gate_i dgate_i)
 * and dl_j = 0 for an unselected head (the top-k choice is piecewise constant
 * in the logits; the fp32 rounding of the logits is not differentiated).  Then
 * l = x . W_r + bias gives dx = dl . W_r^T, dW_r = x^T . dl, dbias = sum dl.
 *
 * x [BT, d_model], W_r [d_model, h] (dtype); idx/gate/dgate [BT, g, k]
 * Out, double: dlogits [BT, h]; dx [BT, d_model], dW [d_model, h] and
 * dbias [h] (each may be NULL to skip it).
 */
int oracle_route_backward(int64_t BT, int d_model, int h, int g, int k, int dtype,
                          const void* x, const void* W_r, const int32_t* idx,
                          const double* gate, const double* dgate, double* dlogits,
                          double* dx, double* dW, double* dbias, int n_threads) {
    if (BT < 0 || d_model < 1 || h < 1 || g < 1 || h % g != 0) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    for (int64_t i = 0; i < BT * g * k; ++i)
        if (idx[i] < 0 || idx[i] >= h || idx[i] / hpg != (int)((i / k) % g)) return 1;
    for (int64_t bt = 0; bt < BT; ++bt) {
        for (int j = 0; j < h; ++j) dlogits[bt * h + j] = 0.0;
        for (int q = 0; q < g; ++q) {
            const size_t base = ((size_t)bt * g + q) * k;
            double mean = 0.0;
            for (int s = 0; s < k; ++s) mean += gate[base + s] * dgate[base + s];
            for (int s = 0; s < k; ++s)
                dlogits[bt * h + idx[base + s]] = gate[base + s] * (dgate[base + s] - mean);
        }
    }
    if (dx) {
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(static)
        for (int64_t bt = 0; bt < BT; ++bt)
            for (int i = 0; i < d_model; ++i) {
                double acc = 0.0;
                for (int j = 0; j < h; ++j)
                    acc += dlogits[bt * h + j] * load_elem(W_r, (size_t)i * h + j, dtype);
                dx[bt * d_model + i] = acc;
            }
    }
    if (dW) {
#pragma omp parallel for num_threads(n_threads > 0 ? n_threads : 1) schedule(static)
        for (int i = 0; i < d_model; ++i)
            for (int j = 0; j < h; ++j) {
                double acc = 0.0;
                for (int64_t bt = 0; bt < BT; ++bt)
                    acc += load_elem(x, (size_t)bt * d_model + i, dtype) * dlogits[bt * h + j];
                dW[(size_t)i * h + j] = acc;
            }
    }
    if (dbias) {
        for (int j = 0; j < h; ++j) {
            double acc = 0.0;
            for (int64_t bt = 0; bt < BT; ++bt) acc += dlogits[bt * h + j];
            dbias[j] = acc;
        }
    }
    return 0;
}

/*
 * Load-balancing auxiliary loss.  The GQE page ("Entrainement et Perte") adds
 * an auxiliary loss that makes the router spread tokens evenly over the experts
 * of each group, and gives no formula.  Reading: the fraction-times-probability
 * form of mixture-of-experts routers, taken per group and averaged over groups.
 * With N tokens, hpg = h/g and p[t,j] the softmax of token t's logits over ALL
 * heads of j's group (not only the selected ones):
 *   f_j = #{t : j in S(t)} / (N k)          share of the group's selections
 *   P_j = sum_t p[t,j] / N                  mean router probability
 *   L   = (1/g) sum_q hpg sum_{j in q} f_j P_j      (= 1 when both are uniform)
 * f is a count and passes no gradient, so
 *   dL/dl[t,j] = hpg/(g N) * p[t,j] * (f_j - sum_{i in q} p[t,i] f_i).
 *
 * logits [N, h] float (the router's fp32 logits, bias included); idx [N, g, k].
 * Out: *loss; dlogits [N, h] (double, may be NULL).
 */
int oracle_aux_loss(int64_t N, int h, int g, int k, const float* logits, const int32_t* idx,
                    double* loss, double* dlogits) {
    if (N < 1 || h < 1 || g < 1 || h % g != 0) return 1;
    const int hpg = h / g;
    if (k < 1 || k > hpg) return 1;
    double* f = (double*)calloc((size_t)h, sizeof(double));
    double* P = (double*)calloc((size_t)h, sizeof(double));
    double* p = (double*)malloc(sizeof(double) * (size_t)hpg);
    if (!f || !P || !p) {
        free(f);
        free(P);
        free(p);
        return 2;
    }
    for (int64_t t = 0; t < N; ++t)
        for (int q = 0; q < g; ++q)
            for (int s = 0; s < k; ++s) {
                const int j = idx[((size_t)t * g + q) * k + s];
                if (j < q * hpg || j >= (q + 1) * hpg) {
                    free(f);
                    free(P);
                    free(p);
                    return 1;
                }
                f[j] += 1.0 / ((double)N * k);
            }
    /* mean probabilities */
    for (int64_t t = 0; t < N; ++t)
        for (int q = 0; q < g; ++q) {
            double m = -INFINITY, den = 0.0;
            for (int jj = 0; jj < hpg; ++jj) {
                const double l = (double)logits[(size_t)t * h + q * hpg + jj];
                if (l > m) m = l;
            }
            for (int jj = 0; jj < hpg; ++jj) {
                p[jj] = exp((double)logits[(size_t)t * h + q * hpg + jj] - m);
                den += p[jj];
            }
            for (int jj = 0; jj < hpg; ++jj) P[q * hpg + jj] += p[jj] / den / (double)N;
        }
    double L = 0.0;
    for (int q = 0; q < g; ++q) {
        double s = 0.0;
        for (int jj = 0; jj < hpg; ++jj) s += f[q * hpg + jj] * P[q * hpg + jj];
        L += (double)hpg * s / (double)g;
    }
    *loss = L;
    if (dlogits) {
        const double c = (double)hpg / ((double)g * (double)N);
        for (int64_t t = 0; t < N; ++t)
            for (int q = 0; q < g; ++q) {
                double m = -INFINITY, den = 0.0, pf = 0.0;
                for (int jj = 0; jj < hpg; ++jj) {
                    const double l = (double)logits[(size_t)t * h + q * hpg + jj];
                    if (l > m) m = l;
                }
                for (int jj = 0; jj < hpg; ++jj) {
                    p[jj] = exp((double)logits[(size_t)t * h + q * hpg + jj] - m);
                    den += p[jj];
                }
                for (int jj = 0; jj < hpg; ++jj) {
                    p[jj] /= den;
                    pf += p[jj] * f[q * hpg + jj];
                }
                for (int jj = 0; jj < hpg; ++jj)
                    dlogits[(size_t)t * h + q * hpg + jj] = c * p[jj] * (f[q * hpg + jj] - pf);
            }
    }
    free(f);
    free(P);
    free(p);
    return 0;
}
