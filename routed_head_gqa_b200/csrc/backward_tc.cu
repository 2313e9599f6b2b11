// backward_tc.cu -- backward of the routed attention on the sm_100a tensor
// cores (bf16 inputs, d_h = 128, fp32 gradients).
//
// The pages give no backward for GQE; this is the chain rule through the
// forward ("Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
// gist.science summary, "Architecture et Routage" and "Somme Ponderee
// Renormalisee"; IBM GQA page for the scaled dot-product attention).  For a
// routed row r = (b, t, j) of group q with gate g_r, weights p_rs over the keys
// s <= t, ungated output o_r and incoming gradient dO_r:
//   D_r   = g_r dO_r . o_r
//   dS_rs = p_rs (g_r dO_r . v_s - D_r)
//   dQ_r  = sum_s dS_rs k_s / sqrt(d),   dK_s = sum_r dS_rs q_r / sqrt(d),
//   dV_s  = sum_r p_rs g_r dO_r,         dlogit_j = D_j - g_j sum_{i in S} D_i.
//
// Launches (after the tensor-core prefill has written o_r in fp32 and the
// row's log2-sum-exp lse_r, so p_rs = 2^(s_rs c - lse_r)):
//  1. bwd_pack_kernel: one block per half-window tile of a group (the
//     prefill's row tiles): the tile's row table, its Q and dO rows packed
//     contiguously (so the tensor-core kernels load a tile with plain TMA
//     boxes), dO_r . o_r, the logit gradients of the tile's positions, and
//     zero dQ rows for the unselected heads.  The table folds the gate into
//     the row's statistics: lse2_r = lse_r - log2 g_r and dl2_r = dO_r . o_r,
//     so that g_r p_rs = 2^(s_rs c - lse2_r) and dS_rs = g_r p_rs (dP_rs - dl2_r)
//     with dP_rs = dO_r . v_s.
//  2. dq_tc_kernel: per 128-row tile of routed rows: S = Q K^T and
//     dP = dO V^T on the tensor cores, dS in registers, dQ += dS K
//     accumulated in TMEM.
//  3. dkdv_tc_kernel: per (b, group, 128-key tile): S^T = K Q^T and
//     dP^T = V dO^T over the group's routed row tiles at or after the keys,
//     then dV += (g p)^T dO and dK += dS^T Q accumulated in TMEM.
// In both tensor-core kernels the elementwise step runs in two phases, the
// exponentials (from S) and dS (from dP), each overlapping an MMA of the
// neighbouring phase, and only tiles that straddle the causal diagonal are
// masked.
// Every sum runs in a fixed order: the gradients are reproducible.
#include <climits>

#include "backward.cuh"
#include "exp2_fma.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"
#include "units.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kD = 128;
constexpr int kBM = 128;                   // rows (or keys) per tile
constexpr int kThreads = 384;              // 4 control warps + 8 elementwise warps
constexpr uint32_t kHalf = 128 * 64 * 2;   // [128][64] bf16 box, 16 KB
constexpr uint32_t kTile = 2 * kHalf;      // [128][128] bf16, 32 KB
constexpr uint32_t kWhereBwdTc = 9;
constexpr int kQT = 2;                     // half-window tiles per window

__device__ __forceinline__ bool aborted(const int32_t* flag) { return *((volatile const int32_t*)flag) != 0; }

// Two elementwise warps share each TMEM lane quarter, one per 64-column half
// [64hh, 64hh + 64) of a 128-column tile.  Each writes its bf16 pairs over the
// first 32 columns of its own half, so the MMA's TMEM operand for K step kk
// (16 elements = 8 columns) sits at column a_col(kk), and neither warp writes
// a column the other reads.
__device__ __forceinline__ uint32_t a_col(int kk) { return (uint32_t)((kk >> 2) * 64 + (kk & 3) * 8); }

// ------------------------------------------------------------------ row tables
// The routed rows of one half-window tile (b, group q, first position w0, W
// positions): the concatenation over the group's heads of each head's slice of
// its packed position list.  Built by one warp; rows past the tile's count
// (and rows whose position falls outside the tile) are padding (t = -1).
struct RowTable {
    int32_t t[kBM];
    int32_t j[kBM];
    float gate[kBM];
    float lse[kBM];
    int32_t qrow[kBM];  // row of Q / dO viewed as [B*T*h, 128]; padding rows name q_rows (zero fill)
};

__device__ void build_rows(const UnitGeom& u, int b, int q, int w0, const int32_t* head_offsets,
                           const int32_t* head_chunk_offsets, const int32_t* head_pos, const int32_t* idx,
                           const float* gate_in, const float* lse, int q_rows, RowTable& rt,
                           int32_t* cut_start, int32_t* cut_prefix, uint32_t* status) {
    const int lane = threadIdx.x & 31;
    const int32_t total = (int32_t)((int64_t)u.B * u.T * u.g * u.k);
    if (lane < u.hpg) {
        const int jh = q * u.hpg + lane;
        int32_t a0 = list_cut(u, head_offsets, head_chunk_offsets, b, jh, w0);
        int32_t a1 = list_cut(u, head_offsets, head_chunk_offsets, b, jh, w0 + u.W);
        if (a0 < 0 || a1 < a0 || a1 > total) {
            report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwdTc, 1);
            a0 = a1 = 0;
        }
        cut_start[lane] = a0;
        cut_prefix[lane + 1] = a1 - a0;
    }
    __syncwarp();
    if (lane == 0) {
        int acc = 0;
        cut_prefix[0] = 0;
        for (int jj = 0; jj < u.hpg; ++jj) {
            acc = min(acc + cut_prefix[jj + 1], kBM);
            cut_prefix[jj + 1] = acc;
        }
    }
    __syncwarp();
    const int nrows = cut_prefix[u.hpg];
    for (int r = lane; r < kBM; r += 32) {
        int tt = -1, jh = 0;
        float gv = 0.f, lv = 0.f;
        if (r < nrows) {
            int jj = 0;
            while (cut_prefix[jj + 1] <= r) ++jj;
            jh = q * u.hpg + jj;
            tt = head_pos[cut_start[jj] + (r - cut_prefix[jj])];
            if (tt < w0 || tt >= min(w0 + u.W, u.T)) {
                report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwdTc, 2);
                tt = -1;
            }
        }
        if (tt >= 0) {
            const int64_t sel = (((int64_t)b * u.T + tt) * u.g + q) * u.k;
            for (int s2 = 0; s2 < u.k; ++s2)
                if (idx[sel + s2] == jh) gv = gate_in[sel + s2];
            const int64_t row = ((int64_t)b * u.T + tt) * u.h + jh;
            lv = lse[row];
        }
        rt.t[r] = tt;
        rt.j[r] = jh;
        rt.gate[r] = gv;
        rt.lse[r] = lv;
        rt.qrow[r] = (tt >= 0) ? (int32_t)(((int64_t)b * u.T + tt) * u.h + jh) : q_rows;
    }
    __syncwarp();
}

// A packed tile's table, in the workspace and in shared memory: per row
// lse2 = lse - log2(gate) (+inf for padding and zero gates), dl2 = dO . o,
// the position t (-1: padding) and the head j.
struct TileTab {
    float lse2[kBM];
    float dl2[kBM];
    int32_t t[kBM];
    int32_t j[kBM];
};
static_assert(sizeof(TileTab) == 2048, "a tile table is 2 KB");

// One warp copies a packed tile's table from the workspace into shared memory.
__device__ __forceinline__ void load_tab(const TileTab* src_tab, TileTab& dst_tab) {
    const int lane = threadIdx.x & 31;
    const int4* src = reinterpret_cast<const int4*>(src_tab);
    int4* dst = reinterpret_cast<int4*>(&dst_tab);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[lane + 32 * i] = src[lane + 32 * i];
}

// ------------------------------------------------------------------ 1. packed tiles
// Block = tile id (b*g + q) * ntiles + ti: positions [ti*W, (ti+1)*W) of group
// q of sequence b.  Every head of the group selected at one of these positions
// has its row in this tile, so the logit gradients of the tile's positions
// (dlogit_j = D_j - g_j sum_i D_i over the selected heads i, 0 for the others)
// are complete here; the sum runs in head order.
constexpr int kPackThreads = 256;
__global__ void __launch_bounds__(kPackThreads)
bwd_pack_kernel(UnitGeom u, int ntiles, const int32_t* __restrict__ head_offsets,
                const int32_t* __restrict__ head_chunk_offsets, const int32_t* __restrict__ head_pos,
                const int32_t* __restrict__ idx, const float* __restrict__ gate, const float* __restrict__ lse,
                const float* __restrict__ o32, const __nv_bfloat16* __restrict__ Q,
                const __nv_bfloat16* __restrict__ dO, TileTab* __restrict__ tabs, __nv_bfloat16* __restrict__ Qc,
                __nv_bfloat16* __restrict__ dOc, float* __restrict__ dlogits, float* __restrict__ dQ,
                uint32_t* status) {
    __shared__ RowTable rt;
    __shared__ int32_t cut_start[32], cut_prefix[33];
    __shared__ float dot_s[kBM];
    __shared__ float dsum[kBM];
    __shared__ int16_t row_of[kBM * 32];  // (position - w0) * hpg + head in group -> row, -1: unselected
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t tile = blockIdx.x;
    const int ti = (int)(tile % ntiles);
    const int bq = (int)(tile / ntiles);
    const int b = bq / u.g, q = bq % u.g, hpg = u.hpg;
    const int w0 = ti * u.W;
    const int npos = max(0, min(u.W, u.T - w0));
    for (int i = tid; i < u.W * hpg; i += kPackThreads) row_of[i] = -1;
    for (int i = tid; i < npos * u.k; i += kPackThreads) {  // every selected head belongs to group q
        const int j = idx[(((int64_t)b * u.T + w0 + i / u.k) * u.g + q) * u.k + i % u.k];
        if (j < q * hpg || j >= (q + 1) * hpg) report_error(status, GQE_ERR_INVALID_ARGUMENT, kWhereBwdTc, 3);
    }
    if (warp == 0)
        build_rows(u, b, q, w0, head_offsets, head_chunk_offsets, head_pos, idx, gate, lse, -1, rt, cut_start,
                   cut_prefix, status);
    __syncthreads();
    // Q and dO rows, and dO . o: 16 lanes per 256-byte row, 16 rows per pass
    const int half = lane >> 4, c = lane & 15;
    for (int r = warp * 2 + half; r < kBM; r += 2 * (kPackThreads / 32)) {
        const int tt = rt.t[r];
        uint4 qv = make_uint4(0, 0, 0, 0), dv = qv;
        float acc = 0.f;
        if (tt >= 0) {
            const int64_t src = rt.qrow[r];
            qv = reinterpret_cast<const uint4*>(Q + src * kD)[c];
            dv = reinterpret_cast<const uint4*>(dO + src * kD)[c];
            const float4 o0 = reinterpret_cast<const float4*>(o32 + src * kD)[2 * c];
            const float4 o1 = reinterpret_cast<const float4*>(o32 + src * kD)[2 * c + 1];
            acc = __uint_as_float(dv.x << 16) * o0.x + __uint_as_float(dv.x & 0xffff0000u) * o0.y +
                  __uint_as_float(dv.y << 16) * o0.z + __uint_as_float(dv.y & 0xffff0000u) * o0.w +
                  __uint_as_float(dv.z << 16) * o1.x + __uint_as_float(dv.z & 0xffff0000u) * o1.y +
                  __uint_as_float(dv.w << 16) * o1.z + __uint_as_float(dv.w & 0xffff0000u) * o1.w;
        }
#pragma unroll
        for (int d = 8; d > 0; d >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, d);  // within the half-warp
        reinterpret_cast<uint4*>(Qc + (tile * kBM + r) * kD)[c] = qv;
        reinterpret_cast<uint4*>(dOc + (tile * kBM + r) * kD)[c] = dv;
        if (c == 0) {
            dot_s[r] = acc;
            if (tt >= 0) row_of[(tt - w0) * hpg + (rt.j[r] - q * hpg)] = (int16_t)r;
        }
    }
    __syncthreads();
    // per position: sum of D = g (dO . o) over its selected heads, in head order
    if (tid < npos) {
        float sum = 0.f;
        for (int jj = 0; jj < hpg; ++jj) {
            const int r = row_of[tid * hpg + jj];
            if (r >= 0) sum += rt.gate[r] * dot_s[r];
        }
        dsum[tid] = sum;
    }
    // the table
    if (tid < kBM) {
        const int tt = rt.t[tid];
        const float gm = rt.gate[tid];
        TileTab& tab = tabs[tile];
        tab.lse2[tid] = (tt >= 0 && gm > 0.f) ? rt.lse[tid] - log2f(gm) : __int_as_float(0x7f800000);
        tab.dl2[tid] = (tt >= 0) ? dot_s[tid] : 0.f;
        tab.t[tid] = tt;
        tab.j[tid] = rt.j[tid];
    }
    __syncthreads();
    for (int i = tid; i < npos * hpg; i += kPackThreads) {
        const int pp = i / hpg, jj = i - pp * hpg;
        const int r = row_of[i];
        float dl = 0.f;
        if (r >= 0) {
            const float gm = rt.gate[r];
            dl = gm * dot_s[r] - gm * dsum[pp];
        }
        dlogits[((int64_t)b * u.T + w0 + pp) * u.h + q * hpg + jj] = dl;
    }
    // dQ of an unselected head is 0: one warp per (position, head)
    for (int i = warp; i < npos * hpg; i += kPackThreads / 32) {
        if (row_of[i] >= 0) continue;
        const int pp = i / hpg, jj = i - pp * hpg;
        float4* dst = reinterpret_cast<float4*>(dQ + (((int64_t)b * u.T + w0 + pp) * u.h + q * hpg + jj) * kD);
        dst[lane] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// ------------------------------------------------------------------ shared pieces
struct Params {
    UnitGeom u;
    const int32_t* idx;
    const float* gate;
    const int32_t* head_offsets;
    const int32_t* head_pos;
    const int32_t* head_chunk_offsets;
    const TileTab* tabs;   // packed tile tables
    int ntiles;            // half-window tiles per (b, group): 2 * ceil(T / 2W)
    float* dQ;
    float* dK;
    float* dV;
    uint32_t* status;
    float scale_log2;  // log2(e) / sqrt(128)
    float scale;       // 1 / sqrt(128)
    int q_rows;        // B*T*h
};

__device__ __forceinline__ void fail(int32_t* abort_flag, uint32_t* status, uint32_t detail) {
    atomicExch(abort_flag, 1);
    report_error(status, GQE_ERR_DEVICE_TIMEOUT, kWhereBwdTc, detail);
}

// Item of wave v for this CTA.  Items are numbered heaviest first; the waves
// alternate direction over the CTAs so that every CTA's share of the work
// comes out nearly even.
__device__ __forceinline__ int64_t snake_item(int64_t v) {
    const int64_t G = gridDim.x, c = blockIdx.x;
    return v * G + ((v & 1) ? (G - 1 - c) : c);
}

// Of every 16 pairs of exponentials in an unmasked chunk, this many run on
// the FMA pipe (exp2_poly2) and the rest on the MUFU unit (a same-box sweep:
// 0 and 2 tie, 1 % ahead of 4; 6 is 2 % behind).
constexpr int kPolyPairs = 2;

// The chunk's masked form (a tile on the causal diagonal) runs all on MUFU.
template <bool MASKED>
__device__ __forceinline__ void exp2_chunk(float (&x)[32]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) {
        if (!MASKED && e < kPolyPairs) {
            up2(exp2_poly2_clamped(x[2 * e], x[2 * e + 1]), x[2 * e], x[2 * e + 1]);
        } else {
            x[2 * e] = fast_exp2(x[2 * e]);
            x[2 * e + 1] = fast_exp2(x[2 * e + 1]);
        }
    }
}

// Exponent phase, thread = routed row: gp = 2^(s c - lse2) for 32 key columns
// starting at key kv0 (MASKED: keys after the row's position t give 0).
template <bool MASKED>
__device__ __forceinline__ void exp_row(const uint32_t (&s)[32], float c, float lse2, int t_row, int kv0,
                                        float (&gp)[32]) {
    const float kNegInf = -__int_as_float(0x7f800000);
#pragma unroll
    for (int e = 0; e < 32; ++e) {
        const float x = __uint_as_float(s[e]) * c - lse2;
        gp[e] = (MASKED && kv0 + e > t_row) ? kNegInf : x;
    }
    exp2_chunk<MASKED>(gp);
}

// Exponent phase, thread = key: gp = 2^(s c - lse2) for 32 row columns starting
// at column col0 of the table (MASKED: rows whose position t precedes the key,
// or padding rows, give 0).
template <bool MASKED>
__device__ __forceinline__ void exp_key(const uint32_t (&s)[32], float c, int key, const TileTab& tab, int col0,
                                        float (&gp)[32]) {
    const float kNegInf = -__int_as_float(0x7f800000);
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
        const float4 l = *reinterpret_cast<const float4*>(&tab.lse2[col0 + 4 * e4]);
        gp[4 * e4 + 0] = __uint_as_float(s[4 * e4 + 0]) * c - l.x;
        gp[4 * e4 + 1] = __uint_as_float(s[4 * e4 + 1]) * c - l.y;
        gp[4 * e4 + 2] = __uint_as_float(s[4 * e4 + 2]) * c - l.z;
        gp[4 * e4 + 3] = __uint_as_float(s[4 * e4 + 3]) * c - l.w;
        if (MASKED) {
            const int4 tv = *reinterpret_cast<const int4*>(&tab.t[col0 + 4 * e4]);
            if (key > tv.x) gp[4 * e4 + 0] = kNegInf;
            if (key > tv.y) gp[4 * e4 + 1] = kNegInf;
            if (key > tv.z) gp[4 * e4 + 2] = kNegInf;
            if (key > tv.w) gp[4 * e4 + 3] = kNegInf;
        }
    }
    exp2_chunk<MASKED>(gp);
}

__device__ __forceinline__ void pack_chunk(const float (&v)[32], uint32_t (&out)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e) out[e] = pack_bf16x2(v[2 * e], v[2 * e + 1]);
}

// dS phase: ds = gp (dp - dl2), as bf16 pairs; dl2 the thread's row's (thread =
// row) or per column from the table (thread = key, col0 >= 0).
__device__ __forceinline__ void ds_row(const float (&gp)[32], const uint32_t (&dp)[32], float dl2,
                                       uint32_t (&ds)[16]) {
#pragma unroll
    for (int e = 0; e < 16; ++e)
        ds[e] = pack_bf16x2(gp[2 * e] * (__uint_as_float(dp[2 * e]) - dl2),
                            gp[2 * e + 1] * (__uint_as_float(dp[2 * e + 1]) - dl2));
}
__device__ __forceinline__ void ds_key(const float (&gp)[32], const uint32_t (&dp)[32], const TileTab& tab, int col0,
                                       uint32_t (&ds)[16]) {
#pragma unroll
    for (int e4 = 0; e4 < 8; ++e4) {
        const float4 d = *reinterpret_cast<const float4*>(&tab.dl2[col0 + 4 * e4]);
        ds[2 * e4] = pack_bf16x2(gp[4 * e4] * (__uint_as_float(dp[4 * e4]) - d.x),
                                 gp[4 * e4 + 1] * (__uint_as_float(dp[4 * e4 + 1]) - d.y));
        ds[2 * e4 + 1] = pack_bf16x2(gp[4 * e4 + 2] * (__uint_as_float(dp[4 * e4 + 2]) - d.z),
                                     gp[4 * e4 + 3] * (__uint_as_float(dp[4 * e4 + 3]) - d.w));
    }
}

// ------------------------------------------------------------------ 2. dQ
// One CTA per SM; work item = one half-window tile of 128 routed rows.
// Roles: warp 0 K/V producer (3-stage K ring, 2-stage V ring), warp 1 MMA
// issuer, warp 2 Q/dO loads, warps 4-11 elementwise + epilogue (thread = row, two
// warps per row, one per 64-column half).  TMEM: S buffers [0,128) and
// [128,256), dP [256,384), dQ [384,512); dS (bf16 pairs) overwrites dP's
// columns a_col(0..7) once dP is in registers.  Per key tile the elementwise
// warps run the dS phase of tile i, then the exponent phase of tile i+1 (its
// S is already in TMEM) while the tensor core runs dQ(i) and dP(i+1).
// K has three stages: K(i) is read by S(i) early and by dQ(i) late, so with
// two the load of K(i+2) could only start after dQ(i) and S(i+2) waited for
// it.  The elementwise warps read their rows' table entries from the
// workspace (the shared memory is full).
constexpr int kDqKStages = 3;
struct DqSmem {
    uint8_t q[kTile];
    uint8_t dO[kTile];
    uint8_t k[kDqKStages][kTile];
    uint8_t v[2][kTile];
    uint64_t kv_full_k[kDqKStages], kv_full_v[2], kv_empty_k[kDqKStages], kv_empty_v[2];
    uint64_t rows_full, rows_empty, s_full[2], dp_full, ew_done, dq_full, dq_empty, drain;
    uint32_t tmem_base;
    int32_t abort_flag;
};

__device__ __forceinline__ int dq_items(const UnitGeom& u) { return (int)(u.count() * kQT); }
// Item i: heaviest windows first (unit order of the prefill), two halves per unit.
__device__ __forceinline__ void dq_item(const UnitGeom& u, int ntiles, int64_t i, int& b, int& q, int& w0, int& nkv,
                                        int64_t& tile) {
    int w;
    unit_coords(u, i / kQT, b, q, w);
    const int half = (int)(i % kQT);
    w0 = (w * kQT + half) * u.W;
    const int end = min(w0 + u.W, u.T);
    nkv = (end + kBM - 1) / kBM;
    tile = ((int64_t)b * u.g + q) * ntiles + (w * kQT + half);
}

__global__ void __launch_bounds__(kThreads, 1)
dq_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
             const __grid_constant__ CUtensorMap mapQc, const __grid_constant__ CUtensorMap mapdOc, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    DqSmem& sm = *smem_align1024<DqSmem>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const UnitGeom& u = p.u;
    const int64_t n_items = dq_items(u);
    if (tid == 0) {
        for (int i = 0; i < kDqKStages; ++i) {
            mbar_init(&sm.kv_full_k[i], 1);
            mbar_init(&sm.kv_empty_k[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.kv_full_v[i], 1);
            mbar_init(&sm.kv_empty_v[i], 1);
            mbar_init(&sm.s_full[i], 1);
        }
        mbar_init(&sm.rows_full, 1);
        // the MMA issuer's commit after the item's last dQ step (Q and dO read)
        mbar_init(&sm.rows_empty, 1);
        mbar_init(&sm.dp_full, 1);
        mbar_init(&sm.ew_done, 256);
        mbar_init(&sm.dq_full, 1);
        mbar_init(&sm.dq_empty, 256);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ K/V producer
        if (lane == 0) {
            uint32_t kv = 0;
            bool ok = true;
            for (int64_t v = 0, it = snake_item(0); it < n_items && ok && !aborted(&sm.abort_flag);
                 it = snake_item(++v)) {
                int b, q, w0, nkv;
                int64_t tile;
                dq_item(u, p.ntiles, it, b, q, w0, nkv, tile);
                for (int i = 0; i < nkv; ++i, ++kv) {
                    const int sk = (int)(kv % kDqKStages), st = kv & 1;
                    const uint32_t par_k = ((kv / kDqKStages) & 1) ^ 1, par = ((kv >> 1) & 1) ^ 1;
                    if (!mbar_wait(&sm.kv_empty_k[sk], par_k)) { fail(&sm.abort_flag, p.status, 1); ok = false; break; }
                    mbar_arrive_expect_tx(&sm.kv_full_k[sk], kTile);
                    tma_load_4d(&mapK, &sm.kv_full_k[sk], sm.k[sk], 0, q, i * kBM, b);
                    tma_load_4d(&mapK, &sm.kv_full_k[sk], sm.k[sk] + kHalf, 64, q, i * kBM, b);
                    if (!mbar_wait(&sm.kv_empty_v[st], par)) { fail(&sm.abort_flag, p.status, 2); ok = false; break; }
                    mbar_arrive_expect_tx(&sm.kv_full_v[st], kTile);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st], 0, q, i * kBM, b);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st] + kHalf, 64, q, i * kBM, b);
                }
            }
            // every issued load lands before the CTA may exit
            for (uint32_t back = 1; back <= kDqKStages && back <= kv; ++back) {
                const uint32_t it = kv - back;
                mbar_wait(&sm.kv_full_k[it % kDqKStages], (it / kDqKStages) & 1);
                if (back <= 2) mbar_wait(&sm.kv_full_v[it & 1], (it >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_ss = idesc_bf16_f32(kBM, kBM, false, false);
            const uint32_t idesc_dq = idesc_bf16_f32(kBM, kD, false, true);
            const uint32_t dhi = smem_desc_hi(1024, kSwizzle128B);
            const uint32_t qlo = smem_desc_lo(smem_u32(sm.q), 16), dolo = smem_desc_lo(smem_u32(sm.dO), 16);
            // K stage x % 3 sits (x % 3) * kTile bytes past stage 0 (start address in 16-byte units)
            const uint32_t klo0 = smem_desc_lo(smem_u32(sm.k[0]), 16);
            const uint32_t kmlo0 = smem_desc_lo(smem_u32(sm.k[0]), kHalf);
            auto kstage = [&](uint32_t x) { return (x % kDqKStages) * (kTile >> 4); };
            const uint32_t vlo0 = smem_desc_lo(smem_u32(sm.v[0]), 16), vlo1 = smem_desc_lo(smem_u32(sm.v[1]), 16);
            const uint32_t c_s = tmem, c_dp = tmem + 256, c_dq = tmem + 384;
            auto desc = [&](uint32_t lo) { return smem_desc_join(lo, dhi); };
            // S(kv tile) into S buffer sb: Q . K^T (both K-major).
            auto issue_s = [&](uint32_t kvi, uint32_t sb) {
                const uint32_t kb = klo0 + kstage(kvi);
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (uint32_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
                    umma_ss(c_s + sb * 128, desc(qlo + off), desc(kb + off), idesc_ss, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sm.s_full[sb]);
            };
            // dP = dO . V^T (V rows as a K-major operand).
            auto issue_dp = [&](uint32_t kvi) {
                const uint32_t vb = (kvi & 1) ? vlo1 : vlo0;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (uint32_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
                    umma_ss(c_dp, desc(dolo + off), desc(vb + off), idesc_ss, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sm.dp_full);
            };
            // dQ (+)= dS . K (dS bf16 pairs in dP's columns a_col(kk); K MN-major).
            auto issue_dq = [&](uint32_t kvi, bool first) {
                const uint32_t kb = kmlo0 + kstage(kvi);
#pragma unroll
                for (int kk = 0; kk < kBM / 16; ++kk)
                    umma_ts(c_dq, c_dp + a_col(kk), desc(kb + (uint32_t)((kk * 2048) >> 4)), idesc_dq,
                            (first && kk == 0) ? 0u : 1u);
            };
            auto wait_k = [&](uint32_t x) { return mbar_wait(&sm.kv_full_k[x % kDqKStages], (x / kDqKStages) & 1); };
            auto wait_v = [&](uint32_t x) { return mbar_wait(&sm.kv_full_v[x & 1], (x >> 1) & 1); };
            uint32_t kv = 0, sc = 0, ec = 0, item_no = 0;  // kv tiles, S issued, elementwise steps, items
            bool ok = true;
            for (int64_t v = 0, it = snake_item(0); it < n_items && ok && !aborted(&sm.abort_flag);
                 it = snake_item(++v), ++item_no) {
                int b, q, w0, nkv;
                int64_t tile;
                dq_item(u, p.ntiles, it, b, q, w0, nkv, tile);
                if (!mbar_wait(&sm.rows_full, item_no & 1)) { fail(&sm.abort_flag, p.status, 10); break; }
                tc_fence_after();
                // prologue: S(0), dP(0), S(1)
                if (!(ok = wait_k(kv))) { fail(&sm.abort_flag, p.status, 11); break; }
                tc_fence_after();
                issue_s(kv, sc & 1);
                ++sc;
                if (!(ok = wait_v(kv))) { fail(&sm.abort_flag, p.status, 12); break; }
                tc_fence_after();
                issue_dp(kv);
                umma_commit(&sm.kv_empty_v[kv & 1]);  // V(0) is only read by dP(0)
                if (nkv > 1) {
                    if (!(ok = wait_k(kv + 1))) { fail(&sm.abort_flag, p.status, 13); break; }
                    tc_fence_after();
                    issue_s(kv + 1, sc & 1);
                    ++sc;
                }
                for (int i = 0; i < nkv; ++i) {
                    const uint32_t x = kv + i;
                    // dS(i) is in dP's columns once the elementwise step i is done
                    if (!(ok = mbar_wait(&sm.ew_done, ec & 1))) { fail(&sm.abort_flag, p.status, 14); break; }
                    ++ec;
                    if (i == 0 && !(ok = mbar_wait(&sm.dq_empty, (item_no & 1) ^ 1))) {
                        fail(&sm.abort_flag, p.status, 15);
                        break;
                    }
                    tc_fence_after();
                    issue_dq(x, i == 0);
                    umma_commit(&sm.kv_empty_k[x % kDqKStages]);  // K(i): read by S(i) and dQ(i)
                    if (i == nkv - 1) {
                        umma_commit(&sm.dq_full);
                        umma_commit(&sm.rows_empty);  // Q, dO and the table of the item are no longer read
                    }
                    if (i + 1 < nkv) {
                        if (!(ok = wait_v(x + 1))) { fail(&sm.abort_flag, p.status, 16); break; }
                        tc_fence_after();
                        issue_dp(x + 1);
                        umma_commit(&sm.kv_empty_v[(x + 1) & 1]);
                    }
                    if (i + 2 < nkv) {
                        if (!(ok = wait_k(x + 2))) { fail(&sm.abort_flag, p.status, 17); break; }
                        tc_fence_after();
                        issue_s(x + 2, sc & 1);
                        ++sc;
                    }
                }
                kv += nkv;
            }
            umma_commit(&sm.drain);
            mbar_wait(&sm.drain, 0);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ row table + Q / dO gather
        uint32_t item_no = 0;
        bool armed = false;
        for (int64_t v = 0, it = snake_item(0); it < n_items && !aborted(&sm.abort_flag);
             it = snake_item(++v), ++item_no) {
            int b, q, w0, nkv;
            int64_t tile;
            dq_item(u, p.ntiles, it, b, q, w0, nkv, tile);
            // the previous item's Q and dO are free
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.rows_empty, (item_no & 1) ^ 1))) {
                if (lane == 0) fail(&sm.abort_flag, p.status, 20);
                break;
            }
            if (lane == 0) {
                mbar_arrive_expect_tx(&sm.rows_full, 2 * kTile);
                const int row0 = (int)(tile * kBM);
                tma_load_2d(&mapQc, &sm.rows_full, sm.q, 0, row0);
                tma_load_2d(&mapQc, &sm.rows_full, sm.q + kHalf, 64, row0);
                tma_load_2d(&mapdOc, &sm.rows_full, sm.dO, 0, row0);
                tma_load_2d(&mapdOc, &sm.rows_full, sm.dO + kHalf, 64, row0);
            }
            armed = true;
        }
        if (armed) mbar_wait(&sm.rows_full, (item_no - 1) & 1);
    } else if (warp >= 4) {
        // ------------------------------------------------------------ elementwise + epilogue (thread = row)
        // Warps 4-7 take key columns 0-63 of their rows, warps 8-11 columns 64-127.
        const int wq = warp & 3;
        const int hh = (warp - 4) >> 2;
        const int r = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t d_addr = tmem + lane_off + 256 + hh * 64;
        uint32_t sc = 0, dc = 0, item_no = 0;
        for (int64_t v = 0, it = snake_item(0); it < n_items && !aborted(&sm.abort_flag);
             it = snake_item(++v), ++item_no) {
            int b, q, w0, nkv;
            int64_t tile;
            dq_item(u, p.ntiles, it, b, q, w0, nkv, tile);
            const TileTab* tab = p.tabs + tile;  // read-only here: loaded while Q and dO arrive
            const int t_row = tab->t[r], j_row = tab->j[r];
            const float lse2 = tab->lse2[r], dl2 = tab->dl2[r];
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.rows_full, item_no & 1))) {
                if (lane == 0) fail(&sm.abort_flag, p.status, 30);
                break;
            }
            float gp0[32], gp1[32];
            bool ok = true;
            for (int i = 0; i <= nkv; ++i) {
                if (i > 0) {
                    // dS phase of key tile i - 1: dS pairs over dP's columns a_col
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.dp_full, dc & 1))) {
                        if (lane == 0) fail(&sm.abort_flag, p.status, 32);
                        ok = false;
                        break;
                    }
                    ++dc;
                    tc_fence_after();
                    uint32_t d0[32], d1[32], ds[16];
                    tmem_ld32(d_addr, d0);
                    tmem_ld32(d_addr + 32, d1);
                    tmem_ld_wait();
                    ds_row(gp0, d0, dl2, ds);
                    tmem_st16(d_addr, ds);
                    ds_row(gp1, d1, dl2, ds);
                    tmem_st16(d_addr + 16, ds);
                    tmem_st_wait();
                    tc_fence_before();
                    mbar_arrive(&sm.ew_done);
                }
                if (i < nkv) {
                    // exponent phase of key tile i (S buffer sc & 1)
                    const uint32_t sb = sc & 1;
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (sc >> 1) & 1))) {
                        if (lane == 0) fail(&sm.abort_flag, p.status, 31);
                        ok = false;
                        break;
                    }
                    ++sc;
                    tc_fence_after();
                    const uint32_t s_addr = tmem + lane_off + sb * 128 + hh * 64;
                    uint32_t s0[32], s1[32];
                    tmem_ld32(s_addr, s0);
                    tmem_ld32(s_addr + 32, s1);
                    tmem_ld_wait();
                    const int kv0 = i * kBM + hh * 64;
                    if ((i + 1) * kBM > w0) {  // the key tile reaches the tile's first position
                        exp_row<true>(s0, p.scale_log2, lse2, t_row, kv0, gp0);
                        exp_row<true>(s1, p.scale_log2, lse2, t_row, kv0 + 32, gp1);
                    } else {
                        exp_row<false>(s0, p.scale_log2, lse2, t_row, kv0, gp0);
                        exp_row<false>(s1, p.scale_log2, lse2, t_row, kv0 + 32, gp1);
                    }
                }
            }
            if (!ok) break;
            // epilogue: dQ = (sum_s dS k_s) / sqrt(d), fp32 rows of the routed heads
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.dq_full, item_no & 1))) {
                if (lane == 0) fail(&sm.abort_flag, p.status, 34);
                break;
            }
            tc_fence_after();
            // a table entry outside [0, T) x group q's heads is reported, not written
            const bool row_ok = t_row >= 0 && t_row < u.T && j_row >= q * u.hpg && j_row < (q + 1) * u.hpg;
            if (t_row >= 0 && !row_ok) report_error(p.status, GQE_ERR_INVALID_ARGUMENT, kWhereBwdTc, 4);
            float* drow = p.dQ + (((int64_t)b * u.T + (row_ok ? t_row : 0)) * u.h + (row_ok ? j_row : 0)) * kD;
#pragma unroll 1
            for (int cb = 2 * hh; cb < 2 * hh + 2; ++cb) {  // this warp's 64 columns
                uint32_t o[32];
                tmem_ld32(tmem + lane_off + 384 + cb * 32, o);
                tmem_ld_wait();
                if (row_ok) {
                    float4* dst = reinterpret_cast<float4*>(drow + cb * 32);
#pragma unroll
                    for (int e = 0; e < 8; ++e)
                        dst[e] = make_float4(__uint_as_float(o[4 * e]) * p.scale, __uint_as_float(o[4 * e + 1]) * p.scale,
                                             __uint_as_float(o[4 * e + 2]) * p.scale,
                                             __uint_as_float(o[4 * e + 3]) * p.scale);
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.dq_empty);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// ------------------------------------------------------------------ 3. dK, dV
// Work item = (b, group q, 128-key tile kt), heaviest (earliest keys) first.
// Its rows are the group's half-window tiles from the one holding key 128*kt
// on.  Roles: warp 0 K/V of the item, warp 1 MMA issuer, warp 2 row tables +
// Q/dO gather (double buffered), warps 4-11 elementwise + epilogue (thread =
// key, two warps per key, one per 64-column half).  TMEM: dK [0,128), dV
// [128,256), S^T [256,384), dP^T [384,512); g p and dS (bf16 pairs) overwrite
// the columns a_col(0..7) of S^T and dP^T.  Per row tile i the tensor core runs
// dV(i), S^T(i+1), dK(i), dP^T(i+1): the exponent phase of tile i+1 overlaps
// dK(i) and dP^T(i+1), the dS phase of tile i overlaps dV(i) and S^T(i+1).
struct KvSmem {
    uint8_t k[kTile];
    uint8_t v[kTile];
    uint8_t q[2][kTile];
    uint8_t dO[2][kTile];
    TileTab tab[2];
    uint64_t kv_full, kv_empty, rows_full[2], rows_empty[2], st_full, dpt_full, exp_done, ds_done, acc_full,
        acc_empty, drain;
    uint32_t tmem_base;
    int32_t abort_flag;
};

__device__ __forceinline__ int64_t kv_items(const UnitGeom& u) {
    return (int64_t)u.B * u.g * ((u.T + kBM - 1) / kBM);
}
__device__ __forceinline__ void kv_item(const UnitGeom& u, int64_t i, int& b, int& q, int& kt, int& tile0,
                                        int& ntiles) {
    const int64_t per = (int64_t)u.B * u.g;
    kt = (int)(i / per);
    const int rem = (int)(i % per);
    b = rem / u.g;
    q = rem % u.g;
    tile0 = (kt * kBM) / u.W;           // first half-window tile holding a position >= 128 kt
    ntiles = (u.T + u.W - 1) / u.W - tile0;
}

__global__ void __launch_bounds__(kThreads, 1)
dkdv_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
               const __grid_constant__ CUtensorMap mapQc, const __grid_constant__ CUtensorMap mapdOc, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    KvSmem& sm = *smem_align1024<KvSmem>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const UnitGeom& u = p.u;
    const int64_t n_items = kv_items(u);
    if (tid == 0) {
        mbar_init(&sm.kv_full, 1);
        mbar_init(&sm.kv_empty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.rows_full[i], 1);
            // the MMA issuer's commit after dK of the tile, which follows both
            // elementwise phases of the tile (and so every read of its table)
            mbar_init(&sm.rows_empty[i], 1);
        }
        mbar_init(&sm.st_full, 1);
        mbar_init(&sm.dpt_full, 1);
        mbar_init(&sm.exp_done, 256);
        mbar_init(&sm.ds_done, 256);
        mbar_init(&sm.acc_full, 1);
        mbar_init(&sm.acc_empty, 256);
        mbar_init(&sm.drain, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    if (warp == 0) {
        // ------------------------------------------------------------ K/V of each item
        if (lane == 0) {
            uint32_t n = 0;
            for (int64_t v = 0, it = snake_item(0); it < n_items && !aborted(&sm.abort_flag);
                 it = snake_item(++v), ++n) {
                int b, q, kt, tile0, ntiles;
                kv_item(u, it, b, q, kt, tile0, ntiles);
                if (!mbar_wait(&sm.kv_empty, (n & 1) ^ 1)) { fail(&sm.abort_flag, p.status, 101); break; }
                mbar_arrive_expect_tx(&sm.kv_full, 2 * kTile);
                tma_load_4d(&mapK, &sm.kv_full, sm.k, 0, q, kt * kBM, b);
                tma_load_4d(&mapK, &sm.kv_full, sm.k + kHalf, 64, q, kt * kBM, b);
                tma_load_4d(&mapV, &sm.kv_full, sm.v, 0, q, kt * kBM, b);
                tma_load_4d(&mapV, &sm.kv_full, sm.v + kHalf, 64, q, kt * kBM, b);
            }
            if (n > 0) mbar_wait(&sm.kv_full, (n - 1) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_ss = idesc_bf16_f32(kBM, kBM, false, false);
            const uint32_t idesc_acc = idesc_bf16_f32(kBM, kD, false, true);
            const uint32_t dhi = smem_desc_hi(1024, kSwizzle128B);
            const uint32_t klo = smem_desc_lo(smem_u32(sm.k), 16), vlo = smem_desc_lo(smem_u32(sm.v), 16);
            const uint32_t qlo0 = smem_desc_lo(smem_u32(sm.q[0]), 16), dolo0 = smem_desc_lo(smem_u32(sm.dO[0]), 16);
            const uint32_t qmlo0 = smem_desc_lo(smem_u32(sm.q[0]), kHalf), domlo0 = smem_desc_lo(smem_u32(sm.dO[0]), kHalf);
            const uint32_t buf_step = kTile >> 4;  // the second Q / dO buffer, in 16-byte units
            const uint32_t c_dk = tmem, c_dv = tmem + 128, c_st = tmem + 256, c_dpt = tmem + 384;
            auto desc = [&](uint32_t lo) { return smem_desc_join(lo, dhi); };
            auto issue_st = [&](uint32_t rb) {  // S^T = K . Q^T
                const uint32_t qb = qlo0 + rb * buf_step;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (uint32_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
                    umma_ss(c_st, desc(klo + off), desc(qb + off), idesc_ss, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sm.st_full);
            };
            auto issue_dpt = [&](uint32_t rb) {  // dP^T = V . dO^T
                const uint32_t dob = dolo0 + rb * buf_step;
#pragma unroll
                for (int kk = 0; kk < kD / 16; ++kk) {
                    const uint32_t off = (uint32_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
                    umma_ss(c_dpt, desc(vlo + off), desc(dob + off), idesc_ss, kk > 0 ? 1u : 0u);
                }
                umma_commit(&sm.dpt_full);
            };
            auto issue_acc = [&](uint32_t c_acc, uint32_t c_a, uint32_t mlo, bool first) {  // (+)= A . B
#pragma unroll
                for (int kk = 0; kk < kBM / 16; ++kk)
                    umma_ts(c_acc, c_a + a_col(kk), desc(mlo + (uint32_t)((kk * 2048) >> 4)), idesc_acc,
                            (first && kk == 0) ? 0u : 1u);
            };
            uint32_t n = 0, rc = 0;  // items, row tiles
            bool ok = true;
            for (int64_t v = 0, it = snake_item(0); it < n_items && ok && !aborted(&sm.abort_flag);
                 it = snake_item(++v), ++n) {
                int b, q, kt, tile0, ntiles;
                kv_item(u, it, b, q, kt, tile0, ntiles);
                if (!mbar_wait(&sm.kv_full, n & 1)) { fail(&sm.abort_flag, p.status, 110); break; }
                if (!mbar_wait(&sm.rows_full[rc & 1], (rc >> 1) & 1)) { fail(&sm.abort_flag, p.status, 112); break; }
                tc_fence_after();
                issue_st(rc & 1);
                issue_dpt(rc & 1);
                if (ntiles == 1) umma_commit(&sm.kv_empty);  // K and V are read by S^T and dP^T only
                for (int i = 0; i < ntiles; ++i, ++rc) {
                    const uint32_t rb = rc & 1, rb1 = (rc + 1) & 1;
                    if (!(ok = mbar_wait(&sm.exp_done, rc & 1))) { fail(&sm.abort_flag, p.status, 113); break; }
                    if (i == 0 && !(ok = mbar_wait(&sm.acc_empty, (n & 1) ^ 1))) {
                        fail(&sm.abort_flag, p.status, 111);
                        break;
                    }
                    tc_fence_after();
                    issue_acc(c_dv, c_st, domlo0 + rb * buf_step, i == 0);  // dV += (g p)^T . dO
                    if (i + 1 < ntiles) {
                        if (!(ok = mbar_wait(&sm.rows_full[rb1], ((rc + 1) >> 1) & 1))) {
                            fail(&sm.abort_flag, p.status, 114);
                            break;
                        }
                        tc_fence_after();
                        issue_st(rb1);
                    }
                    if (!(ok = mbar_wait(&sm.ds_done, rc & 1))) { fail(&sm.abort_flag, p.status, 115); break; }
                    tc_fence_after();
                    issue_acc(c_dk, c_dpt, qmlo0 + rb * buf_step, i == 0);  // dK += dS^T . Q
                    umma_commit(&sm.rows_empty[rb]);
                    if (i + 1 < ntiles) {
                        issue_dpt(rb1);
                        if (i + 2 == ntiles) umma_commit(&sm.kv_empty);
                    }
                }
                if (!ok) break;
                umma_commit(&sm.acc_full);
            }
            umma_commit(&sm.drain);
            mbar_wait(&sm.drain, 0);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ row tables + Q / dO gather
        uint32_t rc = 0;
        int64_t armed = -1;
        for (int64_t v = 0, it = snake_item(0); it < n_items && !aborted(&sm.abort_flag); it = snake_item(++v)) {
            int b, q, kt, tile0, ntiles;
            kv_item(u, it, b, q, kt, tile0, ntiles);
            bool ok = true;
            for (int i = 0; i < ntiles; ++i, ++rc) {
                const uint32_t rb = rc & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.rows_empty[rb], ((rc >> 1) & 1) ^ 1))) {
                    if (lane == 0) fail(&sm.abort_flag, p.status, 120);
                    ok = false;
                    break;
                }
                const int64_t tile = ((int64_t)b * u.g + q) * p.ntiles + (tile0 + i);
                load_tab(p.tabs + tile, sm.tab[rb]);
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive_expect_tx(&sm.rows_full[rb], 2 * kTile);
                    const int row0 = (int)(tile * kBM);
                    tma_load_2d(&mapQc, &sm.rows_full[rb], sm.q[rb], 0, row0);
                    tma_load_2d(&mapQc, &sm.rows_full[rb], sm.q[rb] + kHalf, 64, row0);
                    tma_load_2d(&mapdOc, &sm.rows_full[rb], sm.dO[rb], 0, row0);
                    tma_load_2d(&mapdOc, &sm.rows_full[rb], sm.dO[rb] + kHalf, 64, row0);
                }
                armed = rc;
            }
            if (!ok) break;
        }
        if (armed >= 0) mbar_wait(&sm.rows_full[armed & 1], (armed >> 1) & 1);
    } else if (warp >= 4) {
        // ------------------------------------------------------------ elementwise + epilogue (thread = key)
        // Warps 4-7 take columns (rows of the tile) 0-63, warps 8-11 columns 64-127.
        const int wq = warp & 3;
        const int hh = (warp - 4) >> 2;
        const int kr = wq * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t st_addr = tmem + lane_off + 256 + hh * 64, dpt_addr = tmem + lane_off + 384 + hh * 64;
        const int col0 = hh * 64;
        uint32_t n = 0, rc = 0;
        for (int64_t v = 0, it = snake_item(0); it < n_items && !aborted(&sm.abort_flag);
             it = snake_item(++v), ++n) {
            int b, q, kt, tile0, ntiles;
            kv_item(u, it, b, q, kt, tile0, ntiles);
            const int key = kt * kBM + kr;
            bool ok = true;
            for (int i = 0; i < ntiles; ++i, ++rc) {
                const TileTab& tab = sm.tab[rc & 1];
                // the tile's first position lies before the key tile's end
                const bool masked = (tile0 + i) * u.W < (kt + 1) * kBM;
                // exponent phase: g p, kept in fp32, and as bf16 pairs over S^T's columns a_col
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.st_full, rc & 1))) {
                    if (lane == 0) fail(&sm.abort_flag, p.status, 130);
                    ok = false;
                    break;
                }
                tc_fence_after();
                float gp0[32], gp1[32];
                {
                    uint32_t s0[32], s1[32], pk[16];
                    tmem_ld32(st_addr, s0);
                    tmem_ld32(st_addr + 32, s1);
                    tmem_ld_wait();
                    if (masked) {
                        exp_key<true>(s0, p.scale_log2, key, tab, col0, gp0);
                        exp_key<true>(s1, p.scale_log2, key, tab, col0 + 32, gp1);
                    } else {
                        exp_key<false>(s0, p.scale_log2, key, tab, col0, gp0);
                        exp_key<false>(s1, p.scale_log2, key, tab, col0 + 32, gp1);
                    }
                    pack_chunk(gp0, pk);
                    tmem_st16(st_addr, pk);
                    pack_chunk(gp1, pk);
                    tmem_st16(st_addr + 16, pk);
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&sm.exp_done);
                // dS phase: bf16 pairs over dP^T's columns a_col
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.dpt_full, rc & 1))) {
                    if (lane == 0) fail(&sm.abort_flag, p.status, 131);
                    ok = false;
                    break;
                }
                tc_fence_after();
                {
                    uint32_t d0[32], d1[32], ds[16];
                    tmem_ld32(dpt_addr, d0);
                    tmem_ld32(dpt_addr + 32, d1);
                    tmem_ld_wait();
                    ds_key(gp0, d0, tab, col0, ds);
                    tmem_st16(dpt_addr, ds);
                    ds_key(gp1, d1, tab, col0 + 32, ds);
                    tmem_st16(dpt_addr + 16, ds);
                    tmem_st_wait();
                }
                tc_fence_before();
                mbar_arrive(&sm.ds_done);
            }
            if (!ok) break;
            // epilogue: dK (scaled by 1/sqrt(d)) and dV rows of the item's keys
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.acc_full, n & 1))) {
                if (lane == 0) fail(&sm.abort_flag, p.status, 134);
                break;
            }
            tc_fence_after();
            const bool key_ok = key < u.T;
            const int64_t kv_row = ((int64_t)b * u.T + (key_ok ? key : 0)) * u.g + q;
#pragma unroll 1
            for (int part = 0; part < 2; ++part) {
                float* dst_row = (part == 0 ? p.dK : p.dV) + kv_row * kD;
                const float f = (part == 0) ? p.scale : 1.0f;
#pragma unroll 1
                for (int cb = 2 * hh; cb < 2 * hh + 2; ++cb) {  // this warp's 64 columns
                    uint32_t o[32];
                    tmem_ld32(tmem + lane_off + part * 128 + cb * 32, o);
                    tmem_ld_wait();
                    if (key_ok) {
                        float4* dst = reinterpret_cast<float4*>(dst_row + cb * 32);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            dst[e] = make_float4(__uint_as_float(o[4 * e]) * f, __uint_as_float(o[4 * e + 1]) * f,
                                                 __uint_as_float(o[4 * e + 2]) * f, __uint_as_float(o[4 * e + 3]) * f);
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.acc_empty);
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

size_t a256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

bool attn_backward_tc_supported(const gqe_shape* s) {
    return s->dtype == GQE_BF16 && s->d_h == kD && s->k <= 4 && s->h / s->g <= 32;
}

namespace {
// Workspace of the tensor-core backward: the lse plane [B*T*h] and o
// [B*T*h, 128] (fp32) that the forward recompute writes when the training
// forward's are not given, then the packed tiles: tables [tiles] and the rows
// of Q and dO [tiles * 128, 128] (bf16).
struct BwdLayout {
    size_t plane, o32, tabs, rows, total;
    int64_t ntiles, tiles;
};
BwdLayout bwd_layout(const gqe_shape* s) {
    BwdLayout L;
    const size_t bth = (size_t)s->B * s->T * s->h;
    const int W = 32 * (4 / s->k);
    // every half of every 2W-position window, as the prefill's units and the dQ
    // items name them (the last window's second half may lie past T: empty)
    L.ntiles = 2 * (int64_t)((s->T + 2 * W - 1) / (2 * W));
    L.tiles = (int64_t)s->B * s->g * L.ntiles;
    L.plane = a256(bth * sizeof(float));
    L.o32 = a256(bth * kD * sizeof(float));
    L.tabs = a256((size_t)L.tiles * sizeof(TileTab));
    L.rows = a256((size_t)L.tiles * kBM * kD * 2);
    L.total = L.plane + L.o32 + L.tabs + 2 * L.rows;
    return L;
}
}  // namespace

size_t attn_backward_tc_scratch_bytes(const gqe_shape* s) { return bwd_layout(s).total; }

cudaError_t launch_attn_backward_tc(const AttnBwdArgs& a) {
    const gqe_shape& s = *a.s;
    const int64_t BT = (int64_t)s.B * s.T;
    const BwdLayout L = bwd_layout(a.s);
    char* base = static_cast<char*>(a.scratch);
    float* lse_ws = reinterpret_cast<float*>(base);
    float* o32_ws = reinterpret_cast<float*>(base + L.plane);
    const bool saved = a.o32 != nullptr && a.lse != nullptr;
    const float* lse = saved ? a.lse : lse_ws;
    const float* o32 = saved ? a.o32 : o32_ws;
    TileTab* tabs = reinterpret_cast<TileTab*>(base + L.plane + L.o32);
    __nv_bfloat16* Qc = reinterpret_cast<__nv_bfloat16*>(base + L.plane + L.o32 + L.tabs);
    __nv_bfloat16* dOc = reinterpret_cast<__nv_bfloat16*>(base + L.plane + L.o32 + L.tabs + L.rows);
    const int64_t rows_total = L.tiles * kBM;
    if (rows_total >= ((int64_t)1 << 31) - 1 || BT * s.h >= ((int64_t)1 << 31) - 1) return cudaErrorNotSupported;

    // 0. unless the training forward saved them: the forward again, writing o
    // and the log2-sum-exp of every routed row
    cudaError_t e = cudaSuccess;
    if (!saved) {
        PrefillArgs f;
        f.s = a.s;
        f.Q = a.Q;
        f.K = a.K;
        f.V = a.V;
        f.idx = a.idx;
        f.gate = a.gate;
        f.head_offsets = a.head_offsets;
        f.head_pos = a.head_pos;
        f.head_chunk_offsets = a.head_chunk_offsets;
        f.O = nullptr;
        f.status = a.status;
        f.stream = a.stream;
        f.kv_g = s.g;
        f.kv_q0 = 0;
        f.o32 = o32_ws;
        f.lse = lse_ws;
        e = launch_prefill_tc(f);
        if (e != cudaSuccess) return e;
    }

    Params p;
    p.u.B = s.B;
    p.u.T = s.T;
    p.u.h = s.h;
    p.u.g = s.g;
    p.u.k = s.k;
    p.u.hpg = s.h / s.g;
    p.u.W = 32 * (4 / s.k);
    p.u.nwin = (s.T + kQT * p.u.W - 1) / (kQT * p.u.W);
    p.u.nchunk = gqe_chunk_count(s.T);
    p.idx = a.idx;
    p.gate = a.gate;
    p.head_offsets = a.head_offsets;
    p.head_pos = a.head_pos;
    p.head_chunk_offsets = a.head_chunk_offsets;
    p.tabs = tabs;
    p.ntiles = (int)L.ntiles;
    p.dQ = a.dQ;
    p.dK = a.dK;
    p.dV = a.dV;
    p.status = (uint32_t*)a.status;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    p.scale = 1.0f / sqrtf((float)kD);
    p.q_rows = (int)(BT * s.h);

    // 1. packed tiles (tables, Q and dO rows), logit gradients, dQ of unselected heads
    bwd_pack_kernel<<<(unsigned)L.tiles, kPackThreads, 0, a.stream>>>(
        p.u, p.ntiles, a.head_offsets, a.head_chunk_offsets, a.head_pos, a.idx, a.gate, lse, o32,
        (const __nv_bfloat16*)a.Q, (const __nv_bfloat16*)a.dO, tabs, Qc, dOc, a.dlogits, a.dQ,
        (uint32_t*)a.status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;

    // tensor maps: K, V as [B, T, g, 128] (128-key boxes of 64 columns); the
    // packed rows of Q and dO as [tiles * 128, 128] (128-row boxes)
    CUtensorMap mapK, mapV, mapQc, mapdOc;
    {
        const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.g, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.g * kD * 2, (uint64_t)s.T * s.g * kD * 2};
        const uint32_t box[4] = {64, 1, (uint32_t)kBM, 1};
        if (!make_bf16_map(&mapK, a.K, 4, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_bf16_map(&mapV, a.V, 4, dims, strides, box)) return cudaErrorInvalidValue;
    }
    {
        const uint64_t dims[2] = {(uint64_t)kD, (uint64_t)rows_total};
        const uint64_t strides[1] = {(uint64_t)kD * 2};
        const uint32_t box[2] = {64, (uint32_t)kBM};
        if (!make_bf16_map(&mapQc, Qc, 2, dims, strides, box)) return cudaErrorInvalidValue;
        if (!make_bf16_map(&mapdOc, dOc, 2, dims, strides, box)) return cudaErrorInvalidValue;
    }

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);

    // 2. dQ
    {
        const size_t smem = sizeof(DqSmem) + 1024;
        e = cudaFuncSetAttribute(dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t items = p.u.count() * kQT;
        const int grid = (int)(items < sms ? items : sms);
        dq_tc_kernel<<<grid, kThreads, smem, a.stream>>>(mapK, mapV, mapQc, mapdOc, p);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    // 3. dK, dV
    {
        const size_t smem = sizeof(KvSmem) + 1024;
        e = cudaFuncSetAttribute(dkdv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const int64_t items = (int64_t)s.B * s.g * ((s.T + kBM - 1) / kBM);
        const int grid = (int)(items < sms ? items : sms);
        dkdv_tc_kernel<<<grid, kThreads, smem, a.stream>>>(mapK, mapV, mapQc, mapdOc, p);
        e = cudaGetLastError();
    }
    return e;
}

}  // namespace gqe
