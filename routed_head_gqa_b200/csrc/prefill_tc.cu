// prefill_tc.cu -- routed causal flash attention (bf16, d_h = 128) on the
// sm_100a tensor cores, with the gated zero-filling scatter epilogue.
//
// What it computes (gist.science GQE summary, "Architecture et Routage" and
// "Construction de la Sortie"; IBM GQA page, scaled dot-product attention;
// ml-canon "56 GQA / MQA", shared KV heads): for every routed (b, t, j)
//   O[b,t,j,:] = gate * sum_{s<=t} softmax_s(Q[b,t,j] . K[b,s,j/hpg] / sqrt(128)) V[b,s,j/hpg]
// and O[b,t,j,:] = 0 for the unselected (t, j).
//
// Work unit: (b, KV group q, window of 2W positions), W = 32*floor(4/k).  Every
// token selects exactly k heads per group, so each W-position half of the
// window holds k*W <= 128 routed rows (taken from the per-head packed position
// lists): two M=128 Q tiles.  Both tiles share every K/V tile of the group,
// which is loaded once per unit by TMA.
//
// Roles (384 threads, one persistent CTA per SM):
//   warp 0      TMA producer for K/V tiles; owns the TMEM allocation
//   warp 1      MMA issuer (one thread): S_t = Q_t K^T on tcgen05 (the training
//               instance issues O_t += P_t V here too)
//   warp 2      row tables and Q tiles: one TMA box per head and half when every
//               token of the half-window selected every head of the group (dense
//               GQA), TMA tile::gather4 of the routed rows otherwise (128B-swizzled)
//   warp 3      MMA issuer (one thread): O_t += P_t V (inference instances)
//   warps 4-7   softmax + epilogue of Q tile 0 (one row per thread), and the zero
//               fill of its half-window's unselected output slots
//   warps 8-11  the same for Q tile 1
// TMEM columns (inference instances): one S buffer [0,128) that the tiles take
// in turn, P_0 [128,192) and P_1 [192,256) (bf16 pairs), O_0 [256,384), O_1
// [384,512).  A softmax warpgroup reads S into registers and hands the buffer
// back at once, so the next S is computed while it exponentiates; with P in its
// own slot the next S does not wait for this tile's P.V either.  The training
// instance keeps S_t in [128 t, 128 t + 128) with P_t (and R = p - bf16(p))
// overwriting it, because its P and R need 128 columns per tile.
#include <atomic>
#include <climits>

#include "exp2_fma.cuh"
#include "sm100.cuh"
#include "tma_host.cuh"
#include "units.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kD = 128;          // head width
constexpr int kBM = 128;         // routed rows per Q tile (UMMA M)
constexpr int kBN = 128;         // keys per KV tile (UMMA N of S, K of P.V)
constexpr int kQT = 2;           // Q tiles per unit
constexpr int kThreads = 384;
constexpr uint32_t kHalf = 128 * 64 * 2;   // one [128][64] bf16 box, 16 KB
constexpr uint32_t kTileBytes = 2 * kHalf; // [128][128] bf16, 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // + 128 * tile
// Inference instances: one S buffer that the two tiles take in turn and a P
// slot per tile (bf16 pairs, P_t at kColP + 64 * tile), so a tile's next S is
// computed while its softmax still turns the current one into P.
constexpr uint32_t kColSbuf = 0, kColP = 128;
constexpr float kRescaleThreshold = 8.0f;   // log2 units: p <= 2^8 between rescales
// Of every 16 element pairs of an unmasked tile, exp2 on the FMA pipe
// (exp2_poly2) for this many, on MUFU for the rest.  A same-box sweep with
// both softmax warpgroups active measured 0 fastest (gqe_prefill 0.596 ms
// against 0.607 at 4 and 0.616 at 6; gqe_32k 1.865 against 1.944 ms).
constexpr int kPolyPairs = 0;
constexpr uint32_t kWhereTc = 2;            // status "where" id of this kernel
// Register split (setmaxnreg): 4 control warps at 88, 8 softmax warps at 208.
// 128*88 + 256*208 = 64512 = 384 * 168, the block's registers at launch.
constexpr int kRegsLaunch = 168, kRegsCtl = 88, kRegsSoftmax = 208;
static_assert(128 * kRegsCtl + 256 * kRegsSoftmax <= kThreads * kRegsLaunch, "register split exceeds the launch");

struct Smem {
    uint8_t q[kQT][kTileBytes];      // Q tiles (single buffer, guarded by q_empty)
    uint8_t k[2][kTileBytes];        // K ring
    uint8_t v[2][kTileBytes];        // V ring
    int32_t row_t[2][kQT][kBM];      // row tables, double buffered by unit
    int32_t row_j[2][kQT][kBM];
    float row_gate[2][kQT][kBM];
    int32_t cut_start[2][kQT][32];
    int32_t cut_prefix[2][kQT][33];
    uint64_t kv_full_k[2], kv_full_v[2], kv_empty_k[2], kv_empty_v[2];
    uint64_t s_full[kQT], p_full[kQT], o_full[kQT], o_empty[kQT];
    uint64_t s_free, p_empty[kQT];  // shared-S layout: S buffer read out, P slot consumed
    uint64_t q_full[2], q_empty, rows_free[2], mma_drain, mma_drain2;
    uint32_t tmem_base;
    int32_t abort_flag;
};

// Split-KV partial of one routed row: o = O/l in fp32 and its log2-sum-exp.
constexpr int kPartFloats = 132;  // o[128], lse, 3 pad (16-byte records)

struct Params {
    UnitGeom u;
    const __nv_bfloat16* Q;
    const int32_t* idx;
    const float* gate;
    const int32_t* head_offsets;
    const int32_t* head_pos;
    const int32_t* head_chunk_offsets;
    __nv_bfloat16* O;   // gated bf16 output (null: a recompute for the backward, training outputs only)
    float* o32;         // training: ungated fp32 output of every routed row, [B, T, h, 128]
    float* lse;         // training: log2-sum-exp of every routed row's scaled scores, [B, T, h]
    uint32_t* status;
    float scale_log2;
    int q_rows;  // B*T*h: rows of Q viewed as [B*T*h, 128]
    int kv_q0;   // KV group of the unit's group 0 in the K/V tensor maps
    // Split-KV (nsplit > 1): item = unit * nsplit + s covers KV tiles
    // [s n/nsplit, (s+1) n/nsplit) of the unit's n; each item writes its rows'
    // partials to part, split 0 also the rows' (position, head, gate) to
    // part_rows, and prefill_combine_kernel merges them.
    int nsplit;
    float* part;         // [items][kQT][kBM][kPartFloats]
    int32_t* part_rows;  // [units][kQT][kBM][3]
};

// Keys needed by Q tile t of the unit at window w: 0 .. end-1, end = min(w0 + (t+1)W, T).
__host__ __device__ __forceinline__ int tile_kv_tiles(const UnitGeom& u, int w, int t) {
    const int end = min(w * kQT * u.W + (t + 1) * u.W, u.T);
    return (end + kBN - 1) / kBN;
}

// Item -> unit, split and the split's KV tiles: the first KV tile kv_lo and
// each Q tile's count cnt[t] (the tile's own range clipped to the split's).
// Splits take ceil(n / nsplit) tiles each from the start, so a unit with
// fewer tiles than splits leaves its last splits empty, never split 0 (which
// also zero-fills the window and records the rows for the merge).
__device__ __forceinline__ void item_range(const UnitGeom& u, int nsplit, int64_t item, int64_t& unit, int& split,
                                           int& b, int& q, int& w, int& kv_lo, int (&cnt)[kQT]) {
    unit = item / nsplit;
    split = (int)(item % nsplit);
    unit_coords(u, unit, b, q, w);
    const int n_last = tile_kv_tiles(u, w, kQT - 1);
    const int chunk = (n_last + nsplit - 1) / nsplit;
    kv_lo = min(split * chunk, n_last);
    const int kv_hi = min(kv_lo + chunk, n_last);
#pragma unroll
    for (int t = 0; t < kQT; ++t) cnt[t] = max(0, min(kv_hi, tile_kv_tiles(u, w, t)) - kv_lo);
}

// The j-th unit of this CTA: heavy windows first, zig-zag over the CTAs so that
// each CTA's share pairs heavy and light windows.  Returns -1 past the end.
__device__ __forceinline__ int64_t cta_unit(int64_t j, int64_t n_units) {
    const int64_t base = j * gridDim.x;
    const int64_t unit = base + ((j & 1) ? (int64_t)(gridDim.x - 1 - blockIdx.x) : (int64_t)blockIdx.x);
    return unit < n_units ? unit : -1;
}

__device__ __forceinline__ bool aborted(Smem& sm) { return *((volatile int32_t*)&sm.abort_flag) != 0; }

__device__ __forceinline__ void fail(Smem& sm, const Params& p, uint32_t detail) {
    atomicExch(&sm.abort_flag, 1);
    report_error(p.status, GQE_ERR_DEVICE_TIMEOUT, kWhereTc, detail);
}


// tcgen05.wait::ld that also ties the loaded registers, so no use of them can
// be scheduled before the wait.
__device__ __forceinline__ void ld_wait_bind(uint32_t (&r)[32]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}
__device__ __forceinline__ void ld_bind(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
                   "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
                   "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]),
                   "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]),
                   "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}


// ---------------------------------------------------------------------------
// TMEM columns of S_t and P_t.  The training instance keeps S_t and P_t (with
// R = p - bf16(p) in columns 64-127) in the tile's own 128 columns; the others
// use one S buffer that the tiles take in turn, and a 64-column P slot per tile.
template <bool kSB>
__device__ __forceinline__ uint32_t s_col(int t) { return kSB ? kColSbuf : kColS + 128u * t; }
template <bool kSB>
__device__ __forceinline__ uint32_t p_col(int t) { return kSB ? kColP + 64u * t : kColS + 128u * t; }

// The issuing thread's view of the two GEMMs.  Shared-memory descriptors are
// built once: a K step only moves the start address (16-byte units in the low
// word), so each MMA adds a compile-time offset instead of rebuilding the
// descriptor (the issuing thread's scalar work would otherwise outlast the
// MMAs).  The high word (stride offset 1024, 128-byte swizzle) is shared by
// every operand here.
template <bool kSB, bool kTrain>
struct MmaIssue {
    // scalars, not arrays: a runtime index into a member array would put it in local memory
    uint32_t tmem, dhi, qlo0, qlo1, klo0, klo1, vlo0, vlo1, idesc_s, idesc_pv;
    __device__ MmaIssue(Smem& sm, uint32_t tmem_base)
        : tmem(tmem_base),
          dhi(smem_desc_hi(1024, kSwizzle128B)),
          qlo0(smem_desc_lo(smem_u32(sm.q[0]), 16)),
          qlo1(smem_desc_lo(smem_u32(sm.q[1]), 16)),
          klo0(smem_desc_lo(smem_u32(sm.k[0]), 16)),
          klo1(smem_desc_lo(smem_u32(sm.k[1]), 16)),
          vlo0(smem_desc_lo(smem_u32(sm.v[0]), kHalf)),
          vlo1(smem_desc_lo(smem_u32(sm.v[1]), kHalf)),
          idesc_s(idesc_bf16_f32(kBM, kBN, false, false)),
          idesc_pv(idesc_bf16_f32(kBM, kD, false, true)) {}
    __device__ __forceinline__ uint64_t desc(uint32_t lo) const { return smem_desc_join(lo, dhi); }
    // S_t = Q_t K(it)^T into S_t's columns
    __device__ __forceinline__ void s(int t, uint32_t it) const {
        const uint32_t a0 = t ? qlo1 : qlo0, b0 = (it & 1) ? klo1 : klo0;
        const uint32_t d = tmem + s_col<kSB>(t);
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (uint32_t)(((kk >> 2) * kHalf + (kk & 3) * 32) >> 4);
            umma_ss(d, desc(a0 + off), desc(b0 + off), idesc_s, kk > 0 ? 1u : 0u);
        }
    }
    // O_t += P_t V(it).  For the training outputs P.V runs over [P | R] against
    // V twice: R holds p - bf16(p), so o is accurate far beyond bf16 P (the
    // backward's D = g dO . o needs it).
    __device__ __forceinline__ void pv(int t, uint32_t it, bool first) const {
        const uint32_t b0 = (it & 1) ? vlo1 : vlo0;
        const uint32_t d = tmem + kColO + t * 128, a = tmem + p_col<kSB>(t);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
            umma_ts(d, a + kk * 8, desc(b0 + (uint32_t)((kk * 2048) >> 4)), idesc_pv, (first && kk == 0) ? 0u : 1u);
        if (kTrain) {
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk)
                umma_ts(d, a + 64 + kk * 8, desc(b0 + (uint32_t)((kk * 2048) >> 4)), idesc_pv, 1u);
        }
    }
};

// ---------------------------------------------------------------------------
// kTrain: also write the training outputs (o32, lse); O only when asked.
// kSplit: split-KV items (p.nsplit > 1); the plain instance carries none of it.
template <bool kTrain, bool kSplit>
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                  const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapQB,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *smem_align1024<Smem>(smem_raw);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const UnitGeom& u = p.u;
    const int nsplit = kSplit ? p.nsplit : 1;
    const int64_t n_units = u.count() * nsplit;  // work items (units when not split)
    // TMEM layout: the training instance keeps S_t and P_t (with R = p - bf16(p))
    // in the tile's own 128 columns; the others use the shared S buffer.
    constexpr bool kSB = !kTrain;

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.kv_full_k[i], 1);
            mbar_init(&sm.kv_full_v[i], 1);
            mbar_init(&sm.kv_empty_k[i], 1);
            mbar_init(&sm.kv_empty_v[i], 1);
            mbar_init(&sm.q_full[i], 1);
            mbar_init(&sm.rows_free[i], 256);
        }
        for (int t = 0; t < kQT; ++t) {
            mbar_init(&sm.s_full[t], 1);
            mbar_init(&sm.p_full[t], 128);
            mbar_init(&sm.o_full[t], 1);
            mbar_init(&sm.o_empty[t], 128);
            mbar_init(&sm.p_empty[t], 1);
        }
        mbar_init(&sm.s_free, 4);  // one arrive per warp of the tile's warpgroup
        mbar_init(&sm.q_empty, 1);
        mbar_init(&sm.mma_drain, 1);
        mbar_init(&sm.mma_drain2, 1);
        sm.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 0) {
        tmem_alloc(&sm.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;
    // Launched as a programmatic dependent of the compaction: the set-up above
    // overlaps its tail; nothing it writes is read before this wait.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == 0) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapQB);
            uint32_t kv_it = 0;
            bool k_pending = false;
            for (int64_t j = 0;; ++j) {
                const int64_t item = cta_unit(j, n_units);
                if (item < 0 || aborted(sm)) break;
                int64_t unit;
                int split, b, q, w, kv_lo, cnt[kQT];
                item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
                const int n = cnt[kQT - 1];
                bool ok = true;
                for (int i = 0; i < n; ++i, ++kv_it) {
                    const int st = kv_it & 1;
                    const uint32_t par = ((kv_it >> 1) & 1) ^ 1;
                    if (!mbar_wait(&sm.kv_empty_k[st], par)) { fail(sm, p, 1); ok = false; break; }
                    mbar_arrive_expect_tx(&sm.kv_full_k[st], kTileBytes);
                    tma_load_4d(&mapK, &sm.kv_full_k[st], sm.k[st], 0, p.kv_q0 + q, (kv_lo + i) * kBN, b);
                    tma_load_4d(&mapK, &sm.kv_full_k[st], sm.k[st] + kHalf, 64, p.kv_q0 + q, (kv_lo + i) * kBN, b);
                    k_pending = true;
                    if (!mbar_wait(&sm.kv_empty_v[st], par)) { fail(sm, p, 2); ok = false; break; }
                    mbar_arrive_expect_tx(&sm.kv_full_v[st], kTileBytes);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st], 0, p.kv_q0 + q, (kv_lo + i) * kBN, b);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st] + kHalf, 64, p.kv_q0 + q, (kv_lo + i) * kBN, b);
                    k_pending = false;
                }
                if (!ok) break;
            }
            // Drain: every issued load lands before the CTA may exit.
            if (k_pending) mbar_wait(&sm.kv_full_k[kv_it & 1], (kv_it >> 1) & 1);
            for (uint32_t back = 1; back <= 2 && back <= kv_it; ++back) {
                const uint32_t it = kv_it - back;
                mbar_wait(&sm.kv_full_k[it & 1], (it >> 1) & 1);
                mbar_wait(&sm.kv_full_v[it & 1], (it >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
        // ------------------------------------------------------------ MMA issuer (S; all MMAs when training)
        if (lane == 0) {
            const MmaIssue<kSB, kTrain> mma(sm, tmem);
            uint32_t kv_it = 0, u_it = 0, c[kQT] = {0, 0};
            bool ok = true;
            auto wait_k = [&](uint32_t it) { return mbar_wait(&sm.kv_full_k[it & 1], (it >> 1) & 1); };
            auto wait_v = [&](uint32_t it) { return mbar_wait(&sm.kv_full_v[it & 1], (it >> 1) & 1); };
            if constexpr (kSB) {
                // S_t(i) of every step, tile 0 first, into the shared S buffer:
                // each waits until the previous S has been read out by its
                // softmax (s_free), so S of the next step is computed while the
                // softmax warps still work on the current one.  P.V is issued by
                // warp 3.
                uint32_t s_cnt = 0;
                for (int64_t j = 0; ok; ++j) {
                    const int64_t item = cta_unit(j, n_units);
                    if (item < 0 || aborted(sm)) break;
                    int64_t unit;
                    int split, b, q, w, kv_lo, cnt[kQT];
                    item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
                    const int n0 = cnt[0], n1 = cnt[1];
                    if (n1 == 0) continue;  // an empty split: every role skips it
                    const uint32_t ui = u_it++;
                    if (!mbar_wait(&sm.q_full[ui & 1], (ui >> 1) & 1)) { fail(sm, p, 10); break; }
                    for (int i = 0; i < n1 && ok; ++i, ++kv_it) {
                        if (!wait_k(kv_it)) { fail(sm, p, 11); ok = false; break; }
                        for (int t = (i < n0) ? 0 : 1; t < kQT; ++t) {
                            if (s_cnt > 0 && !mbar_wait(&sm.s_free, (s_cnt - 1) & 1)) { fail(sm, p, 12); ok = false; break; }
                            tc_fence_after();
                            mma.s(t, kv_it);
                            umma_commit(&sm.s_full[t]);
                            ++s_cnt;
                        }
                        if (!ok) break;
                        umma_commit(&sm.kv_empty_k[kv_it & 1]);
                        if (i == n1 - 1) umma_commit(&sm.q_empty);
                    }
                }
            } else {
                for (int64_t j = 0; ok; ++j) {
                    const int64_t item = cta_unit(j, n_units);
                    if (item < 0 || aborted(sm)) break;
                    int64_t unit;
                    int split, b, q, w, kv_lo, cnt[kQT];
                    item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
                    const int n0 = cnt[0], n1 = cnt[1];
                    if (n1 == 0) continue;  // an empty split: every role skips it
                    const uint32_t ui = u_it++;
                    const int qs = ui & 1;
                    if (!mbar_wait(&sm.q_full[qs], (ui >> 1) & 1)) { fail(sm, p, 10); break; }
                    tc_fence_after();
                    if (!wait_k(kv_it)) { fail(sm, p, 11); break; }
                    tc_fence_after();
                    if (n0 > 0) {
                        mma.s(0, kv_it);
                        umma_commit(&sm.s_full[0]);
                    }
                    mma.s(1, kv_it);
                    umma_commit(&sm.s_full[1]);
                    umma_commit(&sm.kv_empty_k[kv_it & 1]);
                    if (n1 == 1) umma_commit(&sm.q_empty);
                    for (int i = 0; i < n1; ++i) {
                        const uint32_t it = kv_it + i;
                        if (i < n0) {
                            ok = mbar_wait(&sm.p_full[0], (c[0] + i) & 1);
                            if (ok && i == 0) ok = mbar_wait(&sm.o_empty[0], (ui & 1) ^ 1);
                            if (ok) ok = wait_v(it);
                            if (!ok) { fail(sm, p, 12); break; }
                            tc_fence_after();
                            mma.pv(0, it, i == 0);
                            if (i == n0 - 1) umma_commit(&sm.o_full[0]);
                            if (i + 1 < n0) {
                                if (!wait_k(it + 1)) { fail(sm, p, 13); ok = false; break; }
                                tc_fence_after();
                                mma.s(0, it + 1);
                                umma_commit(&sm.s_full[0]);
                            }
                        }
                        ok = mbar_wait(&sm.p_full[1], (c[1] + i) & 1);
                        if (ok && i == 0) ok = mbar_wait(&sm.o_empty[1], (ui & 1) ^ 1);
                        if (ok) ok = wait_v(it);
                        if (!ok) { fail(sm, p, 14); break; }
                        tc_fence_after();
                        mma.pv(1, it, i == 0);
                        umma_commit(&sm.kv_empty_v[it & 1]);
                        if (i == n1 - 1) umma_commit(&sm.o_full[1]);
                        if (i + 1 < n1) {
                            if (!wait_k(it + 1)) { fail(sm, p, 15); ok = false; break; }
                            tc_fence_after();
                            mma.s(1, it + 1);
                            umma_commit(&sm.s_full[1]);
                            umma_commit(&sm.kv_empty_k[(it + 1) & 1]);
                            if (i + 1 == n1 - 1) umma_commit(&sm.q_empty);
                        }
                    }
                    kv_it += n1;
                    c[0] += n0;
                    c[1] += n1;
                }
            }
            // Drain: all issued MMAs complete before TMEM is released.
            umma_commit(&sm.mma_drain);
            mbar_wait(&sm.mma_drain, 0);
        }
    } else if (warp == 2) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
        // ------------------------------------------------------------ row tables + Q gather
        uint32_t u_it = 0;
        int64_t armed = -1;  // last unit whose Q loads were issued
        const int32_t total = (int32_t)((int64_t)u.B * u.T * u.g * u.k);
        for (int64_t j = 0;; ++j) {
            const int64_t item = cta_unit(j, n_units);
            if (item < 0 || aborted(sm)) break;
            int64_t unit;
            int split, b, q, w, kv_lo, cnt[kQT];
            item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
            if (cnt[kQT - 1] == 0) continue;  // an empty split
            const uint32_t ui = u_it++;
            const int rs = ui & 1;
            // The row tables are double buffered: build this unit's while the
            // previous unit still computes, then wait for its Q tiles to be free.
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.rows_free[rs], ((ui >> 1) & 1) ^ 1))) {
                if (lane == 0) fail(sm, p, 20);
                break;
            }
            for (int t = 0; t < kQT; ++t) {
                const int w0 = (w * kQT + t) * u.W;  // first position of this tile's half-window
                // 1. per-head slices of the half-window in the packed position lists
                if (lane < u.hpg) {
                    const int jh = q * u.hpg + lane;
                    int32_t a0 = list_cut(u, p.head_offsets, p.head_chunk_offsets, b, jh, w0);
                    int32_t a1 = list_cut(u, p.head_offsets, p.head_chunk_offsets, b, jh, w0 + u.W);
                    if (a0 < 0 || a1 < a0 || a1 > total) {  // malformed lists: report, use none
                        report_error(p.status, GQE_ERR_INVALID_ARGUMENT, kWhereTc, 41);
                        a0 = a1 = 0;
                    }
                    sm.cut_start[rs][t][lane] = a0;
                    sm.cut_prefix[rs][t][lane + 1] = a1 - a0;
                }
                __syncwarp();
                if (lane == 0) {
                    int acc = 0;
                    sm.cut_prefix[rs][t][0] = 0;
                    for (int jj = 0; jj < u.hpg; ++jj) {
                        acc = min(acc + sm.cut_prefix[rs][t][jj + 1], kBM);
                        sm.cut_prefix[rs][t][jj + 1] = acc;
                    }
                }
                __syncwarp();
                const int nrows = sm.cut_prefix[rs][t][u.hpg];
                // 2. row table: position, head and gate of each routed row.  Each
                // lane's 4 rows issue their loads together (two dependent rounds:
                // head_pos, then the token's k (idx, gate) pairs).
                int tt[kBM / 32], jh[kBM / 32];
#pragma unroll
                for (int i = 0; i < kBM / 32; ++i) {
                    const int r = lane + 32 * i;
                    tt[i] = -1;
                    jh[i] = 0;
                    if (r < nrows) {
                        int jj = 0;
                        while (sm.cut_prefix[rs][t][jj + 1] <= r) ++jj;
                        jh[i] = q * u.hpg + jj;
                        tt[i] = p.head_pos[sm.cut_start[rs][t][jj] + (r - sm.cut_prefix[rs][t][jj])];
                    }
                }
#pragma unroll
                for (int i = 0; i < kBM / 32; ++i) {
                    const int r = lane + 32 * i;
                    float gv = 0.f;
                    if (tt[i] >= 0) {
                        if (tt[i] < w0 || tt[i] >= min(w0 + u.W, u.T)) {  // outside the window: report, drop
                            report_error(p.status, GQE_ERR_INVALID_ARGUMENT, kWhereTc, 40);
                            tt[i] = -1;
                        } else {
                            const int64_t sel = (((int64_t)b * u.T + tt[i]) * u.g + q) * u.k;
                            int sj[4];
                            float sg[4];
#pragma unroll
                            for (int s2 = 0; s2 < 4; ++s2) {
                                if (s2 < u.k) {
                                    sj[s2] = p.idx[sel + s2];
                                    sg[s2] = p.gate[sel + s2];
                                }
                            }
#pragma unroll
                            for (int s2 = 0; s2 < 4; ++s2)
                                if (s2 < u.k && sj[s2] == jh[i]) gv = sg[s2];
                        }
                    }
                    sm.row_t[rs][t][r] = tt[i];
                    sm.row_j[rs][t][r] = jh[i];
                    sm.row_gate[rs][t][r] = gv;
                }
            }
            __syncwarp();
            // Pull the unit's Q rows into L2 while the previous unit still computes.
            for (int t = 0; t < kQT; ++t) {
                for (int r = lane; r < kBM; r += 32) {
                    const int tr = sm.row_t[rs][t][r];
                    if (tr >= 0) {
                        const __nv_bfloat16* row = p.Q + (((int64_t)b * u.T + tr) * u.h + sm.row_j[rs][t][r]) * kD;
                        prefetch_l2(row);
                        prefetch_l2(row + 64);
                    }
                }
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_empty, (ui & 1) ^ 1))) {
                if (lane == 0) fail(sm, p, 21);
                break;
            }
            // 3. Q tiles by TMA.  A tile with h/g * W rows holds every position
            // of its half-window for every head of the group (dense GQA): head
            // jj's W rows are W consecutive tokens of Q viewed as [B, T, h, 128],
            // one box per 64-column half.  Any other tile is gathered: each
            // routed row is one row of Q viewed as [B*T*h, 128], and one
            // tile::gather4 copy moves four rows' 64-column halves (box one row
            // high) to rows r..r+3 of a tile half.  Either way the 128-byte
            // swizzle follows the shared-memory address.  Padding rows name an
            // out-of-range row, which the TMA zero-fills.
            if (lane == 0) mbar_arrive_expect_tx(&sm.q_full[rs], kQT * kTileBytes);
            __syncwarp();
#pragma unroll
            for (int t = 0; t < kQT; ++t) {
                // full tile of exactly 128 rows: the boxes deliver the 32 KB the
                // barrier expects (a 96-row full tile, h/g = k = 3, is gathered)
                if (u.hpg * u.W == kBM && sm.cut_prefix[rs][t][u.hpg] == kBM) {
                    if (lane < 2 * u.hpg) {
                        const int jj = lane >> 1, half = lane & 1;
                        uint8_t* dst = sm.q[t] + jj * u.W * 128 + half * kHalf;
                        tma_load_4d(&mapQB, &sm.q_full[rs], dst, half * 64, q * u.hpg + jj, (w * kQT + t) * u.W, b);
                    }
                } else {
                    const int r0 = lane * 4;  // four rows per lane
                    int row[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tr = sm.row_t[rs][t][r0 + e];
                        row[e] = (tr >= 0) ? (int)(((int64_t)b * u.T + tr) * u.h + sm.row_j[rs][t][r0 + e]) : p.q_rows;
                    }
                    uint8_t* dst = sm.q[t] + r0 * 128;
                    tma_gather4_2d(&mapQ, &sm.q_full[rs], dst, 0, row[0], row[1], row[2], row[3]);
                    tma_gather4_2d(&mapQ, &sm.q_full[rs], dst + kHalf, 64, row[0], row[1], row[2], row[3]);
                }
            }
            armed = ui;
        }
        // Drain: the last issued Q loads land before the CTA may exit.
        if (armed >= 0) mbar_wait(&sm.q_full[armed & 1], (armed >> 1) & 1);
    } else if (warp == 3) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsCtl));
        if constexpr (kSB) {
            // -------------------------------------------------------- MMA issuer (P.V)
            // O_t += P_t(i) V(i) once the softmax has written P_t(i) to the
            // tile's P slot; each completion hands the slot back (p_empty).
            if (lane == 0) {
                const MmaIssue<kSB, kTrain> mma(sm, tmem);
                uint32_t kv_it = 0, u_it = 0, c[kQT] = {0, 0};
                bool ok = true;
                for (int64_t j = 0; ok; ++j) {
                    const int64_t item = cta_unit(j, n_units);
                    if (item < 0 || aborted(sm)) break;
                    int64_t unit;
                    int split, b, q, w, kv_lo, cnt[kQT];
                    item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
                    const int n0 = cnt[0], n1 = cnt[1];
                    if (n1 == 0) continue;  // an empty split
                    const uint32_t ui = u_it++;
                    for (int i = 0; i < n1 && ok; ++i, ++kv_it) {
                        if (!mbar_wait(&sm.kv_full_v[kv_it & 1], (kv_it >> 1) & 1)) { fail(sm, p, 17); ok = false; break; }
                        for (int t = (i < n0) ? 0 : 1; t < kQT; ++t) {
                            ok = mbar_wait(&sm.p_full[t], c[t] & 1);
                            if (ok && i == 0) ok = mbar_wait(&sm.o_empty[t], (ui & 1) ^ 1);
                            if (!ok) { fail(sm, p, 18); break; }
                            tc_fence_after();
                            mma.pv(t, kv_it, i == 0);
                            umma_commit(&sm.p_empty[t]);
                            ++c[t];
                            if (i == (t ? n1 : n0) - 1) umma_commit(&sm.o_full[t]);
                        }
                        if (!ok) break;
                        umma_commit(&sm.kv_empty_v[kv_it & 1]);
                    }
                }
                umma_commit(&sm.mma_drain2);
                mbar_wait(&sm.mma_drain2, 0);
            }
        }
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
        // ------------------------------------------------------------ softmax + epilogue (tile t)
        const int t = (warp - 4) >> 2;     // Q tile of this warpgroup
        const int wq = warp & 3;           // TMEM lane quarter of this warp
        const int r = wq * 32 + lane;      // routed row owned by this thread
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        const uint32_t s_addr = tmem + lane_off + s_col<kSB>(t);
        const uint32_t p_addr = tmem + lane_off + p_col<kSB>(t);
        const uint32_t o_addr = tmem + lane_off + kColO + t * 128;
        constexpr bool train = kTrain;  // also write R = p - bf16(p) for the exact P.V
        uint32_t ctile = 0, u_it = 0, o_it = 0;  // S tiles, items, O_t completions waited
        for (int64_t j = 0;; ++j) {
            const int64_t item = cta_unit(j, n_units);
            if (item < 0 || aborted(sm)) break;
            int64_t unit;
            int split, b, q, w, kv_lo, cnt[kQT];
            item_range(u, nsplit, item, unit, split, b, q, w, kv_lo, cnt);
            if (cnt[kQT - 1] == 0) continue;  // an empty split
            const uint32_t ui = u_it++;
            const int n = cnt[t];
            const int rs = ui & 1;
            // Zero fill of the tile's half-window [lo, lo + W): every slot whose
            // head the token did not select is written as zeros (a unit's first
            // split does it; a recompute for the backward leaves O alone).  It
            // needs neither Q nor S, so it runs while the unit's Q tiles load.
            // Each token has 128 / W threads; thread r takes every (128 / W)-th
            // head of the token's complement.
            if (p.O != nullptr && (!kSplit || split == 0)) {
                const int lo = (w * kQT + t) * u.W;
                const int tpt = kBM / u.W;  // threads per token: 1, 2 or 4
                const int tok = lo + r / tpt;
                if (tok < min(lo + u.W, u.T)) {
                    const int64_t sel = (((int64_t)b * u.T + tok) * u.g + q) * u.k;
                    uint64_t chosen = 0;
#pragma unroll
                    for (int s2 = 0; s2 < 4; ++s2) {
                        if (s2 < u.k) {
                            const int a = p.idx[sel + s2] - q * u.hpg;  // head within the group
                            if (a >= 0 && a < u.hpg) chosen |= 1ull << a;
                        }
                    }
                    uint64_t un = ~chosen & ((u.hpg >= 64) ? ~0ull : ((1ull << u.hpg) - 1ull));
                    uint4* orow = reinterpret_cast<uint4*>(p.O + (((int64_t)b * u.T + tok) * u.h + q * u.hpg) * kD);
                    for (int c = 0; un != 0ull; ++c) {
                        const int a = __ffsll((long long)un) - 1;
                        un &= un - 1ull;
                        if (c % tpt != r % tpt) continue;
                        uint4* dst = orow + (int64_t)a * (kD * 2 / 16);
#pragma unroll
                        for (int v = 0; v < kD * 2 / 16; ++v) dst[v] = make_uint4(0, 0, 0, 0);
                    }
                }
            }
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full[rs], (ui >> 1) & 1))) {
                if (lane == 0) fail(sm, p, 30);
                break;
            }
            const int t_row = sm.row_t[rs][t][r];
            const int t_eff = (t_row >= 0) ? t_row : INT_MAX;  // padding rows: unmasked, output dropped
            const int lo = (w * kQT + t) * u.W;               // first position of the tile
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int i = 0; i < n; ++i, ++ctile) {
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[t], ctile & 1))) {
                    if (lane == 0) fail(sm, p, 31);
                    ok = false;
                    break;
                }
                tc_fence_after();
                // The tile's scores, four 32-column chunks.  On an unmasked tile
                // after the first, the exponentials are taken against the running
                // max m while the tile's row max is formed alongside: when no row
                // of the warp grew its max by more than the rescale threshold (the
                // usual case) P is final, else the general path below redoes the
                // tile from the scores, which stay in registers.  The first
                // chunk's exponentials start while the other three load.
                uint32_t s[4][32];
                const int kv0 = (kv_lo + i) * kBN;
                const bool need_mask = kv0 + kBN - 1 > lo;
                const bool spec = !need_mask && i > 0;  // the same for the whole warp
                const uint64_t C2 = pk2(p.scale_log2, p.scale_log2);
                uint64_t sum2[4] = {0, 0, 0, 0};
                float m_use = m;
                bool rescale = false, done = false, slot_ok = true;
                // Shared S buffer: read it out whole and hand it back to the next S.
                if constexpr (kSB) {
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) tmem_ld32(s_addr + cb * 32, s[cb]);
                    ld_wait_bind(s[0]);
                    ld_bind(s[1]);
                    ld_bind(s[2]);
                    ld_bind(s[3]);
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&sm.s_free);
                }
                // P slot of this tile: free once the tile's previous P.V has
                // completed (which also completes O_t up to the previous tile).
                auto wait_slot = [&]() {
                    if (ctile > 0 && !__all_sync(0xffffffffu, mbar_wait(&sm.p_empty[t], (ctile - 1) & 1)))
                        slot_ok = false;
                    tc_fence_after();
                };
                if (spec) {
                    if constexpr (!kSB) {
                        tmem_ld32(s_addr, s[0]);
                        ld_wait_bind(s[0]);
#pragma unroll
                        for (int cb = 1; cb < 4; ++cb) tmem_ld32(s_addr + cb * 32, s[cb]);
                    }
                    const uint64_t NM2 = pk2(-m, -m);
                    float mq[4];
                    uint32_t pk[4][16], rk[4][16];
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        if (!kSB && cb == 1) {
                            ld_wait_bind(s[1]);
                            ld_bind(s[2]);
                            ld_bind(s[3]);
                        }
                        float a0 = __uint_as_float(s[cb][0]);
#pragma unroll
                        for (int e = 1; e < 31; e += 2)
                            a0 = fmax3(a0, __uint_as_float(s[cb][e]), __uint_as_float(s[cb][e + 1]));
                        mq[cb] = fmaxf(a0, __uint_as_float(s[cb][31]));
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            float x0, x1;
                            up2(ffma2(pk2(__uint_as_float(s[cb][2 * e]), __uint_as_float(s[cb][2 * e + 1])), C2, NM2),
                                x0, x1);
                            const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                            sum2[e & 3] = fadd2(sum2[e & 3], pk2(p0, p1));
                            pk[cb][e] = pack_bf16x2(p0, p1);
                            if (train) rk[cb][e] = pack_bf16x2(p0 - __uint_as_float(pk[cb][e] << 16),
                                                               p1 - __uint_as_float(pk[cb][e] & 0xffff0000u));
                        }
                        if constexpr (kSB) {
                            // the first two chunks wait in registers for the slot
                            if (cb == 1) {
                                wait_slot();
                                tmem_st16(p_addr, pk[0]);
                                tmem_st16(p_addr + 16, pk[1]);
                            } else if (cb > 1) {
                                tmem_st16(p_addr + cb * 16, pk[cb]);
                            }
                        } else {
                            tmem_st16(p_addr + cb * 16, pk[cb]);
                            if (train) tmem_st16(s_addr + 64 + cb * 16, rk[cb]);
                        }
                    }
                    const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * p.scale_log2;
                    done = __all_sync(0xffffffffu, mx <= m + kRescaleThreshold);
                    if (!done) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) sum2[e] = 0;
                    }
                } else if constexpr (!kSB) {
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) tmem_ld32(s_addr + cb * 32, s[cb]);
                    ld_wait_bind(s[0]);
                    ld_bind(s[1]);
                    ld_bind(s[2]);
                    ld_bind(s[3]);
                }
                if (!done) {
                    if (need_mask) {
#pragma unroll
                        for (int cb = 0; cb < 4; ++cb)
#pragma unroll
                            for (int e = 0; e < 32; ++e)
                                if (kv0 + cb * 32 + e > t_eff) s[cb][e] = __float_as_uint(-INFINITY);
                    }
                    // row max of the raw scores: four independent 3-input max chains
                    float mq[4];
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        float a0 = __uint_as_float(s[cb][0]);
#pragma unroll
                        for (int e = 1; e < 31; e += 2)
                            a0 = fmax3(a0, __uint_as_float(s[cb][e]), __uint_as_float(s[cb][e + 1]));
                        mq[cb] = fmaxf(a0, __uint_as_float(s[cb][31]));
                    }
                    const float mx = fmax3(mq[0], mq[1], fmaxf(mq[2], mq[3])) * p.scale_log2;
                    // Lazy rescaling: keep the running max unless it grows by more than the threshold.
                    if (mx > m + kRescaleThreshold || m == -INFINITY) {
                        m_use = mx;
                        rescale = (i > 0);
                    }
                    // O_t must hold P.V of every earlier tile: in the shared-S layout
                    // the tile's previous P.V has completed once the slot is free; in
                    // the other, S_t's completion covers it (the same commit).
                    if constexpr (kSB) wait_slot();
                    if (__any_sync(0xffffffffu, rescale)) {
                        const float alpha = rescale ? fast_exp2(m - m_use) : 1.0f;
#pragma unroll 1
                        for (int cb = 0; cb < 4; ++cb) {
                            uint32_t o[32];
                            tmem_ld32(o_addr + cb * 32, o);
                            ld_wait_bind(o);
#pragma unroll
                            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                            tmem_st16(o_addr + cb * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
                            tmem_st16(o_addr + cb * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
                        }
                        l *= alpha;
                    }
                    // p = 2^(s*c - m): one packed FMA per pair; exp2 on MUFU, or for
                    // kPolyPairs of every 16 pairs of an unmasked tile on the FMA pipe.
                    const uint64_t NM2 = pk2(-m_use, -m_use);
                    if (need_mask) {
#pragma unroll
                        for (int cb = 0; cb < 4; ++cb) {
                            uint32_t pk[16], rk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                float x0, x1;
                                up2(ffma2(pk2(__uint_as_float(s[cb][2 * e]), __uint_as_float(s[cb][2 * e + 1])), C2,
                                          NM2),
                                    x0, x1);
                                const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
                                sum2[e & 3] = fadd2(sum2[e & 3], pk2(p0, p1));
                                pk[e] = pack_bf16x2(p0, p1);
                                if (train) rk[e] = pack_bf16x2(p0 - __uint_as_float(pk[e] << 16),
                                                               p1 - __uint_as_float(pk[e] & 0xffff0000u));
                            }
                            tmem_st16(p_addr + cb * 16, pk);
                            if (train) tmem_st16(s_addr + 64 + cb * 16, rk);
                        }
                    } else {
#pragma unroll
                        for (int cb = 0; cb < 4; ++cb) {
                            uint32_t pk[16], rk[16];
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const uint64_t x2 = ffma2(
                                    pk2(__uint_as_float(s[cb][2 * e]), __uint_as_float(s[cb][2 * e + 1])), C2, NM2);
                                float p0, p1;
                                if (e < kPolyPairs) {
                                    float x0, x1;
                                    up2(x2, x0, x1);
                                    up2(exp2_poly2_clamped(x0, x1), p0, p1);
                                } else {
                                    float x0, x1;
                                    up2(x2, x0, x1);
                                    p0 = fast_exp2(x0);
                                    p1 = fast_exp2(x1);
                                }
                                sum2[e & 3] = fadd2(sum2[e & 3], pk2(p0, p1));
                                pk[e] = pack_bf16x2(p0, p1);
                                if (train) rk[e] = pack_bf16x2(p0 - __uint_as_float(pk[e] << 16),
                                                               p1 - __uint_as_float(pk[e] & 0xffff0000u));
                            }
                            tmem_st16(p_addr + cb * 16, pk);
                            if (train) tmem_st16(s_addr + 64 + cb * 16, rk);
                        }
                    }
                }
                float sa, sb;
                up2(fadd2(fadd2(sum2[0], sum2[1]), fadd2(sum2[2], sum2[3])), sa, sb);
                const float rowsum = sa + sb;
                l += rowsum;
                m = m_use;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sm.p_full[t]);
                if (!slot_ok) {
                    if (lane == 0) fail(sm, p, 36);
                    ok = false;
                    break;
                }
            }
            if (!ok) break;
            const int j_row = sm.row_j[rs][t][r];
            if (kSplit) {
                // Split-KV: this split's o = O_t / l and log2-sum-exp m + log2(l)
                // (-inf for a split with no keys for this tile); split 0 also
                // records the row's position, head and gate for the merge.
                float* rec = p.part + ((item * kQT + t) * kBM + r) * kPartFloats;
                if (n > 0) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[t], o_it & 1))) {
                        if (lane == 0) fail(sm, p, 35);
                        break;
                    }
                    ++o_it;
                    tc_fence_after();
                    const float inv = 1.0f / l;
#pragma unroll 1
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t o[32];
                        tmem_ld32(o_addr + cb * 32, o);
                        ld_wait_bind(o);
                        float4* dst = reinterpret_cast<float4*>(rec + cb * 32);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                                 __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
                    }
                    rec[kD] = m + log2f(l);
                } else {
                    rec[kD] = -INFINITY;
                }
                if (split == 0) {
                    int32_t* pr = p.part_rows + ((unit * kQT + t) * kBM + r) * 3;
                    pr[0] = t_row;
                    pr[1] = j_row;
                    pr[2] = __float_as_int(sm.row_gate[rs][t][r]);
                }
                tc_fence_before();
                mbar_arrive(&sm.o_empty[t]);
                mbar_arrive(&sm.rows_free[rs]);
                continue;
            }
            // Epilogue: O_t / l * gate -> bf16 row of O[b, t, j, :].
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full[t], o_it & 1))) {
                if (lane == 0) fail(sm, p, 34);
                break;
            }
            ++o_it;
            tc_fence_after();
            const int64_t orow_idx = ((int64_t)b * u.T + (t_row >= 0 ? t_row : 0)) * u.h + j_row;
            if (kTrain) {
                // Training: the ungated output o = O_t / l in fp32 and the row's
                // log2-sum-exp m + log2(l) (so that p_s = 2^(s_s * c - lse)).
                const float inv = 1.0f / l;
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + cb * 32, o);
                    ld_wait_bind(o);
                    if (t_row >= 0) {
                        float4* dst = reinterpret_cast<float4*>(p.o32 + orow_idx * kD + cb * 32);
#pragma unroll
                        for (int v = 0; v < 8; ++v)
                            dst[v] = make_float4(__uint_as_float(o[4 * v]) * inv, __uint_as_float(o[4 * v + 1]) * inv,
                                                 __uint_as_float(o[4 * v + 2]) * inv, __uint_as_float(o[4 * v + 3]) * inv);
                    }
                }
                if (t_row >= 0) p.lse[orow_idx] = m + log2f(l);
                if (p.O == nullptr) {  // a recompute for the backward: O is not wanted
                    tc_fence_before();
                    mbar_arrive(&sm.o_empty[t]);
                    mbar_arrive(&sm.rows_free[rs]);
                    continue;
                }
            }
            const float f = (t_row >= 0) ? sm.row_gate[rs][t][r] / l : 0.f;
            __nv_bfloat16* orow = p.O + orow_idx * kD;
            if constexpr (kSB) {
                // O_t whole into registers; O_t and the row table go back to the
                // next unit before the global stores.
                uint32_t o[4][32];
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) tmem_ld32(o_addr + cb * 32, o[cb]);
                ld_wait_bind(o[0]);
                ld_bind(o[1]);
                ld_bind(o[2]);
                ld_bind(o[3]);
                tc_fence_before();
                mbar_arrive(&sm.o_empty[t]);
                mbar_arrive(&sm.rows_free[rs]);
                if (t_row >= 0) {
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 pk;
                            pk.x = pack_bf16x2(__uint_as_float(o[cb][8 * v + 0]) * f, __uint_as_float(o[cb][8 * v + 1]) * f);
                            pk.y = pack_bf16x2(__uint_as_float(o[cb][8 * v + 2]) * f, __uint_as_float(o[cb][8 * v + 3]) * f);
                            pk.z = pack_bf16x2(__uint_as_float(o[cb][8 * v + 4]) * f, __uint_as_float(o[cb][8 * v + 5]) * f);
                            pk.w = pack_bf16x2(__uint_as_float(o[cb][8 * v + 6]) * f, __uint_as_float(o[cb][8 * v + 7]) * f);
                            dst[v] = pk;
                        }
                    }
                }
            } else {
#pragma unroll 1
                for (int cb = 0; cb < 4; ++cb) {
                    uint32_t o[32];
                    tmem_ld32(o_addr + cb * 32, o);
                    ld_wait_bind(o);
                    if (t_row >= 0) {
                        uint4* dst = reinterpret_cast<uint4*>(orow + cb * 32);
#pragma unroll
                        for (int v = 0; v < 4; ++v) {
                            uint4 pk;
                            pk.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * f, __uint_as_float(o[8 * v + 1]) * f);
                            pk.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * f, __uint_as_float(o[8 * v + 3]) * f);
                            pk.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * f, __uint_as_float(o[8 * v + 5]) * f);
                            pk.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * f, __uint_as_float(o[8 * v + 7]) * f);
                            dst[v] = pk;
                        }
                    }
                }
                tc_fence_before();
                mbar_arrive(&sm.o_empty[t]);
                mbar_arrive(&sm.rows_free[rs]);
            }
        }
    }

    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// Merge of the split-KV partials, one warp per routed row (unit, Q tile, row):
// O = gate * sum_s 2^(lse_s - LSE) o_s with LSE = log2 sum_s 2^lse_s, over the
// splits that hold keys for the row's tile, in order (reproducible).  Lane s
// reads split s's log-sum-exp.
__global__ void __launch_bounds__(256)
prefill_combine_kernel(UnitGeom u, int nsplit, const float* __restrict__ part, const int32_t* __restrict__ part_rows,
                       __nv_bfloat16* __restrict__ O) {
    const int lane = threadIdx.x & 31;
    const int64_t row = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;  // (unit * kQT + t) * kBM + r
    if (row >= u.count() * kQT * kBM) return;
    const int32_t* pr = part_rows + row * 3;
    const int t_row = pr[0];
    if (t_row < 0) return;  // padding
    const int j_row = pr[1];
    const float gate = __int_as_float(pr[2]);
    const int64_t unit = row / (kQT * kBM);
    const int64_t tr = row % (kQT * kBM);
    const int t = (int)(tr / kBM);
    const float* recs = part + (unit * nsplit * (kQT * kBM) + tr) * kPartFloats;
    const int64_t rstride = (int64_t)kQT * kBM * kPartFloats;  // next split, same row
    float ls = -INFINITY;
    if (lane < nsplit) {
        int64_t un;
        int sp, b, q, w, kv_lo, cnt[kQT];
        item_range(u, nsplit, unit * nsplit + lane, un, sp, b, q, w, kv_lo, cnt);
        if (cnt[t] > 0) ls = recs[lane * rstride + kD];
    }
    float m = ls;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, d));
    const float wl = (ls == -INFINITY) ? 0.f : fast_exp2(ls - m);
    float L = wl;
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) L += __shfl_xor_sync(0xffffffffu, L, d);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp = 0; sp < nsplit; ++sp) {
        const float wt = __shfl_sync(0xffffffffu, wl, sp);
        if (wt == 0.f) continue;
        const float4 v = reinterpret_cast<const float4*>(recs + sp * rstride)[lane];
        acc.x += wt * v.x;
        acc.y += wt * v.y;
        acc.z += wt * v.z;
        acc.w += wt * v.w;
    }
    const float inv = 1.0f / L;
    const float4 o = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    int b, q, w;
    unit_coords(u, unit, b, q, w);
    const int64_t orow = ((int64_t)b * u.T + t_row) * u.h + j_row;
    reinterpret_cast<uint2*>(O + orow * kD)[lane] =
        make_uint2(pack_bf16x2(gate * o.x, gate * o.y), pack_bf16x2(gate * o.z, gate * o.w));
}

UnitGeom prefill_geom(const gqe_shape& s) {
    UnitGeom u;
    u.B = s.B; u.T = s.T; u.h = s.h; u.g = s.g; u.k = s.k; u.hpg = s.h / s.g;
    u.W = 32 * (4 / s.k);  // k*W <= 128 rows per tile, W a multiple of the 32-token chunk
    u.nwin = (s.T + kQT * u.W - 1) / (kQT * u.W);
    u.nchunk = gqe_chunk_count(s.T);
    return u;
}

// Splits per unit: 1 unless the units would leave at least half of the SMs
// idle (measured on the shared head: 128 units on 148 SMs ran 16 % slower
// split, 32 and 64 units 8 % and 1.7x faster), else enough for about two
// items per SM, with at least two KV tiles per split of the longest unit (an
// item's fixed cost, its row table and Q tiles, is a few KV tiles' worth), at
// most 16 (the merge reads one split per lane, at most 32).
int prefill_splits(const UnitGeom& u, int sms) {
    const int64_t units = u.count(), target = 2 * (int64_t)sms;
    if (units <= 0 || 2 * units > sms) return 1;
    int64_t sp = (target + units - 1) / units;
    const int n_max = tile_kv_tiles(u, u.nwin - 1, kQT - 1);
    if (sp > n_max / 2) sp = n_max / 2;
    if (sp > 16) sp = 16;
    return sp < 1 ? 1 : (int)sp;
}

size_t a256b(size_t n) { return (n + 255) & ~size_t(255); }
size_t split_part_bytes(const UnitGeom& u, int nsplit) {
    return a256b((size_t)u.count() * nsplit * kQT * kBM * kPartFloats * sizeof(float));
}
size_t split_rows_bytes(const UnitGeom& u) { return a256b((size_t)u.count() * kQT * kBM * 3 * sizeof(int32_t)); }

int device_sms() {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) != cudaSuccess) return sms;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return sms;
}

}  // namespace

size_t prefill_split_bytes(const gqe_shape* s) {
    if (s->dtype != GQE_BF16 || s->d_h != kD || s->k > 4 || s->h / s->g > 32) return 0;
    const UnitGeom u = prefill_geom(*s);
    const int sp = prefill_splits(u, device_sms());
    return sp > 1 ? split_part_bytes(u, sp) + split_rows_bytes(u) : 0;
}

cudaError_t launch_prefill_tc(const PrefillArgs& a) {
    const gqe_shape& s = *a.s;
    if (s.k > 4 || s.h / s.g > 32) return cudaErrorNotSupported;
    const UnitGeom u = prefill_geom(s);

    // The setmaxnreg split needs exactly kRegsLaunch registers per thread at
    // launch (a property of the compiled kernel: checked once per process).
    static std::atomic<int> regs_checked{0};
    if (regs_checked.load(std::memory_order_acquire) == 0) {
        cudaFuncAttributes fa, fb, fc;
        cudaError_t e = cudaFuncGetAttributes(&fa, prefill_tc_kernel<false, false>);
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fb, prefill_tc_kernel<true, false>);
        if (e == cudaSuccess) e = cudaFuncGetAttributes(&fc, prefill_tc_kernel<false, true>);
        if (e != cudaSuccess) return e;
        const bool all = fa.numRegs == kRegsLaunch && fb.numRegs == kRegsLaunch && fc.numRegs == kRegsLaunch;
        regs_checked.store(all ? 1 : -1, std::memory_order_release);
    }
    if (regs_checked.load(std::memory_order_acquire) != 1) return cudaErrorNotSupported;

    CUtensorMap mapK, mapV;
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)a.kv_g, (uint64_t)s.T, (uint64_t)s.B};
    const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)a.kv_g * kD * 2, (uint64_t)s.T * a.kv_g * kD * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)kBN, 1};
    if (!make_bf16_map(&mapK, a.K, 4, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_bf16_map(&mapV, a.V, 4, dims, strides, box)) return cudaErrorInvalidValue;
    CUtensorMap mapQ;
    const int64_t q_rows = (int64_t)s.B * s.T * s.h;
    if (q_rows >= ((int64_t)1 << 31) - 1) return cudaErrorNotSupported;
    {
        const uint64_t qdims[2] = {(uint64_t)kD, (uint64_t)q_rows};
        const uint64_t qstrides[1] = {(uint64_t)kD * 2};
        const uint32_t qbox[2] = {64, 1};
        if (!make_bf16_map(&mapQ, a.Q, 2, qdims, qstrides, qbox)) return cudaErrorInvalidValue;
    }
    CUtensorMap mapQB;  // Q as [B, T, h, 128]: one head's W consecutive tokens per box
    {
        const uint64_t qdims[4] = {(uint64_t)kD, (uint64_t)s.h, (uint64_t)s.T, (uint64_t)s.B};
        const uint64_t qstrides[3] = {(uint64_t)kD * 2, (uint64_t)s.h * kD * 2, (uint64_t)s.T * s.h * kD * 2};
        const uint32_t qbox[4] = {64, 1, (uint32_t)u.W, 1};
        if (!make_bf16_map(&mapQB, a.Q, 4, qdims, qstrides, qbox)) return cudaErrorInvalidValue;
    }

    Params p;
    p.u = u;
    p.Q = (const __nv_bfloat16*)a.Q;
    p.idx = a.idx;
    p.gate = a.gate;
    p.head_offsets = a.head_offsets;
    p.head_pos = a.head_pos;
    p.head_chunk_offsets = a.head_chunk_offsets;
    p.O = (__nv_bfloat16*)a.O;
    p.o32 = a.o32;
    p.lse = a.lse;
    p.status = (uint32_t*)a.status;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);
    p.q_rows = (int)q_rows;
    p.kv_q0 = a.kv_q0;

    const int sms = device_sms();
    // Split-KV when the units leave SMs idle and the caller's scratch holds the
    // partials (inference only: the training outputs come from one pass).
    p.nsplit = 1;
    p.part = nullptr;
    p.part_rows = nullptr;
    if (a.split_scratch != nullptr && a.o32 == nullptr && a.O != nullptr) {
        const int sp = prefill_splits(u, sms);
        if (sp > 1 && a.split_bytes >= split_part_bytes(u, sp) + split_rows_bytes(u)) {
            p.nsplit = sp;
            p.part = static_cast<float*>(a.split_scratch);
            p.part_rows = reinterpret_cast<int32_t*>(static_cast<char*>(a.split_scratch) + split_part_bytes(u, sp));
        }
    }
    const int64_t units = u.count() * p.nsplit;
    const int grid = (int)(units < sms ? units : sms);
    const size_t smem = sizeof(Smem) + 1024;
    const bool train = a.o32 != nullptr;
    auto kern = train ? prefill_tc_kernel<true, false>
                      : (p.nsplit > 1 ? prefill_tc_kernel<false, true> : prefill_tc_kernel<false, false>);
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = a.stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, kern, mapK, mapV, mapQ, mapQB, p);
    if (err != cudaSuccess || p.nsplit == 1) return err;
    const int64_t rows = u.count() * kQT * kBM;
    prefill_combine_kernel<<<(unsigned)((rows * 32 + 255) / 256), 256, 0, a.stream>>>(
        u, p.nsplit, p.part, p.part_rows, (__nv_bfloat16*)a.O);
    return cudaGetLastError();
}

}  // namespace gqe
