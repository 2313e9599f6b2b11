// prefill_tc.cu -- routed causal flash attention (bf16, d_h = 128) on the
// sm_100a tensor cores, with the gated zero-filling scatter epilogue.
//
// What it computes (gist.science GQE summary, "Architecture et Routage" and
// "Construction de la Sortie"; IBM GQA page, scaled dot-product attention;
// ml-canon "56 GQA / MQA", shared KV heads): for every routed (b, t, j)
//   O[b,t,j,:] = gate * sum_{s<=t} softmax_s(Q[b,t,j] . K[b,s,j/hpg] / sqrt(128)) V[b,s,j/hpg]
// and O[b,t,j,:] = 0 for the unselected (t, j).
//
// Work unit: (b, KV group q, window of W = 128/k.. positions), whose k*W routed
// rows (from the per-head packed position lists) form one M=128 tile.  Each
// K/V tile of group q is loaded once per unit by TMA and used by every routed
// head of the group in that window.
//
// Roles (256 threads, one persistent CTA per SM):
//   warp 0      TMA producer for K/V tiles; owns the TMEM allocation
//   warp 1      MMA issuer (one thread): S = Q K^T and O += P V on tcgen05
//   warp 2      row table and Q gather (cp.async, 128B-swizzled)
//   warp 3      zero fill of the window's unselected output slots
//   warps 4-7   softmax (one row per thread, S read from TMEM, P written back
//               to TMEM as bf16) and the gated epilogue
// TMEM columns: S0 [0,128) S1 [128,256) O [256,384) P0 [384,448) P1 [448,512).
#include <climits>

#include "sm100.cuh"
#include "tma_host.cuh"
#include "units.cuh"

namespace gqe {
namespace {

using namespace sm100;

constexpr int kD = 128;          // head width
constexpr int kBM = 128;         // routed rows per unit (UMMA M)
constexpr int kBN = 128;         // keys per KV tile (UMMA N of S, K of P.V)
constexpr int kThreads = 256;
constexpr uint32_t kHalf = 128 * 64 * 2;   // one [128][64] bf16 box, 16 KB
constexpr uint32_t kTileBytes = 2 * kHalf; // [128][128] bf16, 32 KB
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS0 = 0, kColO = 256, kColP0 = 384;
constexpr float kRescaleThreshold = 8.0f;  // log2 units: p <= 2^8 between rescales
constexpr uint32_t kWhereTc = 2;           // status "where" id of this kernel

struct Smem {
    uint8_t q[2][kTileBytes];
    uint8_t k[2][kTileBytes];
    uint8_t v[2][kTileBytes];
    int32_t row_t[2][kBM];
    int32_t row_j[2][kBM];
    float row_gate[2][kBM];
    int32_t nrows[2];
    int32_t cut_start[2][32];
    int32_t cut_prefix[2][33];
    uint64_t kv_full_k[2], kv_full_v[2], kv_empty_k[2], kv_empty_v[2];
    uint64_t s_full[2], p_full[2], pv_done[2];
    uint64_t q_full[2], q_empty[2], rows_free[2];
    uint64_t o_full, o_empty, mma_drain;
    uint32_t tmem_base;
    int32_t abort_flag;
};

struct Params {
    UnitGeom u;
    const __nv_bfloat16* Q;
    const int32_t* idx;
    const float* gate;
    const int32_t* head_offsets;
    const int32_t* head_pos;
    const int32_t* head_chunk_offsets;
    __nv_bfloat16* O;
    uint32_t* status;
    float scale_log2;
};

__device__ __forceinline__ int unit_kv_tiles(const UnitGeom& u, int w) {
    const int end = min((w + 1) * u.W, u.T);  // keys 0 .. end-1
    return (end + kBN - 1) / kBN;
}

__device__ __forceinline__ bool aborted(Smem& sm) { return *((volatile int32_t*)&sm.abort_flag) != 0; }

__device__ __forceinline__ void fail(Smem& sm, const Params& p, uint32_t detail) {
    atomicExch(&sm.abort_flag, 1);
    report_error(p.status, GQE_ERR_DEVICE_TIMEOUT, kWhereTc, detail);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

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
__global__ void __launch_bounds__(kThreads, 1)
prefill_tc_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                  const Params p) {
    extern __shared__ uint8_t smem_raw[];
    Smem& sm = *reinterpret_cast<Smem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const UnitGeom& u = p.u;
    const int64_t n_units = u.count();

    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&sm.kv_full_k[i], 1);
            mbar_init(&sm.kv_full_v[i], 1);
            mbar_init(&sm.kv_empty_k[i], 1);
            mbar_init(&sm.kv_empty_v[i], 1);
            mbar_init(&sm.s_full[i], 1);
            mbar_init(&sm.p_full[i], 128);
            mbar_init(&sm.pv_done[i], 1);
            mbar_init(&sm.q_full[i], 32);
            mbar_init(&sm.q_empty[i], 1);
            mbar_init(&sm.rows_free[i], 128);
        }
        mbar_init(&sm.o_full, 1);
        mbar_init(&sm.o_empty, 128);
        mbar_init(&sm.mma_drain, 1);
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

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            uint32_t kv_it = 0;
            for (int64_t unit = blockIdx.x; unit < n_units && !aborted(sm); unit += gridDim.x) {
                int b, q, w;
                unit_coords(u, unit, b, q, w);
                const int n = unit_kv_tiles(u, w);
                for (int i = 0; i < n; ++i, ++kv_it) {
                    const int st = kv_it & 1;
                    const uint32_t par = ((kv_it >> 1) & 1) ^ 1;
                    if (!mbar_wait(&sm.kv_empty_k[st], par)) { fail(sm, p, 1); break; }
                    mbar_arrive_expect_tx(&sm.kv_full_k[st], kTileBytes);
                    tma_load_4d(&mapK, &sm.kv_full_k[st], sm.k[st], 0, q, i * kBN, b);
                    tma_load_4d(&mapK, &sm.kv_full_k[st], sm.k[st] + kHalf, 64, q, i * kBN, b);
                    if (!mbar_wait(&sm.kv_empty_v[st], par)) {
                        fail(sm, p, 2);
                        mbar_wait(&sm.kv_full_k[st], (kv_it >> 1) & 1);
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.kv_full_v[st], kTileBytes);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st], 0, q, i * kBN, b);
                    tma_load_4d(&mapV, &sm.kv_full_v[st], sm.v[st] + kHalf, 64, q, i * kBN, b);
                }
            }
            // Drain: every issued load lands before the CTA may exit.
            for (uint32_t back = 1; back <= 2 && back <= kv_it; ++back) {
                const uint32_t it = kv_it - back;
                mbar_wait(&sm.kv_full_k[it & 1], (it >> 1) & 1);
                mbar_wait(&sm.kv_full_v[it & 1], (it >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(kBM, kBN, false, false);
            const uint32_t idesc_pv = idesc_bf16_f32(kBM, kD, false, true);
            uint32_t kv_it = 0, u_it = 0;
            bool ok = true;
            auto issue_pv = [&](uint32_t it, bool first) -> bool {
                const int sb = it & 1;
                if (!mbar_wait(&sm.p_full[sb], (it >> 1) & 1)) return false;
                if (!mbar_wait(&sm.kv_full_v[sb], (it >> 1) & 1)) return false;
                tc_fence_after();
                const uint32_t vaddr = smem_u32(sm.v[sb]);
                for (int kk = 0; kk < kBN / 16; ++kk) {
                    const uint64_t bdesc = smem_desc(vaddr + kk * 2048, kHalf, 1024, kSwizzle128B);
                    umma_ts(tmem + kColO, tmem + kColP0 + sb * 64 + kk * 8, bdesc, idesc_pv,
                            (first && kk == 0) ? 0u : 1u);
                }
                umma_commit(&sm.kv_empty_v[sb]);
                umma_commit(&sm.pv_done[sb]);
                return true;
            };
            for (int64_t unit = blockIdx.x; unit < n_units && ok && !aborted(sm); unit += gridDim.x, ++u_it) {
                int b, q, w;
                unit_coords(u, unit, b, q, w);
                const int n = unit_kv_tiles(u, w);
                const int qs = u_it & 1;
                if (!mbar_wait(&sm.q_full[qs], (u_it >> 1) & 1)) { fail(sm, p, 10); ok = false; break; }
                tc_fence_after();
                const uint32_t qaddr = smem_u32(sm.q[qs]);
                for (int i = 0; i < n; ++i, ++kv_it) {
                    const int st = kv_it & 1;
                    if (!mbar_wait(&sm.kv_full_k[st], (kv_it >> 1) & 1)) { fail(sm, p, 11); ok = false; break; }
                    tc_fence_after();
                    const uint32_t kaddr = smem_u32(sm.k[st]);
                    for (int kk = 0; kk < kD / 16; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
                        const uint64_t adesc = smem_desc(qaddr + off, 16, 1024, kSwizzle128B);
                        const uint64_t bdesc = smem_desc(kaddr + off, 16, 1024, kSwizzle128B);
                        umma_ss(tmem + kColS0 + st * 128, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&sm.kv_empty_k[st]);
                    umma_commit(&sm.s_full[st]);
                    if (i == n - 1) umma_commit(&sm.q_empty[qs]);
                    if (i >= 1) {
                        if (i == 1 && !mbar_wait(&sm.o_empty, (u_it & 1) ^ 1)) { fail(sm, p, 12); ok = false; break; }
                        if (!issue_pv(kv_it - 1, i == 1)) { fail(sm, p, 13); ok = false; break; }
                    }
                }
                if (!ok) break;
                if (n == 1 && !mbar_wait(&sm.o_empty, (u_it & 1) ^ 1)) { fail(sm, p, 14); break; }
                if (!issue_pv(kv_it - 1, n == 1)) { fail(sm, p, 15); break; }
                umma_commit(&sm.o_full);
            }
            // Drain: all issued MMAs complete before TMEM is released.
            umma_commit(&sm.mma_drain);
            mbar_wait(&sm.mma_drain, 0);
        }
    } else if (warp == 2) {
        // ------------------------------------------------------------ row table + Q gather
        uint32_t u_it = 0;
        for (int64_t unit = blockIdx.x; unit < n_units && !aborted(sm); unit += gridDim.x, ++u_it) {
            int b, q, w;
            unit_coords(u, unit, b, q, w);
            const int qs = u_it & 1;
            const uint32_t par = ((u_it >> 1) & 1) ^ 1;
            bool ok = mbar_wait(&sm.q_empty[qs], par);
            ok = ok && mbar_wait(&sm.rows_free[qs], par);
            if (!__all_sync(0xffffffffu, ok)) { if (lane == 0) fail(sm, p, 20); break; }
            const int w0 = w * u.W;
            // 1. per-head slices of the window in the packed position lists
            if (lane < u.hpg) {
                const int j = q * u.hpg + lane;
                const int32_t total = (int32_t)((int64_t)u.B * u.T * u.g * u.k);
                int32_t a0 = list_cut(u, p.head_offsets, p.head_chunk_offsets, b, j, w0);
                int32_t a1 = list_cut(u, p.head_offsets, p.head_chunk_offsets, b, j, w0 + u.W);
                if (a0 < 0 || a1 < a0 || a1 > total) {  // malformed lists: report, use none
                    report_error(p.status, GQE_ERR_INVALID_ARGUMENT, kWhereTc, 41);
                    a0 = a1 = 0;
                }
                sm.cut_start[qs][lane] = a0;
                sm.cut_prefix[qs][lane + 1] = a1 - a0;
            }
            __syncwarp();
            if (lane == 0) {
                int acc = 0;
                sm.cut_prefix[qs][0] = 0;
                for (int jj = 0; jj < u.hpg; ++jj) {
                    acc += sm.cut_prefix[qs][jj + 1];
                    sm.cut_prefix[qs][jj + 1] = acc;
                }
                sm.nrows[qs] = min(acc, kBM);
            }
            __syncwarp();
            const int nrows = sm.nrows[qs];
            // 2. row table: position, head and gate of each routed row
            for (int r = lane; r < kBM; r += 32) {
                int t = -1, j = 0;
                float gv = 0.f;
                if (r < nrows) {
                    int jj = 0;
                    while (sm.cut_prefix[qs][jj + 1] <= r) ++jj;
                    j = q * u.hpg + jj;
                    t = p.head_pos[sm.cut_start[qs][jj] + (r - sm.cut_prefix[qs][jj])];
                    if (t < w0 || t >= min(w0 + u.W, u.T)) {  // outside the window: report, drop the row
                        report_error(p.status, GQE_ERR_INVALID_ARGUMENT, kWhereTc, 40);
                        t = -1;
                    } else {
                        const int64_t sel = (((int64_t)b * u.T + t) * u.g + q) * u.k;
                        for (int s = 0; s < u.k; ++s)
                            if (p.idx[sel + s] == j) gv = p.gate[sel + s];
                    }
                }
                sm.row_t[qs][r] = t;
                sm.row_j[qs][r] = j;
                sm.row_gate[qs][r] = gv;
            }
            __syncwarp();
            // 3. Q gather: row r, 16-byte chunk c -> half c/8, 128B-swizzled slot
            const uint32_t qbase = smem_u32(sm.q[qs]);
            for (int e = lane; e < kBM * 16; e += 32) {
                const int r = e >> 4, c = e & 15;
                const int t = sm.row_t[qs][r];
                const int j = sm.row_j[qs][r];
                const uint32_t dst = qbase + (c >> 3) * kHalf + r * 128 + (((c & 7) ^ (r & 7)) << 4);
                const __nv_bfloat16* src =
                    (t >= 0) ? p.Q + (((int64_t)b * u.T + t) * u.h + j) * kD + c * 8 : p.Q;
                cp_async16(dst, src, t >= 0 ? 16u : 0u);
            }
            cp_async_wait_all();
            fence_proxy_async_smem();
            mbar_arrive(&sm.q_full[qs]);
        }
    } else if (warp == 3) {
        // ------------------------------------------------------------ zero fill of unselected slots
        // Each unit's window [w0, w0+W) x heads of group q: slots whose head the
        // token did not select are written as zeros (16 lanes per 256-byte slot).
        for (int64_t unit = blockIdx.x; unit < n_units && !aborted(sm); unit += gridDim.x) {
            int b, q, w;
            unit_coords(u, unit, b, q, w);
            const int w0 = w * u.W;
            const int wend = min(w0 + u.W, u.T);
            const int slots = (wend - w0) * u.hpg;
            for (int e = lane >> 4; e < slots; e += 2) {
                const int t = w0 + e / u.hpg;
                const int j = q * u.hpg + e % u.hpg;
                const int64_t sel = (((int64_t)b * u.T + t) * u.g + q) * u.k;
                bool hit = false;
                for (int s = 0; s < u.k; ++s) hit |= (p.idx[sel + s] == j);
                if (!hit) {
                    uint4* o = reinterpret_cast<uint4*>(p.O + (((int64_t)b * u.T + t) * u.h + j) * kD);
                    o[lane & 15] = make_uint4(0, 0, 0, 0);
                }
            }
        }
    } else {
        // ------------------------------------------------------------ softmax + epilogue
        const int wq = warp & 3;           // TMEM lane quarter of this warp
        const int r = wq * 32 + lane;      // routed row owned by this thread
        const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
        uint32_t kv_it = 0, u_it = 0;
        for (int64_t unit = blockIdx.x; unit < n_units && !aborted(sm); unit += gridDim.x, ++u_it) {
            int b, q, w;
            unit_coords(u, unit, b, q, w);
            const int n = unit_kv_tiles(u, w);
            const int qs = u_it & 1;
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.q_full[qs], (u_it >> 1) & 1))) { if (lane == 0) fail(sm, p, 30); break; }
            const int t_row = sm.row_t[qs][r];
            const int t_eff = (t_row >= 0) ? t_row : INT_MAX;  // padding rows: unmasked, output dropped
            const int w0 = w * u.W;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int i = 0; i < n; ++i, ++kv_it) {
                const int sb = kv_it & 1;
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.s_full[sb], (kv_it >> 1) & 1))) { if (lane == 0) fail(sm, p, 31); ok = false; break; }
                tc_fence_after();
                uint32_t s[4][32];
                const uint32_t sa = tmem + lane_off + kColS0 + sb * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32(sa + c * 32, s[c]);
                ld_wait_bind(s[0]);
                ld_bind(s[1]);
                ld_bind(s[2]);
                ld_bind(s[3]);
                const int kv0 = i * kBN;
                const bool need_mask = kv0 + kBN - 1 > w0;
                float mx = -INFINITY;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        float v = __uint_as_float(s[c][e]) * p.scale_log2;
                        if (need_mask && kv0 + c * 32 + e > t_eff) v = -INFINITY;
                        s[c][e] = __float_as_uint(v);
                        mx = fmaxf(mx, v);
                    }
                }
                // Lazy rescaling: keep the running max unless it grows by more than the threshold.
                float m_use = m;
                bool rescale = false;
                if (mx > m + kRescaleThreshold || m == -INFINITY) {
                    m_use = mx;
                    rescale = (i > 0);
                }
                // P buffer sb is free once P.V of tile kv_it-2 is done.
                if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[sb], ((kv_it >> 1) & 1) ^ 1))) { if (lane == 0) fail(sm, p, 32); ok = false; break; }
                float rowsum = 0.f;
                const uint32_t pa = tmem + lane_off + kColP0 + sb * 64;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float p0 = fast_exp2(__uint_as_float(s[c][2 * e]) - m_use);
                        const float p1 = fast_exp2(__uint_as_float(s[c][2 * e + 1]) - m_use);
                        rowsum += p0 + p1;
                        pk[e] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(pa + c * 16, pk);
                }
                if (__any_sync(0xffffffffu, rescale)) {
                    // O holds P.V of tiles < i once P.V of tile kv_it-1 is done.
                    const uint32_t prev = kv_it - 1;
                    if (!__all_sync(0xffffffffu, mbar_wait(&sm.pv_done[prev & 1], (prev >> 1) & 1))) { if (lane == 0) fail(sm, p, 33); ok = false; break; }
                    tc_fence_after();
                    const float alpha = rescale ? fast_exp2(m - m_use) : 1.0f;
                    const uint32_t oa = tmem + lane_off + kColO;
#pragma unroll 1
                    for (int c = 0; c < 4; ++c) {
                        uint32_t o[32];
                        tmem_ld32(oa + c * 32, o);
                        ld_wait_bind(o);
#pragma unroll
                        for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                        tmem_st16(oa + c * 32, *reinterpret_cast<uint32_t(*)[16]>(&o[0]));
                        tmem_st16(oa + c * 32 + 16, *reinterpret_cast<uint32_t(*)[16]>(&o[16]));
                    }
                    l *= alpha;
                }
                l += rowsum;
                m = m_use;
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&sm.p_full[sb]);
            }
            if (!ok) break;
            // Epilogue: O / l * gate -> bf16 row of O[b, t, j, :].
            if (!__all_sync(0xffffffffu, mbar_wait(&sm.o_full, u_it & 1))) { if (lane == 0) fail(sm, p, 34); break; }
            tc_fence_after();
            const int j_row = sm.row_j[qs][r];
            const float f = (t_row >= 0) ? sm.row_gate[qs][r] / l : 0.f;
            __nv_bfloat16* orow = p.O + (((int64_t)b * u.T + (t_row >= 0 ? t_row : 0)) * u.h + j_row) * kD;
            const uint32_t oa = tmem + lane_off + kColO;
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                uint32_t o[32];
                tmem_ld32(oa + c * 32, o);
                ld_wait_bind(o);
                if (t_row >= 0) {
                    uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
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
            mbar_arrive(&sm.o_empty);
            mbar_arrive(&sm.rows_free[qs]);
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

}  // namespace

cudaError_t launch_prefill_tc(const PrefillArgs& a) {
    const gqe_shape& s = *a.s;
    if (s.k > 4 || s.h / s.g > 32) return cudaErrorNotSupported;
    UnitGeom u;
    u.B = s.B; u.T = s.T; u.h = s.h; u.g = s.g; u.k = s.k; u.hpg = s.h / s.g;
    u.W = 32 * (4 / s.k);  // k*W <= 128 rows, W a multiple of the 32-token chunk
    u.nwin = (s.T + u.W - 1) / u.W;
    u.nchunk = gqe_chunk_count(s.T);

    CUtensorMap mapK, mapV;
    const uint64_t dims[4] = {(uint64_t)kD, (uint64_t)s.g, (uint64_t)s.T, (uint64_t)s.B};
    const uint64_t strides[3] = {(uint64_t)kD * 2, (uint64_t)s.g * kD * 2, (uint64_t)s.T * s.g * kD * 2};
    const uint32_t box[4] = {64, 1, (uint32_t)kBN, 1};
    if (!make_bf16_map(&mapK, a.K, 4, dims, strides, box)) return cudaErrorInvalidValue;
    if (!make_bf16_map(&mapV, a.V, 4, dims, strides, box)) return cudaErrorInvalidValue;

    Params p;
    p.u = u;
    p.Q = (const __nv_bfloat16*)a.Q;
    p.idx = a.idx;
    p.gate = a.gate;
    p.head_offsets = a.head_offsets;
    p.head_pos = a.head_pos;
    p.head_chunk_offsets = a.head_chunk_offsets;
    p.O = (__nv_bfloat16*)a.O;
    p.status = (uint32_t*)a.status;
    p.scale_log2 = 1.4426950408889634f / sqrtf((float)kD);

    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t units = u.count();
    const int grid = (int)(units < sms ? units : sms);
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t err = cudaFuncSetAttribute(prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (err != cudaSuccess) return err;
    prefill_tc_kernel<<<grid, kThreads, smem, a.stream>>>(mapK, mapV, p);
    return cudaGetLastError();
}

}  // namespace gqe
