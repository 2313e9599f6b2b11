// units.cuh -- work units of the routed prefill.
//
// A unit is (batch b, KV group q, window of W consecutive positions [w0, w0+W)).
// Every token selects exactly k heads of every group, so a full window holds
// exactly k*W routed rows (t, j) whatever the router's skew: the grid is
// static.  The rows are the concatenation, over the group's heads, of each
// head's slice of its packed position list (compaction output) that falls in
// the window.  The unit also owns the zero-fill of the window's unselected
// (t, j) output slots, so the units tile O exactly.
#pragma once

#include "common.cuh"

namespace gqe {

struct UnitGeom {
    int B, T, h, g, k, hpg, W, nwin, nchunk;
    __host__ __device__ int64_t count() const { return (int64_t)B * g * nwin; }
};

// Unit order: heaviest windows (largest w0) first, so the causal triangle's
// long rows start early; within a window rank, (b, q) vary fastest.
__device__ __forceinline__ void unit_coords(const UnitGeom& u, int64_t unit, int& b, int& q, int& w) {
    const int64_t per_win = (int64_t)u.B * u.g;
    const int wr = (int)(unit / per_win);
    const int rem = (int)(unit % per_win);
    w = u.nwin - 1 - wr;
    b = rem / u.g;
    q = rem % u.g;
}

// Start index in head_pos of head j's entries with t >= w0 (w0 a multiple of 32),
// or the end of its list when w0 >= T.
__device__ __forceinline__ int32_t list_cut(const UnitGeom& u, const int32_t* head_offsets,
                                            const int32_t* head_chunk_offsets, int b, int j, int w0) {
    const int c = w0 / kChunk;
    if (c >= u.nchunk) return head_offsets[(int64_t)b * u.h + j + 1];
    return head_chunk_offsets[((int64_t)b * u.h + j) * u.nchunk + c];
}

}  // namespace gqe
