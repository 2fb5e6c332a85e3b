// grouped.cuh -- tile scheduling over variable-size expert groups.
//
// Group e owns rows [offsets[e], offsets[e+1]) of the grouped activations
// (the contiguous per-expert blocks input encode produces).  Its output tile
// grid is ceil(m_e / BM) x ceil(N / BN).  Every CTA builds the prefix of tile
// counts over groups in shared memory from the device-side offsets (no host
// round trip), then maps a linear tile index to (group, m-block, n-block),
// m-block fastest so that CTAs running side by side share one weight tile
// through L2.
#pragma once

#include "common.cuh"

namespace moe {

struct TileCoord {
    int e;       // group
    int row0;    // first row of the tile in the grouped activations
    int rows;    // valid rows in the tile (<= BM)
    int n0;      // first output column
};

// Group bounds: offsets[e], or a single group [0, single_M) when offsets is
// null (the gate projection is one group).
__device__ __forceinline__ int group_off(const int32_t* __restrict__ offsets, int e, int single_M) {
    return offsets ? offsets[e] : (e == 0 ? 0 : single_M);
}

// Which rows of each group a launch covers: all of them (PART_ALL), the whole
// kSplitRows-row blocks from the group's start (PART_BLOCKS), or the rows after
// the last whole block (PART_TAIL).  A dense grouped GEMM runs the blocks on
// 2-CTA 256-row tiles and the tails on 128-row tiles, so a group pads to 128
// rows instead of 256.
enum { PART_ALL = 0, PART_BLOCKS = 1, PART_TAIL = 2 };
constexpr int kSplitRows = 256;

// First row and row count of group e's part (groups with invalid bounds get no
// tiles from build_tile_table, so tile_coord never lands on them).
__device__ __forceinline__ void group_part(const int32_t* __restrict__ offsets, int e,
                                           int single_M, int part, int& a, int& m) {
    a = group_off(offsets, e, single_M);
    m = group_off(offsets, e + 1, single_M) - a;
    if (part == PART_BLOCKS) {
        m = (m / kSplitRows) * kSplitRows;
    } else if (part == PART_TAIL) {
        const int whole = (m / kSplitRows) * kSplitRows;
        a += whole;
        m -= whole;
    }
}

// Builds s_prefix[0..E] (exclusive prefix of tiles per group) with all threads
// of the block; returns the total tile count.  Invalid offsets (negative,
// decreasing, or beyond R_max) give that group no tiles and flag an error.
// s_prefix must hold E + 1 ints, s_warp 32 ints.  Must be called by every
// thread of the block (contains __syncthreads).
__device__ inline int build_tile_table(const int32_t* __restrict__ offsets, int single_M, int E,
                                       int nt, int BM, int R_max, int32_t* s_prefix,
                                       int32_t* s_warp, int32_t* err, int part = PART_ALL) {
    const int tid = threadIdx.x, nthr = blockDim.x;
    const int lane = tid & 31, wid = tid >> 5, nw = nthr >> 5;
    int carry = 0;
    for (int base = 0; base < E; base += nthr) {
        const int e = base + tid;
        int tiles = 0;
        if (e < E) {
            const int a = group_off(offsets, e, single_M), b = group_off(offsets, e + 1, single_M);
            if (a < 0 || b < a || b > R_max) {
                if (blockIdx.x == 0) flag_error(err, MOE_DEVERR_OFFSETS);
            } else {
                int pa, pm;
                group_part(offsets, e, single_M, part, pa, pm);
                tiles = ((pm + BM - 1) / BM) * nt;
            }
        }
        int incl = tiles;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int o = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += o;
        }
        if (lane == 31) s_warp[wid] = incl;
        __syncthreads();
        if (wid == 0) {
            int v = lane < nw ? s_warp[lane] : 0;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int o = __shfl_up_sync(0xffffffffu, v, off);
                if (lane >= off) v += o;
            }
            if (lane < nw) s_warp[lane] = v;
        }
        __syncthreads();
        const int before = carry + (wid > 0 ? s_warp[wid - 1] : 0) + incl - tiles;
        if (e < E) s_prefix[e] = before;
        carry += s_warp[nw - 1];
        __syncthreads();
    }
    if (tid == 0) s_prefix[E] = carry;
    __syncthreads();
    return carry;
}

// Maps a linear tile index to its coordinates, given the prefix of M-tiles per
// group (s_prefix from build_tile_table with nt = 1 and the same part) and nt
// N-tiles per group: group e owns tiles [nt * s_prefix[e], nt * s_prefix[e+1]),
// its M-tiles fastest.
__device__ __forceinline__ TileCoord tile_coord(int tile, const int32_t* s_prefix, int E,
                                                const int32_t* __restrict__ offsets, int single_M,
                                                int BM, int BN, int nt, int part = PART_ALL) {
    int lo = 0, hi = E - 1;  // largest e with nt * s_prefix[e] <= tile
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (nt * s_prefix[mid] <= tile) lo = mid; else hi = mid - 1;
    }
    const int e = lo;
    const int mt = s_prefix[e + 1] - s_prefix[e];
    const int local = tile - nt * s_prefix[e];
    const int mb = local % mt, nb = local / mt;
    int a, m;
    group_part(offsets, e, single_M, part, a, m);
    TileCoord c;
    c.e = e;
    c.row0 = a + mb * BM;
    c.rows = min(BM, m - mb * BM);
    c.n0 = nb * BN;
    return c;
}

}  // namespace moe
