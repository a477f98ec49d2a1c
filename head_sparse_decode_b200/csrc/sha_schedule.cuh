// sha_schedule.cuh -- how one call's work is cut across thread blocks.
//
// The work of a call is B*top_k units (one per selected (batch row, head));
// each unit's N_kv keys are cut into tiles of kTile keys (the last one
// partial, as in the pages' tiling of Algorithm 1, "Selective Head Flash
// Attention (Decode)": kend = min(j*Bc, N_kv)).  All tiles of all units are
// numbered unit-major, t = unit*tiles_per_unit + j, and the range [0, total)
// is cut into num_ctas contiguous pieces of equal size (to within one tile),
// one per thread block.  Every block therefore streams the same number of
// K/V bytes whatever B, top_k and N_kv are.  A unit whose tiles fall in more
// than one piece is finished by a log-sum-exp merge of the pieces' partial
// (m, l, O) states (see the kernels).  When units are only a few tiles long
// the merges cost more than an uneven cut, and the host may instead cut at
// unit boundaries: whole units per block, or each unit in p equal pieces,
// or (the clustered cut) each unit in p pieces held by the p blocks of one
// thread-block cluster, which merge them in distributed shared memory.
//
// A unit split across blocks c_first..c_last is merged by whichever of them
// finishes last, found with an arrival counter.  Counter c_first belongs to
// it alone: a block can be the first of at most one split unit (two units
// starting inside one block's range would put the earlier one wholly inside
// it).  So one counter per block suffices, in a fixed-size region at the
// start of the workspace that only ever holds counters, whatever the shape
// of the call that used the workspace before.
//
// Everything here is integer arithmetic shared by the host planner and the
// device code, so both agree on every boundary.
#pragma once

#include <stdint.h>

namespace sha {

constexpr int kMaxBlocks = 4096;                       // cap on blocks of one call
constexpr int kCounterBytes = kMaxBlocks * 4;          // counter region, zero between calls

struct Schedule {
    int tiles_per_unit;      // ceil(N_kv / kTile)
    long long total_tiles;   // units * tiles_per_unit
    int num_ctas;            // 1 <= num_ctas <= total_tiles
    // 0: the tiles are cut evenly across the blocks, whatever the unit
    // boundaries.  p >= 1: each unit is cut into p equal pieces (by tiles) and
    // block c takes the whole pieces [c P / num_ctas, (c+1) P / num_ctas) of
    // the P = units * p pieces, so no block starts or ends inside a piece.
    int pieces;
    // >= 2: the clustered cut.  Blocks form thread-block clusters of this many;
    // cluster k takes the units [k * units_per_cluster, (k+1) * units_per_cluster).
    // The first cluster * whole_per_block of them go whole, whole_per_block to
    // each block in rank order; the block of rank r streams piece r of each of
    // the others (tiles [r * tiles_per_unit / cluster, (r+1) * tiles_per_unit /
    // cluster)), before its whole units, and the pieces meet in the cluster's
    // shared memory, not in the workspace.
    int cluster;
    int units_per_cluster;
    int whole_per_block;

    // First tile of piece i of the unit-aligned cut (pieces >= 1).
    __host__ __device__ __forceinline__ long long piece_start(long long i) const
    {
        const long long u = i / pieces;
        const long long k = i - u * pieces;
        return u * tiles_per_unit + k * tiles_per_unit / pieces;
    }
    // First tile of block c (c in [0, num_ctas]); begin(num_ctas) == total_tiles.
    __host__ __device__ __forceinline__ long long begin(int c) const
    {
        if (pieces == 0) return (long long)c * total_tiles / num_ctas;
        const long long P = total_tiles / tiles_per_unit * pieces;
        return piece_start((long long)c * P / num_ctas);
    }
    // The block whose range holds tile t: the largest c with begin(c) <= t.
    __host__ __device__ __forceinline__ int cta_of(long long t) const
    {
        if (pieces == 0) return (int)(((t + 1) * (long long)num_ctas - 1) / total_tiles);
        const long long P = total_tiles / tiles_per_unit * pieces;
        const long long u = t / tiles_per_unit, j = t - u * tiles_per_unit;
        // the last piece of the unit that starts at or before tile j
        const long long i = u * pieces + ((j + 1) * pieces - 1) / tiles_per_unit;
        return (int)(((i + 1) * (long long)num_ctas - 1) / P);
    }
    __host__ __device__ __forceinline__ long long unit_of(long long t) const
    {
        return t / tiles_per_unit;
    }
    // Partial-state slot of block c's piece of unit u.  A block holds at most
    // two pieces that are not whole units: the tail of the unit it starts in
    // (slot 2c) and the head of the unit it ends in (slot 2c+1).
    __host__ __device__ __forceinline__ int slot_of(int c, long long u) const
    {
        return 2 * c + (unit_of(begin(c)) == u ? 0 : 1);
    }
};

// One maximal run of a block's tiles that belongs to a single unit.
struct Segment {
    long long unit;
    int first_tile;   // tile index within the unit
    int num_tiles;
    bool whole;       // the run covers the whole unit
};

__host__ __device__ __forceinline__ Segment segment_at(const Schedule &s, long long t,
                                                       long long t_end)
{
    Segment seg;
    seg.unit = s.unit_of(t);
    long long unit_begin = seg.unit * s.tiles_per_unit;
    long long unit_end = unit_begin + s.tiles_per_unit;
    long long end = unit_end < t_end ? unit_end : t_end;
    seg.first_tile = (int)(t - unit_begin);
    seg.num_tiles = (int)(end - t);
    seg.whole = (t == unit_begin) && (end == unit_end);
    return seg;
}

}  // namespace sha
