// sha_walk.cuh -- how a block walks its tile range, unit by unit.
//
// Fixed length (every row has N_kv keys): the host plans the call (see
// sha_schedule.cuh) and a block's segments follow from integer arithmetic.
//
// Per-row lengths (row b attends to its first seqlens[b] keys, as in a decode
// batch whose sequences differ in length): the lengths live on the device, so
// each block plans for itself in its prologue.  One pass over seqlens gives
// the total tile count and the longest row; the tiles are then cut into
// equal contiguous ranges exactly as for fixed lengths, and a second pass (a
// block-wide prefix sum over rows) finds the row, slot and tile at which this
// block's range begins.  From there the walk only needs seqlens[b] of the
// rows it reaches.  Rows with a length outside [1, N_max] hold no tiles; they
// raise the bad-input flag and their outputs stay untouched.
#pragma once

#include "sha_device.cuh"
#include "sha_merge.cuh"
#include "sha_schedule.cuh"

namespace sha {

// One run of a block's tiles inside a single unit, with what the kernels need
// to know about that unit.
struct Seg {
    long long unit;        // b * top_k + k
    int first_tile;        // tile index within the unit
    int num_tiles;
    bool whole;            // the run is the whole unit
    long long unit_start;  // global index of the unit's first tile
    int unit_tiles;        // tiles of the unit
    int n_keys;            // keys of the unit (its row's length)
};

// Blocks first..last that share a unit, and the slot of block `first`'s part.
__device__ __forceinline__ void unit_parts(const Schedule &S, const Seg &seg, int &first,
                                           int &last, int &first_slot)
{
    first = S.cta_of(seg.unit_start);
    last = S.cta_of(seg.unit_start + seg.unit_tiles - 1);
    // the first block's part is its first unit only if its range starts there
    first_slot = 2 * first + (S.begin(first) == seg.unit_start ? 0 : 1);
}

struct UniformWalk {
    Schedule S;
    long long t, t_end;
    int n_keys;

    __device__ __forceinline__ bool next(Seg &s)
    {
        if (t >= t_end) return false;
        const Segment g = segment_at(S, t, t_end);
        s.unit = g.unit;
        s.first_tile = g.first_tile;
        s.num_tiles = g.num_tiles;
        s.whole = g.whole;
        s.unit_start = g.unit * S.tiles_per_unit;
        s.unit_tiles = S.tiles_per_unit;
        s.n_keys = n_keys;
        t += g.num_tiles;
        return true;
    }
};

// Clustered cut (Schedule::cluster >= 2): this block's piece of each unit the
// cluster shares, then its whole units.  Every block of a cluster visits the
// same shared units in the same order; taking them first lets their merges
// overlap the streaming of the whole units.
struct ClusterWalk {
    int tiles_per_unit, cluster, rank;
    long long s, s_end;           // the cluster's shared units
    long long u, u_end;           // this block's whole units
    int n_keys;

    __device__ __forceinline__ void start(const Schedule &S, long long units, int keys)
    {
        tiles_per_unit = S.tiles_per_unit;
        cluster = S.cluster;
        rank = (int)cluster_ctarank();
        const long long base = (long long)(blockIdx.x / S.cluster) * S.units_per_cluster;
        const long long end =
            base + S.units_per_cluster < units ? base + S.units_per_cluster : units;
        const long long shared0 = base + (long long)S.cluster * S.whole_per_block;
        u = base + (long long)rank * S.whole_per_block;
        u_end = u + S.whole_per_block;
        if (u_end > end) u_end = end;
        s = shared0 < end ? shared0 : end;
        s_end = end;
        n_keys = keys;
    }
    __device__ __forceinline__ bool next(Seg &g)
    {
        g.unit_tiles = tiles_per_unit;
        g.n_keys = n_keys;
        if (s < s_end) {
            const int j0 = rank * tiles_per_unit / cluster;
            const int j1 = (rank + 1) * tiles_per_unit / cluster;
            g.unit = s;
            g.first_tile = j0;
            g.num_tiles = j1 - j0;
            g.whole = false;
            g.unit_start = s * tiles_per_unit;
            ++s;
            return true;
        }
        if (u >= u_end) return false;
        g.unit = u;
        g.first_tile = 0;
        g.num_tiles = tiles_per_unit;
        g.whole = true;
        g.unit_start = u * tiles_per_unit;
        ++u;
        return true;
    }
};

__device__ __forceinline__ int varlen_tiles(int len, int n_max, int tile)
{
    return (len >= 1 && len <= n_max) ? (len + tile - 1) / tile : 0;
}

struct VarlenWalk {
    const int32_t *seqlens;
    int B, top_k, n_max, tile;
    long long t, t_end;
    int b, k, j, T, n;          // position: row, slot, tile in unit; row's tiles and keys
    long long unit_start;

    __device__ __forceinline__ bool next(Seg &s)
    {
        if (t >= t_end) return false;
        const long long left = t_end - t;
        const int run = (long long)(T - j) < left ? T - j : (int)left;
        s.unit = (long long)b * top_k + k;
        s.first_tile = j;
        s.num_tiles = run;
        s.whole = (j == 0 && run == T);
        s.unit_start = unit_start;
        s.unit_tiles = T;
        s.n_keys = n;
        t += run;
        j += run;
        if (j == T && t < t_end) {        // step to the next unit that has tiles
            j = 0;
            unit_start = t;
            if (++k == top_k) {
                k = 0;
                do {
                    ++b;
                    n = seqlens[b];
                    T = varlen_tiles(n, n_max, tile);
                } while (T == 0);
            }
        }
        return true;
    }
};

// Block-wide prologue for per-row lengths: fills S (total tiles, blocks in
// use), this block's range and the walk's starting position.  Every thread of
// the block calls it (it synchronises with __syncthreads).  Returns false if
// this block has nothing to do.  scratch: shared, >= 2 * (NT/32) + 8 longs.
template <int NT>
__device__ bool varlen_plan(const int32_t *seqlens, int B, int top_k, int n_max, int tile,
                            int max_blocks, long long *scratch, Schedule &S, VarlenWalk &w)
{
    constexpr int kWarps = NT / 32;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const unsigned FULL = 0xffffffffu;

    // pass 1: total tiles and the longest row (in tiles)
    long long sum = 0;
    int tmax = 0;
    for (int r = tid; r < B; r += NT) {
        const int len = seqlens[r];
        const int T = varlen_tiles(len, n_max, tile);
        if (T == 0 && blockIdx.x == 0) atomicOr(&g_sha_status, kStatusBadIndex);
        sum += (long long)top_k * T;
        tmax = max(tmax, T);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
        sum += __shfl_xor_sync(FULL, sum, off);
        tmax = max(tmax, __shfl_xor_sync(FULL, tmax, off));
    }
    if (lane == 0) {
        scratch[warp] = sum;
        scratch[kWarps + warp] = tmax;
    }
    __syncthreads();
    long long total = 0;
    int longest = 0;
    for (int i = 0; i < kWarps; ++i) {
        total += scratch[i];
        longest = max(longest, (int)scratch[kWarps + i]);
    }
    __syncthreads();
    if (total == 0) return false;

    // blocks in use: at most one per tile, and no unit shared by more than
    // kMaxMergeParts blocks
    long long ctas = max_blocks;
    if (ctas > total) ctas = total;
    const long long min_tiles = (longest - 1 + kMaxMergeParts - 2) / (kMaxMergeParts - 1);
    if (min_tiles > 1 && ctas > total / min_tiles) ctas = total / min_tiles;
    if (ctas < 1) ctas = 1;
    S.tiles_per_unit = 0;                  // units differ; the walk carries their size
    S.total_tiles = total;
    S.num_ctas = (int)ctas;
    S.pieces = 0;                          // tiles cut evenly
    if ((int)blockIdx.x >= S.num_ctas) return false;
    const long long t0 = S.begin(blockIdx.x);

    // pass 2: the row holding tile t0 (prefix sum over rows, NT rows at a time)
    long long base = 0;
    for (int r0 = 0; r0 < B; r0 += NT) {
        const int r = r0 + tid;
        const int len = r < B ? seqlens[r] : 0;
        const int T = r < B ? varlen_tiles(len, n_max, tile) : 0;
        const long long val = (long long)top_k * T;
        long long incl = val;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const long long x = __shfl_up_sync(FULL, incl, off);
            if (lane >= off) incl += x;
        }
        if (lane == 31) scratch[warp] = incl;
        __syncthreads();
        long long before = base, chunk = 0;
        for (int i = 0; i < kWarps; ++i) {
            if (i < warp) before += scratch[i];
            chunk += scratch[i];
        }
        const long long row_start = before + incl - val;
        if (val > 0 && row_start <= t0 && t0 < row_start + val) {
            const long long off = t0 - row_start;
            scratch[2 * kWarps + 0] = r;
            scratch[2 * kWarps + 1] = off / T;          // slot k
            scratch[2 * kWarps + 2] = off % T;          // tile j
            scratch[2 * kWarps + 3] = T;
            scratch[2 * kWarps + 4] = len;
            scratch[2 * kWarps + 5] = t0 - off % T;     // the unit's first tile
        }
        __syncthreads();
        base += chunk;
        if (base > t0) break;                           // the same for every thread
    }
    w.seqlens = seqlens;
    w.B = B;
    w.top_k = top_k;
    w.n_max = n_max;
    w.tile = tile;
    w.t = t0;
    w.t_end = S.begin(blockIdx.x + 1);
    w.b = (int)scratch[2 * kWarps + 0];
    w.k = (int)scratch[2 * kWarps + 1];
    w.j = (int)scratch[2 * kWarps + 2];
    w.T = (int)scratch[2 * kWarps + 3];
    w.n = (int)scratch[2 * kWarps + 4];
    w.unit_start = scratch[2 * kWarps + 5];
    __syncthreads();
    return true;
}

}  // namespace sha
