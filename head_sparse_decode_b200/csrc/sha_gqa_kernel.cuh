// sha_gqa_kernel.cuh -- selective decode for grouped-query attention (G > 1),
// and for multi-head attention (G = 1) at d = 128 with one length per row.
//
// What one thread block does.  As in the multi-head kernel, it walks a
// contiguous range of key tiles (sha_schedule.cuh).  Here a unit is a batch
// row b and a selected KV group h (Polar Sparsity, papernotes.org summary,
// "Selective Head Attention (SHA) Kernel": GQA models select groups); all G
// query heads h*G .. h*G+G-1 of the group are computed from each K/V tile
// while it is in shared memory, so the group's cache is read from HBM once.
//
// How, on sm_100a.  With G query rows sharing every key, a tile is a small
// dense contraction (about G flops per byte: 8 for LLaMA-3.1-70B), so the
// scores and P.V run on the tensor cores with fp32 accumulation:
//   * one producer lane loads each K and V tile with TMA tensor copies
//     (cp.async.bulk.tensor, a 3-D map [planes = B*H_kv][N_kv][d] with
//     64-element boxes and 128-byte swizzle) into a kStages-deep ring; keys
//     past N_kv are outside the map and arrive as zeros;
//   * 4 consumer warps take 16 keys of every 64-key slice of a tile each and
//     keep their own online-softmax state for up to 16 query rows;
//   * S = Q K^T: mma.sync m16n8k16 with Q (G rows, zero-padded to 16) as the
//     A operand held in registers and K fragments read by ldmatrix from the
//     swizzled tile (conflict-free);
//   * P V: the S accumulators, exponentiated, are reused in registers as the
//     A operand (16 keys = one k-step); V fragments come from ldmatrix.trans;
//   * with G = 1, fifteen of the sixteen MMA rows are padding, yet the path
//     issues far fewer instructions per byte than the multi-head FMA kernel
//     and holds its speed under the power cap of a sustained load, so the host
//     sends multi-head calls with d = 128 and one length per row here;
//   * warps merge once per unit; units split across blocks merge in the
//     workspace exactly as in the multi-head kernel, and with G <= 8 the block
//     finishes the split unit it ends with on chip (sha_lookahead.cuh), its
//     parts kept in the rows G..15 that the warps' state areas leave free.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "sha_device.cuh"
#include "sha_lookahead.cuh"
#include "sha_merge.cuh"
#include "sha_mha_kernel.cuh"
#include "sha_mma.cuh"
#include "sha_schedule.cuh"
#include "sha_walk.cuh"

namespace sha {

// Build-time tuning of the grouped-query kernel (default measured best on B200).
#ifndef SHA_GQA_TILE_KEYS
#define SHA_GQA_TILE_KEYS 128
#endif
#ifndef SHA_GQA_STAGES
#define SHA_GQA_STAGES 3
#endif
#ifndef SHA_GQA_GATHER_WARPS
#define SHA_GQA_GATHER_WARPS 4
#endif

template <int D>
struct GqaConfig {
    static constexpr int kConsumerWarps = 4;
    static constexpr int kConsumers = kConsumerWarps * 32;
    static constexpr int kThreads = kConsumers + 32;   // + one producer warp
    // ... and a scout warp in the builds that finish a block's last unit on chip
    static constexpr int threads(bool look) { return kThreads + (look ? 32 : 0); }
    // A gathered layout (listed key positions) is copied by kGatherWarps
    // warps, each owning whole 32-row blocks of a tile: one warp's 16-byte
    // copies in flight reach only about 2.6 TB/s, four about 6 TB/s.  That
    // build has no scout warp (the register file holds 8 warps at this size).
    static constexpr int kGatherWarps = SHA_GQA_GATHER_WARPS;
    static constexpr int block_threads(bool look, bool gather)
    {
        return gather ? kThreads + 32 * (kGatherWarps - 1) : threads(look);
    }
    static constexpr int kTile = SHA_GQA_TILE_KEYS;    // keys per tile (one pipeline stage)
    static constexpr int kSlices = kTile / 64;         // 64-key slices per tile
    static constexpr int kKeysPerWarp = 64 / kConsumerWarps;      // 16 per slice: one m16n8k16 k-step
    static constexpr int kStages = SHA_GQA_STAGES;
    static constexpr int kRows = 16;                   // query rows per MMA (G padded)
    static constexpr int kBoxes = D / 64;              // 128-byte boxes across d
    static constexpr int kBoxBytes = kTile * 128;
    static constexpr int kTileBytes = kBoxes * kBoxBytes;
    static constexpr int kKSteps = D / 16;
    static constexpr int kONTiles = D / 8;
    static constexpr int kStateFloats = kRows * (D + 2);
    static constexpr int kAlignPad = 1024;             // 128-byte swizzle wants 1 KiB alignment
    static constexpr int kKOffset = 0;
    static constexpr int kVOffset = kStages * kTileBytes;
    static constexpr int kBarOffset = 2 * kStages * kTileBytes;
    // ring barriers (full, empty), then the copy barrier of the on-chip merge,
    // then the clustered cut's barriers (parts ready x2, parts read x2)
    static constexpr int kClusterBarOffset = kBarOffset + 2 * kStages * 8 + 16;
    static constexpr int kFlagOffset = kClusterBarOffset + 32;
    static constexpr int kPlanOffset = kFlagOffset + 16;       // 32 longs: per-row-length plan
    static constexpr int kStateOffset = kPlanOffset + 256;
    // on-chip merge (G <= 8): part i (0 = this block's) in rows 8..15 of warp
    // i+1's state area, so at most 2 other parts
    static constexpr int kMaxPartRows = 8;
    static constexpr int kPartFloats = kStateFloats;
    static constexpr int kPartRowOffset = kMaxPartRows * (D + 2);
    // clustered cut (G <= 8): the slices of a unit's parts that the cluster's
    // blocks store into this block, double-buffered by unit, in rows 8..15 of
    // the warps' state areas (warps 0, 1 for even units, 2, 3 for odd ones)
    static constexpr int kClusterMax = 8;                 // blocks per cluster (portable)
    static constexpr int kRegionFloats = kPartRowOffset;  // rows 8..15 of one warp
    // per query row: the warps' weights 2^(m_w - M), then M and L
    static constexpr int kCombineFloats = kConsumerWarps + 2;
    static constexpr int kCombineOffset = kStateOffset + kConsumerWarps * kStateFloats * 4;
    // clustered cut: per 4-element group of a unit's outputs, the block that
    // finishes it and the group's offset in that block's slice
    static constexpr int kOwnerOffset = kCombineOffset + kRows * kCombineFloats * 4;
    static constexpr int kOwnerGroups = kMaxPartRows * D / 4;
    static constexpr int kSmemBytes = kAlignPad + kOwnerOffset + kOwnerGroups * 2;
    static_assert(2 * (threads(true) / 32) + 8 <= 32, "plan scratch fits");
    static_assert(kKeysPerWarp == 16, "one k-step of 16 keys per warp and slice");
    static_assert((kTile / 32) % kGatherWarps == 0, "whole 32-row blocks per gather warp");
    static_assert(kTile % 64 == 0 && kTile <= 256, "whole 64-key slices, TMA box <= 256 rows");
    static_assert(kBoxBytes % 1024 == 0, "boxes stay 1 KiB aligned");
    static_assert(kConsumerWarps * kStateFloats >= 3 * kMaxMergeParts * kRows,
                  "merge staging fits");
    static_assert(kStateOffset % 16 == 0 && (kStateFloats * 4) % 16 == 0 &&
                      (kPartRowOffset * 4) % 16 == 0,
                  "bulk-copy alignment");
    static_assert(3 * kMaxMergeParts * kMaxPartRows <= kStateFloats + kPartRowOffset,
                  "merge staging for G <= 8 ends before the first part's rows");
};

// TMA tiled load of one box of a 3-D tensor map into shared memory.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, int x, int y,
                                            int z, uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar)),
        "l"(policy)
        : "memory");
}

// Shared address of 16-byte chunk `chunk` (of d/8) of key row `key` in a
// tile stored as 128-byte-swizzled boxes of 64 elements.
template <int D>
__device__ __forceinline__ uint32_t swizzled(uint32_t tile, int key, int chunk)
{
    using C = GqaConfig<D>;
    const int box = chunk >> 3, c = chunk & 7;
    return tile + box * C::kBoxBytes + key * 128 + ((c ^ (key & 7)) << 4);
}

template <typename T, int D, int kLayout, bool kLook>
__global__ void __launch_bounds__(GqaConfig<D>::block_threads(kLook, kLayout == kLayoutTokens), 1)
    sha_gqa_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v)
{
    constexpr bool kVarlen = layout_varlen(kLayout);
    constexpr bool kCluster = kLayout == kLayoutCluster;
    using Walk = typename std::conditional<
        kVarlen, VarlenWalk,
        typename std::conditional<kCluster, ClusterWalk, UniformWalk>::type>::type;
    using C = GqaConfig<D>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = reinterpret_cast<unsigned char *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    unsigned char *k_ring = smem + C::kKOffset;
    unsigned char *v_ring = smem + C::kVOffset;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    uint64_t *part_bar = empty + C::kStages;
    volatile int *flags = reinterpret_cast<volatile int *>(smem + C::kFlagOffset);
    float *wstate = reinterpret_cast<float *>(smem + C::kStateOffset);
    float *own_part = wstate + C::kStateFloats + C::kPartRowOffset;
    // clustered cut: one barrier per unit buffer; it completes when all the
    // cluster's slices of the unit have landed here
    uint64_t *cbar = reinterpret_cast<uint64_t *>(smem + C::kClusterBarOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int G = p.H_q / p.H_kv;
    const int max_partners = G <= C::kMaxPartRows ? C::kConsumerWarps - 2 : 0;
    // a part's bytes rounded up to 16: within the slot (padded to 32 floats) and
    // within rows 8..15 (G <= 7 whenever G * (D + 2) is not a multiple of 4)
    const uint32_t part_bytes = (uint32_t)((G * (D + 2) * 4 + 15) & ~15);

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // a gathered tile is filled by every gather lane's copies
            mbar_init(&full[s], kLayout == kLayoutTokens ? 32 * C::kGatherWarps : 1);
            mbar_init(&empty[s], C::kConsumerWarps);
        }
        mbar_init(part_bar, 1);
        if constexpr (kCluster)
            for (int i = 0; i < 2; ++i) mbar_init(&cbar[i], 1);
        flags[0] = 0;
        flags[1] = 0;
        flags[kFlagClaim] = 0;
        flags[kFlagOnChip] = 0;
        mbar_init_fence();
    }
    __syncthreads();
    // the cluster's barriers are initialised before any block signals another's
    if constexpr (kCluster) cluster_arrive();
    // the tensor maps are kernel parameters: fetch them while the previous
    // kernel finishes
    if (warp == C::kConsumerWarps && lane == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k))
                     : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v))
                     : "memory");
    }
    // inputs, workspace and the output may come from the previous kernel
    pdl_wait();
    pdl_launch_dependents();
    if constexpr (kCluster) cluster_wait();

    Schedule S = p.sched;
    Walk walk;
    if constexpr (kVarlen) {
        if (!varlen_plan<C::threads(kLook)>(p.seqlens, p.B, p.top_k, p.N_kv, C::kTile, gridDim.x,
                                      reinterpret_cast<long long *>(smem + C::kPlanOffset), S,
                                      walk))
            return;
    } else if constexpr (kCluster) {
        walk.start(S, (long long)p.B * p.top_k, p.N_kv);
    } else {
        walk.S = S;
        walk.t = S.begin(blockIdx.x);
        walk.t_end = S.begin(blockIdx.x + 1);
        walk.n_keys = kLayout == kLayoutTokens ? p.n_sel : p.N_kv;
    }

    // ------------------------------------------------------------ scout
    if constexpr (kLook) {
        if (warp == C::kConsumerWarps + 1) {
            if (lane == 0)
                lookahead_scout(walk, S, max_partners, p.counters, p.slots, p.slot_floats,
                                part_bytes, own_part, C::kPartFloats, flags, part_bar);
            return;
        }
    }

    // ------------------------------------------------------------ producer
    // gw: this warp's share of a gathered tile (0 for the producer warp; in the
    // token layout's build, which has no scout, gather warps 1.. follow it)
    static_assert(!(kLook && kLayout == kLayoutTokens), "the gathered build has no scout");
    int gw = warp == C::kConsumerWarps ? 0 : -1;
    if constexpr (kLayout == kLayoutTokens)
        if (warp > C::kConsumerWarps) gw = warp - C::kConsumerWarps;
    if (gw >= 0) {
        // A paged cache needs several page ids per tile: the whole warp gathers
        // them (one page box per lane).  Otherwise one lane drives the pipeline.
        constexpr bool kWarpProducer = kLayout == kLayoutPaged || kLayout == kLayoutTokens;
        if (!kWarpProducer && lane != 0) {
            if constexpr (kCluster) cluster_sync_unaligned();
            return;
        }
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t last_parity = 0, used = 0;
        bool ok = true;
        Walk wk = walk;
        Seg seg;
        // gathered layout: the raw positions of this warp's row blocks of the
        // next tile (lane l holding rows i*32 + l), loaded while the current
        // tile's copies go out; a unit's first tile is loaded beside its head id
        int pos_next[C::kTile / 32];
        auto load_pos = [&](long long unit, int tile) {
            const int n0 = tile * C::kTile;
            const int rows = min(C::kTile, p.n_sel - n0);
            const int32_t *tk = p.tokens + (size_t)unit * p.n_sel + n0;
#pragma unroll
            for (int i = 0; i < C::kTile / 32; ++i) {
                const int r = i * 32 + lane;
                pos_next[i] = (i % C::kGatherWarps == gw && r < rows) ? tk[r] : 0;
            }
        };
        (void)load_pos;
        while (ok && wk.next(seg)) {
            const int b = (int)(seg.unit / p.top_k);
            const int h = p.idx[seg.unit];
            if constexpr (kLayout == kLayoutTokens) load_pos(seg.unit, seg.first_tile);
            if ((unsigned)h >= (unsigned)p.H_kv) continue;
            const int plane = b * p.H_kv + h;
            for (int j = seg.first_tile; j < seg.first_tile + seg.num_tiles; ++j) {
                bool go = true;
                if (lane == 0) {
                    if (flags[0]) {
                        go = false;
                    } else if (!mbar_wait(&empty[stage], phase ^ 1)) {
                        atomicOr(&g_sha_status, kStatusTimeout);
                        flags[0] = 1;
                        go = false;
                    } else if (flags[0]) {
                        // a consumer that gave up raised the flag before releasing
                        // this stage: its last copy may still be landing
                        go = false;
                    }
                }
                if constexpr (kWarpProducer) go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                if constexpr (kLayout == kLayoutPaged) {
                    // boxes of min(page_size, tile) keys, each inside one page,
                    // landing at 1 KiB-aligned rows of the swizzled tile
                    const int n0 = j * C::kTile;
                    const int rows = min(C::kTile, seg.n_keys - n0);
                    const int box_rows = min(p.page_size, C::kTile);
                    const int chunks = (rows + box_rows - 1) / box_rows;
                    if (lane == 0)
                        mbar_arrive_expect_tx(
                            &full[stage], (uint32_t)(2 * chunks * C::kBoxes * box_rows * 128));
                    __syncwarp();
                    const int32_t *bt = p.block_table + (size_t)b * p.max_pages;
                    for (int c = lane; c < chunks; c += 32) {
                        const int key = n0 + c * box_rows;
                        const int pi = key / p.page_size, off = key - pi * p.page_size;
                        int page = bt[pi];
                        if ((unsigned)page >= (unsigned)p.num_pages) {
                            atomicOr(&g_sha_status, kStatusBadIndex);
                            page = 0;                   // stay inside the pool
                        }
                        const int pplane = page * p.H_kv + h;
                        for (int bx = 0; bx < C::kBoxes; ++bx) {
                            tma_load_3d(k_ring + stage * C::kTileBytes + bx * C::kBoxBytes +
                                            c * box_rows * 128,
                                        &tm_k, bx * 64, off, pplane, &full[stage], policy);
                            tma_load_3d(v_ring + stage * C::kTileBytes + bx * C::kBoxBytes +
                                            c * box_rows * 128,
                                        &tm_v, bx * 64, off, pplane, &full[stage], policy);
                        }
                    }
                } else if constexpr (kLayout == kLayoutTokens) {
                    // the unit's listed keys, gathered into the swizzled tile with
                    // 16-byte cp.async: 8 lanes copy the 128 bytes of one row's box,
                    // so an instruction moves 4 whole lines of 4 rows; rows past the
                    // list are zero-filled (and masked by the consumers).  Gather
                    // warp gw takes the tile's 32-row blocks gw, gw + kGatherWarps,
                    // ..., and each lane arrives on the stage once its copies have
                    // landed.
                    const int n0 = j * C::kTile;
                    const int rows = min(C::kTile, seg.n_keys - n0);
                    const T *kb = static_cast<const T *>(p.k) + (size_t)plane * p.N_kv * D;
                    const T *vb = static_cast<const T *>(p.v) + (size_t)plane * p.N_kv * D;
                    const uint32_t kt = smem_addr(k_ring + stage * C::kTileBytes);
                    const uint32_t vt = smem_addr(v_ring + stage * C::kTileBytes);
                    // this tile's positions (loaded a tile ahead), checked
                    int ids[C::kTile / 32];
#pragma unroll
                    for (int i = 0; i < C::kTile / 32; ++i) {
                        int t = pos_next[i];
                        if ((unsigned)t >= (unsigned)p.N_kv) {
                            atomicOr(&g_sha_status, kStatusBadIndex);
                            t = 0;                      // stay inside the head's cache
                        }
                        ids[i] = t;
                    }
                    if (j + 1 < seg.first_tile + seg.num_tiles) load_pos(seg.unit, j + 1);
                    const int sub = lane >> 3, ch = lane & 7;
#pragma unroll
                    for (int i = 0; i < C::kTile / 32; ++i) {
                        if (i % C::kGatherWarps != gw) continue;
#pragma unroll 2
                        for (int r1 = 0; r1 < 32; r1 += 4) {
                            const int r = i * 32 + r1 + sub;
                            const int t = __shfl_sync(0xffffffffu, ids[i], r1 + sub);
                            const uint32_t src_bytes = r < rows ? 16u : 0u;
                            const T *krow = kb + (size_t)t * D;
                            const T *vrow = vb + (size_t)t * D;
#pragma unroll
                            for (int bx = 0; bx < C::kBoxes; ++bx) {
                                const int c = bx * 8 + ch;
                                cp_async16_zfill(swizzled<D>(kt, r, c), krow + c * 8, src_bytes,
                                                 policy);
                                cp_async16_zfill(swizzled<D>(vt, r, c), vrow + c * 8, src_bytes,
                                                 policy);
                            }
                        }
                    }
                    cp_async_arrive_noinc(&full[stage]);
                } else if constexpr (layout_strided(kLayout)) {
                    // boxes of a 4-D map whose outer dimensions follow the caller's strides
                    int c[3];
                    strided_coords(p, j * C::kTile, h, b, c);
                    mbar_arrive_expect_tx(&full[stage], 2 * C::kTileBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_load_4d(k_ring + stage * C::kTileBytes + bx * C::kBoxBytes, &tm_k,
                                    bx * 64, c[0], c[1], c[2], &full[stage], policy);
                        tma_load_4d(v_ring + stage * C::kTileBytes + bx * C::kBoxBytes, &tm_v,
                                    bx * 64, c[0], c[1], c[2], &full[stage], policy);
                    }
                } else {
                    mbar_arrive_expect_tx(&full[stage], 2 * C::kTileBytes);
#pragma unroll
                    for (int bx = 0; bx < C::kBoxes; ++bx) {
                        tma_load_3d(k_ring + stage * C::kTileBytes + bx * C::kBoxBytes, &tm_k,
                                    bx * 64, j * C::kTile, plane, &full[stage], policy);
                        tma_load_3d(v_ring + stage * C::kTileBytes + bx * C::kBoxBytes, &tm_v,
                                    bx * 64, j * C::kTile, plane, &full[stage], policy);
                    }
                }
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        if constexpr (kLayout == kLayoutTokens) cp_async_wait_all();
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        if constexpr (kWarpProducer) __syncwarp();
        if constexpr (kCluster) cluster_sync_unaligned();
        return;
    }

    // ------------------------------------------------------------ consumers
    const int tid = threadIdx.x;
    const int g = lane >> 2;          // accumulator rows g and g+8
    const int qd = lane & 3;          // column pair within an 8-wide n-tile
    const unsigned FULL = 0xffffffffu;
    const uint32_t k_base = smem_addr(k_ring), v_base = smem_addr(v_ring);
    // ldmatrix row addresses: lane -> (matrix lane>>3, row lane&7)
    const int mi = lane >> 3, mr = lane & 7;
    const int key_k = warp * C::kKeysPerWarp + (mi >> 1) * 8 + mr;   // K: matrices (keys, d-chunk)
    const int key_v = warp * C::kKeysPerWarp + (mi & 1) * 8 + mr;    // V: matrices (keys, d-chunk)

    int stage = 0;
    uint32_t phase = 0;

    // Clustered cut: block r of the P-block cluster finishes the 4-element
    // groups [r*groups/P, (r+1)*groups/P) of a unit's G x D outputs, and every
    // block stores each part's slices (and its m, l) where their finishers
    // stage them: part i of a unit at cstage(buf, i) in every block, the
    // first (P+1)/2 parts in one warp's rows 8..15, the others in the next's.
    // All of it is fixed for the kernel: worked out here once.
    const int P = kCluster ? S.cluster : 1;
    const int groups = G * D / 4;
    const int slice_max = 4 * ((groups + P - 1) / P);
    const int part_stride = slice_max + 4 * ((2 * G + 3) / 4);
    const int half = (P + 1) / 2;
    auto cstage = [=](int buf, int i) {
        const bool hi = i >= half;
        return wstate + (2 * buf + (hi ? 1 : 0)) * C::kStateFloats + C::kPartRowOffset +
               (hi ? i - half : i) * part_stride;
    };
    uint16_t *owner_tab = reinterpret_cast<uint16_t *>(smem + C::kOwnerOffset);
    int crank = 0, e0 = 0, e1 = 0;
    uint32_t cluster_bytes = 0;
    if constexpr (kCluster) {
        crank = walk.rank;
        e0 = 4 * (crank * groups / P);
        e1 = 4 * ((crank + 1) * groups / P);
        cluster_bytes = (uint32_t)(P * (e1 - e0 + 2 * G) * 4);
        // owner (high 4 bits) and offset within its slice (floats) per group;
        // read after the consumers' first named barrier
        for (int g4 = tid; g4 < groups; g4 += C::kConsumers) {
            const int r = ((g4 + 1) * P - 1) / groups;
            owner_tab[g4] = (uint16_t)((r << 12) | (4 * g4 - 4 * (r * groups / P)));
        }
    }

    Walk wk = walk;
    Seg seg;
    int n_done = 0;   // clustered cut: units this block has finished (its buffers' parity)
    for (bool first_seg = true; wk.next(seg); first_seg = false) {
        const long long u = seg.unit;
        const int b = (int)(u / p.top_k);
        const int h = p.idx[u];
        if ((unsigned)h >= (unsigned)p.H_kv) {
            if (tid == 0) atomicOr(&g_sha_status, kStatusBadIndex);
            continue;
        }

        // Q of the group as the MMA's A operand: rows g, g+8 (zero past G)
        uint32_t qa[C::kKSteps][4];
        {
            const T *qg = static_cast<const T *>(p.q) + ((size_t)b * p.H_q + (size_t)h * G) * D;
            const bool r0 = g < G, r1 = g + 8 < G;
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
                const int c0 = ks * 16 + qd * 2;
                qa[ks][0] = r0 ? *reinterpret_cast<const uint32_t *>(qg + g * D + c0) : 0u;
                qa[ks][1] = r1 ? *reinterpret_cast<const uint32_t *>(qg + (g + 8) * D + c0) : 0u;
                qa[ks][2] = r0 ? *reinterpret_cast<const uint32_t *>(qg + g * D + c0 + 8) : 0u;
                qa[ks][3] =
                    r1 ? *reinterpret_cast<const uint32_t *>(qg + (g + 8) * D + c0 + 8) : 0u;
            }
        }

        float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
        float o[C::kONTiles][4];
#pragma unroll
        for (int n = 0; n < C::kONTiles; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

        for (int j = seg.first_tile; j < seg.first_tile + seg.num_tiles; ++j) {
            bool live = !__any_sync(FULL, flags[0] != 0);
            if (live) {
                live = __all_sync(FULL, mbar_wait(&full[stage], phase));
                if (!live && lane == 0) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    flags[0] = 1;
                }
            }
            if (live) {
                const uint32_t kt = k_base + stage * C::kTileBytes;
                const uint32_t vt = v_base + stage * C::kTileBytes;
                const int rows = min(C::kTile, seg.n_keys - j * C::kTile);
                if constexpr (kVarlen) {
                    // keys past this row's length but inside the cache hold stale
                    // values: zero this warp's V rows there (0 * NaN would poison P V)
                    if (rows < C::kTile) {
                        unsigned char *vtile = v_ring + stage * C::kTileBytes;
                        for (int i = lane; i < C::kSlices * 16 * C::kBoxes * 8; i += 32) {
                            const int chunk = i & 7, bx = (i >> 3) % C::kBoxes;
                            const int rr = (i >> 3) / C::kBoxes;      // 0 .. kSlices*16-1
                            const int key = (rr >> 4) * 64 + warp * C::kKeysPerWarp + (rr & 15);
                            if (key >= rows)
                                *reinterpret_cast<uint4 *>(vtile + bx * C::kBoxBytes + key * 128 +
                                                           chunk * 16) = make_uint4(0, 0, 0, 0);
                        }
                        fence_proxy_async_shared();   // before the stage is refilled by TMA
                        __syncwarp();
                    }
                }

                // S = Q K^T over this warp's 16 keys of each 64-key slice:
                // two 8-key n-tiles per slice
                float s[C::kSlices][2][4];
#pragma unroll
                for (int sl = 0; sl < C::kSlices; ++sl) {
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
                        s[sl][nt][0] = s[sl][nt][1] = s[sl][nt][2] = s[sl][nt][3] = 0.f;
#pragma unroll
                    for (int ks = 0; ks < C::kKSteps; ++ks) {
                        uint32_t kb[4];
                        ldmatrix_x4(swizzled<D>(kt, sl * 64 + key_k, ks * 2 + (mi & 1)), kb);
                        mma_16816<T>(s[sl][0], qa[ks], kb[0], kb[1]);
                        mma_16816<T>(s[sl][1], qa[ks], kb[2], kb[3]);
                    }
                }

                // online softmax on rows g (entries 0,1) and g+8 (entries 2,3)
                float mt[2] = {-INFINITY, -INFINITY};
#pragma unroll
                for (int sl = 0; sl < C::kSlices; ++sl)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int key = sl * 64 + warp * C::kKeysPerWarp + nt * 8 + qd * 2 +
                                            (e & 1);
                            s[sl][nt][e] = key < rows ? s[sl][nt][e] * p.scale_log2 : -INFINITY;
                            mt[e >> 1] = fmaxf(mt[e >> 1], s[sl][nt][e]);
                        }
                float alpha[2], ref[2];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    mt[r] = fmaxf(mt[r], __shfl_xor_sync(FULL, mt[r], 1));
                    mt[r] = fmaxf(mt[r], __shfl_xor_sync(FULL, mt[r], 2));
                    const float m_new = fmaxf(m_run[r], mt[r]);
                    ref[r] = (m_new == -INFINITY) ? 0.f : m_new;
                    alpha[r] = exp2f(m_run[r] - ref[r]);
                    m_run[r] = m_new;
                    l_run[r] *= alpha[r];
                }
#pragma unroll
                for (int sl = 0; sl < C::kSlices; ++sl)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            s[sl][nt][e] = exp2f(s[sl][nt][e] - ref[e >> 1]);
                            l_run[e >> 1] += s[sl][nt][e];
                        }
#pragma unroll
                for (int n = 0; n < C::kONTiles; ++n) {
                    o[n][0] *= alpha[0];
                    o[n][1] *= alpha[0];
                    o[n][2] *= alpha[1];
                    o[n][3] *= alpha[1];
                }

                // O += P V: per slice, 16 keys x d, two 8-wide n-tiles per ldmatrix
#pragma unroll
                for (int sl = 0; sl < C::kSlices; ++sl) {
                    uint32_t pa[4];
                    pa[0] = pack2<T>(s[sl][0][0], s[sl][0][1]);
                    pa[1] = pack2<T>(s[sl][0][2], s[sl][0][3]);
                    pa[2] = pack2<T>(s[sl][1][0], s[sl][1][1]);
                    pa[3] = pack2<T>(s[sl][1][2], s[sl][1][3]);
#pragma unroll
                    for (int dn = 0; dn < D / 16; ++dn) {
                        uint32_t vb[4];
                        ldmatrix_x4_trans(swizzled<D>(vt, sl * 64 + key_v, dn * 2 + (mi >> 1)), vb);
                        mma_16816<T>(o[2 * dn], pa, vb[0], vb[1]);
                        mma_16816<T>(o[2 * dn + 1], pa, vb[2], vb[3]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }

        // ---- merge: the quad's partial sums, then warps, then (maybe) blocks
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            l_run[r] += __shfl_xor_sync(FULL, l_run[r], 1);
            l_run[r] += __shfl_xor_sync(FULL, l_run[r], 2);
        }
        float *ws = wstate + warp * C::kStateFloats;
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int row = g + 8 * r;
            if (row < G) {
#pragma unroll
                for (int n = 0; n < C::kONTiles; ++n) {
                    ws[row * (D + 2) + n * 8 + qd * 2] = o[n][2 * r];
                    ws[row * (D + 2) + n * 8 + qd * 2 + 1] = o[n][2 * r + 1];
                }
                if (qd == 0) {
                    ws[row * (D + 2) + D] = m_run[r];
                    ws[row * (D + 2) + D + 1] = l_run[r];
                }
            }
        }
        // blocks first..last share a split unit; the one the block ends with may
        // be finished on chip
        int first = 0, last = 0, first_slot = 0;
        if (!kCluster && !seg.whole) unit_parts(S, seg, first, last, first_slot);
        int la_parts = 0;
        if constexpr (kLook)
            if (wk.t >= wk.t_end) la_parts = lookahead_parts(seg, first, last, max_partners);
        if (la_parts && tid == 0) flags[kFlagOnChip] = lookahead_claim(flags);
        named_barrier(1, C::kConsumers);
        const bool on_chip = la_parts && flags[kFlagOnChip];

        // the warps' weights of each query row, once: c_w = 2^(m_w - M), L = sum_w c_w l_w
        float *cw = reinterpret_cast<float *>(smem + C::kCombineOffset);
        if (tid < G) {
            const float *st = wstate + tid * (D + 2);
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) M = fmaxf(M, st[w * C::kStateFloats + D]);
            const float M_ref = (M == -INFINITY) ? 0.f : M;
            float L = 0.f;
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) {
                const float c = exp2f(st[w * C::kStateFloats + D] - M_ref);
                cw[tid * C::kCombineFloats + w] = c;
                L = fmaf(c, st[w * C::kStateFloats + D + 1], L);
            }
            cw[tid * C::kCombineFloats + C::kConsumerWarps] = M;
            cw[tid * C::kCombineFloats + C::kConsumerWarps + 1] = L;
        }
        named_barrier(1, C::kConsumers);

        T *out_g = static_cast<T *>(p.out) + ((size_t)b * p.H_q + (size_t)h * G) * D;
        const bool aborted = flags[0] != 0;
        // this block's first unit goes to slot 2c, any later partial one to 2c+1;
        // on chip it is part 0, beside the copies of the others
        float *slot = on_chip   ? own_part
                    : p.slots ? p.slots + (size_t)(2 * blockIdx.x + (first_seg ? 0 : 1)) *
                                              p.slot_floats
                              : nullptr;
        // under the clustered cut, a unit that is not whole here is shared by
        // the cluster's blocks
        bool shared = false;
        if constexpr (kCluster) shared = !seg.whole;
        if (shared) {
            // this block's part of the unit, slice by slice, to the blocks that
            // finish them (always, so that every block's byte count completes)
            const int buf = n_done & 1;
            float *mine = cstage(buf, crank);
            for (int e = 2 * tid; e < G * D; e += 2 * C::kConsumers) {
                const uint32_t code = owner_tab[e >> 2];
                const int row = e / D, c = e - row * D;
                const float *cr = cw + row * C::kCombineFloats;
                float2 O = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < C::kConsumerWarps; ++w) {
                    const float2 x = *reinterpret_cast<const float2 *>(
                        wstate + w * C::kStateFloats + row * (D + 2) + c);
                    O.x = fmaf(cr[w], x.x, O.x);
                    O.y = fmaf(cr[w], x.y, O.y);
                }
                st_async_f32x2(mine + (code & 0xfff) + (e & 3), code >> 12, O.x, O.y,
                               &cbar[buf]);
            }
            // every row's (m, l) to every block: one pair per thread
            if (tid < P * G) {
                const int r = tid / G, row = tid - r * G;
                const float *cr = cw + row * C::kCombineFloats;
                st_async_f32x2(mine + slice_max + 2 * row, (uint32_t)r, cr[C::kConsumerWarps],
                               cr[C::kConsumerWarps + 1], &cbar[buf]);
            }
        } else if (!aborted) {
            // two neighbouring elements of a row per thread (D is even)
            for (int e = 2 * tid; e < G * D; e += 2 * C::kConsumers) {
                const int row = e / D, c = e - row * D;
                const float *cr = cw + row * C::kCombineFloats;
                float2 O = make_float2(0.f, 0.f);
#pragma unroll
                for (int w = 0; w < C::kConsumerWarps; ++w) {
                    const float2 x = *reinterpret_cast<const float2 *>(
                        wstate + w * C::kStateFloats + row * (D + 2) + c);
                    O.x = fmaf(cr[w], x.x, O.x);
                    O.y = fmaf(cr[w], x.y, O.y);
                }
                const float L = cr[C::kConsumerWarps + 1];
                if (seg.whole) {
                    *reinterpret_cast<uint32_t *>(out_g + e) = pack2<T>(O.x / L, O.y / L);
                } else {
                    *reinterpret_cast<float2 *>(slot + e) = O;
                    if (c == 0) {
                        slot[G * D + row] = cr[C::kConsumerWarps];
                        slot[G * D + G + row] = L;
                    }
                }
            }
            if (!kCluster && !seg.whole && !on_chip) __threadfence();
        }
        named_barrier(1, C::kConsumers);

        if (shared) {
            // wait for this block's slices of every part (its own included), then
            // write them out merged in block order
            const int buf = n_done & 1;
            if (tid == 0) mbar_arrive_expect_tx(&cbar[buf], cluster_bytes);
            if (!mbar_wait_cluster(&cbar[buf], (n_done >> 1) & 1)) {
                atomicOr(&g_sha_status, kStatusTimeout);
                flags[0] = 1;
            }
            named_barrier(1, C::kConsumers);
            if (tid == 0) flags[1] = !flags[0];
            named_barrier(1, C::kConsumers);
            if (flags[1]) {
                auto part_at = [=](int i) { return cstage(buf, i); };
                merge_parts<T, D, C::kConsumers>(
                    StagedParts<decltype(part_at)>{part_at, e0, slice_max}, P, G, out_g, wstate,
                    tid, e0, e1);
            }
            ++n_done;
        } else if (on_chip) {
            // every other part has arrived and none merged: this block merges
            if (!mbar_wait(part_bar, 0)) {
                atomicOr(&g_sha_status, kStatusTimeout);
                flags[0] = 1;
            }
            named_barrier(1, C::kConsumers);
            if (tid == 0) flags[1] = !flags[0];
            named_barrier(1, C::kConsumers);
            if (flags[1]) {
                merge_parts<T, D, C::kConsumers>(SharedParts{own_part, C::kPartFloats, G * D}, la_parts,
                                                  G, out_g, wstate, tid);
                if (tid == 0) p.counters[first] = 0;
            }
        } else if (!seg.whole) {
            if (tid == 0) {
                int merge = 0;
                if (!flags[0]) {
                    const int prev = atomicAdd(&p.counters[first], 1);
                    merge = (prev == last - first);
                }
                flags[1] = merge;
            }
            named_barrier(1, C::kConsumers);
            if (flags[1]) {
                __threadfence();
                merge_parts<T, D, C::kConsumers>(
                    GlobalParts{p.slots, p.slot_floats, first, first_slot, G * D}, last - first + 1, G,
                    out_g, wstate, tid);
                if (tid == 0) p.counters[first] = 0;
            }
        }
    }
    if (kLook && tid == 0) lookahead_claim(flags);   // the scout stops looking
    // no block of a cluster leaves while another may still store into it
    if constexpr (kCluster) cluster_sync_unaligned();
}

}  // namespace sha
