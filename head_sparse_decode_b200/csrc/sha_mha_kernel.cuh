// sha_mha_kernel.cuh -- selective head decode for multi-head attention (G = 1)
// with d = 64, per-row lengths or a paged cache (the host sends d = 128 calls
// with one length per row to the grouped kernel's tensor cores, sha_gqa_kernel.cuh).
//
// What one thread block does.  It owns a contiguous range of key tiles (see
// sha_schedule.cuh) and walks it one unit (batch row b, selected head h) at a
// time, as in Algorithm 1, "Selective Head Flash Attention (Decode)" (Polar
// Sparsity, ri.k117.org reproducibility record): head id lookup
// h = batch_head_index[b, k], query row Q[b, h], then the tiles of
// K[b, h], V[b, h] with an online softmax, and finally O written to
// out[b, h] only.  Heads that are not selected are never touched.
//
// How, on sm_100a.  The kernel is bound by HBM bandwidth (about one flop per
// byte), so the design is about keeping bytes in flight:
//   * one producer lane issues 1-D bulk async copies (cp.async.bulk) of each
//     K and V tile -- kTile rows of the head's contiguous [N_kv, d] block --
//     into a kStages-deep shared-memory ring, completion counted on an
//     mbarrier per stage; the ring refills while consumers compute and
//     across unit boundaries;
//   * kConsumerWarps warps each take kTile/kConsumerWarps rows of every tile
//     and keep their OWN running (m, l, O) state for the unit, so a tile
//     needs no block-wide reduction; the warps' states are merged once per
//     unit (log-sum-exp);
//   * scores q.k: 8 lanes per key row, each lane holding 8*(d/64) elements of
//     q in registers, reduced with 3 shuffles; the 16-byte shared loads of 8
//     lanes cover 128 consecutive bytes, so they are free of bank conflicts;
//   * P.V: d/8 lanes per row, one 16-byte vector each, fp32 accumulators;
//   * q is pre-multiplied by scale*log2(e) so every weight is one exp2f;
//   * the block finishes the split unit it ends with on chip when the other
//     parts are done in time (sha_lookahead.cuh).
// The pages' Algorithm 1 renormalises O after every tile; this kernel keeps
// O unnormalised and divides once at the end, which is the same quantity.
#pragma once

#include <cuda.h>
#include <type_traits>

#include "sha_device.cuh"
#include "sha_lookahead.cuh"
#include "sha_merge.cuh"
#include "sha_schedule.cuh"
#include "sha_walk.cuh"

namespace sha {

struct DecodeParams {
    const void *q;
    const void *k;
    const void *v;
    const int32_t *idx;
    void *out;
    int B, H_q, H_kv, N_kv, top_k;
    float scale_log2;        // scale * log2(e)
    Schedule sched;
    float *slots;            // 2*num_ctas partial states of slot_floats floats
    int slot_floats;
    int *counters;           // arrival counters, one per block, zero between calls
    const int32_t *seqlens;  // per-row cache lengths (variable-length calls), else null
    // paged cache: k, v are page pools [num_pages, H_kv, page_size, d] and key n
    // of row b sits in page block_table[b, n / page_size]
    const int32_t *block_table;
    int page_size, max_pages, num_pages;
    // strided cache: K and V are read through 4-D tensor maps [d, ., ., .] whose
    // three outer dimensions are the token, head and batch dimensions in the
    // order of increasing stride; these give each one's position (0..2)
    int tok_dim, head_dim, batch_dim;
    // head x token sparsity: unit u attends only to the keys tokens[u * n_sel ..
    // u * n_sel + n_sel) of its head (positions in [0, N_kv))
    const int32_t *tokens;
    int n_sel;
};

// How K/V of a unit are found: one padded [N_kv] block per (b, h) with every
// row N_kv long or with per-row lengths, pages of a shared pool, or any
// (batch, head, token) strides with d contiguous (every row N_kv long, or
// per-row lengths within N_kv).
enum : int {
    kLayoutFixed = 0,
    kLayoutVarlen = 1,
    kLayoutPaged = 2,
    kLayoutStrided = 3,
    kLayoutStridedVarlen = 4,
    // the padded layout of kLayoutFixed under the clustered cut (grouped kernel
    // only): thread-block clusters, split units merged in distributed shared memory
    kLayoutCluster = 5,
    // the padded layout, each unit restricted to a listed subset of its keys,
    // gathered row by row (grouped kernel only)
    kLayoutTokens = 6
};

// Layouts whose rows have their own lengths (planned on the device) and that
// read K/V through strided 4-D tensor maps.
constexpr bool layout_varlen(int layout)
{
    return layout == kLayoutVarlen || layout == kLayoutPaged || layout == kLayoutStridedVarlen;
}
constexpr bool layout_strided(int layout)
{
    return layout == kLayoutStrided || layout == kLayoutStridedVarlen;
}

// TMA tiled load of one box of a 4-D tensor map into shared memory.
__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, int x, int c1,
                                            int c2, int c3, uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// Tile (keys n0.., head h, row b) of a strided cache: the box's outer coordinates.
__device__ __forceinline__ void strided_coords(const DecodeParams &p, int n0, int h, int b,
                                               int (&c)[3])
{
    c[p.tok_dim] = n0;
    c[p.head_dim] = h;
    c[p.batch_dim] = b;
}

// Build-time tuning of the multi-head kernel (defaults measured best on B200).
#ifndef SHA_MHA_TILE_KEYS
#define SHA_MHA_TILE_KEYS 128
#endif
#ifndef SHA_MHA_STAGES
#define SHA_MHA_STAGES 3
#endif
// Blocks per SM the multi-head kernel is planned and compiled for.
#ifndef SHA_MHA_BLOCKS_PER_SM
#define SHA_MHA_BLOCKS_PER_SM 1
#endif

template <int D>
struct MhaConfig {
    static constexpr int kConsumerWarps = 8;
    static constexpr int kConsumers = kConsumerWarps * 32;
    static constexpr int kThreads = kConsumers + 32;   // + one producer warp
    // ... and a scout warp in the builds that finish a block's last unit on chip
    static constexpr int threads(bool look) { return kThreads + (look ? 32 : 0); }
    static constexpr int kTile = SHA_MHA_TILE_KEYS;    // keys per tile
    static constexpr int kStages = SHA_MHA_STAGES;
    static constexpr int kRowsPerWarp = kTile / kConsumerWarps;
    static constexpr int kPasses = kRowsPerWarp / 4;   // score passes of 4 rows
    static constexpr int kQkChunks = D / 64;           // 16-byte chunks per lane (scores)
    static constexpr int kPvLanesPerRow = D / 8;
    static constexpr int kPvRowsPerIter = 32 / kPvLanesPerRow;
    static constexpr int kPvIters = kRowsPerWarp / kPvRowsPerIter;
    static constexpr int kRowBytes = D * 2;
    static constexpr int kTileBytes = kTile * kRowBytes;
    static constexpr int kStateFloats = D + 2;         // O[0..D), m, l
    static constexpr int kKOffset = 0;
    static constexpr int kVOffset = kStages * kTileBytes;
    static constexpr int kBarOffset = 2 * kStages * kTileBytes;
    // ring barriers (full, empty), then the copy barrier of the on-chip merge
    static constexpr int kFlagOffset = kBarOffset + 2 * kStages * 8 + 16;
    static constexpr int kPlanOffset = kFlagOffset + 16;       // 32 longs: per-row-length plan
    static constexpr int kStateOffset = kPlanOffset + 256;
    // the block's own part and up to kMaxPartners others, for an on-chip merge
    static constexpr int kMaxPartners = 3;
    static constexpr int kPartFloats = (kStateFloats + 3) / 4 * 4;
    static constexpr uint32_t kPartBytes = kPartFloats * 4;
    static constexpr int kPartOffset = kStateOffset + kConsumerWarps * kStateFloats * 4;
    static constexpr int kSmemBytes = kPartOffset + (1 + kMaxPartners) * kPartBytes;
    static_assert(kStateOffset % 16 == 0 && kPartOffset % 16 == 0, "bulk-copy alignment");
    static_assert(2 * (threads(true) / 32) + 8 <= 32, "plan scratch fits");
    static_assert(kRowsPerWarp % 4 == 0, "score passes cover 4 rows");
    static_assert(kRowsPerWarp % kPvRowsPerIter == 0, "P.V iterations");
    static_assert(kConsumers >= D, "one consumer thread per output element");
    static_assert(kConsumerWarps * kStateFloats >= 3 * kMaxMergeParts, "merge staging fits");
};

template <typename T, int D, int kLayout, bool kLook>
__global__ void __launch_bounds__(MhaConfig<D>::threads(kLook), SHA_MHA_BLOCKS_PER_SM)
    sha_mha_decode_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v)
{
    constexpr bool kVarlen = layout_varlen(kLayout);
    using Walk = typename std::conditional<kVarlen, VarlenWalk, UniformWalk>::type;
    using C = MhaConfig<D>;
    extern __shared__ __align__(1024) unsigned char smem[];
    unsigned char *k_ring = smem + C::kKOffset;
    unsigned char *v_ring = smem + C::kVOffset;
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    uint64_t *part_bar = empty + C::kStages;
    volatile int *flags = reinterpret_cast<volatile int *>(smem + C::kFlagOffset);
    float *wstate = reinterpret_cast<float *>(smem + C::kStateOffset);
    float *own_part = reinterpret_cast<float *>(smem + C::kPartOffset);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::kConsumerWarps);
        }
        mbar_init(part_bar, 1);
        flags[0] = 0;   // abort: a wait gave up
        flags[1] = 0;   // this block merges the current unit
        flags[kFlagClaim] = 0;
        flags[kFlagOnChip] = 0;
        mbar_init_fence();
    }
    __syncthreads();
    // inputs, workspace and the output may come from the previous kernel
    pdl_wait();
    pdl_launch_dependents();

    Schedule S = p.sched;
    Walk walk;
    if constexpr (kVarlen) {
        if (!varlen_plan<C::threads(kLook)>(p.seqlens, p.B, p.top_k, p.N_kv, C::kTile, gridDim.x,
                                      reinterpret_cast<long long *>(smem + C::kPlanOffset), S,
                                      walk))
            return;
    } else {
        walk.S = S;
        walk.t = S.begin(blockIdx.x);
        walk.t_end = S.begin(blockIdx.x + 1);
        walk.n_keys = p.N_kv;
    }

    // ------------------------------------------------------------ scout
    if constexpr (kLook) {
        if (warp == C::kConsumerWarps + 1) {
            if (lane == 0)
                lookahead_scout(walk, S, C::kMaxPartners, p.counters, p.slots, p.slot_floats,
                                C::kPartBytes, own_part, C::kPartFloats, flags, part_bar);
            return;
        }
    }

    // ------------------------------------------------------------ producer
    if (warp == C::kConsumerWarps) {
        // A paged cache needs several page ids per tile: the whole warp gathers
        // them (one page run per lane) so a tile costs one round trip to the
        // block table.  Otherwise one lane drives the pipeline.
        constexpr bool kWarpProducer = kLayout == kLayoutPaged;
        if (!kWarpProducer && lane != 0) return;
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0;
        uint32_t last_parity = 0, used = 0;   // per-stage parity of the last copy, stages used
        bool ok = true;
        Walk wk = walk;
        Seg seg;
        while (ok && wk.next(seg)) {
            const int b = (int)(seg.unit / p.top_k);
            const int h = p.idx[seg.unit];
            if ((unsigned)h >= (unsigned)p.H_kv) continue;
            const size_t head = ((size_t)b * p.H_kv + h) * (size_t)p.N_kv * D;
            const T *kbase = static_cast<const T *>(p.k) + head;
            const T *vbase = static_cast<const T *>(p.v) + head;
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
                const int n0 = j * C::kTile;
                const int rows = min(C::kTile, seg.n_keys - n0);
                const uint32_t bytes = (uint32_t)rows * C::kRowBytes;
                if constexpr (layout_strided(kLayout)) {
                    // one [kTile][d] box per tensor (rows past N_kv arrive as zeros)
                    int c[3];
                    strided_coords(p, n0, h, b, c);
                    mbar_arrive_expect_tx(&full[stage], 2 * C::kTileBytes);
                    tma_load_4d(k_ring + stage * C::kTileBytes, &tm_k, 0, c[0], c[1], c[2],
                                &full[stage], policy);
                    tma_load_4d(v_ring + stage * C::kTileBytes, &tm_v, 0, c[0], c[1], c[2],
                                &full[stage], policy);
                } else if constexpr (kLayout == kLayoutPaged) {
                    // one copy per run of keys that lie in one page, a run per lane
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], 2 * bytes);
                    __syncwarp();
                    const int32_t *bt = p.block_table + (size_t)b * p.max_pages;
                    const int ps = p.page_size;
                    const int pi0 = n0 / ps, runs = (n0 + rows - 1) / ps - pi0 + 1;
                    for (int r = lane; r < runs; r += 32) {
                        const int pi = pi0 + r;
                        const int k0 = max(n0, pi * ps), k1 = min(n0 + rows, (pi + 1) * ps);
                        int page = bt[pi];
                        if ((unsigned)page >= (unsigned)p.num_pages) {
                            atomicOr(&g_sha_status, kStatusBadIndex);
                            page = 0;                   // stay inside the pool
                        }
                        const size_t src =
                            (((size_t)page * p.H_kv + h) * ps + (k0 - pi * ps)) * D;
                        const int dst = k0 - n0;
                        bulk_copy_g2s(k_ring + stage * C::kTileBytes + dst * C::kRowBytes,
                                      static_cast<const T *>(p.k) + src,
                                      (uint32_t)(k1 - k0) * C::kRowBytes, &full[stage], policy);
                        bulk_copy_g2s(v_ring + stage * C::kTileBytes + dst * C::kRowBytes,
                                      static_cast<const T *>(p.v) + src,
                                      (uint32_t)(k1 - k0) * C::kRowBytes, &full[stage], policy);
                    }
                } else {
                    mbar_arrive_expect_tx(&full[stage], 2 * bytes);
                    bulk_copy_g2s(k_ring + stage * C::kTileBytes, kbase + (size_t)n0 * D,
                                  bytes, &full[stage], policy);
                    bulk_copy_g2s(v_ring + stage * C::kTileBytes, vbase + (size_t)n0 * D,
                                  bytes, &full[stage], policy);
                }
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        // Never leave the block with a copy still landing in shared memory.
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        if constexpr (kWarpProducer) __syncwarp();
        return;
    }

    // ------------------------------------------------------------ consumers
    const int tid = threadIdx.x;            // 0 .. kConsumers-1
    const int part = lane & 7;              // score lanes: 8 per row
    const int grp = lane >> 3;
    const int pv_chunk = lane % C::kPvLanesPerRow;
    const int pv_row = lane / C::kPvLanesPerRow;
    const unsigned FULL = 0xffffffffu;

    int stage = 0;
    uint32_t phase = 0;

    Walk wk = walk;
    Seg seg;
    for (bool first_seg = true; wk.next(seg); first_seg = false) {
        const long long u = seg.unit;
        const int b = (int)(u / p.top_k);
        const int h = p.idx[u];
        if ((unsigned)h >= (unsigned)p.H_kv) {
            if (tid == 0) atomicOr(&g_sha_status, kStatusBadIndex);
            continue;
        }

        // query row of head h, pre-scaled by scale*log2(e)
        float q[C::kQkChunks * 8];
        {
            const T *qrow = static_cast<const T *>(p.q) + ((size_t)b * p.H_q + h) * D;
#pragma unroll
            for (int i = 0; i < C::kQkChunks; ++i) {
                const uint4 raw = *reinterpret_cast<const uint4 *>(qrow + (part + 8 * i) * 8);
                float f[8];
                widen8<T>(raw, f);
#pragma unroll
                for (int e = 0; e < 8; ++e) q[i * 8 + e] = f[e] * p.scale_log2;
            }
        }

        float m_run = -INFINITY, l_run = 0.f;
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = 0.f;

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
                const int rows = min(C::kTile, seg.n_keys - j * C::kTile);
                const unsigned char *kt = k_ring + stage * C::kTileBytes;
                const unsigned char *vt = v_ring + stage * C::kTileBytes;
                const int row0 = warp * C::kRowsPerWarp;

                // scores, already in log2 units
                float sc[C::kPasses];
#pragma unroll
                for (int ps = 0; ps < C::kPasses; ++ps) {
                    const int r = row0 + ps * 4 + grp;
                    float acc = 0.f;
#pragma unroll
                    for (int i = 0; i < C::kQkChunks; ++i) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(
                            kt + r * C::kRowBytes + (part + 8 * i) * 16);
                        float f[8];
                        widen8<T>(raw, f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) acc = fmaf(q[i * 8 + e], f[e], acc);
                    }
                    acc += __shfl_xor_sync(FULL, acc, 1);
                    acc += __shfl_xor_sync(FULL, acc, 2);
                    acc += __shfl_xor_sync(FULL, acc, 4);
                    sc[ps] = (r < rows) ? acc : -INFINITY;
                }

                // online softmax over this warp's rows of the tile
                float mt = sc[0];
#pragma unroll
                for (int ps = 1; ps < C::kPasses; ++ps) mt = fmaxf(mt, sc[ps]);
                mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 8));
                mt = fmaxf(mt, __shfl_xor_sync(FULL, mt, 16));
                const float m_new = fmaxf(m_run, mt);
                const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
                const float alpha = exp2f(m_run - m_ref);
                float pw[C::kPasses];
                float ls = 0.f;
#pragma unroll
                for (int ps = 0; ps < C::kPasses; ++ps) {
                    pw[ps] = exp2f(sc[ps] - m_ref);
                    ls += pw[ps];
                }
                ls += __shfl_xor_sync(FULL, ls, 8);
                ls += __shfl_xor_sync(FULL, ls, 16);
                l_run = l_run * alpha + ls;
                m_run = m_new;
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] *= alpha;

                // O += P V over this warp's rows
#pragma unroll
                for (int it = 0; it < C::kPvIters; ++it) {
                    const int lr = it * C::kPvRowsPerIter + pv_row;
                    const int ps = (it * C::kPvRowsPerIter) / 4;
                    const float pr = __shfl_sync(FULL, pw[ps], (lr & 3) * 8);
                    const int r = row0 + lr;
                    if (r < rows) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(
                            vt + r * C::kRowBytes + pv_chunk * 16);
                        float f[8];
                        widen8<T>(raw, f);
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = fmaf(pr, f[e], o[e]);
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }

        // ---- merge: lanes of one warp, then the warps, then (maybe) blocks
#pragma unroll
        for (int off = C::kPvLanesPerRow; off < 32; off <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(FULL, o[e], off);
        float *ws = wstate + warp * C::kStateFloats;
        if (lane < C::kPvLanesPerRow) {
#pragma unroll
            for (int e = 0; e < 8; ++e) ws[lane * 8 + e] = o[e];
        }
        if (lane == 0) {
            ws[D] = m_run;
            ws[D + 1] = l_run;
        }
        // blocks first..last share a split unit; the one the block ends with may
        // be finished on chip
        int first = 0, last = 0, first_slot = 0;
        if (!seg.whole) unit_parts(S, seg, first, last, first_slot);
        const int la_parts =
            kLook && wk.t >= wk.t_end ? lookahead_parts(seg, first, last, C::kMaxPartners) : 0;
        if (la_parts && tid == 0) flags[kFlagOnChip] = lookahead_claim(flags);
        named_barrier(1, C::kConsumers);
        const bool on_chip = la_parts && flags[kFlagOnChip];

        const bool aborted = flags[0] != 0;
        if (tid < D && !aborted) {
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) M = fmaxf(M, wstate[w * C::kStateFloats + D]);
            const float M_ref = (M == -INFINITY) ? 0.f : M;
            float L = 0.f, O = 0.f;
#pragma unroll
            for (int w = 0; w < C::kConsumerWarps; ++w) {
                const float c = exp2f(wstate[w * C::kStateFloats + D] - M_ref);
                L = fmaf(c, wstate[w * C::kStateFloats + D + 1], L);
                O = fmaf(c, wstate[w * C::kStateFloats + tid], O);
            }
            if (seg.whole) {
                T *orow = static_cast<T *>(p.out) + ((size_t)b * p.H_q + h) * D;
                orow[tid] = Elem<T>::from_float(O / L);
            } else if (on_chip) {
                // part 0 of the unit, beside the copies of the others
                own_part[tid] = O;
                if (tid == 0) {
                    own_part[D] = M;
                    own_part[D + 1] = L;
                }
            } else {
                // this block's first unit goes to slot 2c, any later partial one to 2c+1
                float *slot = p.slots + (size_t)(2 * blockIdx.x + (first_seg ? 0 : 1)) *
                                            p.slot_floats;
                slot[tid] = O;
                if (tid == 0) {
                    slot[D] = M;
                    slot[D + 1] = L;
                }
                __threadfence();
            }
        }
        named_barrier(1, C::kConsumers);

        if (on_chip) {
            // every other part has arrived and none merged: this block merges
            if (!mbar_wait(part_bar, 0)) {
                atomicOr(&g_sha_status, kStatusTimeout);
                flags[0] = 1;
            }
            named_barrier(1, C::kConsumers);
            if (tid == 0) flags[1] = !flags[0];
            named_barrier(1, C::kConsumers);
            if (flags[1]) {
                T *orow = static_cast<T *>(p.out) + ((size_t)b * p.H_q + h) * D;
                merge_parts<T, D, C::kConsumers>(SharedParts{own_part, C::kPartFloats, D}, la_parts,
                                                  1, orow, wstate, tid);
                if (tid == 0) p.counters[first] = 0;
            }
        } else if (!seg.whole) {
            if (tid == 0) {
                int merge = 0;
                if (!flags[0]) {
                    // a split unit's first block is unique to it: its counter slot
                    const int prev = atomicAdd(&p.counters[first], 1);
                    merge = (prev == last - first);
                }
                flags[1] = merge;
            }
            named_barrier(1, C::kConsumers);
            if (flags[1]) {
                // Last block to finish its piece: merge all pieces in block order.
                __threadfence();
                T *orow = static_cast<T *>(p.out) + ((size_t)b * p.H_q + h) * D;
                merge_parts<T, D, C::kConsumers>(
                    GlobalParts{p.slots, p.slot_floats, first, first_slot, D}, last - first + 1, 1,
                    orow, wstate, tid);
                if (tid == 0) p.counters[first] = 0;
            }
        }
    }
    if (kLook && tid == 0) lookahead_claim(flags);   // the scout stops looking
}

}  // namespace sha
