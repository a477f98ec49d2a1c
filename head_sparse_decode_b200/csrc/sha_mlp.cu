// sha_mlp.cu -- Selective GEMM, the MLP half of Polar Sparsity (papernotes.org
// summary, "MLP 层动态稀疏"): for a decode batch x [B, d] and the union S_B of
// the neurons active for any of its rows,
//     MLP_{S_B}(x) = sigma(x W1[:, S_B]) W2[:, S_B]^T,
// computed by reading only the selected neurons' weights, with the index
// gather fused into the GEMMs (no gathered copy of the weights is made).
// Weights are stored neuron-major: W1t = W1^T and W2t = W2^T, [D, d], so
// neuron j's weights are one contiguous row in each.
//
// The union size n_S is produced on the device and never read by the host:
// every kernel reads it from device memory and sizes its work from it, so the
// whole layer is one stream of launches (capturable, no host round trip).
//
// Kernels (each launched with programmatic stream serialization):
//   mlp_union_flags / mlp_union_write -- S_B as sorted neuron ids + n_S
// Batches up to 8 (and the down-projection of batches up to 16), on
// warp-level tensor-core MMAs (mma.sync m16n8k16, fp32 accumulate):
//   mlp_up    -- partial x . W1t[S]^T (fp32): M = 16 gathered neurons, N =
//                batch, K = d streamed in long row segments
//   mlp_act   -- Ht = sigma(sum of the partials), rounded to the input dtype,
//                neuron-major
//   mlp_down  -- partial Ht^T . W2t[S] over a range of neurons (fp32): M =
//                batch, N = up to 1024 output columns, K = neurons
//   mlp_out   -- y = sum of the partials, in a fixed order
// These stream weight-row segments into shared-memory rows padded by 16
// bytes, so ldmatrix reads are free of bank conflicts: 1-D bulk copies (one
// per row and stage, up to 4.5 KiB) for the up-projection, 16-byte cp.async
// copies from four producer warps for the down-projection.
// Batches of 9 to 64, on tcgen05 with fp32 accumulators in tensor memory:
//   mlp_up_tc   -- D[128 neurons x batch] = W1t[S] . x^T, stream-K over
//                  (neuron group, K tile); whole groups write Ht directly
//   mlp_act_tc  -- Ht of the groups split across blocks
//   mlp_down_tc -- D[128 output columns x batch] = W2t[S]^T . Ht^T (from batch
//                  32), stream-K over (512-column block, 64-neuron tile)
//   mlp_out_tc  -- y of the column blocks split across blocks
// Their gathered weight rows are copied by 16-byte cp.async into 128-byte
// swizzled operand tiles (a TMA gather moves too little per operation), the
// dense operand (x, Ht) by one TMA box per stage.
// All of them are bound by HBM: every selected weight byte is read once, and
// the arithmetic intensity is about B flops per weight byte.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <mutex>
#include <type_traits>
#include <utility>

#include <cudaTypedefs.h>

#include "sha_decode.h"
#include "sha_device.cuh"
#include "sha_mma.cuh"
#include "sha_tcgen05.cuh"

namespace {

using namespace sha;

#ifndef SHA_USE_PDL
#define SHA_USE_PDL 1
#endif

// GEMMs of batches above 8 on tcgen05 (1) or on warp-level MMAs (0); the
// down-projection joins from padded batch SHA_MLP_TC_DOWN_MIN_BATCH up.
#ifndef SHA_MLP_TC
#define SHA_MLP_TC 1
#endif
#ifndef SHA_MLP_TC_DOWN_MIN_BATCH
#define SHA_MLP_TC_DOWN_MIN_BATCH 32
#endif

constexpr int kMaxDevicesMlp = 64;
constexpr int kMlpMaxBatch = 64;        // batch rows per call (MMA tiles cover 64)
constexpr int kUnionChunk = 256;        // neurons per block in the union kernels
constexpr int kUnionThreads = 256;
constexpr int kUnionRowGroups = kUnionThreads / (kUnionChunk / 4);   // batch rows split 4 ways

// ---------------------------------------------------------------- union

// flags[j] = 1 if any row of the batch has neuron j active; counts[block] =
// the number of such neurons in the block's chunk.  A thread ORs four
// neighbouring neurons over every fourth batch row (one 32-bit load per row
// when the mask rows are 4-byte aligned).
__global__ void __launch_bounds__(kUnionThreads)
    mlp_union_flags_kernel(const uint8_t *__restrict__ active, int B, int D, int words,
                           uint8_t *__restrict__ flags, int *__restrict__ counts)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ uint32_t part[kUnionRowGroups][kUnionChunk / 4];
    __shared__ int warp_sum[kUnionThreads / 32];
    const int quad = threadIdx.x % (kUnionChunk / 4), rg = threadIdx.x / (kUnionChunk / 4);
    const int j = blockIdx.x * kUnionChunk + quad * 4;
    uint32_t any = 0;
    if (j < D) {
        if (words) {
            for (int b = rg; b < B; b += kUnionRowGroups)
                any |= __ldg(reinterpret_cast<const uint32_t *>(active + (size_t)b * D + j));
        } else {
            const int n = min(4, D - j);
            for (int b = rg; b < B; b += kUnionRowGroups)
                for (int i = 0; i < n; ++i)
                    any |= (uint32_t)active[(size_t)b * D + j + i] << (8 * i);
        }
    }
    part[rg][quad] = any;
    __syncthreads();
    int cnt = 0;
    if (rg == 0 && j < D) {
        for (int r = 1; r < kUnionRowGroups; ++r) any |= part[r][quad];
        uint32_t f = 0;
        for (int i = 0; i < 4; ++i)
            if (j + i < D && ((any >> (8 * i)) & 0xffu)) {
                f |= 1u << (8 * i);
                ++cnt;
            }
        if (words)
            *reinterpret_cast<uint32_t *>(flags + j) = f;
        else
            for (int i = 0; i < min(4, D - j); ++i) flags[j + i] = (f >> (8 * i)) & 1u;
    }
    for (int off = 16; off > 0; off >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, off);
    if ((threadIdx.x & 31) == 0) warp_sum[threadIdx.x >> 5] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        int total = 0;
        for (int w = 0; w < kUnionThreads / 32; ++w) total += warp_sum[w];
        counts[blockIdx.x] = total;
    }
}

// S = the flagged neuron ids in increasing order, n_S = their number.  Each
// block adds up the counts of the blocks before it, then writes its chunk at
// that offset in thread order.
__global__ void __launch_bounds__(kUnionThreads)
    mlp_union_write_kernel(const uint8_t *__restrict__ flags, const int *__restrict__ counts,
                           int D, int32_t *__restrict__ S, int32_t *__restrict__ n_S)
{
    pdl_wait();
    pdl_launch_dependents();
    static_assert(kUnionChunk == kUnionThreads, "one neuron per thread");
    __shared__ int warp_sum[kUnionThreads / 32];
    __shared__ int s_base;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int before = 0;
    for (int i = threadIdx.x; i < (int)blockIdx.x; i += kUnionThreads) before += counts[i];
    for (int off = 16; off > 0; off >>= 1) before += __shfl_xor_sync(0xffffffffu, before, off);
    if (lane == 0) warp_sum[warp] = before;
    __syncthreads();
    if (threadIdx.x == 0) {
        int base = 0;
        for (int w = 0; w < kUnionThreads / 32; ++w) base += warp_sum[w];
        s_base = base;
        if (blockIdx.x == gridDim.x - 1) *n_S = base + counts[blockIdx.x];
    }
    __syncthreads();
    const int j = blockIdx.x * kUnionChunk + threadIdx.x;
    const int f = j < D ? flags[j] : 0;
    // exclusive prefix of the flags over the block, in thread order
    int incl = f;
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += x;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int pos = s_base + incl - f;
    for (int w = 0; w < warp; ++w) pos += warp_sum[w];
    if (f) S[pos] = j;
}

// The union size and ids come from device memory (the union kernel or the
// caller): keep every access inside the weight arrays whatever they hold.
__device__ __forceinline__ int union_size(const int32_t *n_S_ptr, int D)
{
    const int n = *n_S_ptr;
    return n < 0 ? 0 : (n > D ? D : n);
}

__device__ __forceinline__ int neuron_id(const int32_t *S, int t, int D)
{
    const int j = S[t];
    if ((unsigned)j >= (unsigned)D) {
        atomicOr(&g_sha_status, kStatusBadIndex);
        return 0;
    }
    return j;
}

// ---------------------------------------------------------------- up-projection
//
// An item is kUpRows gathered neurons x the whole hidden width d (or a range
// of it when the union is too small to give every block several items).
// Each stage holds kUpRows weight-row segments and the matching x segments,
// kstage elements long (2 KiB for batches up to 16), so DRAM sees long
// contiguous runs of each selected row.  The four consumer warps split a
// stage's columns; their partial products go to the workspace separately
// and the activation kernel adds them up.

constexpr int kUpRows = 16;

// Build-time tuning of the up-projection for batches up to 8.
#ifndef SHA_MLP_UP8_K
#define SHA_MLP_UP8_K 2304
#endif
#ifndef SHA_MLP_UP8_STAGES
#define SHA_MLP_UP8_STAGES 2
#endif

template <int BP>
struct UpCfg {
    static constexpr int kConsumerWarps = 4;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    // d per stage and stages: the longest weight-row segments that fit two
    // (or three) stages next to the matching x rows
    static constexpr int kKMax =
        BP == 8 ? SHA_MLP_UP8_K : (BP == 16 ? 1536 : (BP == 32 ? 1024 : 512));
    static constexpr int kStages = BP == 8 ? SHA_MLP_UP8_STAGES : 2;
    static constexpr int kRow = kKMax * 2 + 16;        // padded row: conflict-free ldmatrix
    static constexpr int kStage = (kUpRows + BP) * kRow;
    static constexpr int kBarOffset = kStages * kStage;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8;
};

// Width of a stage along d (or of an output-column range): the largest
// multiple of 256 not above kmax that divides d (d is a multiple of 256).
__host__ __device__ __forceinline__ int stage_width(int d, int kmax)
{
    int k = kmax / 256 * 256;
    while (k > 256 && d % k != 0) k -= 256;
    return k;
}

// Items of the up-projection: groups of kUpRows neurons, each over `splits`
// ranges of d; the partial buffer holds splits * 4 (warps) sums per neuron.
__host__ __device__ __forceinline__ void up_plan(int n_S, int d, int kstage, int blocks,
                                                 int &groups, int &splits)
{
    groups = (n_S + kUpRows - 1) / kUpRows;
    const int ktiles = d / kstage;
    splits = groups > 0 ? (4 * blocks + groups - 1) / groups : 1;
    if (splits > ktiles) splits = ktiles;
    if (splits < 1) splits = 1;
}

template <typename T, int BP>
__global__ void __launch_bounds__(UpCfg<BP>::kThreads, 1)
    mlp_up_kernel(const T *__restrict__ x, const T *__restrict__ W1t,
                  const int32_t *__restrict__ S, const int32_t *__restrict__ n_S_ptr, int B,
                  int d, int D, float *__restrict__ part)
{
    using C = UpCfg<BP>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::kConsumerWarps);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    const int n_S = union_size(n_S_ptr, D);
    const int kstage = stage_width(d, C::kKMax);
    int groups, splits;
    up_plan(n_S, d, kstage, gridDim.x, groups, splits);
    const int items = groups * splits, ktiles = d / kstage;
    const int n_pad = groups * kUpRows;

    if (warp == C::kConsumerWarps) {
        // producer warp: lanes 0..15 fetch weight-row segments, all lanes x rows
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        // the ids of an item's neurons are loaded one item ahead, so the
        // pipeline never waits on them at an item boundary
        auto item_id = [&](int it) {
            const int t = (it / splits) * kUpRows + lane;
            return (it < items && lane < kUpRows && t < n_S) ? neuron_id(S, t, D) : -1;
        };
        int id_next = item_id(blockIdx.x);
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const int grp = item / splits, split = item % splits;
            const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
            const int id = id_next;
            id_next = item_id(item + gridDim.x);
            const int valid = min(kUpRows, n_S - grp * kUpRows);
            for (int kt = kt0; kt < kt1; ++kt) {
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                if (lane == 0)
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)((valid + B) * kstage * 2));
                __syncwarp();
                unsigned char *ws = smem + stage * C::kStage;
                unsigned char *xs = ws + kUpRows * C::kRow;
                const size_t k0 = (size_t)kt * kstage;
                if (id >= 0)
                    bulk_copy_g2s(ws + lane * C::kRow, W1t + (size_t)id * d + k0, kstage * 2,
                                  &full[stage], policy);
                for (int b = lane; b < B; b += 32)
                    bulk_copy_g2s(xs + b * C::kRow, x + (size_t)b * d + k0, kstage * 2,
                                  &full[stage], policy);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
        return;
    }

    // consumers: all kUpRows neurons x the batch, over a quarter of each stage
    const int g = lane >> 2, qd = lane & 3, mi = lane >> 3;
    constexpr int kNT = BP / 8;                       // 8-row batch tiles
    const int ntiles = (B + 7) / 8;
    static_assert(BP == 8 || kNT % 2 == 0, "batch tiles come in pairs above 8 rows");
    const int k16_per_warp = kstage / 16 / C::kConsumerWarps;
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t base = smem_addr(smem);
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int grp = item / splits, split = item % splits;
        const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
        float acc[kNT][4];
#pragma unroll
        for (int nt = 0; nt < kNT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
        for (int kt = kt0; kt < kt1; ++kt) {
            const bool live = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase));
            if (live) {
                const uint32_t ws = base + stage * C::kStage, xs = ws + kUpRows * C::kRow;
                for (int kk = 0; kk < k16_per_warp; ++kk) {
                    const int k16 = warp * k16_per_warp + kk;
                    uint32_t a[4];
                    ldmatrix_x4(ws + (lane & 15) * C::kRow + (k16 * 16 + (lane >> 4) * 8) * 2, a);
                    if constexpr (BP == 8) {
                        // one 8-row batch tile: x rows 0-7 at k and k+8
                        uint32_t kb[2];
                        ldmatrix_x2(xs + (lane & 7) * C::kRow + (k16 * 16 + ((lane >> 3) & 1) * 8) * 2,
                                    kb);
                        mma_16816<T>(acc[0], a, kb[0], kb[1]);
                    } else {
#pragma unroll
                        for (int np = 0; np < kNT / 2; ++np) {
                            if (np * 2 >= ntiles) break;             // warp-uniform
                            uint32_t kb[4];
                            ldmatrix_x4(xs + (np * 16 + (mi >> 1) * 8 + (lane & 7)) * C::kRow +
                                            (k16 * 16 + (mi & 1) * 8) * 2,
                                        kb);
                            mma_16816<T>(acc[2 * np], a, kb[0], kb[1]);
                            mma_16816<T>(acc[2 * np + 1], a, kb[2], kb[3]);
                        }
                    }
                }
            } else if (lane == 0) {
                atomicOr(&g_sha_status, kStatusTimeout);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        // part[(split*4 + warp)][neuron][batch], batch padded to BP
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const int t = grp * kUpRows + g + 8 * r;
            if (t >= n_S) continue;
            float *dst = part + ((size_t)(split * C::kConsumerWarps + warp) * n_pad + t) * BP;
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt)
                if (nt < ntiles)
                    *reinterpret_cast<float2 *>(dst + nt * 8 + qd * 2) =
                        make_float2(acc[nt][2 * r], acc[nt][2 * r + 1]);
        }
    }
}

// Ht[t, b] = sigma(sum of the partial products), rounded to T, neuron-major
// ([n rows][BP]); zero outside the batch and the union.
template <typename T, int BP>
__global__ void mlp_act_kernel(const float *__restrict__ part, const int32_t *__restrict__ n_S_ptr,
                               int B, int d, int D, int h_rows, int up_blocks, int act,
                               T *__restrict__ Ht)
{
    pdl_wait();
    pdl_launch_dependents();
    const int n_S = union_size(n_S_ptr, D);
    const int kstage = stage_width(d, UpCfg<BP>::kKMax);
    int groups, splits;
    up_plan(n_S, d, kstage, up_blocks, groups, splits);
    const int n_pad = groups * kUpRows;
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)h_rows * BP) return;
    const int t = (int)(i / BP), b = (int)(i % BP);
    float v = 0.f;
    if (t < n_S && b < B) {
        for (int s = 0; s < splits * UpCfg<BP>::kConsumerWarps; ++s)
            v += part[((size_t)s * n_pad + t) * BP + b];
        if (act == 1) v = fmaxf(v, 0.f);
    }
    Ht[i] = Elem<T>::from_float(v);
}

// ---------------------------------------------------------------- up-projection on tcgen05
//
// For batches of 9 to 64 rows the arithmetic per weight byte (about B flops)
// is more than warp-level MMAs sustain at HBM speed, so the up-projection of
// those batches runs on the fifth-generation tensor cores:
//     D [128 neurons x BP] (fp32, in TMEM) = W1t[S rows] . x^T
// A = 128 gathered weight rows and B = the batch's x rows, both K-major with
// 128-byte swizzle, four 64-element K atoms (256 elements) per stage.  Four
// producer warps copy the rows with 16-byte cp.async (a TMA four-row gather
// moves at most 512 bytes per operation, too little to keep HBM busy); x is
// one TMA box per atom.  One thread issues the MMAs; four epilogue warps read
// the accumulator (double-buffered in TMEM) back.
//
// Work units are (group of 128 neurons, 256-element K tile); block b takes the
// contiguous unit range [b U / NB, (b+1) U / NB) (stream-K), so every block
// streams the same number of weight bytes at any union size.  A group whose
// K tiles all fall in one block is finished there: the activation is applied
// and its Ht rows written.  A group split across blocks leaves fp32 partial
// sums in slot 0 (the block's first group) or slot 1 (its last group) of the
// block, and mlp_act_tc adds them up in block order.

namespace uptc {
constexpr int kM = 128;                    // neurons per group (MMA M)
constexpr int kAtomK = 64;                 // elements per 128-byte swizzled row
constexpr int kAtoms = 4;                  // K atoms per stage
constexpr int kStageK = kAtoms * kAtomK;   // elements of K per stage
constexpr int kProducerWarps = 4;        // cp.async copies of the gathered rows
constexpr int kMmaWarp = kProducerWarps;   // then four epilogue warps
constexpr int kThreads = (kProducerWarps + 5) * 32;
}  // namespace uptc

template <int BP>
struct UpTcCfg {
    static constexpr int kAAtom = uptc::kM * 128;             // bytes of one A K atom
    static constexpr int kABytes = uptc::kAtoms * kAAtom;
    static constexpr int kBAtom = BP * 128;
    static constexpr int kBBytes = uptc::kAtoms * kBAtom;
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kStages = BP == 16 ? 3 : 2;
    static constexpr int kBarOffset = kStages * kStage;
    // full[s], empty[s], acc_full[2], acc_empty[2], mma_done; the TMEM address
    static constexpr int kBarBytes = (2 * kStages + 5) * 8 + 8;
    static constexpr int kSmemBytes = 1024 + kBarOffset + kBarBytes;   // + alignment slack
    static constexpr uint32_t kTmemCols = 2 * BP < 32 ? 32 : 2 * BP;   // two accumulators
    static_assert(BP % 16 == 0 && BP <= 64, "N = BP: a multiple of 16 up to 64");
    static_assert(kAAtom % 1024 == 0 && kBAtom % 1024 == 0 && kStage % 1024 == 0,
                  "swizzle atoms stay 1 KiB aligned");
    static_assert(kSmemBytes <= 232448, "fits the shared-memory opt-in");
};

// Stream-K split of U units over NB blocks.
struct UnitSplit {
    long long U;
    int NB;
    __device__ __forceinline__ long long begin(int b) const { return U * b / NB; }
};

__device__ __forceinline__ uint64_t l2_policy_evict_last()
{
    uint64_t policy;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(policy));
    return policy;
}

// kBatchMajor: Ht stored [BP][h_rows] (the tcgen05 down-projection's K-major
// operand); otherwise [h_rows][BP] (the warp-level down-projection's).
template <typename T, int BP, bool kBatchMajor>
__global__ void __launch_bounds__(uptc::kThreads, 1)
    mlp_up_tc_kernel(const __grid_constant__ CUtensorMap tm_x,
                     const T *__restrict__ W1t, const int32_t *__restrict__ S,
                     const int32_t *__restrict__ n_S_ptr, int B, int d, int D, int act, int h_rows,
                     float *__restrict__ part, T *__restrict__ Ht)
{
    using C = UpTcCfg<BP>;
    using namespace uptc;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // the x box's expect-tx arrival, plus one cp.async arrival per producer thread
            mbar_init(&full[s], 1 + 32 * kProducerWarps);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(mma_done, 1);
        mbar_init_fence();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    pdl_wait();
    pdl_launch_dependents();

    const int n_S = union_size(n_S_ptr, D);
    const int KT = d / kStageK;
    const UnitSplit split{(long long)((n_S + kM - 1) / kM) * KT, (int)gridDim.x};
    const long long u0 = split.begin(blockIdx.x), u1 = split.begin(blockIdx.x + 1);
    const int g_first = (int)(u0 / KT);

    if (warp < kProducerWarps) {
        const uint64_t pol_w = l2_policy_evict_first(), pol_x = l2_policy_evict_last();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        for (long long u = u0; u < u1 && ok;) {
            const int g = (int)(u / KT);
            const int kt0 = (int)(u - (long long)g * KT);
            const int kt1 = (int)min((long long)KT, u1 - (long long)g * KT);
            // warp p copies rows 32p..32p+31: copy i of a k atom moves 128 bytes of
            // rows 32p+4i .. +3 (eight lanes per row, one 16-byte chunk each) to
            // their swizzled places (ids past the union repeat its last neuron;
            // their rows are computed and dropped)
            const int chunk = lane & 7;
            int row[8];
            const T *src[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                row[i] = 32 * warp + 4 * i + (lane >> 3);
                const int id = neuron_id(S, min(g * kM + row[i], n_S - 1), D);
                src[i] = W1t + (size_t)id * d + chunk * 8;
            }
            for (int kt = kt0; kt < kt1; ++kt) {
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                unsigned char *sa = smem + stage * C::kStage;
                unsigned char *sb = sa + C::kABytes;
                const int k0 = kt * kStageK;
                if (warp == 0) {
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], (uint32_t)C::kBBytes);
                    __syncwarp();
                    if (lane < kAtoms)
                        tma_load_2d(sb + lane * C::kBAtom, &tm_x, k0 + lane * kAtomK, 0,
                                    &full[stage], pol_x);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
#pragma unroll
                    for (int j = 0; j < kAtoms; ++j)
                        cp_async16(sa + j * C::kAAtom + row[i] * 128 + ((chunk ^ (row[i] & 7)) << 4),
                                   src[i] + k0 + j * kAtomK, pol_w);
                cp_async_arrive_noinc(&full[stage]);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
            u = (long long)(g + 1) * KT;
        }
        // no copy may be in flight when the block exits
        cp_async_wait_all();
        if (warp == 0 && lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_f16(!std::is_same<T, __half>::value, kM, BP);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const int g = (int)(u / KT);
                const int kt0 = (int)(u - (long long)g * KT);
                const int kt1 = (int)min((long long)KT, u1 - (long long)g * KT);
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t dt = tmem + (uint32_t)(acc * BP);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!mbar_wait(&full[stage], phase)) {
                        atomicOr(&g_sha_status, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    fence_proxy_async_shared();    // copied rows -> tensor-core reads
                    tc_fence_after_sync();
                    const uint32_t sa = smem_addr(smem + stage * C::kStage);
                    const uint32_t sb = sa + C::kABytes;
#pragma unroll
                    for (int j = 0; j < kAtoms; ++j)
#pragma unroll
                        for (int kk = 0; kk < kAtomK / 16; ++kk)
                            umma_f16(dt, umma_desc_k_sw128(sa + j * C::kAAtom + kk * 32),
                                     umma_desc_k_sw128(sb + j * C::kBAtom + kk * 32), idesc,
                                     (kt > kt0 || j > 0 || kk > 0) ? 1u : 0u);
                    umma_commit(&empty[stage]);          // stage reusable once read
                    if (++stage == C::kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
                u = (long long)(g + 1) * KT;
            }
            // every issued MMA has finished before TMEM is released
            if (u1 > u0) {
                umma_commit(mma_done);
                if (!mbar_wait_drain(mma_done, 0)) atomicOr(&g_sha_status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4)..+31 = neuron rows of the group
        const int quarter = warp & 3, row = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (long long u = u0; u < u1;) {
            const int g = (int)(u / KT);
            const int kt0 = (int)(u - (long long)g * KT);
            const int kt1 = (int)min((long long)KT, u1 - (long long)g * KT);
            const bool live = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase));
            if (!live) {
                if (lane == 0) atomicOr(&g_sha_status, kStatusTimeout);
                break;
            }
            tc_fence_after_sync();
            float v[BP / 16][16];
#pragma unroll
            for (int c = 0; c < BP / 16; ++c)
                tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * BP + c * 16),
                          v[c]);
            tmem_ld_wait();
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            const int t = g * kM + row;
            if (kt0 == 0 && kt1 == KT) {
                // whole group here: Ht = sigma(D), zero outside the union and batch
                if constexpr (kBatchMajor) {
#pragma unroll
                    for (int col = 0; col < BP; ++col) {
                        float x = v[col / 16][col % 16];
                        if (act == 1) x = fmaxf(x, 0.f);
                        Ht[(size_t)col * h_rows + t] =
                            Elem<T>::from_float((t < n_S && col < B) ? x : 0.f);
                    }
                } else {
#pragma unroll
                    for (int c8 = 0; c8 < BP / 8; ++c8) {
                        __align__(16) T h[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = c8 * 8 + e;
                            float x = v[col / 16][col % 16];
                            if (act == 1) x = fmaxf(x, 0.f);
                            h[e] = Elem<T>::from_float((t < n_S && col < B) ? x : 0.f);
                        }
                        *reinterpret_cast<uint4 *>(Ht + (size_t)t * BP + c8 * 8) =
                            *reinterpret_cast<const uint4 *>(h);
                    }
                }
            } else {
                // partial sums, column-major per slot: [slot][col][row]
                const int slot = g == g_first ? 0 : 1;
                float *dst = part + (size_t)(blockIdx.x * 2 + slot) * BP * kM + row;
#pragma unroll
                for (int col = 0; col < BP; ++col) dst[(size_t)col * kM] = v[col / 16][col % 16];
            }
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            u = (long long)(g + 1) * KT;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// The split as the fix-up kernels compute it: 32-bit arithmetic (the host
// keeps U * NB below 2^32), so the per-block setup stays cheap.
struct UnitSplit32 {
    uint32_t U, NB;
    __device__ __forceinline__ uint32_t begin(uint32_t b) const { return U * b / NB; }
    __device__ __forceinline__ uint32_t owner(uint32_t u) const
    {
        return ((u + 1) * NB + U - 1) / U - 1;
    }
};

// Fills, for item `item` (units item*per_item .. +per_item) of a split, the
// blocks that hold part of it in block order -- blk[k] = bf + k, slot[k] = 0
// if the item is that block's first, 1 if not, -1 for a block with no units
// -- one entry per thread of the calling block, and returns how many (0 when
// one block holds the whole item).  Ends with a block barrier.
__device__ __forceinline__ int split_contributors(const UnitSplit32 &split, uint32_t item,
                                                  uint32_t per_item, int *slot, int *s_bf,
                                                  int *s_n)
{
    if (threadIdx.x == 0) {
        const uint32_t bf = split.owner(item * per_item);
        const uint32_t bl = split.owner((item + 1) * per_item - 1);
        *s_bf = (int)bf;
        *s_n = bf == bl ? 0 : (int)(bl - bf + 1);
    }
    __syncthreads();
    const int n = *s_n;
    for (int k = threadIdx.x; k < n; k += blockDim.x) {
        const uint32_t b = (uint32_t)(*s_bf + k), a = split.begin(b);
        slot[k] = a == split.begin(b + 1) ? -1 : (item == a / per_item ? 0 : 1);
    }
    __syncthreads();
    return n;
}

constexpr int kMaxContributors = 256;     // >= the blocks of a split (one per SM)

// Ht entries (layout as in mlp_up_tc) of the groups mlp_up_tc split across
// blocks: the blocks' partial sums added in block order, then sigma; zero
// outside the union and batch.  Block (g, j) covers columns kActCols*j ..
// +kActCols of group g, two columns at a time, one thread per (column, neuron).
constexpr int kActCols = 8;

template <typename T, int BP, bool kBatchMajor>
__global__ void __launch_bounds__(2 * uptc::kM)
    mlp_act_tc_kernel(const float *__restrict__ part, const int32_t *__restrict__ n_S_ptr, int B,
                      int d, int D, int up_blocks, int act, int h_rows, T *__restrict__ Ht)
{
    using namespace uptc;
    __shared__ int s_slot[kMaxContributors], s_bf, s_n;
    pdl_wait();
    pdl_launch_dependents();
    const int n_S = union_size(n_S_ptr, D);
    const int KT = d / kStageK, G = (n_S + kM - 1) / kM, g = blockIdx.x;
    if (g >= G) return;
    const UnitSplit32 split{(uint32_t)(G * KT), (uint32_t)up_blocks};
    const int n = split_contributors(split, (uint32_t)g, (uint32_t)KT, s_slot, &s_bf, &s_n);
    if (n == 0) return;                         // finished by the up-projection
    // this thread: neuron `row`, columns col0, col0 + 2, ... (kActCols / 2 of
    // them, summed side by side so their loads are in flight together)
    constexpr int kPer = kActCols / 2;
    const int row = threadIdx.x % kM, t = g * kM + row;
    const int col0 = blockIdx.y * kActCols + threadIdx.x / kM;
    float v[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) v[j] = 0.f;
    for (int k = 0; k < n; ++k) {
        if (s_slot[k] < 0) continue;
        const float *src = part + (size_t)((s_bf + k) * 2 + s_slot[k]) * BP * kM + row;
#pragma unroll
        for (int j = 0; j < kPer; ++j) v[j] += src[(size_t)(col0 + 2 * j) * kM];
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int col = col0 + 2 * j;
        const float x = act == 1 ? fmaxf(v[j], 0.f) : v[j];
        Ht[kBatchMajor ? (size_t)col * h_rows + t : (size_t)t * BP + col] =
            Elem<T>::from_float((t < n_S && col < B) ? x : 0.f);
    }
}

// ---------------------------------------------------------------- down-projection on tcgen05
//
// y[b][c] = sum over the union of Ht[b][t] W2t[S_t][c], for batches of 9 to 64
// rows, on the fifth-generation tensor cores:
//     D [128 output columns x BP] (fp32, TMEM) = W2t[S rows][columns]^T . Ht^T
// An item is 256 output columns (two accumulators, so each selected weight
// row is read in 512-byte runs) over a range of the union in stages of 64
// neurons.  A = the stage's weight-row segments, MN-major (output columns
// contiguous) with 128-byte swizzle, copied by four producer warps with
// 16-byte cp.async (one 512-byte row segment per warp instruction); B = the
// stage's 64 x BP block of the batch-major activations (one TMA box, K-major).
// Units are (256-column block, 64-neuron tile), split over the blocks as in
// the up-projection: a column block whose tiles all fall in one block is
// written to y there; a split one leaves fp32 partial sums in the block's
// slot 0 (first column block) or 1 (last) and mlp_out_tc adds them in block
// order.

// Output columns per item: 512 (four accumulators, 1 KiB runs of each weight
// row) when they divide d, else 256.
#ifndef SHA_MLP_DOWN_TC_WIDE
#define SHA_MLP_DOWN_TC_WIDE 1
#endif

// Neurons per stage of the down-projection: 64 (Ht tile one 128-byte swizzle
// atom) or 32 (64-byte swizzle; twice the stages in the same shared memory).
#ifndef SHA_MLP_DOWN_TC_ROWS
#define SHA_MLP_DOWN_TC_ROWS 64
#endif

namespace downtc {
constexpr int kM = 128;                    // output columns per accumulator (MMA M)
constexpr int kR = SHA_MLP_DOWN_TC_ROWS;   // neurons per stage (K steps of 16)
static_assert(kR == 32 || kR == 64, "a stage's Ht tile is one 64- or 128-byte swizzle row");
constexpr int kProducerWarps = 4;
constexpr int kMmaWarp = kProducerWarps;   // then four epilogue warps
constexpr int kThreads = (kProducerWarps + 5) * 32;
}  // namespace downtc

template <int BP, int kHalves>
struct DownTcCfg {
    static constexpr int kCols = downtc::kM * kHalves;                 // output columns per item
    static constexpr int kABytes = downtc::kR * kCols * 2;
    static constexpr int kBBytes = BP * downtc::kR * 2;               // the stage's Ht tile
    static constexpr int kStage = kABytes + kBBytes;
    static constexpr int kStages = (200 * 1024) / kStage;
    static constexpr int kBarOffset = kStages * kStage;
    static constexpr int kBarBytes = (2 * kStages + 5) * 8 + 8;
    static constexpr int kSmemBytes = 1024 + kBarOffset + kBarBytes;
    static constexpr uint32_t kTmemCols = 2 * kHalves * BP;   // two items in flight
    static_assert(kABytes % 1024 == 0 && kStage % 1024 == 0, "swizzle atoms stay 1 KiB aligned");
    static_assert(kTmemCols >= 32 && (kTmemCols & (kTmemCols - 1)) == 0, "TMEM allocation size");
    static_assert(kSmemBytes <= 232448, "fits the shared-memory opt-in");
};

// Work of the down-projection's blocks.  With no more column blocks (CB) than
// blocks (NB), each column block gets its own NB/CB or NB/CB + 1 blocks (the
// first NB % CB column blocks one more), which split its K tiles evenly: a
// block then leaves at most one partial slot.  Otherwise the units are split
// evenly over the blocks (stream-K).  Returns block b's unit range [u0, u1),
// a unit being (column block, tile) = cb * KT + tile.
struct ColumnSplit {
    int CB, KT, NB;
    __host__ __device__ bool aligned() const { return CB <= NB; }
    __host__ __device__ int blocks_of(int cb) const
    {
        return NB / CB + (cb < NB % CB ? 1 : 0);
    }
    __host__ __device__ int first_block(int cb) const
    {
        const int per = NB / CB, extra = NB % CB;
        return cb * per + (cb < extra ? cb : extra);
    }
    __device__ void range(int b, long long &u0, long long &u1) const
    {
        if (!aligned()) {
            const UnitSplit split{(long long)CB * KT, NB};
            u0 = split.begin(b);
            u1 = split.begin(b + 1);
            return;
        }
        const int per = NB / CB, extra = NB % CB;
        int cb, sp, nsp;
        if (b < extra * (per + 1)) {
            cb = b / (per + 1);
            sp = b % (per + 1);
            nsp = per + 1;
        } else {
            const int bb = b - extra * (per + 1);
            cb = extra + bb / per;
            sp = bb % per;
            nsp = per;
        }
        u0 = (long long)cb * KT + (long long)sp * KT / nsp;
        u1 = (long long)cb * KT + (long long)(sp + 1) * KT / nsp;
    }
};

template <typename T, int BP, int kHalves>
__global__ void __launch_bounds__(downtc::kThreads, 1)
    mlp_down_tc_kernel(const __grid_constant__ CUtensorMap tm_h, const T *__restrict__ W2t,
                       const int32_t *__restrict__ S, const int32_t *__restrict__ n_S_ptr, int B,
                       int d, int D, float *__restrict__ part, T *__restrict__ y)
{
    using C = DownTcCfg<BP, kHalves>;
    using namespace downtc;
    constexpr int kCols = C::kCols;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char *smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    uint64_t *acc_full = empty + C::kStages;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *mma_done = acc_empty + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // the Ht box's expect-tx arrival, plus one cp.async arrival per producer thread
            mbar_init(&full[s], 1 + 32 * kProducerWarps);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&acc_full[a], 1);
            mbar_init(&acc_empty[a], 4);
        }
        mbar_init(mma_done, 1);
        mbar_init_fence();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    pdl_wait();
    pdl_launch_dependents();

    const int n_S = union_size(n_S_ptr, D);
    const int KT = (n_S + uptc::kM - 1) / uptc::kM * (uptc::kM / kR);   // tiles of the padded union
    long long u0 = 0, u1 = 0;
    if (KT > 0) ColumnSplit{d / kCols, KT, (int)gridDim.x}.range(blockIdx.x, u0, u1);
    const int cb_first = KT > 0 ? (int)(u0 / KT) : 0;

    if (warp < kProducerWarps) {
        // warp p copies neurons (kR/4)p .. +kR/4 of each stage.  An instruction
        // moves 64 output columns (128 bytes) of four neurons: lane l takes
        // neuron 4j + l/8 of the warp's quad j and 16-byte chunk l%8, so the
        // four rows land as four consecutive 128-byte K rows of one swizzle atom
        // (512 contiguous bytes of shared memory); the 2*kHalves pieces of the
        // same four rows follow back to back.
        const uint64_t pol_w = l2_policy_evict_first(), pol_h = l2_policy_evict_last();
        constexpr int kQuads = kR / 16;                    // neuron quads per warp and stage
        const int rsub = lane >> 3, cc = lane & 7;
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        // this lane's neuron ids of a stage (rows past the union repeat its last
        // neuron: their activations are zero)
        auto stage_ids = [&](int kt, int (&ids)[kQuads]) {
#pragma unroll
            for (int j = 0; j < kQuads; ++j)
                ids[j] = neuron_id(S, min(kt * kR + (kR / 4) * warp + 4 * j + rsub, n_S - 1), D);
        };
        for (long long u = u0; u < u1 && ok;) {
            const int cb = (int)(u / KT);
            const int kt0 = (int)(u - (long long)cb * KT);
            const int kt1 = (int)min((long long)KT, u1 - (long long)cb * KT);
            const T *col_src = W2t + (size_t)cb * kCols + cc * 8;
            int ids_next[kQuads];
            stage_ids(kt0, ids_next);
            for (int kt = kt0; kt < kt1; ++kt) {
                int ids[kQuads];
#pragma unroll
                for (int j = 0; j < kQuads; ++j) ids[j] = ids_next[j];
                if (kt + 1 < kt1) stage_ids(kt + 1, ids_next);
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                unsigned char *sa = smem + stage * C::kStage;
                unsigned char *sb = sa + C::kABytes;
                if (warp == 0) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[stage], (uint32_t)C::kBBytes);
                        tma_load_2d(sb, &tm_h, kt * kR, 0, &full[stage], pol_h);
                    }
                    __syncwarp();
                }
#pragma unroll
                for (int j = 0; j < kQuads; ++j) {
                    const int t = (kR / 4) * warp + 4 * j + rsub, kb = t >> 3, kr = t & 7;
                    const T *src = col_src + (size_t)ids[j] * d;
                    unsigned char *dst = sa + kb * 2048 + kr * 128 + ((cc ^ kr) << 4);
#pragma unroll
                    for (int pc = 0; pc < 2 * kHalves; ++pc)     // accumulator pc/2, 64-column block pc%2
                        cp_async16(dst + ((pc >> 1) * (kR / 8) * 2 + (pc & 1)) * 1024,
                                   src + pc * 64, pol_w);
                }
                cp_async_arrive_noinc(&full[stage]);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
            u = (long long)(cb + 1) * KT;
        }
        // no copy may be in flight when the block exits
        cp_async_wait_all();
        if (warp == 0 && lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
    } else if (warp == kMmaWarp) {
        if (lane == 0) {
            constexpr uint32_t idesc =
                umma_idesc_f16(!std::is_same<T, __half>::value, kM, BP, /*a_mn=*/true);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (long long u = u0; u < u1 && ok;) {
                const int cb = (int)(u / KT);
                const int kt0 = (int)(u - (long long)cb * KT);
                const int kt1 = (int)min((long long)KT, u1 - (long long)cb * KT);
                if (!mbar_wait(&acc_empty[acc], acc_phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    break;
                }
                tc_fence_after_sync();
                const uint32_t dt = tmem + (uint32_t)(acc * kHalves * BP);
                for (int kt = kt0; kt < kt1; ++kt) {
                    if (!mbar_wait(&full[stage], phase)) {
                        atomicOr(&g_sha_status, kStatusTimeout);
                        ok = false;
                        break;
                    }
                    fence_proxy_async_shared();    // copied rows -> tensor-core reads
                    tc_fence_after_sync();
                    const uint32_t sa = smem_addr(smem + stage * C::kStage);
                    const uint32_t sb = sa + C::kABytes;
#pragma unroll
                    for (int ks = 0; ks < kR / 16; ++ks) {
                        const uint64_t bdesc = kR == 64 ? umma_desc_k_sw128(sb + ks * 32)
                                                        : umma_desc_k_sw64(sb + ks * 32);
#pragma unroll
                        for (int h = 0; h < kHalves; ++h)
                            umma_f16(dt + (uint32_t)(h * BP),
                                     umma_desc_mn_sw128(sa + (h * (kR / 8) + 2 * ks) * 2 * 1024, 1024,
                                                        2048),
                                     bdesc, idesc, (kt > kt0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty[stage]);
                    if (++stage == C::kStages) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(&acc_full[acc]);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
                u = (long long)(cb + 1) * KT;
            }
            if (u1 > u0) {
                umma_commit(mma_done);
                if (!mbar_wait_drain(mma_done, 0)) atomicOr(&g_sha_status, kStatusTimeout);
            }
        }
        __syncwarp();
    } else {
        // epilogue: warp w reads TMEM lanes 32*(w%4)..+31 = output columns of each half
        const int quarter = warp & 3, row = quarter * 32 + lane;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (long long u = u0; u < u1;) {
            const int cb = (int)(u / KT);
            const int kt0 = (int)(u - (long long)cb * KT);
            const int kt1 = (int)min((long long)KT, u1 - (long long)cb * KT);
            const bool live = __all_sync(0xffffffffu, mbar_wait(&acc_full[acc], acc_phase));
            if (!live) {
                if (lane == 0) atomicOr(&g_sha_status, kStatusTimeout);
                break;
            }
            tc_fence_after_sync();
            const bool whole = kt0 == 0 && kt1 == KT;
            const int slot = cb == cb_first ? 0 : 1;
#pragma unroll 1
            for (int h = 0; h < kHalves; ++h) {
                float v[BP / 16][16];
#pragma unroll
                for (int c = 0; c < BP / 16; ++c)
                    tmem_ld16(tmem + ((uint32_t)(quarter * 32) << 16) +
                                  (uint32_t)(acc * kHalves * BP + h * BP + c * 16),
                              v[c]);
                tmem_ld_wait();
                const int col = h * kM + row;             // within the item
                if (whole) {
                    T *dst = y + (size_t)cb * kCols + col;
#pragma unroll
                    for (int b = 0; b < BP; ++b)
                        if (b < B) dst[(size_t)b * d] = Elem<T>::from_float(v[b / 16][b % 16]);
                } else {
                    float *dst = part + (size_t)(blockIdx.x * 2 + slot) * BP * kCols + col;
#pragma unroll
                    for (int b = 0; b < BP; ++b) dst[(size_t)b * kCols] = v[b / 16][b % 16];
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            u = (long long)(cb + 1) * KT;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after_sync();
        tmem_dealloc(tmem, C::kTmemCols);
    }
}

// y entries of the column blocks mlp_down_tc split across blocks: the blocks'
// partial sums added in block order; all of y when the union is empty.  Block
// (cb, j) covers batch rows 8j..8j+7 of column block cb, one thread per column.
constexpr int kOutRows = 8;

template <typename T, int BP, int kCols>
__global__ void __launch_bounds__(kCols)
    mlp_out_tc_kernel(const float *__restrict__ part, const int32_t *__restrict__ n_S_ptr, int B,
                      int d, int D, int down_blocks, T *__restrict__ y)
{
    using namespace downtc;
    __shared__ int s_slot[kMaxContributors], s_bf, s_n;
    pdl_wait();
    pdl_launch_dependents();
    const int cb = blockIdx.x, c = cb * kCols + threadIdx.x;
    const int b0 = blockIdx.y * kOutRows, b1 = min(B, b0 + kOutRows);
    const int n_S = union_size(n_S_ptr, D);
    const int KT = (n_S + uptc::kM - 1) / uptc::kM * (uptc::kM / kR);
    if (KT == 0) {
        for (int b = b0; b < b1; ++b) y[(size_t)b * d + c] = Elem<T>::from_float(0.f);
        return;
    }
    const ColumnSplit cs{d / kCols, KT, down_blocks};
    int n;
    if (cs.aligned()) {
        // this column block's own blocks, one partial slot each (none for an
        // empty K range).  An even split of KT tiles over nsp blocks leaves
        // min(nsp, KT) of them non-empty; when that is one, its block covered
        // the whole column block and wrote y itself.
        const int nsp = cs.blocks_of(cb);
        if (threadIdx.x == 0) s_bf = cs.first_block(cb);
        for (int k = threadIdx.x; k < nsp; k += blockDim.x)
            s_slot[k] = (long long)(k + 1) * KT / nsp > (long long)k * KT / nsp ? 0 : -1;
        n = min(nsp, KT) == 1 ? 0 : nsp;
        __syncthreads();
    } else {
        const UnitSplit32 split{(uint32_t)((d / kCols) * KT), (uint32_t)down_blocks};
        n = split_contributors(split, (uint32_t)cb, (uint32_t)KT, s_slot, &s_bf, &s_n);
    }
    if (n == 0) return;                         // written by the down-projection
    // the block's batch rows summed side by side, so their loads are in flight together
    float v[kOutRows];
#pragma unroll
    for (int r = 0; r < kOutRows; ++r) v[r] = 0.f;
    for (int k = 0; k < n; ++k) {
        if (s_slot[k] < 0) continue;
        const float *src = part + ((size_t)((s_bf + k) * 2 + s_slot[k]) * BP + b0) * kCols + threadIdx.x;
#pragma unroll
        for (int r = 0; r < kOutRows; ++r)
            if (b0 + r < b1) v[r] += src[(size_t)r * kCols];
    }
#pragma unroll
    for (int r = 0; r < kOutRows; ++r)
        if (b0 + r < b1) y[(size_t)(b0 + r) * d + c] = Elem<T>::from_float(v[r]);
}

// ---------------------------------------------------------------- down-projection
//
// An item is a range of wc output columns (2 KiB of each weight row for
// batches up to 16) over a range of the union's neurons; stages hold
// kRows weight-row segments and the matching kRows x BP block of the
// neuron-major activations (one contiguous copy).  The weight rows arrive by
// 16-byte cp.async from four producer warps (or, with SHA_MLP_DOWN_CPASYNC=0,
// by one bulk copy per row segment).  Eight consumer warps own wc/8 columns
// each.  Partial sums over the neuron ranges go to the workspace and mlp_out
// adds them in a fixed order.

// Build-time tuning of the down-projection (the feed; widths for batches up to 8).
#ifndef SHA_MLP_DOWN_CPASYNC
#define SHA_MLP_DOWN_CPASYNC 1
#endif
#ifndef SHA_MLP_DOWN8_W
#define SHA_MLP_DOWN8_W 1024
#endif
#ifndef SHA_MLP_DOWN8_ROWS
#define SHA_MLP_DOWN8_ROWS 32
#endif

template <int BP>
struct DownCfg {
    static constexpr int kConsumerWarps = 8;
    // weight rows: one bulk copy per row segment from one producer warp, or
    // 16-byte cp.async copies (128 bytes of four rows per instruction) from four
    static constexpr int kProducerWarps = SHA_MLP_DOWN_CPASYNC ? 4 : 1;
    static constexpr int kThreads = (kConsumerWarps + kProducerWarps) * 32;
    static constexpr int kWMax =                        // columns per item
        BP == 8 ? SHA_MLP_DOWN8_W : (BP == 16 ? 1024 : (BP == 32 ? 1024 : 512));
    static constexpr int kRows = BP == 8 ? SHA_MLP_DOWN8_ROWS : 32;   // neurons per stage
    static constexpr int kStages = 3;
    static constexpr int kWRow = kWMax * 2 + 16;       // padded rows
    static constexpr int kHBytes = kRows * BP * 2;
    static constexpr int kStage = kRows * kWRow + kHBytes;
    static_assert(kRows == 16 || kRows == 32, "one or two k-steps per stage");
    static constexpr int kBarOffset = kStages * kStage;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8;
};

template <typename T, int BP>
__global__ void __launch_bounds__(DownCfg<BP>::kThreads, 1)
    mlp_down_kernel(const T *__restrict__ Ht, const T *__restrict__ W2t,
                    const int32_t *__restrict__ S, const int32_t *__restrict__ n_S_ptr, int B,
                    int d, int D, int splits, float *__restrict__ part)
{
    using C = DownCfg<BP>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + C::kBarOffset);
    uint64_t *empty = full + C::kStages;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::kStages; ++s) {
            // the Ht tile's expect-tx arrival (+ one cp.async arrival per producer thread)
            mbar_init(&full[s], SHA_MLP_DOWN_CPASYNC ? 1 + 32 * C::kProducerWarps : 1);
            mbar_init(&empty[s], C::kConsumerWarps);
        }
        mbar_init_fence();
    }
    __syncthreads();
    pdl_wait();
    pdl_launch_dependents();

    const int n_S = union_size(n_S_ptr, D);
    const int wc = stage_width(d, C::kWMax);
    const int ktiles = (n_S + C::kRows - 1) / C::kRows;
    const int wchunks = d / wc;
    const int items = wchunks * splits;

#if SHA_MLP_DOWN_CPASYNC
    if (warp >= C::kConsumerWarps) {
        // producer warp p (of 4) copies row quads p, p+4, ... of each stage: an
        // instruction moves 128 bytes (64 columns) of four rows, lane l taking
        // row 4q + l/8 and 16-byte chunk l%8; the stage's Ht tile is one bulk
        // copy.  Rows past the union repeat its last neuron (finite values times
        // an activation of 0 add nothing, where stale shared memory could hold NaN).
        constexpr int kQuads = C::kRows / 4 / C::kProducerWarps;   // row quads per warp
        const int pw = warp - C::kConsumerWarps, chunk = lane & 7;
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        auto stage_ids = [&](int kt, int (&ids)[kQuads]) {
#pragma unroll
            for (int j = 0; j < kQuads; ++j)
                ids[j] = neuron_id(
                    S, min(kt * C::kRows + 4 * (pw + C::kProducerWarps * j) + (lane >> 3), n_S - 1), D);
        };
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const int wcn = item / splits, split = item % splits;
            const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
            const size_t c0 = (size_t)wcn * wc;
            int ids_next[kQuads];
            if (kt0 < kt1) stage_ids(kt0, ids_next);
            for (int kt = kt0; kt < kt1; ++kt) {
                int ids[kQuads];
#pragma unroll
                for (int j = 0; j < kQuads; ++j) ids[j] = ids_next[j];
                if (kt + 1 < kt1) stage_ids(kt + 1, ids_next);
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                unsigned char *ws = smem + stage * C::kStage;
                unsigned char *hs = ws + C::kRows * C::kWRow;
                if (pw == 0 && lane == 0) {
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)C::kHBytes);
                    bulk_copy_g2s(hs, Ht + (size_t)kt * C::kRows * BP, C::kHBytes, &full[stage],
                                  policy);
                }
#pragma unroll
                for (int j = 0; j < kQuads; ++j) {
                    const int row = 4 * (pw + C::kProducerWarps * j) + (lane >> 3);
                    const T *src = W2t + (size_t)ids[j] * d + c0 + chunk * 8;
                    unsigned char *dst = ws + row * C::kWRow + chunk * 16;
                    for (int piece = 0; piece < wc / 64; ++piece)
                        cp_async16(dst + piece * 128, src + piece * 64, policy);
                }
                cp_async_arrive_noinc(&full[stage]);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        // no copy may be in flight when the block exits
        cp_async_wait_all();
        if (pw == 0 && lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
        return;
    }
#else
    if (warp == C::kConsumerWarps) {
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        // one weight row per lane and tile; its neuron id is loaded one tile
        // ahead (rows past the union repeat its last neuron: finite values
        // times an activation of 0 add nothing, where stale shared memory
        // could hold NaN)
        auto tile_id = [&](int kt) {
            return (kt < ktiles && lane < C::kRows)
                       ? neuron_id(S, min(kt * C::kRows + lane, n_S - 1), D)
                       : 0;
        };
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const int wcn = item / splits, split = item % splits;
            const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
            const size_t c0 = (size_t)wcn * wc;
            int id_next = tile_id(kt0 < kt1 ? kt0 : ktiles);
            for (int kt = kt0; kt < kt1; ++kt) {
                const int id = id_next;
                id_next = tile_id(kt + 1 < kt1 ? kt + 1 : ktiles);
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                if (lane == 0)
                    mbar_arrive_expect_tx(&full[stage],
                                          (uint32_t)(C::kRows * wc * 2 + C::kHBytes));
                __syncwarp();
                unsigned char *ws = smem + stage * C::kStage;
                unsigned char *hs = ws + C::kRows * C::kWRow;
                const int t0 = kt * C::kRows;
                if (lane < C::kRows)
                    bulk_copy_g2s(ws + lane * C::kWRow, W2t + (size_t)id * d + c0, wc * 2,
                                  &full[stage], policy);
                if (lane == 0)
                    bulk_copy_g2s(hs, Ht + (size_t)t0 * BP, C::kHBytes, &full[stage], policy);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait_drain(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
        return;
    }

#endif

    // consumers: warp w owns output columns [w*wc/8, (w+1)*wc/8) x the batch
    const int g = lane >> 2, qd = lane & 3, mi = lane >> 3;
    constexpr int kMT = BP >= 16 ? BP / 16 : 1;     // 16-row batch tiles (8 rows padded)
    constexpr int kNT = C::kWMax / C::kConsumerWarps / 8;   // 8-column tiles per warp
    const int mtiles = (B + 15) / 16;
    const int nt_used = wc / C::kConsumerWarps / 8;
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t base = smem_addr(smem);
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int wcn = item / splits, split = item % splits;
        const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
        float acc[kMT][kNT][4];
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int nt = 0; nt < kNT; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] =
                                                acc[mt][nt][3] = 0.f;
        const int col0 = warp * (wc / C::kConsumerWarps);
        for (int kt = kt0; kt < kt1; ++kt) {
            const bool live = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase));
            if (live) {
                const uint32_t ws = base + stage * C::kStage, hs = ws + C::kRows * C::kWRow;
#pragma unroll
                for (int k16 = 0; k16 < C::kRows / 16; ++k16) {
                    // activations, neuron-major in shared memory: A = Ht^T via ldmatrix.trans
                    uint32_t a[kMT][4];
                    if constexpr (BP == 8) {
                        // batch rows 0-7 only: the A rows 8-15 are zero
                        uint32_t h2[2];
                        ldmatrix_x2_trans(hs + (k16 * 16 + ((lane >> 3) & 1) * 8 + (lane & 7)) * BP * 2,
                                          h2);
                        a[0][0] = h2[0];
                        a[0][1] = 0u;
                        a[0][2] = h2[1];
                        a[0][3] = 0u;
                    } else {
#pragma unroll
                        for (int mt = 0; mt < kMT; ++mt)
                            if (mt < mtiles)
                                ldmatrix_x4_trans(hs + (k16 * 16 + (mi >> 1) * 8 + (lane & 7)) * BP * 2 +
                                                      (mt * 16 + (mi & 1) * 8) * 2,
                                                  a[mt]);
                    }
#pragma unroll
                    for (int np = 0; np < kNT / 2; ++np) {
                        if (np * 2 >= nt_used) break;               // warp-uniform
                        uint32_t vb[4];
                        ldmatrix_x4_trans(ws + (k16 * 16 + (mi & 1) * 8 + (lane & 7)) * C::kWRow +
                                              (col0 + np * 16 + (mi >> 1) * 8) * 2,
                                          vb);
#pragma unroll
                        for (int mt = 0; mt < kMT; ++mt) {
                            if (mt >= mtiles) break;                 // warp-uniform
                            mma_16816<T>(acc[mt][2 * np], a[mt], vb[0], vb[1]);
                            mma_16816<T>(acc[mt][2 * np + 1], a[mt], vb[2], vb[3]);
                        }
                    }
                }
            } else if (lane == 0) {
                atomicOr(&g_sha_status, kStatusTimeout);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (++stage == C::kStages) { stage = 0; phase ^= 1; }
        }
        // partial sums of this range of neurons: part[split][b][column]
#pragma unroll
        for (int mt = 0; mt < kMT; ++mt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int b = mt * 16 + g + 8 * r;
                if (b >= B) continue;
                float *dst = part + ((size_t)split * kMlpMaxBatch + b) * d + (size_t)wcn * wc + col0;
#pragma unroll
                for (int nt = 0; nt < kNT; ++nt)
                    if (nt < nt_used)
                        *reinterpret_cast<float2 *>(dst + nt * 8 + qd * 2) =
                            make_float2(acc[mt][nt][2 * r], acc[mt][nt][2 * r + 1]);
            }
    }
}

template <typename T>
__global__ void mlp_out_kernel(const float *__restrict__ part, int B, int d, int splits,
                               T *__restrict__ y)
{
    pdl_wait();
    pdl_launch_dependents();
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)B * d) return;
    float v = 0.f;
    for (int s = 0; s < splits; ++s) v += part[(size_t)s * kMlpMaxBatch * d + i];
    y[i] = Elem<T>::from_float(v);
}

// ---------------------------------------------------------------- host

thread_local char g_mlp_error[256] = "no error";

sha_status_t mlp_launch_error(cudaError_t e)
{
    std::snprintf(g_mlp_error, sizeof g_mlp_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return SHA_ERR_LAUNCH;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, int block, size_t smem,
                       cudaStream_t stream, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = SHA_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

bool aligned_to(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int device_sms(int *dev)
{
    if (cudaGetDevice(dev) != cudaSuccess) return 0;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, *dev) != cudaSuccess)
        return 0;
    return sms;
}

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// cuTensorMapEncodeTiled from the driver, found through the runtime so the
// library does not link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 mlp_tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D view [rows][d] of a row-major fp16/bf16 matrix, boxes of box_cols (64
// or 32) elements x box_rows rows with 128- (or 64-) byte swizzle; rows past
// the end read as zero.
sha_status_t mlp_tensor_map(CUtensorMap *map, const void *base, bool bf16, int d, int rows,
                            int box_rows, int box_cols = uptc::kAtomK)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = mlp_tensor_map_encoder();
    if (!encode) {
        std::snprintf(g_mlp_error, sizeof g_mlp_error,
                      "cuTensorMapEncodeTiled is not available from the driver");
        return SHA_ERR_LAUNCH;
    }
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
    cuuint32_t elem[2] = {1, 1};
    CUresult r = encode(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        2, const_cast<void *>(base), dims, strides, box, elem,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_mlp_error, sizeof g_mlp_error,
                      "cuTensorMapEncodeTiled failed with CUresult %d", (int)r);
        return SHA_ERR_LAUNCH;
    }
    return SHA_OK;
}

// Workspace of sha_selective_mlp for these sizes on a device with `sms` SMs.
struct MlpPlan {
    int bp;                // batch padded to 16, 32 or 64
    int h_rows;            // rows of the neuron-major activations (union padded)
    bool tc_up;            // up-projection on tcgen05 (batches above 8)
    bool tc;               // down-projection on tcgen05 as well
    int down_splits, down_blocks;
    int down_wc;           // output columns per warp-level down-projection item
    size_t up_bytes, h_bytes, down_bytes;
    size_t total() const { return up_bytes + h_bytes + down_bytes; }
};

// Batches up to 8 run padded to 8 on warp-level MMAs (1) or padded to 16 on the
// tcgen05 path (0).
#ifndef SHA_MLP_PAD8
#define SHA_MLP_PAD8 1
#endif

int batch_pad(int B)
{
    if (B <= 8) return SHA_MLP_PAD8 ? 8 : 16;
    return B <= 16 ? 16 : (B <= 32 ? 32 : 64);
}

MlpPlan mlp_plan(int B, int d, int D, int sms)
{
    MlpPlan pl;
    pl.bp = batch_pad(B);
    const int kmax = pl.bp == 8 ? DownCfg<8>::kWMax
                                : (pl.bp == 16 ? DownCfg<16>::kWMax
                                               : (pl.bp == 32 ? DownCfg<32>::kWMax : DownCfg<64>::kWMax));
    pl.h_rows = (int)round_up((size_t)D, (size_t)uptc::kM);   // whole neuron groups
    // split sizes the fix-up kernels compute in 32 bits: U * NB < 2^32
    const size_t max_units = ((size_t)D + uptc::kM - 1) / uptc::kM * ((size_t)d / 128);
    pl.tc_up = pl.bp >= 16 && SHA_MLP_TC && sms <= kMaxContributors &&
               max_units * (size_t)(sms + 1) < (1ull << 32);
    pl.tc = pl.tc_up && pl.bp >= SHA_MLP_TC_DOWN_MIN_BATCH;
    if (pl.tc_up) {
        // two partial slots of 128 x BP per block
        pl.up_bytes = round_up((size_t)sms * 2 * uptc::kM * pl.bp * 4, 256);
    } else {
        // splits * 4 warps sums of n_pad neurons; splits * groups <= 4*sms + groups
        const size_t max_groups = (D + kUpRows - 1) / kUpRows;
        pl.up_bytes = round_up((4 * (size_t)sms + max_groups) * 4 * kUpRows * pl.bp * 4, 256);
    }
    pl.h_bytes = round_up((size_t)pl.h_rows * pl.bp * 2, 256);
    const int wc = stage_width(d, kmax);
    pl.down_wc = wc;
    const int wchunks = d / wc;
    pl.down_splits = sms / wchunks > 0 ? sms / wchunks : 1;
    const int items = wchunks * pl.down_splits;
    pl.down_blocks = items < sms ? items : sms;
    pl.down_bytes = round_up((size_t)pl.down_splits * kMlpMaxBatch * d * 4, 256);
    if (pl.tc)   // two partial slots of BP x (up to 512) columns per block
        pl.down_bytes = round_up((size_t)sms * 2 * pl.bp * 512 * 4, 256);
    return pl;
}

template <typename T, int BP>
sha_status_t run_mlp_bp(const void *x, const void *W1t, const void *W2t, const int32_t *S,
                        const int32_t *n_S, int B, int d, int D, int act, void *y, void *ws,
                        int dev, int sms, cudaStream_t s)
{
    static std::atomic<bool> configured[kMaxDevicesMlp];
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(mlp_up_kernel<T, BP>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             UpCfg<BP>::kSmemBytes);
        if constexpr (BP >= 16) {
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(mlp_up_tc_kernel<T, BP, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         UpTcCfg<BP>::kSmemBytes);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(mlp_up_tc_kernel<T, BP, false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         UpTcCfg<BP>::kSmemBytes);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(mlp_down_tc_kernel<T, BP, 2>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DownTcCfg<BP, 2>::kSmemBytes);
            if (e == cudaSuccess)
                e = cudaFuncSetAttribute(mlp_down_tc_kernel<T, BP, 4>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DownTcCfg<BP, 4>::kSmemBytes);
        }
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(mlp_down_kernel<T, BP>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     DownCfg<BP>::kSmemBytes);
        if (e != cudaSuccess) return mlp_launch_error(e);
        configured[dev].store(true, std::memory_order_release);
    }
    const MlpPlan pl = mlp_plan(B, d, D, sms);
    char *w = static_cast<char *>(ws);
    float *up_part = reinterpret_cast<float *>(w);
    T *Ht = reinterpret_cast<T *>(w + pl.up_bytes);
    float *down_part = reinterpret_cast<float *>(w + pl.up_bytes + pl.h_bytes);

    const size_t hn = (size_t)pl.h_rows * BP;
    const size_t n = (size_t)B * d;
    cudaError_t e;
    bool up_done = false;
    if constexpr (BP >= 16) {
        if (pl.tc_up) {
            constexpr bool bf16 = !std::is_same<T, __half>::value;
            CUtensorMap tm_x, tm_h;
            sha_status_t st = mlp_tensor_map(&tm_x, x, bf16, d, B, BP);
            if (st == SHA_OK && pl.tc)
                st = mlp_tensor_map(&tm_h, Ht, bf16, pl.h_rows, BP, BP, downtc::kR);
            if (st != SHA_OK) return st;
            const dim3 act_grid((unsigned)(pl.h_rows / uptc::kM), BP / kActCols);
            if (pl.tc) {
                e = launch_pdl(mlp_up_tc_kernel<T, BP, true>, dim3(sms), uptc::kThreads,
                               UpTcCfg<BP>::kSmemBytes, s, tm_x, static_cast<const T *>(W1t),
                               S, n_S, B, d, D, act, pl.h_rows, up_part, Ht);
                if (e != cudaSuccess) return mlp_launch_error(e);
                e = launch_pdl(mlp_act_tc_kernel<T, BP, true>, act_grid, 2 * uptc::kM, 0, s,
                               (const float *)up_part, n_S, B, d, D, sms, act, pl.h_rows, Ht);
                if (e != cudaSuccess) return mlp_launch_error(e);
                if (SHA_MLP_DOWN_TC_WIDE && d % 512 == 0) {
                    e = launch_pdl(mlp_down_tc_kernel<T, BP, 4>, dim3(sms), downtc::kThreads,
                                   DownTcCfg<BP, 4>::kSmemBytes, s, tm_h,
                                   static_cast<const T *>(W2t), S, n_S, B, d, D, down_part,
                                   static_cast<T *>(y));
                    if (e != cudaSuccess) return mlp_launch_error(e);
                    e = launch_pdl(mlp_out_tc_kernel<T, BP, 512>,
                                   dim3((unsigned)(d / 512), (B + kOutRows - 1) / kOutRows), 512, 0,
                                   s, (const float *)down_part, n_S, B, d, D, sms,
                                   static_cast<T *>(y));
                } else {
                    e = launch_pdl(mlp_down_tc_kernel<T, BP, 2>, dim3(sms), downtc::kThreads,
                                   DownTcCfg<BP, 2>::kSmemBytes, s, tm_h,
                                   static_cast<const T *>(W2t), S, n_S, B, d, D, down_part,
                                   static_cast<T *>(y));
                    if (e != cudaSuccess) return mlp_launch_error(e);
                    e = launch_pdl(mlp_out_tc_kernel<T, BP, 256>,
                                   dim3((unsigned)(d / 256), (B + kOutRows - 1) / kOutRows), 256, 0,
                                   s, (const float *)down_part, n_S, B, d, D, sms,
                                   static_cast<T *>(y));
                }
                if (e != cudaSuccess) return mlp_launch_error(e);
                return SHA_OK;
            }
            e = launch_pdl(mlp_up_tc_kernel<T, BP, false>, dim3(sms), uptc::kThreads,
                           UpTcCfg<BP>::kSmemBytes, s, tm_x, static_cast<const T *>(W1t), S,
                           n_S, B, d, D, act, pl.h_rows, up_part, Ht);
            if (e != cudaSuccess) return mlp_launch_error(e);
            e = launch_pdl(mlp_act_tc_kernel<T, BP, false>, act_grid, 2 * uptc::kM, 0, s,
                           (const float *)up_part, n_S, B, d, D, sms, act, pl.h_rows, Ht);
            if (e != cudaSuccess) return mlp_launch_error(e);
            up_done = true;
        }
    }
    if (!up_done) {
        e = launch_pdl(mlp_up_kernel<T, BP>, dim3(sms), UpCfg<BP>::kThreads,
                       UpCfg<BP>::kSmemBytes, s, static_cast<const T *>(x),
                       static_cast<const T *>(W1t), S, n_S, B, d, D, up_part);
        if (e != cudaSuccess) return mlp_launch_error(e);
        e = launch_pdl(mlp_act_kernel<T, BP>, dim3((unsigned)((hn + 255) / 256)), 256, 0, s,
                       (const float *)up_part, n_S, B, d, D, pl.h_rows, sms, act, Ht);
        if (e != cudaSuccess) return mlp_launch_error(e);
    }
    e = launch_pdl(mlp_down_kernel<T, BP>, dim3(pl.down_blocks), DownCfg<BP>::kThreads,
                   DownCfg<BP>::kSmemBytes, s, (const T *)Ht, static_cast<const T *>(W2t), S, n_S,
                   B, d, D, pl.down_splits, down_part);
    if (e != cudaSuccess) return mlp_launch_error(e);
    e = launch_pdl(mlp_out_kernel<T>, dim3((unsigned)((n + 255) / 256)), 256, 0, s,
                   (const float *)down_part, B, d, pl.down_splits, static_cast<T *>(y));
    if (e != cudaSuccess) return mlp_launch_error(e);
    return SHA_OK;
}

template <typename T>
sha_status_t run_mlp(const void *x, const void *W1t, const void *W2t, const int32_t *S,
                     const int32_t *n_S, int B, int d, int D, int act, void *y, void *ws,
                     int dev, int sms, cudaStream_t s)
{
    switch (batch_pad(B)) {
    case 8: return run_mlp_bp<T, 8>(x, W1t, W2t, S, n_S, B, d, D, act, y, ws, dev, sms, s);
    case 16: return run_mlp_bp<T, 16>(x, W1t, W2t, S, n_S, B, d, D, act, y, ws, dev, sms, s);
    case 32: return run_mlp_bp<T, 32>(x, W1t, W2t, S, n_S, B, d, D, act, y, ws, dev, sms, s);
    default: return run_mlp_bp<T, 64>(x, W1t, W2t, S, n_S, B, d, D, act, y, ws, dev, sms, s);
    }
}

}  // namespace

// Read and clear this translation unit's device status word (the decode
// library's sha_get_device_status() merges it with its own).  Internal.
extern "C" __attribute__((visibility("hidden"))) unsigned sha_mlp_take_status()
{
    unsigned flags = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&flags, g_sha_status, sizeof flags) != cudaSuccess) return 0;
    cudaMemcpyToSymbol(g_sha_status, &zero, sizeof zero);
    return flags;
}

extern "C" {

size_t sha_mlp_union_workspace_size(int D)
{
    if (D < 1) return 0;
    const size_t blocks = (D + kUnionChunk - 1) / kUnionChunk;
    return round_up((size_t)D, 256) + round_up(blocks * 4, 256);
}

sha_status_t sha_mlp_union(const uint8_t *active, int B, int D, int32_t *S, int32_t *n_S,
                           void *workspace, size_t workspace_bytes, void *stream)
{
    if (B < 1 || D < 1 || !active || !S || !n_S || !workspace) return SHA_ERR_INVALID_ARG;
    if (!aligned_to(S, 4) || !aligned_to(n_S, 4) || !aligned_to(workspace, 256))
        return SHA_ERR_MISALIGNED;
    if (workspace_bytes < sha_mlp_union_workspace_size(D)) return SHA_ERR_WORKSPACE;
    const int blocks = (D + kUnionChunk - 1) / kUnionChunk;
    uint8_t *flags = static_cast<uint8_t *>(workspace);
    int *counts = reinterpret_cast<int *>(static_cast<char *>(workspace) + round_up(D, 256));
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int words = (D % 4 == 0 && aligned_to(active, 4)) ? 1 : 0;
    cudaError_t e = launch_pdl(mlp_union_flags_kernel, dim3(blocks), kUnionThreads, 0, s, active,
                               B, D, words, flags, counts);
    if (e != cudaSuccess) return mlp_launch_error(e);
    e = launch_pdl(mlp_union_write_kernel, dim3(blocks), kUnionThreads, 0, s,
                   (const uint8_t *)flags, (const int *)counts, D, S, n_S);
    if (e != cudaSuccess) return mlp_launch_error(e);
    return SHA_OK;
}

size_t sha_selective_mlp_workspace_size(int B, int d, int D)
{
    if (B < 1 || B > kMlpMaxBatch || d < 256 || d % 256 || D < 1) return 0;
    int dev;
    const int sms = device_sms(&dev);
    if (sms == 0) return 0;
    return mlp_plan(B, d, D, sms).total();
}

sha_status_t sha_selective_mlp_plan(int B, int d, int D, int num_sms, int64_t plan[8])
{
    if (!plan || B < 1 || D < 1 || d < 1 || num_sms < 1) return SHA_ERR_INVALID_ARG;
    if (B > kMlpMaxBatch || d % 256 != 0) return SHA_ERR_UNSUPPORTED;
    const MlpPlan pl = mlp_plan(B, d, D, num_sms);
    plan[0] = pl.bp;
    plan[1] = pl.tc_up ? 1 : 0;
    plan[2] = pl.tc ? 1 : 0;
    plan[3] = pl.h_rows;
    plan[4] = pl.down_splits;
    plan[5] = pl.down_blocks;
    plan[6] = pl.down_wc;
    plan[7] = (int64_t)pl.total();
    return SHA_OK;
}

sha_status_t sha_selective_mlp(const void *x, const void *W1t, const void *W2t,
                               const int32_t *S, const int32_t *n_S, int B, int d, int D,
                               int activation, sha_dtype_t dtype, void *y, void *workspace,
                               size_t workspace_bytes, void *stream)
{
    if (dtype != SHA_FP16 && dtype != SHA_BF16) return SHA_ERR_UNSUPPORTED;
    if (B < 1 || D < 1 || d < 1 || (activation != 0 && activation != 1))
        return SHA_ERR_INVALID_ARG;
    if (B > kMlpMaxBatch || d % 256 != 0) return SHA_ERR_UNSUPPORTED;
    if (!x || !W1t || !W2t || !S || !n_S || !y || !workspace) return SHA_ERR_INVALID_ARG;
    if (!aligned_to(x, 16) || !aligned_to(W1t, 16) || !aligned_to(W2t, 16) ||
        !aligned_to(y, 16) || !aligned_to(S, 4) || !aligned_to(n_S, 4) ||
        !aligned_to(workspace, 256))
        return SHA_ERR_MISALIGNED;
    int dev;
    const int sms = device_sms(&dev);
    if (sms == 0 || dev >= kMaxDevicesMlp) return SHA_ERR_LAUNCH;
    if (workspace_bytes < mlp_plan(B, d, D, sms).total()) return SHA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SHA_FP16)
        return run_mlp<__half>(x, W1t, W2t, S, n_S, B, d, D, activation, y, workspace, dev, sms, s);
    return run_mlp<__nv_bfloat16>(x, W1t, W2t, S, n_S, B, d, D, activation, y, workspace, dev,
                                  sms, s);
}

}  // extern "C"
