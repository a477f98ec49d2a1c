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
//   mlp_up    -- P[split] = x . W1t[S]^T over a range of d (fp32 partials):
//                M = 128 gathered neurons, N = batch, K = d in 128-wide tiles
//   mlp_act   -- H = sigma(sum of the splits), rounded to the input dtype
//   mlp_down  -- Q[split] = H . W2t[S] over a range of neurons (fp32):
//                M = batch, N = 256 output columns, K = neurons in 64-row tiles
//   mlp_out   -- y = sum of the splits, in a fixed order
// The GEMMs stream weight rows with 1-D bulk copies (one per row) into
// shared-memory rows padded by 16 bytes, so ldmatrix reads are free of bank
// conflicts, and run on the tensor cores (mma.sync m16n8k16, fp32 accumulate).
// They are bound by HBM: every selected weight byte is read once, and the
// arithmetic intensity is about B flops per weight byte.
#include <cmath>
#include <cstdio>
#include <mutex>
#include <utility>

#include "sha_decode.h"
#include "sha_device.cuh"
#include "sha_mma.cuh"

namespace {

using namespace sha;

constexpr int kMaxDevicesMlp = 64;
constexpr int kMlpMaxBatch = 64;        // batch rows per call (MMA tiles cover 64)
constexpr int kUnionChunk = 1024;       // neurons per block in the union kernels
constexpr int kUnionThreads = 256;

// ---------------------------------------------------------------- union

__global__ void __launch_bounds__(kUnionThreads)
    mlp_union_flags_kernel(const uint8_t *__restrict__ active, int B, int D,
                           uint8_t *__restrict__ flags, int *__restrict__ counts)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ int warp_sum[kUnionThreads / 32];
    const int j0 = blockIdx.x * kUnionChunk;
    int cnt = 0;
    for (int j = j0 + threadIdx.x; j < min(D, j0 + kUnionChunk); j += kUnionThreads) {
        uint8_t any = 0;
        for (int b = 0; b < B; ++b) any |= active[(size_t)b * D + j];
        flags[j] = any != 0;
        cnt += any != 0;
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

__global__ void __launch_bounds__(kUnionThreads)
    mlp_union_write_kernel(const uint8_t *__restrict__ flags, const int *__restrict__ counts,
                           int D, int32_t *__restrict__ S, int32_t *__restrict__ n_S)
{
    pdl_wait();
    pdl_launch_dependents();
    constexpr int kPer = kUnionChunk / kUnionThreads;   // 4 neurons per thread
    __shared__ int warp_sum[kUnionThreads / 32];
    int base = 0;
    for (int i = 0; i < (int)blockIdx.x; ++i) base += counts[i];
    if (blockIdx.x == gridDim.x - 1 && threadIdx.x == 0) *n_S = base + counts[blockIdx.x];
    const int j0 = blockIdx.x * kUnionChunk + threadIdx.x * kPer;
    int f[kPer], mine = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        f[i] = (j0 + i < D) ? flags[j0 + i] : 0;
        mine += f[i];
    }
    // exclusive prefix of `mine` over the block, in thread order
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = mine;
    for (int off = 1; off < 32; off <<= 1) {
        const int x = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += x;
    }
    if (lane == 31) warp_sum[warp] = incl;
    __syncthreads();
    int pos = base + incl - mine;
    for (int w = 0; w < warp; ++w) pos += warp_sum[w];
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (f[i]) S[pos++] = j0 + i;
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

struct UpCfg {
    static constexpr int kConsumerWarps = 4;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    static constexpr int kM = 128;                      // gathered neurons per item
    static constexpr int kK = 128;                      // d per tile
    static constexpr int kStages = 3;
    static constexpr int kRow = kK * 2 + 16;            // padded row: conflict-free ldmatrix
    static constexpr int kWBytes = kM * kRow;
    static constexpr int kXBytes = kMlpMaxBatch * kRow;
    static constexpr int kStage = kWBytes + kXBytes;
    static constexpr int kBarOffset = kStages * kStage;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8;
};

// Work of the up-projection for n_S selected neurons on `blocks` blocks:
// chunks of kM neurons, each split over `splits` ranges of d.
__device__ __forceinline__ void up_plan(int n_S, int d, int blocks, int &chunks, int &splits)
{
    chunks = (n_S + UpCfg::kM - 1) / UpCfg::kM;
    const int ktiles = d / UpCfg::kK;
    splits = chunks > 0 ? (blocks + chunks - 1) / chunks : 1;
    if (splits > ktiles) splits = ktiles;
    if (splits < 1) splits = 1;
}

template <typename T>
__global__ void __launch_bounds__(UpCfg::kThreads, 1)
    mlp_up_kernel(const T *__restrict__ x, const T *__restrict__ W1t,
                  const int32_t *__restrict__ S, const int32_t *__restrict__ n_S_ptr, int B,
                  int d, int D, float *__restrict__ part)
{
    using C = UpCfg;
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
    int chunks, splits;
    up_plan(n_S, d, gridDim.x, chunks, splits);
    const int items = chunks * splits, ktiles = d / C::kK;
    const int n_pad = chunks * C::kM;

    if (warp == C::kConsumerWarps) {
        // producer warp: lanes gather weight rows and batch rows of each tile
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const int chunk = item / splits, split = item % splits;
            const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
            int ids[C::kM / 32];
#pragma unroll
            for (int i = 0; i < C::kM / 32; ++i) {
                const int t = chunk * C::kM + lane + 32 * i;
                ids[i] = t < n_S ? neuron_id(S, t, D) : -1;
            }
            int valid = min(C::kM, n_S - chunk * C::kM);
            for (int kt = kt0; kt < kt1; ++kt) {
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                if (lane == 0)
                    mbar_arrive_expect_tx(&full[stage], (uint32_t)((valid + B) * C::kK * 2));
                __syncwarp();
                unsigned char *ws = smem + stage * C::kStage;
                unsigned char *xs = ws + C::kWBytes;
                const size_t k0 = (size_t)kt * C::kK;
#pragma unroll
                for (int i = 0; i < C::kM / 32; ++i)
                    if (ids[i] >= 0)
                        bulk_copy_g2s(ws + (lane + 32 * i) * C::kRow, W1t + (size_t)ids[i] * d + k0,
                                      C::kK * 2, &full[stage], policy);
                for (int b = lane; b < B; b += 32)
                    bulk_copy_g2s(xs + b * C::kRow, x + (size_t)b * d + k0, C::kK * 2,
                                  &full[stage], policy);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
        return;
    }

    // consumers: warp w computes neurons [32w, 32w+32) of the chunk x all batch rows
    const int g = lane >> 2, qd = lane & 3;
    const int ntiles = (B + 7) / 8;          // 8-row batch tiles in use
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t base = smem_addr(smem);
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int chunk = item / splits, split = item % splits;
        const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
        float acc[2][8][4];
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] =
                                                acc[mt][nt][3] = 0.f;
        for (int kt = kt0; kt < kt1; ++kt) {
            const bool live = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase));
            if (live) {
                const uint32_t ws = base + stage * C::kStage, xs = ws + C::kWBytes;
#pragma unroll
                for (int k16 = 0; k16 < C::kK / 16; ++k16) {
                    uint32_t a[2][4];
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt)
                        ldmatrix_x4(ws + (warp * 32 + mt * 16 + (lane & 15)) * C::kRow +
                                        (k16 * 16 + (lane >> 4) * 8) * 2,
                                    a[mt]);
#pragma unroll
                    for (int np = 0; np < 4; ++np) {
                        if (np * 2 >= ntiles) break;                 // warp-uniform
                        const int mi = lane >> 3;
                        uint32_t kb[4];
                        ldmatrix_x4(xs + (np * 16 + (mi >> 1) * 8 + (lane & 7)) * C::kRow +
                                        (k16 * 16 + (mi & 1) * 8) * 2,
                                    kb);
#pragma unroll
                        for (int mt = 0; mt < 2; ++mt) {
                            mma_16816<T>(acc[mt][2 * np], a[mt], kb[0], kb[1]);
                            mma_16816<T>(acc[mt][2 * np + 1], a[mt], kb[2], kb[3]);
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
        // partial sums of this range of d: part[split][neuron][batch]
#pragma unroll
        for (int mt = 0; mt < 2; ++mt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int t = chunk * C::kM + warp * 32 + mt * 16 + g + 8 * r;
                if (t >= n_S) continue;
                float *dst = part + ((size_t)split * n_pad + t) * kMlpMaxBatch;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
                    if (nt < ntiles)
                        *reinterpret_cast<float2 *>(dst + nt * 8 + qd * 2) =
                            make_float2(acc[mt][nt][2 * r], acc[mt][nt][2 * r + 1]);
            }
    }
}

// H[b, t] = sigma(sum over splits), rounded to T; zero outside the batch and the union.
template <typename T>
__global__ void mlp_act_kernel(const float *__restrict__ part, const int32_t *__restrict__ n_S_ptr,
                               int B, int d, int D, int h_stride, int up_blocks, int act,
                               T *__restrict__ H)
{
    pdl_wait();
    pdl_launch_dependents();
    const int n_S = union_size(n_S_ptr, D);
    int chunks, splits;
    up_plan(n_S, d, up_blocks, chunks, splits);
    const int n_pad = chunks * UpCfg::kM;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    const int b = blockIdx.y;
    if (t >= h_stride) return;
    float v = 0.f;
    if (t < n_S && b < B) {
        for (int s = 0; s < splits; ++s) v += part[((size_t)s * n_pad + t) * kMlpMaxBatch + b];
        if (act == 1) v = fmaxf(v, 0.f);
    }
    H[(size_t)b * h_stride + t] = Elem<T>::from_float(v);
}

// ---------------------------------------------------------------- down-projection

struct DownCfg {
    static constexpr int kConsumerWarps = 8;
    static constexpr int kThreads = (kConsumerWarps + 1) * 32;
    static constexpr int kN = 256;                      // output columns per item
    static constexpr int kK = 64;                       // neurons per tile
    static constexpr int kStages = 4;
    static constexpr int kWRow = kN * 2 + 16;           // padded rows
    static constexpr int kHRow = kK * 2 + 16;
    static constexpr int kWBytes = kK * kWRow;
    static constexpr int kHBytes = kMlpMaxBatch * kHRow;
    static constexpr int kStage = kWBytes + kHBytes;
    static constexpr int kBarOffset = kStages * kStage;
    static constexpr int kSmemBytes = kBarOffset + 2 * kStages * 8;
};

template <typename T>
__global__ void __launch_bounds__(DownCfg::kThreads, 1)
    mlp_down_kernel(const T *__restrict__ H, const T *__restrict__ W2t,
                    const int32_t *__restrict__ S, const int32_t *__restrict__ n_S_ptr, int B,
                    int d, int D, int h_stride, int splits, float *__restrict__ part)
{
    using C = DownCfg;
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
    const int ktiles = (n_S + C::kK - 1) / C::kK;
    const int dchunks = d / C::kN;
    const int items = dchunks * splits;

    if (warp == C::kConsumerWarps) {
        const uint64_t policy = l2_policy_evict_first();
        int stage = 0;
        uint32_t phase = 0, last_parity = 0, used = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            const int dc = item / splits, split = item % splits;
            const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
            const size_t c0 = (size_t)dc * C::kN;
            for (int kt = kt0; kt < kt1; ++kt) {
                bool go = true;
                if (lane == 0 && !mbar_wait(&empty[stage], phase ^ 1)) {
                    atomicOr(&g_sha_status, kStatusTimeout);
                    go = false;
                }
                go = __shfl_sync(0xffffffffu, go, 0);
                if (!go) { ok = false; break; }
                if (lane == 0)
                    mbar_arrive_expect_tx(&full[stage],
                                          (uint32_t)(C::kK * C::kN * 2 + kMlpMaxBatch * C::kK * 2));
                __syncwarp();
                unsigned char *ws = smem + stage * C::kStage;
                unsigned char *hs = ws + C::kWBytes;
                const int t0 = kt * C::kK;
                for (int r = lane; r < C::kK; r += 32) {
                    // rows past the union repeat its last neuron: finite values
                    // times H = 0 add nothing (stale shared memory could be NaN)
                    const int t = min(t0 + r, n_S - 1);
                    bulk_copy_g2s(ws + r * C::kWRow, W2t + (size_t)neuron_id(S, t, D) * d + c0,
                                  C::kN * 2, &full[stage], policy);
                }
                for (int b = lane; b < kMlpMaxBatch; b += 32)
                    bulk_copy_g2s(hs + b * C::kHRow, H + (size_t)b * h_stride + t0, C::kK * 2,
                                  &full[stage], policy);
                last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                used |= 1u << stage;
                if (++stage == C::kStages) { stage = 0; phase ^= 1; }
            }
        }
        if (lane == 0)
            for (int s = 0; s < C::kStages; ++s)
                if (used & (1u << s)) mbar_wait(&full[s], (last_parity >> s) & 1u);
        __syncwarp();
        return;
    }

    // consumers: warp w owns output columns [32w, 32w+32) of the item x all batch rows
    const int g = lane >> 2, qd = lane & 3, mi = lane >> 3;
    const int mtiles = (B + 15) / 16;
    int stage = 0;
    uint32_t phase = 0;
    const uint32_t base = smem_addr(smem);
    for (int item = blockIdx.x; item < items; item += gridDim.x) {
        const int dc = item / splits, split = item % splits;
        const int kt0 = split * ktiles / splits, kt1 = (split + 1) * ktiles / splits;
        float acc[4][4][4];
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] =
                                                acc[mt][nt][3] = 0.f;
        for (int kt = kt0; kt < kt1; ++kt) {
            const bool live = __all_sync(0xffffffffu, mbar_wait(&full[stage], phase));
            if (live) {
                const uint32_t ws = base + stage * C::kStage, hs = ws + C::kWBytes;
#pragma unroll
                for (int k16 = 0; k16 < C::kK / 16; ++k16) {
                    uint32_t vb[2][4];
#pragma unroll
                    for (int np = 0; np < 2; ++np)
                        ldmatrix_x4_trans(ws + (k16 * 16 + (mi & 1) * 8 + (lane & 7)) * C::kWRow +
                                              (warp * 32 + np * 16 + (mi >> 1) * 8) * 2,
                                          vb[np]);
#pragma unroll
                    for (int mt = 0; mt < 4; ++mt) {
                        if (mt >= mtiles) break;                     // warp-uniform
                        uint32_t a[4];
                        ldmatrix_x4(hs + (mt * 16 + (lane & 15)) * C::kHRow +
                                        (k16 * 16 + (lane >> 4) * 8) * 2,
                                    a);
#pragma unroll
                        for (int np = 0; np < 2; ++np) {
                            mma_16816<T>(acc[mt][2 * np], a, vb[np][0], vb[np][1]);
                            mma_16816<T>(acc[mt][2 * np + 1], a, vb[np][2], vb[np][3]);
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
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int r = 0; r < 2; ++r) {
                const int b = mt * 16 + g + 8 * r;
                if (b >= B) continue;
                float *dst = part + ((size_t)split * kMlpMaxBatch + b) * d + (size_t)dc * C::kN +
                             warp * 32;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt)
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
    attr[0].val.programmaticStreamSerializationAllowed = 1;
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

// Workspace of sha_selective_mlp for these sizes on a device with `sms` SMs.
struct MlpPlan {
    int h_stride;          // padded union length (H row stride)
    int down_splits;
    size_t up_bytes, h_bytes, down_bytes;
    size_t total() const { return up_bytes + h_bytes + down_bytes; }
};

MlpPlan mlp_plan(int d, int D, int sms)
{
    MlpPlan pl;
    pl.h_stride = (int)round_up((size_t)D, UpCfg::kM);
    const int max_chunks = pl.h_stride / UpCfg::kM;
    // splits * chunks <= blocks + chunks for any union size
    pl.up_bytes = round_up((size_t)(sms + max_chunks) * UpCfg::kM * kMlpMaxBatch * 4, 256);
    pl.h_bytes = round_up((size_t)kMlpMaxBatch * pl.h_stride * 2, 256);
    const int dchunks = d / DownCfg::kN;
    pl.down_splits = sms / dchunks > 0 ? sms / dchunks : 1;
    pl.down_bytes = round_up((size_t)pl.down_splits * kMlpMaxBatch * d * 4, 256);
    return pl;
}

template <typename T>
sha_status_t run_mlp(const void *x, const void *W1t, const void *W2t, const int32_t *S,
                     const int32_t *n_S, int B, int d, int D, int act, void *y, void *ws,
                     int dev, int sms, cudaStream_t s)
{
    static bool configured[kMaxDevicesMlp] = {};
    if (!configured[dev]) {
        cudaError_t e = cudaFuncSetAttribute(mlp_up_kernel<T>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             UpCfg::kSmemBytes);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(mlp_down_kernel<T>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     DownCfg::kSmemBytes);
        if (e != cudaSuccess) return mlp_launch_error(e);
        configured[dev] = true;
    }
    const MlpPlan pl = mlp_plan(d, D, sms);
    char *w = static_cast<char *>(ws);
    float *up_part = reinterpret_cast<float *>(w);
    T *H = reinterpret_cast<T *>(w + pl.up_bytes);
    float *down_part = reinterpret_cast<float *>(w + pl.up_bytes + pl.h_bytes);

    cudaError_t e = launch_pdl(mlp_up_kernel<T>, dim3(sms), UpCfg::kThreads, UpCfg::kSmemBytes, s,
                               static_cast<const T *>(x), static_cast<const T *>(W1t), S, n_S, B, d,
                               D, up_part);
    if (e != cudaSuccess) return mlp_launch_error(e);
    e = launch_pdl(mlp_act_kernel<T>, dim3((pl.h_stride + 255) / 256, kMlpMaxBatch), 256, 0, s,
                   (const float *)up_part, n_S, B, d, D, pl.h_stride, sms, act, H);
    if (e != cudaSuccess) return mlp_launch_error(e);
    const int items = (d / DownCfg::kN) * pl.down_splits;
    e = launch_pdl(mlp_down_kernel<T>, dim3(items < sms ? items : sms), DownCfg::kThreads,
                   DownCfg::kSmemBytes, s, (const T *)H, static_cast<const T *>(W2t), S, n_S, B,
                   d, D, pl.h_stride, pl.down_splits, down_part);
    if (e != cudaSuccess) return mlp_launch_error(e);
    const size_t n = (size_t)B * d;
    e = launch_pdl(mlp_out_kernel<T>, dim3((unsigned)((n + 255) / 256)), 256, 0, s,
                   (const float *)down_part, B, d, pl.down_splits, static_cast<T *>(y));
    if (e != cudaSuccess) return mlp_launch_error(e);
    return SHA_OK;
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
    cudaError_t e = launch_pdl(mlp_union_flags_kernel, dim3(blocks), kUnionThreads, 0, s, active,
                               B, D, flags, counts);
    if (e != cudaSuccess) return mlp_launch_error(e);
    e = launch_pdl(mlp_union_write_kernel, dim3(blocks), kUnionThreads, 0, s,
                   (const uint8_t *)flags, (const int *)counts, D, S, n_S);
    if (e != cudaSuccess) return mlp_launch_error(e);
    return SHA_OK;
}

size_t sha_selective_mlp_workspace_size(int B, int d, int D)
{
    if (B < 1 || B > kMlpMaxBatch || d < DownCfg::kN || d % DownCfg::kN || D < 1) return 0;
    int dev;
    const int sms = device_sms(&dev);
    if (sms == 0) return 0;
    return mlp_plan(d, D, sms).total();
}

sha_status_t sha_selective_mlp(const void *x, const void *W1t, const void *W2t,
                               const int32_t *S, const int32_t *n_S, int B, int d, int D,
                               int activation, sha_dtype_t dtype, void *y, void *workspace,
                               size_t workspace_bytes, void *stream)
{
    if (dtype != SHA_FP16 && dtype != SHA_BF16) return SHA_ERR_UNSUPPORTED;
    if (B < 1 || D < 1 || d < 1 || (activation != 0 && activation != 1))
        return SHA_ERR_INVALID_ARG;
    if (B > kMlpMaxBatch || d % DownCfg::kN != 0) return SHA_ERR_UNSUPPORTED;
    if (!x || !W1t || !W2t || !S || !n_S || !y || !workspace) return SHA_ERR_INVALID_ARG;
    if (!aligned_to(x, 16) || !aligned_to(W1t, 16) || !aligned_to(W2t, 16) ||
        !aligned_to(y, 16) || !aligned_to(S, 4) || !aligned_to(n_S, 4) ||
        !aligned_to(workspace, 256))
        return SHA_ERR_MISALIGNED;
    int dev;
    const int sms = device_sms(&dev);
    if (sms == 0 || dev >= kMaxDevicesMlp) return SHA_ERR_LAUNCH;
    if (workspace_bytes < mlp_plan(d, D, sms).total()) return SHA_ERR_WORKSPACE;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (dtype == SHA_FP16)
        return run_mlp<__half>(x, W1t, W2t, S, n_S, B, d, D, activation, y, workspace, dev, sms, s);
    return run_mlp<__nv_bfloat16>(x, W1t, W2t, S, n_S, B, d, D, activation, y, workspace, dev,
                                  sms, s);
}

}  // extern "C"
