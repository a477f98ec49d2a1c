// sha_decode.cu -- C ABI of the Selective Head Attention decode library:
// argument checks, the work planner, workspace handling and kernel launches.
// The operation and every argument are specified in include/sha_decode.h.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <utility>

#include <cudaTypedefs.h>

#include "sha_decode.h"
#include "sha_device.cuh"
#include "sha_gqa_kernel.cuh"
#include "sha_mha_kernel.cuh"
#include "sha_schedule.cuh"
#include "sha_select_kernel.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxG = 16;

thread_local char g_last_cuda_error[256] = "no error";

sha_status_t launch_error(cudaError_t e)
{
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e),
                  cudaGetErrorString(e));
    return SHA_ERR_LAUNCH;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Shape checks shared by every entry point; no CUDA call is made here.
sha_status_t check_shape(int B, int H_q, int H_kv, int N_kv, int d, int top_k, float scale)
{
    if (B < 0 || H_q < 1 || H_kv < 1 || N_kv < 1 || top_k < 0 || top_k > H_kv)
        return SHA_ERR_INVALID_ARG;
    if (H_q % H_kv != 0) return SHA_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return SHA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SHA_ERR_UNSUPPORTED;
    if (H_q / H_kv > kMaxG) return SHA_ERR_UNSUPPORTED;
    return SHA_OK;
}

struct DeviceInfo {
    int num_sms = 0;
};

std::mutex g_mutex;
DeviceInfo g_devices[kMaxDevices];

// Workspace of sha_decode / sha_decode_bf16, one per device, grown on demand.
struct OwnedWorkspace {
    void *ptr;
    size_t bytes;
};
OwnedWorkspace g_owned[kMaxDevices];

sha_status_t current_device(int *dev, DeviceInfo **info)
{
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return launch_error(e);
    if (*dev < 0 || *dev >= kMaxDevices) return SHA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mutex);
    DeviceInfo &di = g_devices[*dev];
    if (di.num_sms == 0) {
        e = cudaDeviceGetAttribute(&di.num_sms, cudaDevAttrMultiProcessorCount, *dev);
        if (e != cudaSuccess) {
            di.num_sms = 0;
            return launch_error(e);
        }
    }
    *info = &di;
    return SHA_OK;
}

// Co-resident thread-block clusters of each size of the clustered grouped
// kernel (index = blocks per cluster, 2..kClusterMax; 0 where none fit).
struct ClusterCaps {
    int n[sha::GqaConfig<128>::kClusterMax + 1];
};

// The call's plan: tile schedule and workspace layout.
struct Plan {
    sha::Schedule sched;
    int slot_floats;
    size_t counter_bytes;   // fixed region of sha::kMaxBlocks int32 counters
    size_t slot_bytes;      // 2*num_ctas slots
    size_t workspace_bytes() const { return counter_bytes + slot_bytes; }
};

// Whether the host may cut a call at unit boundaries (see make_plan), and
// what a split unit's merge is taken to cost, in key tiles of streaming.
#ifndef SHA_ALIGN_UNITS
#define SHA_ALIGN_UNITS 1
#endif
#ifndef SHA_MERGE_COST_TILES
#define SHA_MERGE_COST_TILES 2
#endif
constexpr long long kMergeCostTiles = SHA_MERGE_COST_TILES;

// The clustered cut (Schedule::cluster): 1 lets the planner choose it for the
// grouped kernel's fixed-length calls where it is estimated faster, 0 never.
#ifndef SHA_CLUSTER_CUT
#define SHA_CLUSTER_CUT 1
#endif

// Cost model of a call's cuts (ns), measured on B200 with per-block timer
// stamps and CUDA-graph timings: a block streams a 64 KiB K+V tile in about
// kBlockTileNs at best (80 blocks of a GQA call at 16K context streamed at
// 64 GB/s each); all blocks together share the HBM rate; a unit split across
// blocks and merged through the workspace adds kSlotMergeNs at the end of the
// call (partial write, fence, arrival atomic, reading the parts back), and a
// unit merged in a cluster's shared memory adds kClusterMergeNs.
constexpr double kBlockTileNs = 1000.0;
constexpr double kHbmBytesPerNs = 6500.0;
#ifndef SHA_SLOT_MERGE_NS
#define SHA_SLOT_MERGE_NS 3500
#endif
#ifndef SHA_CLUSTER_MERGE_NS
#define SHA_CLUSTER_MERGE_NS 2000
#endif

// Whether the clustered kernel can stage a unit's parts for clusters of c
// blocks: each block receives every part's slice of its share of the G x d
// outputs (plus m and l), two units' worth, in the rows 8..15 of its four
// warps' state areas (two per unit, the first (c+1)/2 parts in one).
bool cluster_stage_fits(int G, int d, int c)
{
    const int groups = G * d / 4;
    const int stride = 4 * ((groups + c - 1) / c) + 4 * ((2 * G + 3) / 4);
    const int region = sha::GqaConfig<128>::kMaxPartRows * (d + 2);
    return G <= sha::GqaConfig<128>::kMaxPartRows && (c + 1) / 2 * stride <= region;
}

// Streaming time of a cut whose busiest of `active` blocks streams max_tiles
// tiles of tile_bytes each.
double stream_ns(long long max_tiles, long long active, double tile_bytes)
{
    const double per_tile = std::fmax(kBlockTileNs * tile_bytes / 65536.0,
                                      (double)active * tile_bytes / kHbmBytesPerNs);
    return (double)max_tiles * per_tile;
}

// Multi-head calls (G = 1) with d = 128 and one length for every row run on
// the grouped kernel's tensor-core path, one query row of the 16 an MMA
// covers.  On the OPT-66B step both kernels read exactly the algorithmic
// bytes; the tensor-core path executes 2.25x fewer instructions and keeps the
// issue slots half as busy.  Timed under the power cap that a sustained decode
// load holds the GPU at, the two have come out within 0.2 % of each other on
// some boxes and 3.5 % apart in the tensor-core path's favour on others; in
// bursts at full clock the FMA kernel is 1-3 % faster.  The FMA kernel keeps
// d = 64 and per-row lengths (paged caches included), where it is faster.
#ifndef SHA_MHA_TENSOR_CORES
#define SHA_MHA_TENSOR_CORES 1
#endif

// whether a call runs on the multi-head FMA kernel
bool fma_path(int G, int d, bool per_row_lengths)
{
    return G == 1 && !(SHA_MHA_TENSOR_CORES && d == 128 && !per_row_lengths);
}

// pages the grouped kernel loads as whole TMA boxes: powers of two from 8 keys
bool boxable_pages(int page_size) { return page_size >= 8 && (page_size & (page_size - 1)) == 0; }

// resident blocks per SM each kernel is planned for
int blocks_per_sm(int G, int d, bool per_row_lengths)
{
    return fma_path(G, d, per_row_lengths) ? SHA_MHA_BLOCKS_PER_SM : 1;
}

// keys per tile of the kernel that serves the call
int tile_keys(int G, int d, bool per_row_lengths)
{
    return fma_path(G, d, per_row_lengths) ? sha::MhaConfig<128>::kTile
                                           : sha::GqaConfig<128>::kTile;
}

Plan make_plan(int B, int H_q, int H_kv, int N_kv, int d, int top_k, int num_splits,
               int num_sms, bool per_row_lengths = false, const ClusterCaps *caps = nullptr)
{
    Plan pl;
    const int G = H_q / H_kv;
    const long long units = (long long)B * top_k;
    const int tile = tile_keys(G, d, per_row_lengths);
    pl.sched.tiles_per_unit = (N_kv + tile - 1) / tile;
    pl.sched.total_tiles = units * pl.sched.tiles_per_unit;
    pl.sched.pieces = 0;
    pl.sched.cluster = 0;
    pl.sched.units_per_cluster = 0;
    pl.sched.whole_per_block = 0;
    long long ctas =
        num_splits > 0 ? num_splits : (long long)num_sms * blocks_per_sm(G, d, per_row_lengths);
    if (ctas > sha::kMaxBlocks) ctas = sha::kMaxBlocks;
    if (ctas > pl.sched.total_tiles) ctas = pl.sched.total_tiles;
    // every block gets at least ceil((Tu-1)/(kMaxMergeParts-1)) tiles, so a
    // unit of Tu tiles is shared by at most kMaxMergeParts blocks
    const long long min_tiles =
        (pl.sched.tiles_per_unit - 1 + sha::kMaxMergeParts - 2) / (sha::kMaxMergeParts - 1);
    if (min_tiles > 1 && ctas > pl.sched.total_tiles / min_tiles)
        ctas = pl.sched.total_tiles / min_tiles;
    if (ctas < 1) ctas = 1;
    if (num_splits == 0 && SHA_ALIGN_UNITS) {
        // Cut at unit boundaries when the busiest block then streams no more
        // tiles than under the even cut plus what the merges of split units
        // cost (kMergeCostTiles): whole units per block when there are at
        // least as many units as blocks, else each unit in p equal pieces.
        // (the merges sit on the critical path at the end of a short call; in a
        // long one the other blocks' streaming hides all but about a tile)
        const long long tpu = pl.sched.tiles_per_unit;
        const long long even_tiles = (pl.sched.total_tiles + ctas - 1) / ctas;
        const long long even = even_tiles + (even_tiles < 32 ? kMergeCostTiles : 1);
        const long long blocks = (long long)num_sms * blocks_per_sm(G, d, per_row_lengths);
        if (units >= blocks) {
            if ((units + blocks - 1) / blocks * tpu <= even && blocks <= sha::kMaxBlocks) {
                pl.sched.pieces = 1;
                ctas = blocks;
            }
        } else {
            long long p = blocks / units;
            if (p > tpu) p = tpu;
            if (p > sha::kMaxMergeParts) p = sha::kMaxMergeParts;
            // pieces of one or two tiles merge as often as the even cut does:
            // take fewer, longer pieces
            while (p > 1 && tpu < 3 * p) --p;
            // pieces still merge, so they must keep most blocks streaming to
            // beat the even cut; whole units (p = 1) merge nothing
            if (p > 1 && 5 * units * p < 4 * blocks) p = 1;
            if ((tpu + p - 1) / p <= even) {
                pl.sched.pieces = (int)p;
                ctas = units * p;
            }
        }
    }
    pl.sched.num_ctas = (int)ctas;
    // The clustered cut.  Clusters of c blocks take upc units each: w whole
    // units per block, and s = upc - c*w units split into c pieces whose parts
    // merge in the cluster's shared memory, with every cluster in one wave.
    // It pays where whole units per block would leave SMs idle (fewer units
    // than blocks: w = 0, one unit per cluster) or stream unevenly in a short
    // call (a few units per block: the leftover units shared), and is taken
    // where the cost model rates it faster than the cut chosen so far.
    const long long blocks_avail = (long long)num_sms * blocks_per_sm(G, d, per_row_lengths);
    if (num_splits == 0 && SHA_CLUSTER_CUT && caps && G <= sha::GqaConfig<128>::kMaxPartRows &&
        !fma_path(G, d, per_row_lengths)) {
        const long long tpu = pl.sched.tiles_per_unit;
        const double tile_bytes = 2.0 * tile * d * 2;
        const long long n = pl.sched.num_ctas;
        long long busiest;
        bool merges;
        if (pl.sched.pieces >= 1) {
            const long long P = units * pl.sched.pieces;
            busiest = 0;
            for (long long c = 0; c < n; ++c) {
                const long long t =
                    pl.sched.piece_start((c + 1) * P / n) - pl.sched.piece_start(c * P / n);
                busiest = t > busiest ? t : busiest;
            }
            merges = pl.sched.pieces > 1;
        } else {
            busiest = (pl.sched.total_tiles + n - 1) / n;
            merges = !(pl.sched.total_tiles % n == 0 && (pl.sched.total_tiles / n) % tpu == 0);
        }
        // with fewer units than blocks the cluster cut is weighed against whole
        // units per block (the merges of pieces through the workspace cost more
        // than the model can say); otherwise against the cut chosen so far
        const bool few_units = units < blocks_avail;
        double best = few_units ? stream_ns(tpu, units, tile_bytes)
                                : stream_ns(busiest, n, tile_bytes) + (merges ? SHA_SLOT_MERGE_NS : 0);
        if (few_units || busiest < 32) {
            for (int c = 2; c <= sha::GqaConfig<128>::kClusterMax && c <= tpu; ++c) {
                if (caps->n[c] < 1 || !cluster_stage_fits(G, d, c)) continue;
                const long long upc_min = (units + caps->n[c] - 1) / caps->n[c];
                for (long long upc = upc_min; upc <= upc_min + 1; ++upc) {
                    const long long w = upc / c, shared = upc - c * w;
                    if (shared == 0) continue;              // whole units: not clustered
                    const long long clusters = (units + upc - 1) / upc;
                    if (clusters > caps->n[c] || clusters * c > sha::kMaxBlocks) continue;
                    const long long tiles = w * tpu + shared * ((tpu + c - 1) / c);
                    const double est = stream_ns(tiles, clusters * c, tile_bytes) +
                                       (double)shared * SHA_CLUSTER_MERGE_NS;
                    // a cut that also holds whole units must win clearly: the
                    // model's error is about a tenth of a short call
                    if (est < (w > 0 ? 0.9 : 1.0) * best) {
                        best = est;
                        pl.sched.cluster = c;
                        pl.sched.units_per_cluster = (int)upc;
                        pl.sched.whole_per_block = (int)w;
                        pl.sched.num_ctas = (int)(clusters * c);
                        pl.sched.pieces = 0;
                    }
                }
            }
        }
    }
    // one partial state: G rows of (O[d], m, l), padded to 128 bytes
    pl.slot_floats = ((G * (d + 2)) + 31) / 32 * 32;
    pl.counter_bytes = sha::kCounterBytes;
    pl.slot_bytes = (size_t)2 * pl.sched.num_ctas * pl.slot_floats * sizeof(float);
    // every unit held whole by one block, or merged on chip: no workspace
    if (pl.sched.pieces == 1 || pl.sched.cluster >= 2 ||
        (pl.sched.total_tiles % pl.sched.num_ctas == 0 &&
         (pl.sched.total_tiles / pl.sched.num_ctas) % pl.sched.tiles_per_unit == 0)) {
        pl.counter_bytes = 0;
        pl.slot_bytes = 0;
    }
    return pl;
}

// A clustered cut chosen by the caller: clusters of `cluster` blocks, each
// taking `units_per_cluster` whole units.  SHA_ERR_UNSUPPORTED where the
// clustered kernel cannot serve the call, SHA_ERR_INVALID_ARG for sizes out
// of range.
sha_status_t forced_cluster_plan(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                                 int cluster, int units_per_cluster, int whole_per_block,
                                 Plan &pl)
{
    const int G = H_q / H_kv;
    if (G > sha::GqaConfig<128>::kMaxPartRows || fma_path(G, d, false)) return SHA_ERR_UNSUPPORTED;
    pl = make_plan(B, H_q, H_kv, N_kv, d, top_k, 0, 1);
    const long long units = (long long)B * top_k;
    if (cluster < 2 || cluster > sha::GqaConfig<128>::kClusterMax || units_per_cluster < 1 ||
        whole_per_block < 0 || (long long)cluster * whole_per_block > units_per_cluster)
        return SHA_ERR_INVALID_ARG;
    // units split into pieces need a tile per piece
    if ((long long)cluster * whole_per_block < units_per_cluster && cluster > pl.sched.tiles_per_unit)
        return SHA_ERR_INVALID_ARG;
    if (!cluster_stage_fits(G, d, cluster)) return SHA_ERR_UNSUPPORTED;
    const long long clusters = (units + units_per_cluster - 1) / units_per_cluster;
    if (clusters * cluster > sha::kMaxBlocks) return SHA_ERR_INVALID_ARG;
    pl.sched.cluster = cluster;
    pl.sched.units_per_cluster = units_per_cluster;
    pl.sched.whole_per_block = whole_per_block;
    pl.sched.num_ctas = (int)(clusters * cluster);
    pl.sched.pieces = 0;
    pl.counter_bytes = 0;
    pl.slot_bytes = 0;
    return SHA_OK;
}

static_assert(sha::MhaConfig<128>::kTile == sha::MhaConfig<64>::kTile &&
                  sha::GqaConfig<128>::kTile == sha::GqaConfig<64>::kTile,
              "one tile size per kernel, whatever d");

#ifndef SHA_USE_PDL
#define SHA_USE_PDL 1
#endif

// Launch with programmatic stream serialization: the kernel may be scheduled
// while the previous kernel in the stream finishes, and waits for it on the
// device (griddepcontrol.wait) before reading any input.
// cluster > 1: the grid is launched as thread-block clusters of that many blocks.
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel_cluster(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                                  cudaStream_t stream, int cluster, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = SHA_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cluster > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = cluster;
        attr[1].val.clusterDim.y = 1;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kernel)(KArgs...), int grid, int block, size_t smem,
                          cudaStream_t stream, Args &&...args)
{
    return launch_kernel_cluster(kernel, grid, block, smem, stream, 0,
                                 std::forward<Args>(args)...);
}

// cuTensorMapEncodeTiled from the driver, found through the runtime so the
// library does not link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
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

// 3-D view [B*H_kv][N_kv][d] of a K or V cache, 64x64-element boxes with
// 128-byte swizzle; rows past N_kv read as zero.
sha_status_t kv_tensor_map(CUtensorMap *map, const void *base, sha_dtype_t dtype, int d,
                           int N_kv, long long planes, int box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled is not available from the driver");
        return SHA_ERR_LAUNCH;
    }
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N_kv, (cuuint64_t)planes};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N_kv * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t elem[3] = {1, 1, 1};
    CUresult r = encode(map,
                        dtype == SHA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        3, const_cast<void *>(base), dims, strides, box, elem,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled failed with CUresult %d", (int)r);
        return SHA_ERR_LAUNCH;
    }
    return SHA_OK;
}

// 4-D view [d, o1, o2, o3] of a strided K or V cache: d contiguous, the outer
// dimensions (token, head, batch in the order of increasing stride) with the
// given sizes and byte strides, boxes of box_d x box_rows tokens (1 along the
// other dimensions), 128-byte swizzled (64-element boxes of the grouped-query
// kernel) or not (whole rows for the multi-head kernel).  Tokens past the end
// read as zero.
sha_status_t kv_tensor_map_4d(CUtensorMap *map, const void *base, sha_dtype_t dtype, int d,
                              const long long (&size)[3], const long long (&stride_bytes)[3],
                              int tok_dim, int box_d, int box_rows, bool swizzle128)
{
    PFN_cuTensorMapEncodeTiled_v12000 encode = tensor_map_encoder();
    if (!encode) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled is not available from the driver");
        return SHA_ERR_LAUNCH;
    }
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)size[0], (cuuint64_t)size[1],
                          (cuuint64_t)size[2]};
    cuuint64_t strides[3] = {(cuuint64_t)stride_bytes[0], (cuuint64_t)stride_bytes[1],
                             (cuuint64_t)stride_bytes[2]};
    cuuint32_t box[4] = {(cuuint32_t)box_d, 1, 1, 1};
    box[1 + tok_dim] = (cuuint32_t)box_rows;
    cuuint32_t elem[4] = {1, 1, 1, 1};
    CUresult r = encode(map,
                        dtype == SHA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                          : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
                        4, const_cast<void *>(base), dims, strides, box, elem,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                      "cuTensorMapEncodeTiled failed with CUresult %d", (int)r);
        return SHA_ERR_LAUNCH;
    }
    return SHA_OK;
}

// Strides of a strided K or V cache in elements: batch, head, token.
struct KvStrides {
    long long batch, head, token;
};

// Sizes and byte strides of the outer dimensions in the order of increasing
// stride (ties keep token, head, batch order) and each dimension's position.
void order_outer_dims(const KvStrides &st, int B, int H_kv, int N_kv, long long (&size)[3],
                      long long (&stride_bytes)[3], int &tok_dim, int &head_dim,
                      int &batch_dim)
{
    long long sv[3] = {st.token, st.head, st.batch};
    long long nv[3] = {N_kv, H_kv, B};
    int order[3] = {0, 1, 2};
    for (int i = 1; i < 3; ++i)
        for (int j = i; j > 0 && sv[order[j]] < sv[order[j - 1]]; --j)
            std::swap(order[j], order[j - 1]);
    int pos[3];
    for (int i = 0; i < 3; ++i) {
        size[i] = nv[order[i]];
        stride_bytes[i] = sv[order[i]] * 2;
        pos[order[i]] = i;
    }
    tok_dim = pos[0];
    head_dim = pos[1];
    batch_dim = pos[2];
}

// Per-row lengths: the kernel plans its own split from the lengths on the
// device, using at most this many blocks; the workspace covers any split.
Plan make_varlen_plan(int B, int H_q, int H_kv, int N_kv, int d, int top_k, int num_splits,
                      int num_sms)
{
    Plan pl = make_plan(B, H_q, H_kv, N_kv, d, top_k, 0, num_sms, true);
    pl.sched.pieces = 0;                    // the device plans an even cut
    long long ctas = num_splits > 0 ? num_splits
                                    : (long long)num_sms * blocks_per_sm(H_q / H_kv, d, true);
    if (ctas > sha::kMaxBlocks) ctas = sha::kMaxBlocks;
    if (ctas > pl.sched.total_tiles) ctas = pl.sched.total_tiles;
    if (ctas < 1) ctas = 1;
    pl.sched.num_ctas = (int)ctas;
    pl.counter_bytes = sha::kCounterBytes;
    pl.slot_bytes = (size_t)2 * pl.sched.num_ctas * pl.slot_floats * sizeof(float);
    return pl;
}

// Tensor-map shapes of a strided cache (outer dimensions ordered by stride).
struct StridedMaps {
    long long k_size[3], k_stride[3], v_size[3], v_stride[3];
};

template <typename T, int D, int kLayout, bool kLook>
sha_status_t launch_gqa(const sha::DecodeParams &prm, sha_dtype_t dtype, int dev,
                        cudaStream_t stream, const StridedMaps *kv)
{
    using C = sha::GqaConfig<D>;
    static std::atomic<bool> configured[kMaxDevices];
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(sha::sha_gqa_decode_kernel<T, D, kLayout, kLook>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return launch_error(e);
        configured[dev].store(true, std::memory_order_release);
    }
    CUtensorMap tm_k, tm_v;
    if constexpr (sha::layout_strided(kLayout)) {
        sha_status_t st = kv_tensor_map_4d(&tm_k, prm.k, dtype, D, kv->k_size, kv->k_stride,
                                           prm.tok_dim, 64, C::kTile, true);
        if (st == SHA_OK)
            st = kv_tensor_map_4d(&tm_v, prm.v, dtype, D, kv->v_size, kv->v_stride, prm.tok_dim,
                                  64, C::kTile, true);
        if (st != SHA_OK) return st;
        cudaError_t e = launch_kernel(sha::sha_gqa_decode_kernel<T, D, kLayout, kLook>,
                                      prm.sched.num_ctas, C::threads(kLook), C::kSmemBytes, stream,
                                      prm, tm_k, tm_v);
        if (e != cudaSuccess) return launch_error(e);
        return SHA_OK;
    }
    // a padded cache: [B*H_kv][N_kv][d]; a page pool: [num_pages*H_kv][page_size][d]
    const bool paged = kLayout == sha::kLayoutPaged;
    const long long planes = paged ? (long long)prm.num_pages * prm.H_kv : (long long)prm.B * prm.H_kv;
    const int rows = paged ? prm.page_size : prm.N_kv;
    const int box_rows = paged && prm.page_size < C::kTile ? prm.page_size : C::kTile;
    sha_status_t st = kv_tensor_map(&tm_k, prm.k, dtype, D, rows, planes, box_rows);
    if (st != SHA_OK) return st;
    st = kv_tensor_map(&tm_v, prm.v, dtype, D, rows, planes, box_rows);
    if (st != SHA_OK) return st;
    cudaError_t e = launch_kernel_cluster(
        sha::sha_gqa_decode_kernel<T, D, kLayout, kLook>, prm.sched.num_ctas,
        C::block_threads(kLook, kLayout == sha::kLayoutTokens), C::kSmemBytes, stream,
        kLayout == sha::kLayoutCluster ? prm.sched.cluster : 0, prm, tm_k, tm_v);
    if (e != cudaSuccess) return launch_error(e);
    return SHA_OK;
}

template <typename T, int D, int kLayout, bool kLook>
sha_status_t launch_mha(const sha::DecodeParams &prm, sha_dtype_t dtype, int dev,
                        cudaStream_t stream, const StridedMaps *kv)
{
    using C = sha::MhaConfig<D>;
    static std::atomic<bool> configured[kMaxDevices];
    if (!configured[dev].load(std::memory_order_acquire)) {
        cudaError_t e = cudaFuncSetAttribute(sha::sha_mha_decode_kernel<T, D, kLayout, kLook>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return launch_error(e);
        configured[dev].store(true, std::memory_order_release);
    }
    CUtensorMap tm_k, tm_v;                 // used by the strided layout only
    std::memset(&tm_k, 0, sizeof tm_k);
    std::memset(&tm_v, 0, sizeof tm_v);
    if constexpr (sha::layout_strided(kLayout)) {
        // whole [kTile][d] rows, unswizzled: the same tile layout as a bulk copy
        sha_status_t st = kv_tensor_map_4d(&tm_k, prm.k, dtype, D, kv->k_size, kv->k_stride,
                                           prm.tok_dim, D, C::kTile, false);
        if (st == SHA_OK)
            st = kv_tensor_map_4d(&tm_v, prm.v, dtype, D, kv->v_size, kv->v_stride, prm.tok_dim,
                                  D, C::kTile, false);
        if (st != SHA_OK) return st;
    }
    cudaError_t e = launch_kernel(sha::sha_mha_decode_kernel<T, D, kLayout, kLook>, prm.sched.num_ctas,
                                  C::threads(kLook), C::kSmemBytes, stream, prm, tm_k, tm_v);
    if (e != cudaSuccess) return launch_error(e);
    return SHA_OK;
}

template <typename T, int D, int kLayout, bool kLook>
sha_status_t launch_one(const sha::DecodeParams &prm, sha_dtype_t dtype, bool fma, int dev,
                        cudaStream_t s, const StridedMaps *kv)
{
    return fma ? launch_mha<T, D, kLayout, kLook>(prm, dtype, dev, s, kv)
               : launch_gqa<T, D, kLayout, kLook>(prm, dtype, dev, s, kv);
}

template <typename T, int D, int kLayout>
sha_status_t launch_look(const sha::DecodeParams &prm, sha_dtype_t dtype, bool fma, bool look,
                         int dev, cudaStream_t s, const StridedMaps *kv)
{
    return look ? launch_one<T, D, kLayout, true>(prm, dtype, fma, dev, s, kv)
                : launch_one<T, D, kLayout, false>(prm, dtype, fma, dev, s, kv);
}

// Head x token sparsity: the grouped kernel's gathering build.
template <typename T>
sha_status_t launch_tokens(const sha::DecodeParams &prm, sha_dtype_t dtype, int d, int dev,
                           cudaStream_t s)
{
    // the gathered build: extra gather warps, no scout
    return d == 128 ? launch_gqa<T, 128, sha::kLayoutTokens, false>(prm, dtype, dev, s, nullptr)
                    : launch_gqa<T, 64, sha::kLayoutTokens, false>(prm, dtype, dev, s, nullptr);
}

// The clustered cut: the grouped kernel only, no scout.
template <typename T>
sha_status_t launch_cluster(const sha::DecodeParams &prm, sha_dtype_t dtype, int d, int dev,
                            cudaStream_t s)
{
    return d == 128 ? launch_gqa<T, 128, sha::kLayoutCluster, false>(prm, dtype, dev, s, nullptr)
                    : launch_gqa<T, 64, sha::kLayoutCluster, false>(prm, dtype, dev, s, nullptr);
}

// fma: the multi-head FMA kernel, else the grouped kernel; look: its scout build
template <int kLayout>
sha_status_t launch_decode(const sha::DecodeParams &prm, sha_dtype_t dtype, int d, bool fma,
                           bool look, int dev, cudaStream_t s, const StridedMaps *kv = nullptr)
{
    if (dtype == SHA_FP16)
        return d == 128 ? launch_look<__half, 128, kLayout>(prm, dtype, fma, look, dev, s, kv)
                        : launch_look<__half, 64, kLayout>(prm, dtype, fma, look, dev, s, kv);
    return d == 128 ? launch_look<__nv_bfloat16, 128, kLayout>(prm, dtype, fma, look, dev, s, kv)
                    : launch_look<__nv_bfloat16, 64, kLayout>(prm, dtype, fma, look, dev, s, kv);
}

// Co-resident clusters of the clustered grouped kernel at head dim D, from the
// occupancy calculator (the same for both element types).
template <int D>
void query_cluster_caps(ClusterCaps &caps)
{
    using C = sha::GqaConfig<D>;
    auto kernel = sha::sha_gqa_decode_kernel<__half, D, sha::kLayoutCluster, false>;
    for (int c = 0; c <= C::kClusterMax; ++c) caps.n[c] = 0;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             C::kSmemBytes) != cudaSuccess) {
        (void)cudaGetLastError();
        return;                               // no clustered cut on this device
    }
    for (int c = 2; c <= C::kClusterMax; ++c) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(c * 64);
        cfg.blockDim = dim3(C::threads(false));
        cfg.dynamicSmemBytes = C::kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = c;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
            (void)cudaGetLastError();
            n = 0;
        }
        caps.n[c] = n;
    }
}

// The cluster capacities of device `dev` (looked up once), or null where the
// clustered cut does not apply: per-row lengths, paged or strided caches.
const ClusterCaps *cluster_caps(int dev, int d, bool fixed_layout)
{
    if (!SHA_CLUSTER_CUT || !fixed_layout) return nullptr;
    static ClusterCaps caps[kMaxDevices][2];
    static bool known[kMaxDevices][2];
    const int i = d == 128 ? 1 : 0;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!known[dev][i]) {
        if (d == 128) query_cluster_caps<128>(caps[dev][i]);
        else query_cluster_caps<64>(caps[dev][i]);
        known[dev][i] = true;
    }
    return &caps[dev][i];
}

// Whether to launch the build with a scout warp (sha_lookahead.cuh): it pays
// when blocks end with the head of a split unit whose other parts were done
// early, as under the even cut when a unit meets at most 1 + max_partners
// blocks and each block streams a few tiles (with one or two, every part
// finishes at the same moment).  Pieces of the unit-aligned cut all finish
// together, so they do not qualify.  Calls with per-row lengths are planned
// on the device and take it whenever the kernel can hold a partner's state.
bool lookahead_pays(const Plan &pl, int G, bool fma, bool device_planned)
{
    if (!SHA_LOOKAHEAD) return false;
    const int max_partners = fma ? sha::MhaConfig<128>::kMaxPartners
                           : G <= sha::GqaConfig<128>::kMaxPartRows
                               ? sha::GqaConfig<128>::kConsumerWarps - 2
                               : 0;
    if (max_partners == 0) return false;
    if (device_planned) return true;
    if (pl.sched.pieces != 0) return false;
    const long long per_block = pl.sched.total_tiles / pl.sched.num_ctas;
    if (per_block < 4) return false;
    const long long parts = (pl.sched.tiles_per_unit - 1 + per_block - 1) / per_block + 1;
    return parts >= 2 && parts - 1 <= max_partners;
}

// Where the keys of a call live beyond the plain [B, H_kv, N_kv, d] cache.
struct KvLayout {
    const int32_t *seqlens = nullptr;       // per-row lengths (device), or null
    const int32_t *block_table = nullptr;   // paged pool: [B, max_pages] (device), or null
    int page_size = 0, max_pages = 0, num_pages = 0;
    bool strided = false;                   // K, V with the strides below (elements)
    KvStrides k_strides{}, v_strides{};
    const int32_t *tokens = nullptr;        // head x token sparsity: [B, top_k, n_sel] (device)
    int n_sel = 0;
};

// N_kv is the padded length (per-row lengths) or max_pages * page_size (paged).
// A caller's choice of the clustered cut (sha_decode_clustered); 0: the planner's.
struct ForcedCluster {
    int cluster = 0, units_per_cluster = 0, whole_per_block = 0;
};

sha_status_t decode_impl(const void *q, const void *k, const void *v, const int32_t *idx,
                         int B, int H_q, int H_kv, int N_kv, int d, int top_k, float scale,
                         void *out, sha_dtype_t dtype, void *workspace,
                         size_t workspace_bytes, int num_splits, void *stream,
                         bool library_workspace, const KvLayout &lay = KvLayout(),
                         ForcedCluster force = ForcedCluster())
{
    const int32_t *seqlens = lay.seqlens;
    if (dtype != SHA_FP16 && dtype != SHA_BF16) return SHA_ERR_UNSUPPORTED;
    sha_status_t st = check_shape(B, H_q, H_kv, N_kv, d, top_k, scale);
    if (st != SHA_OK) return st;
    if (num_splits < 0) return SHA_ERR_INVALID_ARG;
    if (B == 0 || top_k == 0) return SHA_OK;
    if (!q || !k || !v || !idx || !out) return SHA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(idx, 4))
        return SHA_ERR_MISALIGNED;
    if (workspace && !aligned(workspace, 256)) return SHA_ERR_MISALIGNED;
    if (seqlens && !aligned(seqlens, 4)) return SHA_ERR_MISALIGNED;
    if (lay.tokens && !aligned(lay.tokens, 4)) return SHA_ERR_MISALIGNED;
    if (lay.block_table && !aligned(lay.block_table, 4)) return SHA_ERR_MISALIGNED;
    const int G = H_q / H_kv;

    int dev;
    DeviceInfo *info;
    st = current_device(&dev, &info);
    if (st != SHA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const ClusterCaps *caps =
        cluster_caps(dev, d, !seqlens && !lay.strided && !lay.block_table && !lay.tokens);
    Plan pl;
    if (force.cluster) {
        st = forced_cluster_plan(B, H_q, H_kv, N_kv, d, top_k, force.cluster,
                                 force.units_per_cluster, force.whole_per_block, pl);
        if (st != SHA_OK) return st;
    } else if (lay.tokens) {
        // the call streams n_sel keys per unit: plan it as a cache that long
        pl = make_plan(B, H_q, H_kv, lay.n_sel, d, top_k, num_splits, info->num_sms, false,
                       nullptr);
    } else {
        pl = seqlens ? make_varlen_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, info->num_sms)
                     : make_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, info->num_sms, false,
                                 caps);
    }
    const size_t need = pl.workspace_bytes();
    // paged calls carry lengths too; gathered keys take the grouped kernel
    const bool fma = !lay.tokens && fma_path(G, d, seqlens != nullptr);
    const bool look = pl.sched.cluster < 2 && lookahead_pays(pl, G, fma, seqlens != nullptr);

    if (library_workspace && need > 0) {
        OwnedWorkspace *owned = g_owned;
        std::lock_guard<std::mutex> lock(g_mutex);
        if (owned[dev].bytes < need) {
            size_t bytes = need < (1u << 20) ? (1u << 20) : need;
            if (owned[dev].ptr) {
                cudaError_t e = cudaFree(owned[dev].ptr);
                owned[dev].ptr = nullptr;
                owned[dev].bytes = 0;
                if (e != cudaSuccess) return launch_error(e);
            }
            cudaError_t e = cudaMalloc(&owned[dev].ptr, bytes);
            if (e != cudaSuccess) return launch_error(e);
            e = cudaMemsetAsync(owned[dev].ptr, 0, bytes, s);
            if (e != cudaSuccess) return launch_error(e);
            owned[dev].bytes = bytes;
        }
        workspace = owned[dev].ptr;
        workspace_bytes = owned[dev].bytes;
    }
    if (need > 0 && (!workspace || workspace_bytes < need)) return SHA_ERR_WORKSPACE;

    sha::DecodeParams prm;
    prm.q = q;
    prm.k = k;
    prm.v = v;
    prm.idx = idx;
    prm.out = out;
    prm.B = B;
    prm.H_q = H_q;
    prm.H_kv = H_kv;
    prm.N_kv = N_kv;
    prm.top_k = top_k;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.sched = pl.sched;
    prm.slot_floats = pl.slot_floats;
    prm.counters = need ? static_cast<int *>(workspace) : nullptr;
    prm.slots = need ? reinterpret_cast<float *>(static_cast<char *>(workspace) +
                                                 pl.counter_bytes)
                     : nullptr;
    prm.seqlens = seqlens;
    prm.block_table = lay.block_table;
    prm.page_size = lay.page_size;
    prm.max_pages = lay.max_pages;
    prm.num_pages = lay.num_pages;
    prm.tok_dim = 0;
    prm.head_dim = 1;
    prm.batch_dim = 2;
    prm.tokens = lay.tokens;
    prm.n_sel = lay.n_sel;
    if (lay.strided) {
        StridedMaps kv;
        int vt, vh, vb;
        order_outer_dims(lay.k_strides, B, H_kv, N_kv, kv.k_size, kv.k_stride, prm.tok_dim,
                         prm.head_dim, prm.batch_dim);
        order_outer_dims(lay.v_strides, B, H_kv, N_kv, kv.v_size, kv.v_stride, vt, vh, vb);
        // one set of coordinates serves both maps
        if (vt != prm.tok_dim || vh != prm.head_dim || vb != prm.batch_dim)
            return SHA_ERR_UNSUPPORTED;
        if (seqlens)
            return launch_decode<sha::kLayoutStridedVarlen>(prm, dtype, d, fma, look, dev, s, &kv);
        return launch_decode<sha::kLayoutStrided>(prm, dtype, d, fma, look, dev, s, &kv);
    }
    if (lay.tokens)
        return dtype == SHA_FP16 ? launch_tokens<__half>(prm, dtype, d, dev, s)
                                 : launch_tokens<__nv_bfloat16>(prm, dtype, d, dev, s);
    if (pl.sched.cluster >= 2)
        return dtype == SHA_FP16 ? launch_cluster<__half>(prm, dtype, d, dev, s)
                                 : launch_cluster<__nv_bfloat16>(prm, dtype, d, dev, s);
    if (lay.block_table) return launch_decode<sha::kLayoutPaged>(prm, dtype, d, fma, look, dev, s);
    if (seqlens) return launch_decode<sha::kLayoutVarlen>(prm, dtype, d, fma, look, dev, s);
    return launch_decode<sha::kLayoutFixed>(prm, dtype, d, fma, look, dev, s);
}

__global__ void copy_probe_kernel(uint4 *__restrict__ dst, const uint4 *__restrict__ src,
                                  size_t n)
{
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    for (; i + 3 * stride < n; i += 4 * stride) {
        const uint4 a = __ldcs(src + i);
        const uint4 b = __ldcs(src + i + stride);
        const uint4 c = __ldcs(src + i + 2 * stride);
        const uint4 d = __ldcs(src + i + 3 * stride);
        __stcs(dst + i, a);
        __stcs(dst + i + stride, b);
        __stcs(dst + i + 2 * stride, c);
        __stcs(dst + i + 3 * stride, d);
    }
    for (; i < n; i += stride) __stcs(dst + i, __ldcs(src + i));
}

}  // namespace

extern "C" {

sha_status_t sha_decode(const void *q, const void *k, const void *v,
                        const int32_t *batch_head_index, int B, int H_q, int H_kv, int N_kv,
                        int d, int top_k, float scale, void *out, void *stream)
{
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       SHA_FP16, nullptr, 0, 0, stream, true);
}

sha_status_t sha_decode_bf16(const void *q, const void *k, const void *v,
                             const int32_t *batch_head_index, int B, int H_q, int H_kv,
                             int N_kv, int d, int top_k, float scale, void *out, void *stream)
{
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       SHA_BF16, nullptr, 0, 0, stream, true);
}

sha_status_t sha_decode_ex(const void *q, const void *k, const void *v,
                           const int32_t *batch_head_index, int B, int H_q, int H_kv,
                           int N_kv, int d, int top_k, float scale, void *out,
                           sha_dtype_t dtype, void *workspace, size_t workspace_bytes,
                           int num_splits, void *stream)
{
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       dtype, workspace, workspace_bytes, num_splits, stream, false);
}

sha_status_t sha_decode_varlen(const void *q, const void *k, const void *v,
                               const int32_t *batch_head_index, const int32_t *seqlens, int B,
                               int H_q, int H_kv, int N_max, int d, int top_k, float scale,
                               void *out, sha_dtype_t dtype, void *stream)
{
    if (B > 0 && top_k > 0 && !seqlens) return SHA_ERR_INVALID_ARG;
    KvLayout lay;
    lay.seqlens = seqlens;
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_max, d, top_k, scale, out,
                       dtype, nullptr, 0, 0, stream, true, lay);
}

sha_status_t sha_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                              const int32_t *batch_head_index, const int32_t *seqlens,
                              const int32_t *block_table, int B, int H_q, int H_kv,
                              int num_pages, int page_size, int max_pages, int d, int top_k,
                              float scale, void *out, sha_dtype_t dtype, void *stream)
{
    if (num_pages < 1 || page_size < 1 || max_pages < 1) return SHA_ERR_INVALID_ARG;
    if ((long long)max_pages * page_size > (1 << 30)) return SHA_ERR_INVALID_ARG;
    if (H_kv >= 1 && H_q % H_kv == 0 && H_q / H_kv > 1 && !boxable_pages(page_size))
        return SHA_ERR_UNSUPPORTED;   // TMA boxes of whole pages: powers of two >= 8
    if (B > 0 && top_k > 0 && (!seqlens || !block_table)) return SHA_ERR_INVALID_ARG;
    KvLayout lay;
    lay.seqlens = seqlens;
    lay.block_table = block_table;
    lay.page_size = page_size;
    lay.max_pages = max_pages;
    lay.num_pages = num_pages;
    return decode_impl(q, k_pages, v_pages, batch_head_index, B, H_q, H_kv,
                       max_pages * page_size, d, top_k, scale, out, dtype, nullptr, 0, 0,
                       stream, true, lay);
}

sha_status_t sha_decode_strided(const void *q, const void *k, const void *v,
                                const int32_t *batch_head_index, const int32_t *seqlens, int B,
                                int H_q, int H_kv, int N_kv, int d, int top_k, float scale,
                                void *out, const int64_t k_strides[3], const int64_t v_strides[3],
                                sha_dtype_t dtype, void *stream)
{
    if (!k_strides || !v_strides) return SHA_ERR_INVALID_ARG;
    KvLayout lay;
    lay.strided = true;
    lay.seqlens = seqlens;
    lay.k_strides = {k_strides[0], k_strides[1], k_strides[2]};
    lay.v_strides = {v_strides[0], v_strides[1], v_strides[2]};
    for (int i = 0; i < 3; ++i) {
        if (k_strides[i] < 1 || v_strides[i] < 1) return SHA_ERR_INVALID_ARG;
        // TMA: every stride a multiple of 16 bytes, below 2^40 bytes
        if (k_strides[i] % 8 || v_strides[i] % 8) return SHA_ERR_MISALIGNED;
        if (k_strides[i] >= (1ll << 39) || v_strides[i] >= (1ll << 39)) return SHA_ERR_INVALID_ARG;
    }
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       dtype, nullptr, 0, 0, stream, true, lay);
}

sha_status_t sha_decode_tokens(const void *q, const void *k, const void *v,
                               const int32_t *batch_head_index, const int32_t *tokens, int B,
                               int H_q, int H_kv, int N_kv, int d, int top_k, int n_sel,
                               float scale, void *out, sha_dtype_t dtype, void *stream)
{
    if (n_sel < 1) return SHA_ERR_INVALID_ARG;
    if (B > 0 && top_k > 0 && !tokens) return SHA_ERR_INVALID_ARG;
    KvLayout lay;
    lay.tokens = tokens;
    lay.n_sel = n_sel;
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       dtype, nullptr, 0, 0, stream, true, lay);
}

size_t sha_decode_workspace_size(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                                 int num_splits)
{
    if (check_shape(B, H_q, H_kv, N_kv, d, top_k, 1.0f) != SHA_OK || num_splits < 0) return 0;
    if (B == 0 || top_k == 0) return 0;
    int dev;
    DeviceInfo *info;
    if (current_device(&dev, &info) != SHA_OK) return 0;
    return make_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, info->num_sms)
        .workspace_bytes();
}

sha_status_t sha_decode_plan(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                             int num_splits, int num_sms, int64_t plan[5])
{
    sha_status_t st = check_shape(B, H_q, H_kv, N_kv, d, top_k, 1.0f);
    if (st != SHA_OK) return st;
    if (num_splits < 0 || num_sms < 1 || !plan) return SHA_ERR_INVALID_ARG;
    const int tile = tile_keys(H_q / H_kv, d, false);
    if (B == 0 || top_k == 0) {
        plan[0] = (N_kv + tile - 1) / tile;
        plan[1] = plan[2] = plan[3] = 0;
        plan[4] = tile;
        return SHA_OK;
    }
    const Plan pl = make_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, num_sms);
    plan[0] = pl.sched.tiles_per_unit;
    plan[1] = pl.sched.total_tiles;
    plan[2] = pl.sched.num_ctas;
    plan[3] = (int64_t)pl.workspace_bytes();
    plan[4] = tile;
    return SHA_OK;
}

sha_status_t sha_decode_plan_ex(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                                int num_splits, int num_sms, const int32_t cluster_capacity[9],
                                int64_t plan[9])
{
    sha_status_t st = check_shape(B, H_q, H_kv, N_kv, d, top_k, 1.0f);
    if (st != SHA_OK) return st;
    if (num_splits < 0 || num_sms < 1 || !plan) return SHA_ERR_INVALID_ARG;
    const int tile = tile_keys(H_q / H_kv, d, false);
    for (int i = 0; i < 9; ++i) plan[i] = 0;
    plan[4] = tile;
    if (B == 0 || top_k == 0) {
        plan[0] = (N_kv + tile - 1) / tile;
        return SHA_OK;
    }
    ClusterCaps caps;
    for (int c = 0; c <= sha::GqaConfig<128>::kClusterMax; ++c)
        caps.n[c] = cluster_capacity && c >= 2 ? cluster_capacity[c] : 0;
    const Plan pl = make_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, num_sms, false,
                              cluster_capacity ? &caps : nullptr);
    plan[0] = pl.sched.tiles_per_unit;
    plan[1] = pl.sched.total_tiles;
    plan[2] = pl.sched.num_ctas;
    plan[3] = (int64_t)pl.workspace_bytes();
    plan[5] = pl.sched.cluster;
    plan[6] = pl.sched.units_per_cluster;
    plan[7] = pl.sched.pieces;
    plan[8] = pl.sched.whole_per_block;
    return SHA_OK;
}

sha_status_t sha_decode_cluster_capacity(int d, int32_t cluster_capacity[9])
{
    if (!cluster_capacity) return SHA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return SHA_ERR_UNSUPPORTED;
    int dev;
    DeviceInfo *info;
    sha_status_t st = current_device(&dev, &info);
    if (st != SHA_OK) return st;
    const ClusterCaps *caps = cluster_caps(dev, d, true);
    for (int c = 0; c < 9; ++c)
        cluster_capacity[c] = caps && c <= sha::GqaConfig<128>::kClusterMax ? caps->n[c] : 0;
    return SHA_OK;
}

sha_status_t sha_decode_clustered(const void *q, const void *k, const void *v,
                                  const int32_t *batch_head_index, int B, int H_q, int H_kv,
                                  int N_kv, int d, int top_k, float scale, void *out,
                                  sha_dtype_t dtype, int cluster, int units_per_cluster,
                                  int whole_per_block, void *stream)
{
    if (cluster < 2) return SHA_ERR_INVALID_ARG;
    ForcedCluster force;
    force.cluster = cluster;
    force.units_per_cluster = units_per_cluster;
    force.whole_per_block = whole_per_block;
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       dtype, nullptr, 0, 0, stream, false, KvLayout(), force);
}

sha_status_t sha_select_heads(const float *scores, int B, int H, int top_k,
                              int32_t *batch_head_index, void *stream)
{
    if (B < 0 || H < 1 || top_k < 0 || top_k > H) return SHA_ERR_INVALID_ARG;
    if (H > sha::kSelectMaxHeads) return SHA_ERR_UNSUPPORTED;
    if (B == 0 || top_k == 0) return SHA_OK;
    if (!scores || !batch_head_index) return SHA_ERR_INVALID_ARG;
    if (!aligned(scores, 4) || !aligned(batch_head_index, 4)) return SHA_ERR_MISALIGNED;
    const int grid = (B + sha::kSelectRowsPerBlock - 1) / sha::kSelectRowsPerBlock;
    cudaError_t e = launch_kernel(sha::sha_select_heads_kernel, grid,
                                  sha::kSelectRowsPerBlock * 32, 0,
                                  static_cast<cudaStream_t>(stream), scores, B, H, top_k,
                                  batch_head_index);
    if (e != cudaSuccess) return launch_error(e);
    return SHA_OK;
}

unsigned sha_mlp_take_status();   // sha_mlp.cu

sha_status_t sha_get_device_status(void *stream)
{
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return launch_error(e);
    unsigned int flags = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&flags, sha::g_sha_status, sizeof flags);
    if (e != cudaSuccess) return launch_error(e);
    e = cudaMemcpyToSymbol(sha::g_sha_status, &zero, sizeof zero);
    if (e != cudaSuccess) return launch_error(e);
    flags |= sha_mlp_take_status();
    if (flags & sha::kStatusTimeout) {
        // an abandoned merge can leave arrival counters raised: clear the
        // library workspace's, in order on `stream`
        int dev;
        if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < kMaxDevices) {
            std::lock_guard<std::mutex> lock(g_mutex);
            if (g_owned[dev].ptr) {
                e = cudaMemsetAsync(g_owned[dev].ptr, 0, sha::kCounterBytes, s);
                if (e == cudaSuccess) e = cudaStreamSynchronize(s);
                if (e != cudaSuccess) return launch_error(e);
            }
        }
        return SHA_ERR_TIMEOUT;
    }
    if (flags & sha::kStatusBadIndex) return SHA_ERR_BAD_INDEX;
    return SHA_OK;
}

const char *sha_status_string(sha_status_t status)
{
    switch (status) {
    case SHA_OK: return "SHA_OK";
    case SHA_ERR_INVALID_ARG: return "SHA_ERR_INVALID_ARG";
    case SHA_ERR_UNSUPPORTED: return "SHA_ERR_UNSUPPORTED";
    case SHA_ERR_MISALIGNED: return "SHA_ERR_MISALIGNED";
    case SHA_ERR_LAUNCH: return "SHA_ERR_LAUNCH";
    case SHA_ERR_BAD_INDEX: return "SHA_ERR_BAD_INDEX";
    case SHA_ERR_TIMEOUT: return "SHA_ERR_TIMEOUT";
    case SHA_ERR_WORKSPACE: return "SHA_ERR_WORKSPACE";
    }
    return "unknown sha_status_t";
}

const char *sha_last_cuda_error(void) { return g_last_cuda_error; }

#ifdef SHA_TEST_HOOKS
// Test builds only (not part of the ABI): lower the pipeline wait limit of
// the current device, so that a test can make waits give up on purpose.
sha_status_t sha_test_set_wait_limit(unsigned long long ns)
{
    cudaError_t e = cudaMemcpyToSymbol(sha::g_wait_limit_ns, &ns, sizeof ns);
    if (e != cudaSuccess) return launch_error(e);
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return launch_error(e);
    return SHA_OK;
}
#endif

sha_status_t sha_copy_bandwidth_probe(void *dst, const void *src, size_t bytes, void *stream)
{
    if (!dst || !src || bytes % 16 != 0) return SHA_ERR_INVALID_ARG;
    if (!aligned(dst, 16) || !aligned(src, 16)) return SHA_ERR_MISALIGNED;
    if (bytes == 0) return SHA_OK;
    int dev;
    DeviceInfo *info;
    sha_status_t st = current_device(&dev, &info);
    if (st != SHA_OK) return st;
    copy_probe_kernel<<<info->num_sms * 4, 512, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4 *>(dst), static_cast<const uint4 *>(src), bytes / 16);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return launch_error(e);
    return SHA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode without allocation: the multi-head kernel with its split-merge
// scratch (arrival counters + partial states) in a fixed static device array
// instead of a cudaMalloc'd workspace.  Every GPU that loads this library
// holds the array until the process exits.

namespace {

// Scratch of sha_decode_noalloc.  In host code this name is only a stand-in
// for the symbol: the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[SHA_NOALLOC_SCRATCH_BYTES];

void *g_noalloc_scratch_ptr[kMaxDevices];

// Once per device, with that device current: the array's device address.
sha_status_t noalloc_scratch_address(int dev, void **ptr)
{
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_noalloc_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return launch_error(e);
        g_noalloc_scratch_ptr[dev] = p;
    }
    *ptr = g_noalloc_scratch_ptr[dev];
    return SHA_OK;
}

}  // namespace

extern "C" size_t sha_noalloc_scratch_bytes(void) { return SHA_NOALLOC_SCRATCH_BYTES; }

extern "C" sha_status_t sha_decode_noalloc(const void *q, const void *k, const void *v,
                                           const int32_t *batch_head_index, int B, int H_q,
                                           int H_kv, int N_kv, int d, int top_k, float scale,
                                           void *out, sha_dtype_t dtype, int num_splits,
                                           void *stream)
{
    // every host-side check before the first CUDA call
    if (dtype != SHA_FP16 && dtype != SHA_BF16) return SHA_ERR_UNSUPPORTED;
    sha_status_t st = check_shape(B, H_q, H_kv, N_kv, d, top_k, scale);
    if (st != SHA_OK) return st;
    if (num_splits < 0) return SHA_ERR_INVALID_ARG;
    if (H_q != H_kv) return SHA_ERR_UNSUPPORTED;   // multi-head calls (G = 1) only
    if (B == 0 || top_k == 0) return SHA_OK;
    if (!q || !k || !v || !batch_head_index || !out) return SHA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
        !aligned(batch_head_index, 4))
        return SHA_ERR_MISALIGNED;

    int dev;
    DeviceInfo *info;
    st = current_device(&dev, &info);
    if (st != SHA_OK) return st;
    const Plan pl = make_plan(B, H_q, H_kv, N_kv, d, top_k, num_splits, info->num_sms, false,
                              cluster_caps(dev, d, true));
    const size_t need = pl.workspace_bytes();
    if (need > (size_t)SHA_NOALLOC_SCRATCH_BYTES) return SHA_ERR_WORKSPACE;
    void *scratch = nullptr;
    st = noalloc_scratch_address(dev, &scratch);
    if (st != SHA_OK) return st;
    if (need > 0) {
        // the arrival counters must start at zero whatever an earlier call left
        cudaError_t e = cudaMemsetAsync(scratch, 0, (size_t)pl.sched.num_ctas * sizeof(int),
                                        static_cast<cudaStream_t>(stream));
        if (e != cudaSuccess) return launch_error(e);
    }
    return decode_impl(q, k, v, batch_head_index, B, H_q, H_kv, N_kv, d, top_k, scale, out,
                       dtype, scratch, SHA_NOALLOC_SCRATCH_BYTES, num_splits, stream, false);
}
