/*
 * sha_decode.h -- C ABI of the Selective Head Attention (SHA) decode library
 * (libsha_decode.so, CUDA kernels for sm_100a).
 *
 * The operation.  Polar Sparsity (papernotes.org summary, section "Selective
 * Head Attention (SHA) Kernel"; ri.k117.org reproducibility record,
 * "Pseudocode" row, Algorithm 1 "Selective Head Flash Attention (Decode)"):
 * for every batch row b and every slot k < top_k the kernel reads
 * h = batch_head_index[b, k], streams only that head's K/V cache and writes
 *
 *     out[b, h*G + j, :] = softmax(scale * q K^T) V,   q = Q[b, h*G + j, :],
 *     K = K[b, h, :, :],  V = V[b, h, :, :],  j = 0 .. G-1,  G = H_q / H_kv,
 *
 * i.e. the attention equation under "Attention Head 稀疏性" (papernotes.org
 * summary) for one decode token.  G = 1 is multi-head attention with head
 * sparsity; G > 1 is grouped-query attention with group sparsity (the pages:
 * GQA models select KV groups, and a selected group computes all of its query
 * heads).  Rows of heads that are not selected are neither read nor written:
 * they keep the caller's contents bit for bit.
 *
 * Layout (all row-major, contiguous, one dtype for q, k, v and out):
 *     q   : [B, H_q, d]            (the decode token's query; [B, H_q, 1, d] is the same memory)
 *     k,v : [B, H_kv, N_kv, d]     (KV cache)
 *     out : [B, H_q, d]
 *     batch_head_index : [B, top_k] int32, KV-head (group) ids in [0, H_kv)
 * All pointers are DEVICE pointers owned by the caller and must be 16-byte
 * aligned.  Arithmetic: fp32 accumulation; the result is rounded to the
 * tensor dtype (round to nearest even).
 *
 * Asynchrony.  Every launching call enqueues its kernel(s) on `stream`
 * (a cudaStream_t; NULL = the legacy default stream) and returns without
 * synchronising.  Argument errors are detected on the host before any launch
 * and nothing is enqueued then.
 *
 * Head ids out of [0, H_kv) are a device-side condition: that (b, k) slot is
 * skipped (nothing read, nothing written) and a sticky flag is raised, which
 * sha_get_device_status() reports.  No kernel traps.
 *
 * Determinism.  Repeated calls with the same arguments on the same device
 * give bit-identical outputs: a head split across thread blocks is merged in
 * a fixed block order, never in arrival order.  The result does depend, at
 * the level of rounding, on where a head's id sits in its row of
 * batch_head_index: the key tiles of a call are cut in slot order, so
 * permuting a row can move a head's tiles to other blocks and change the
 * order of its fp32 sums.  A caller that reorders the ids of a row between
 * steps gets outputs equal within the fp32-accumulation tolerance, not bit
 * for bit.
 */
#ifndef SHA_DECODE_H
#define SHA_DECODE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SHA_OK = 0,
    SHA_ERR_INVALID_ARG = 1,   /* null pointer, negative or inconsistent size, non-finite scale */
    SHA_ERR_UNSUPPORTED = 2,   /* d not in {64, 128}, G = H_q/H_kv > 16, unknown dtype */
    SHA_ERR_MISALIGNED = 3,    /* a pointer is not 16-byte aligned */
    SHA_ERR_LAUNCH = 4,        /* a CUDA runtime call failed (see sha_last_cuda_error) */
    SHA_ERR_BAD_INDEX = 5,     /* device flag: a head id was out of range */
    SHA_ERR_TIMEOUT = 6,       /* device flag: a pipeline wait gave up (should never happen) */
    SHA_ERR_WORKSPACE = 7      /* caller workspace too small */
} sha_status_t;

typedef enum { SHA_FP16 = 0, SHA_BF16 = 1 } sha_dtype_t;

/*
 * sha_decode -- fp16 selective head decode, the operation above.
 *   q, k, v, out       : device pointers, fp16, layout above.
 *   batch_head_index   : device pointer, int32 [B, top_k].
 *   B >= 0, H_q >= 1, H_kv >= 1 with H_q % H_kv == 0 and H_q / H_kv <= 16,
 *   N_kv >= 1, d in {64, 128}, 0 <= top_k <= H_kv, scale finite
 *   (1/sqrt(d) reproduces the pages' softmax(Q K^T / sqrt(d_h))).
 *   B == 0 or top_k == 0 is a no-op returning SHA_OK.
 * Scratch: the call may split one head's key range across thread blocks and
 * then needs a small device workspace (sha_decode_workspace_size bytes); this
 * entry point keeps one per device, allocated on the first call that needs
 * it (or a larger one) and reused after.  Calls that share a device and
 * overlap in time on different streams therefore race on it; use
 * sha_decode_ex with one workspace per stream for that.
 * Returns SHA_OK once the kernel is enqueued.
 */
sha_status_t sha_decode(const void *q, const void *k, const void *v,
                        const int32_t *batch_head_index, int B, int H_q,
                        int H_kv, int N_kv, int d, int top_k, float scale,
                        void *out, void *stream);

/* sha_decode_bf16 -- the same operation on bfloat16 tensors. */
sha_status_t sha_decode_bf16(const void *q, const void *k, const void *v,
                             const int32_t *batch_head_index, int B, int H_q,
                             int H_kv, int N_kv, int d, int top_k, float scale,
                             void *out, void *stream);

/*
 * sha_decode_ex -- explicit dtype, caller-owned workspace, forced partition count.
 *   dtype           : SHA_FP16 or SHA_BF16.
 *   workspace       : device pointer, 256-byte aligned, at least
 *                     sha_decode_workspace_size(...) bytes for the same sizes
 *                     and num_splits, or NULL when that size is 0.  Its
 *                     first 16 KiB hold arrival counters that must be zero
 *                     before the first use; every call leaves them zero
 *                     again when it completes (whatever the sizes of the
 *                     calls that share the workspace), so one cudaMemset
 *                     after allocation is enough -- unless a call reported
 *                     SHA_ERR_TIMEOUT, after which the workspace must be
 *                     zeroed again.  Calls that use one workspace must not
 *                     overlap on the device.
 *   num_splits      : 0 = automatic.  Otherwise the B*top_k*ceil(N_kv/tile)
 *                     key tiles of the call are cut into exactly this many
 *                     contiguous, equal (to within one tile) ranges, one per
 *                     thread block (clamped to the tile count and to 4096).  A head whose
 *                     tiles straddle ranges is finished by the last block to
 *                     complete its part (log-sum-exp merge of the parts, in a
 *                     fixed order, so results do not depend on timing).
 * The library allocates nothing here.
 */
sha_status_t sha_decode_ex(const void *q, const void *k, const void *v,
                           const int32_t *batch_head_index, int B, int H_q,
                           int H_kv, int N_kv, int d, int top_k, float scale,
                           void *out, sha_dtype_t dtype, void *workspace,
                           size_t workspace_bytes, int num_splits,
                           void *stream);

/*
 * sha_decode_varlen -- the same operation when every batch row has its own
 * cache length, as in a decode batch of sequences of different lengths:
 * row b attends to keys [0, seqlens[b]) of its cache.
 *   k, v     : [B, H_kv, N_max, d] (rows padded to N_max; keys at or past
 *              seqlens[b] are never used and may hold anything)
 *   seqlens  : device pointer, int32 [B], each in [1, N_max]; a row whose
 *              length is outside that range is skipped (its outputs stay
 *              untouched) and raises the SHA_ERR_BAD_INDEX flag
 *   dtype    : SHA_FP16 or SHA_BF16; other arguments as for sha_decode.
 * The lengths stay on the device: the kernel plans its own balanced split
 * from them (every block streams the same number of key tiles).  Uses the
 * library-owned per-device workspace, like sha_decode.
 */
sha_status_t sha_decode_varlen(const void *q, const void *k, const void *v,
                               const int32_t *batch_head_index, const int32_t *seqlens,
                               int B, int H_q, int H_kv, int N_max, int d, int top_k,
                               float scale, void *out, sha_dtype_t dtype, void *stream);

/*
 * sha_decode_strided -- the same operation over K and V caches laid out with
 * any strides, d contiguous: element (b, h, n, c) of K is at
 *   k + b*k_strides[0] + h*k_strides[1] + n*k_strides[2] + c
 * (strides in elements; likewise for V).  This covers a token-major cache
 * [B, N, H_kv, d] (strides N*H_kv*d, d, H_kv*d), a head-major cache padded
 * to N_max > N_kv (strides H_kv*N_max*d, N_max*d, d), and the K and V views
 * of one fused buffer.  Each key tile is one TMA tensor box.
 *   seqlens              : NULL (every row N_kv keys long) or a device pointer,
 *                          int32 [B], each in [1, N_kv]: row b attends to its
 *                          first seqlens[b] keys, as in sha_decode_varlen
 *   k_strides, v_strides : host arrays of 3 int64 (batch, head, token), each
 *                          >= 1 and a multiple of 8 elements (16 bytes;
 *                          SHA_ERR_MISALIGNED otherwise); K and V strides must
 *                          rank their dimensions in the same order
 *                          (SHA_ERR_UNSUPPORTED otherwise)
 *   dtype                : SHA_FP16 or SHA_BF16; other arguments as for sha_decode.
 * The caller guarantees that the addressed elements lie inside its buffers.
 * Uses the library-owned per-device workspace, like sha_decode.
 */
sha_status_t sha_decode_strided(const void *q, const void *k, const void *v,
                                const int32_t *batch_head_index, const int32_t *seqlens, int B,
                                int H_q, int H_kv, int N_kv, int d, int top_k, float scale,
                                void *out, const int64_t k_strides[3], const int64_t v_strides[3],
                                sha_dtype_t dtype, void *stream);

/*
 * sha_decode_paged -- the same operation over a paged KV cache, the serving
 * layout in which each sequence's keys live in fixed-size pages of a pool:
 *   k_pages, v_pages : [num_pages, H_kv, page_size, d]
 *   block_table      : device pointer, int32 [B, max_pages]; key n of row b
 *                      sits at page block_table[b, n / page_size], position
 *                      n % page_size
 *   seqlens          : device pointer, int32 [B], each in
 *                      [1, max_pages * page_size]
 *   page_size >= 1; for G = H_q/H_kv > 1 a power of two >= 8
 *   (SHA_ERR_UNSUPPORTED otherwise).
 * Rows with a bad length are skipped and flagged as in sha_decode_varlen.
 * A page id outside [0, num_pages) is bad input: the flag is raised, no
 * memory outside the pool is read, and that unit's output is unspecified.
 * Uses the library-owned per-device workspace, like sha_decode.
 */
sha_status_t sha_decode_paged(const void *q, const void *k_pages, const void *v_pages,
                              const int32_t *batch_head_index, const int32_t *seqlens,
                              const int32_t *block_table, int B, int H_q, int H_kv,
                              int num_pages, int page_size, int max_pages, int d, int top_k,
                              float scale, void *out, sha_dtype_t dtype, void *stream);

/*
 * sha_decode_tokens -- head x token sparsity.  Polar Sparsity names the
 * combination of head sparsity with token sparsity as future work
 * (papernotes.org summary, "局限与展望"); this entry point is its plainest
 * form: each selected (row b, slot k) unit attends only to a caller-given
 * list of its head's keys,
 *     out[b, h*G + j, :] = softmax over i of (scale * q K[t_i]^T) V[t_i],
 *     t_i = tokens[b, k, i],  i < n_sel,  h = batch_head_index[b, k],
 * a listed position counting once per listing.
 *   tokens : device pointer, int32 [B, top_k, n_sel], positions in [0, N_kv);
 *            any order, repeats allowed
 *   n_sel  : keys per unit, >= 1 (it need not be <= N_kv)
 *   k, v   : [B, H_kv, N_kv, d] as for sha_decode; dtype SHA_FP16 or SHA_BF16.
 * A position outside [0, N_kv) is bad input: the SHA_ERR_BAD_INDEX flag is
 * raised, no memory outside the head's cache is read, and that unit's output
 * is unspecified.  The listed K and V rows are gathered with 16-byte copies
 * (each key row is read once per listing) and run on the grouped kernel for
 * every G (d = 64 or 128).  Uses the library-owned per-device workspace, like
 * sha_decode.
 */
sha_status_t sha_decode_tokens(const void *q, const void *k, const void *v,
                               const int32_t *batch_head_index, const int32_t *tokens, int B,
                               int H_q, int H_kv, int N_kv, int d, int top_k, int n_sel,
                               float scale, void *out, sha_dtype_t dtype, void *stream);

/*
 * sha_decode_workspace_size -- bytes of workspace sha_decode_ex needs for
 * these sizes and num_splits (0 = automatic) on the current device.  Host
 * only; reads the device's SM count.  Returns 0 for sizes sha_decode_ex
 * would reject.
 */
size_t sha_decode_workspace_size(int B, int H_q, int H_kv, int N_kv, int d,
                                 int top_k, int num_splits);

/*
 * sha_decode_plan -- how a call with these sizes is cut into thread blocks on
 * a device with num_sms SMs (host only, no CUDA call).  Writes
 *   plan[0] = key tiles per selected head   (ceil(N_kv / tile))
 *   plan[1] = key tiles of the whole call   (B * top_k * plan[0])
 *   plan[2] = thread blocks launched        (one contiguous tile range each)
 *   plan[3] = workspace bytes               (0: every head lies in one range)
 *   plan[4] = keys per tile
 * Returns the status sha_decode_ex would return for these sizes before any
 * launch (SHA_OK when they are valid).
 */
sha_status_t sha_decode_plan(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                             int num_splits, int num_sms, int64_t plan[5]);

/*
 * The clustered cut.  A short call -- few (batch row, head) units, or few key
 * tiles per unit -- keeps most SMs idle if every unit stays in one thread
 * block, and if a unit's tiles are spread over several blocks, merging the
 * parts through global memory (write, fence, arrival counter, read back) adds
 * microseconds at the end of the call.  Under the clustered cut the blocks
 * form thread-block clusters of c blocks (2 <= c <= 8); each cluster takes
 * units_per_cluster units.  The first c * w of them go whole, w to each
 * block; block r of the cluster streams piece r of each of the others (its
 * tiles [r*T/c, (r+1)*T/c) of T = ceil(N_kv/tile)), and the c parts of such a
 * unit are merged in the cluster's distributed shared memory, each block
 * writing 1/c of the unit's output.  It serves the grouped kernel:
 * G = H_q/H_kv <= 8 with d = 128 (G = 1 included) or G >= 2 with d = 64, one
 * length per row, the contiguous [B, H_kv, N_kv, d] layout.  With
 * num_splits = 0 the planner of sha_decode, sha_decode_bf16, sha_decode_ex
 * and sha_decode_noalloc takes it where a cost model of the call's streaming
 * time and merge tail, with the device's cluster capacities, rates it faster
 * than the other cuts; it needs no workspace.
 *
 * sha_decode_plan_ex -- sha_decode_plan with the clustered cut: the planner's
 * choice on a device with num_sms SMs that holds cluster_capacity[c] clusters
 * of c blocks at once (c = 2..8; entries 0 and 1 ignored; NULL = no clustered
 * cut, as in sha_decode_plan).  Host only, no CUDA call.  Writes plan[0..4]
 * as sha_decode_plan, and
 *   plan[5] = blocks per cluster (0: not the clustered cut)
 *   plan[6] = units per cluster
 *   plan[7] = 0 (tiles cut evenly), 1 (whole units per block),
 *             p >= 2 (each unit in p equal pieces) -- 0 under the clustered cut
 *   plan[8] = whole units per block of a cluster (the clustered cut's w)
 */
sha_status_t sha_decode_plan_ex(int B, int H_q, int H_kv, int N_kv, int d, int top_k,
                                int num_splits, int num_sms, const int32_t cluster_capacity[9],
                                int64_t plan[9]);

/*
 * sha_decode_cluster_capacity -- the current device's cluster capacities for
 * head dim d (64 or 128), as the planner uses them: cluster_capacity[c] =
 * clusters of c blocks of the clustered kernel that fit on the device at once
 * (from cudaOccupancyMaxActiveClusters), c = 2..8; [0] = [1] = 0.  Queried
 * once per device and cached.
 */
sha_status_t sha_decode_cluster_capacity(int d, int32_t cluster_capacity[9]);

/*
 * sha_decode_clustered -- sha_decode_ex with the clustered cut chosen by the
 * caller (for tests and measurements): clusters of `cluster` blocks, each
 * taking `units_per_cluster` units (the last cluster the rest), of which
 * `whole_per_block` go whole to each block and the rest are split into
 * `cluster` pieces.
 *   2 <= cluster <= 8, units_per_cluster >= 1, 0 <= cluster * whole_per_block
 *   <= units_per_cluster, cluster <= ceil(N_kv / tile) when any unit is split,
 *   at most 4096 blocks in all (SHA_ERR_INVALID_ARG otherwise); calls the
 *   clustered kernel cannot serve (above) return SHA_ERR_UNSUPPORTED.
 * Clusters beyond the device's capacity run in further waves.  The result is
 * the same as sha_decode_ex's to within rounding (the parts are merged in
 * block order by the same log-sum-exp arithmetic).  Allocates nothing.
 */
sha_status_t sha_decode_clustered(const void *q, const void *k, const void *v,
                                  const int32_t *batch_head_index, int B, int H_q, int H_kv,
                                  int N_kv, int d, int top_k, float scale, void *out,
                                  sha_dtype_t dtype, int cluster, int units_per_cluster,
                                  int whole_per_block, void *stream);

/*
 * sha_select_heads -- router scores to batch_head_index on the device.
 * Polar Sparsity (papernotes.org summary, "Router 训练"; atlas.scime.ai
 * summary): an attention router scores the heads (or GQA groups) of each
 * token and the top_k are kept.  This call does that selection:
 *   scores           : device pointer, fp32 [B, H] (finite or +-inf; no NaN)
 *   batch_head_index : device pointer, int32 [B, top_k], written in order of
 *                      decreasing score, equal scores by increasing head id
 *   1 <= H <= 256 (SHA_ERR_UNSUPPORTED above), 0 <= top_k <= H.
 * Enqueued on `stream`; a decode enqueued after it on the same stream reads
 * the indices it wrote, with no host synchronisation in between.
 */
sha_status_t sha_select_heads(const float *scores, int B, int H, int top_k,
                              int32_t *batch_head_index, void *stream);

/*
 * ---- Selective GEMM (the MLP half of Polar Sparsity) ----------------------
 * papernotes.org summary, "MLP 层动态稀疏": for a decode batch x [B, d] and the
 * union S_B of the neurons active for any of its rows,
 *     MLP_{S_B}(x) = sigma(x W1[:, S_B]) W2[:, S_B]^T,
 * read only the selected neurons' weights, the index gather fused into the
 * GEMMs.  Weights are neuron-major: W1t = W1^T and W2t = W2^T, each [D, d]
 * row-major, so neuron j's weights are row j.
 */

/* Bytes of workspace sha_mlp_union needs for D neurons. */
size_t sha_mlp_union_workspace_size(int D);

/*
 * sha_mlp_union -- S_B from per-row activity: active [B, D] (uint8, nonzero =
 * active, e.g. a router's thresholded predictions) -> S [D] int32 holding the
 * ids of neurons active in any row in increasing order (first *n_S entries),
 * and n_S (one int32 on the device).  All pointers are device pointers; the
 * union size stays on the device for sha_selective_mlp.  Enqueued on `stream`.
 */
sha_status_t sha_mlp_union(const uint8_t *active, int B, int D, int32_t *S, int32_t *n_S,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace sha_selective_mlp needs (current device); 0 if unsupported. */
size_t sha_selective_mlp_workspace_size(int B, int d, int D);

/*
 * sha_selective_mlp_plan -- how sha_selective_mlp runs a layer of these sizes
 * on a device with num_sms SMs (host only, no CUDA call).  Writes
 *   plan[0] = batch rows the MMA tiles are padded to   (8, 16, 32 or 64)
 *   plan[1] = 1 if the up-projection runs on tcgen05, 0 on warp-level MMAs
 *   plan[2] = 1 if the down-projection runs on tcgen05 as well
 *   plan[3] = rows of the neuron-major activation buffer (D rounded up to 128)
 *   plan[4] = neuron ranges per column chunk of the warp-level down-projection
 *   plan[5] = thread blocks of the warp-level down-projection
 *   plan[6] = output columns per warp-level down-projection item
 *   plan[7] = workspace bytes (what sha_selective_mlp_workspace_size returns on
 *             such a device)
 * plan[4..6] describe the warp-level down-projection, which runs when
 * plan[2] = 0.  The union size is only known on the device, so nothing here
 * depends on it.  Returns SHA_ERR_INVALID_ARG (B, d, D or num_sms below 1, or
 * plan NULL) or SHA_ERR_UNSUPPORTED (B > 64, d not a multiple of 256) as
 * sha_selective_mlp would, SHA_OK otherwise.
 */
sha_status_t sha_selective_mlp_plan(int B, int d, int D, int num_sms, int64_t plan[8]);

/*
 * sha_selective_mlp -- y [B, d] = sigma(x W1t[S]^T) W2t[S] over the first *n_S
 * ids of S (device memory; typically written by sha_mlp_union on the same
 * stream, so no host synchronisation is needed).
 *   x, y      : device, [B, d], fp16 or bf16 (dtype); W1t, W2t: [D, d]
 *   1 <= B <= 64, d a multiple of 256 (SHA_ERR_UNSUPPORTED otherwise)
 *   activation: 1 = ReLU (OPT's MLP), 0 = identity
 *   workspace : device, 256-byte aligned, >= sha_selective_mlp_workspace_size;
 *               scratch only (no contents carried between calls), owned by the
 *               caller; calls that share it must not overlap on the device
 *   x, W1t, W2t, y 16-byte aligned; S, n_S 4-byte aligned (SHA_ERR_MISALIGNED)
 * The hidden activations are rounded to the input dtype before the second
 * product (tensor-core operands); all sums are fp32, and y is rounded to the
 * input dtype.  Partial sums of neuron ranges split across thread blocks are
 * added in a fixed order, so results do not depend on timing.  Batches up to
 * 8 run on warp-level MMAs; larger batches run the up-projection (and from 17
 * rows the down-projection) on tcgen05 with tensor-memory accumulators.  Ids
 * outside [0, D) are bad input: the flag is raised (SHA_ERR_BAD_INDEX from
 * sha_get_device_status), no memory outside the weights is read.
 */
sha_status_t sha_selective_mlp(const void *x, const void *W1t, const void *W2t,
                               const int32_t *S, const int32_t *n_S, int B, int d, int D,
                               int activation, sha_dtype_t dtype, void *y, void *workspace,
                               size_t workspace_bytes, void *stream);

/*
 * sha_get_device_status -- synchronises `stream`, then reads and clears the
 * current device's sticky flags: SHA_ERR_BAD_INDEX if any call since the last
 * read met an out-of-range head id, SHA_ERR_TIMEOUT if a pipeline wait gave
 * up, SHA_OK otherwise (SHA_ERR_LAUNCH if the read itself failed).  After a
 * timeout it also zeroes the arrival counters of the library-owned workspace
 * (sha_decode, _bf16, _varlen, _paged, _strided), enqueued on `stream` and
 * waited for: no call that uses that workspace may then be running on
 * another stream.  A caller-owned workspace (sha_decode_ex) must be zeroed by
 * its owner.
 */
sha_status_t sha_get_device_status(void *stream);

/* Static, human-readable name of a status code. */
const char *sha_status_string(sha_status_t status);

/* The CUDA error string behind the last SHA_ERR_LAUNCH on this thread. */
const char *sha_last_cuda_error(void);

/*
 * sha_copy_bandwidth_probe -- not part of the method: a plain 16-byte
 * vectorised device copy dst[i] = src[i] over `bytes` bytes (a multiple of
 * 16, both pointers 16-byte aligned), grid sized to the SM count.  The
 * benchmark times it in the same process to measure the HBM bandwidth the
 * SHA kernels are compared against.
 */
sha_status_t sha_copy_bandwidth_probe(void *dst, const void *src, size_t bytes,
                                      void *stream);

/*
 * sha_decode_noalloc -- the multi-head (H_q == H_kv) decode above for callers
 * that cannot allocate device memory: for example a serving engine whose
 * allocator has reserved all of HBM for its KV cache and hands out nothing
 * else, or a caller that must not pay cudaMalloc's device-wide
 * synchronisation and latency inside a decode step.  The polar-sparsity
 * pages have no counterpart to this entry point; it exists only for them.
 *
 * It computes what sha_decode_ex computes with the same arguments, but the
 * scratch that merges a head split across thread blocks lives in a fixed
 * device array of SHA_NOALLOC_SCRATCH_BYTES inside this library (each GPU
 * that loads the library holds it until the process exits).  The call makes
 * no cudaMalloc, cudaFree or other allocating call; q, k, v, the index and
 * out are still the caller's device buffers, as for sha_decode.
 *   dtype, num_splits : as for sha_decode_ex.
 * Limits and rules:
 *   - G = H_q / H_kv must be 1 (SHA_ERR_UNSUPPORTED otherwise);
 *   - a call whose scratch (sha_decode_workspace_size for the same sizes and
 *     num_splits) exceeds SHA_NOALLOC_SCRATCH_BYTES is rejected with
 *     SHA_ERR_WORKSPACE before anything is enqueued; with num_splits = 0 this
 *     happens only on GPUs with more than 396 SMs (d = 128);
 *   - the first call on a device looks the array's address up once
 *     (cudaGetSymbolAddress) with that device current and keeps it for the
 *     life of the process; make that first call before any stream capture.
 *     The kept address does not survive cudaDeviceReset: do not call this
 *     entry point on a device after resetting it;
 *   - every call on a device shares the one array, which keeps whatever the
 *     last call left in it.  Each call clears the arrival counters it uses
 *     (a cudaMemsetAsync on `stream`) before its kernel; partial states need
 *     no clearing.  Calls that overlap on the GPU (other streams, other host
 *     threads) race on the array and give wrong results: serialise them.
 */
#define SHA_NOALLOC_SCRATCH_BYTES (512 * 1024)
/* The size of that array in the library as built (SHA_NOALLOC_SCRATCH_BYTES). */
size_t sha_noalloc_scratch_bytes(void);
sha_status_t sha_decode_noalloc(const void *q, const void *k, const void *v,
                                const int32_t *batch_head_index, int B, int H_q,
                                int H_kv, int N_kv, int d, int top_k, float scale,
                                void *out, sha_dtype_t dtype, int num_splits,
                                void *stream);

#ifdef __cplusplus
}
#endif

#endif /* SHA_DECODE_H */
