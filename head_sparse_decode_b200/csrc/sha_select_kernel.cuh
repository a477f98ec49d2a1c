// sha_select_kernel.cuh -- router scores -> batch_head_index on the device.
//
// The step just before selective head decode in Polar Sparsity: the attention
// router (one fully connected layer; papernotes.org summary, "Router 训练")
// scores every head of every batch row and the top_k heads are kept.  This
// kernel turns scores [B, H] (fp32) into batch_head_index [B, top_k] (int32)
// without a host round trip, so the decode that follows on the same stream
// reads indices produced on the device.
//
// Order within a row: decreasing score, equal scores by increasing head id.
// One warp per row.  Every head's rank -- the number of heads that beat it --
// is counted against all H scores broadcast by shuffles; a head whose rank is
// below top_k is written at that rank.  H <= 256 (8 scores per lane).
#pragma once

#include "sha_device.cuh"

namespace sha {

constexpr int kSelectMaxHeads = 256;
constexpr int kSelectRowsPerBlock = 8;

__global__ void __launch_bounds__(kSelectRowsPerBlock * 32)
    sha_select_heads_kernel(const float *__restrict__ scores, int B, int H, int top_k,
                            int32_t *__restrict__ batch_head_index)
{
    constexpr int kPer = kSelectMaxHeads / 32;
    const unsigned FULL = 0xffffffffu;
    const int lane = threadIdx.x & 31;
    const int row = blockIdx.x * kSelectRowsPerBlock + (threadIdx.x >> 5);
    pdl_wait();                 // the scores may come from the previous kernel
    pdl_launch_dependents();
    if (row >= B) return;

    const float *s = scores + (size_t)row * H;
    float v[kPer];
    int rank[kPer];
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int h = lane + 32 * j;
        v[j] = h < H ? s[h] : 0.f;
        rank[j] = 0;
    }
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        if (32 * i >= H) break;                   // warp-uniform
        for (int l = 0; l < 32; ++l) {
            const int src = 32 * i + l;
            if (src >= H) break;                  // warp-uniform
            const float x = __shfl_sync(FULL, v[i], l);
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int h = lane + 32 * j;
                rank[j] += (x > v[j] || (x == v[j] && src < h)) ? 1 : 0;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPer; ++j) {
        const int h = lane + 32 * j;
        if (h < H && rank[j] < top_k) batch_head_index[(size_t)row * top_k + rank[j]] = h;
    }
}

}  // namespace sha
