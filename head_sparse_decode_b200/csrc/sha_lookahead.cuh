// sha_lookahead.cuh -- finishing a block's last split unit on chip.
//
// Under the even tile cut a unit that straddles blocks c and c+1 is finished
// early by c+1, whose range starts with the unit's tail, and late by c, whose
// range ends with the unit's head.  So the last thing most blocks do is the
// head of a split unit whose other parts were done long before.  Through the
// slots that still costs four dependent trips to memory at the very end of
// the call: write the partial state, fence, count the arrival, read the
// other parts back (the merge of the log-sum-exp rule, sha_merge.cuh).
//
// A scout warp takes those trips off the critical path.  It polls the unit's
// arrival counter while the block streams its last segment.  Once every
// other part has arrived, it claims the unit for the on-chip path and
// bulk-copies their partial states into shared memory.  At the end of the
// segment the block merges them with its own state, which never leaves the
// chip, and writes the output.  The claim is one compare-and-swap on a shared
// word: if the consumers reach the end of the segment first, they claim it
// for the slots instead and carry on at once.  No block ever waits for
// another: the scout only looks.
//
// Exactly one block merges either way.  A block that takes the on-chip path
// has seen every other part's arrival and adds none of its own, so no other
// block can count itself last; it then clears the counter for the next call.
// The merge arithmetic is the same on both paths (merge_parts), so the result
// does not depend on which one ran.
//
// The scout pays only where blocks end with the head of a unit whose other
// parts were done early, which is how the even cut splits units no longer
// than a few blocks' ranges; the kernels come in two builds and the host
// planner picks (kLook).
#pragma once

#include "sha_device.cuh"
#include "sha_merge.cuh"
#include "sha_walk.cuh"

// Build-time switch: 0 never launches the scout builds (every split unit
// goes through the slots).
#ifndef SHA_LOOKAHEAD
#define SHA_LOOKAHEAD 1
#endif

namespace sha {

// Shared control words of a block (after the abort and merge flags).
enum : int {
    kFlagClaim = 2,    // the last unit's path: 0 open, 1 on chip (scout), 2 slots (consumers)
    kFlagOnChip = 3    // the consumers' reading of the claim, taken once
};

// If `seg`, a block's last segment, is the head of a unit held by blocks
// first..last (unit_parts) and at most max_partners other blocks hold the
// rest: the number of parts of the unit.  Else 0.
__device__ __forceinline__ int lookahead_parts(const Seg &seg, int first, int last,
                                               int max_partners)
{
    if (seg.whole || seg.first_tile != 0 || max_partners <= 0) return 0;
    const int parts = last - first + 1;
    return (parts >= 2 && parts - 1 <= max_partners) ? parts : 0;
}

__device__ __forceinline__ int load_relaxed_gpu(const int *p)
{
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acquire_gpu()
{
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// Orders this thread's earlier generic-proxy accesses of global memory (and
// what they synchronised with) before its later bulk copies from it.
__device__ __forceinline__ void fence_proxy_async_global()
{
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// One lane of the scout warp runs this.  walk: the block's own walk (copied);
// parts 1.. of the unit go to dst + i * stride floats, each 16-byte aligned;
// copy_bytes: the bytes of a part (a 16-byte multiple within a slot).
// Returns once the claim is taken and no copy is in flight.
template <class Walk>
__device__ void lookahead_scout(Walk wk, const Schedule &S, int max_partners,
                                const int *counters, const float *slots, int slot_floats,
                                uint32_t copy_bytes, float *dst, int stride,
                                volatile int *flags, uint64_t *bar)
{
    Seg seg, last_seg;
    bool any = false;
    while (wk.next(seg)) {
        last_seg = seg;
        any = true;
    }
    if (!any || last_seg.whole || last_seg.first_tile != 0) return;
    int first, last, first_slot;
    unit_parts(S, last_seg, first, last, first_slot);
    const int parts = lookahead_parts(last_seg, first, last, max_partners);
    if (parts == 0) return;

    int *claim = const_cast<int *>(flags + kFlagClaim);
    bool copied = false;
    const unsigned long long t0 = global_timer_ns();
    // the consumers always take the claim by the time they leave
    while (flags[kFlagClaim] == 0 && global_timer_ns() - t0 <= wait_limit_ns()) {
        if (load_relaxed_gpu(counters + first) == parts - 1) {
            if (atomicCAS(claim, 0, 1) == 0) {
                fence_acquire_gpu();          // the other parts' slots, as they arrived
                fence_proxy_async_global();   // ... are what the bulk copies read
                const uint64_t policy = l2_policy_evict_first();
                mbar_arrive_expect_tx(bar, (uint32_t)(parts - 1) * copy_bytes);
                for (int i = 1; i < parts; ++i)
                    bulk_copy_g2s(dst + (size_t)i * stride,
                                  slots + (size_t)merge_slot(first, first_slot, i) * slot_floats,
                                  copy_bytes, bar, policy);
                copied = true;
            }
            break;
        }
        __nanosleep(500);
    }
    if (copied && !mbar_wait_drain(bar, 0)) atomicOr(&g_sha_status, kStatusTimeout);
}

// The consumers' side (one thread).  At the end of the block's last segment:
// true if the scout has claimed the unit for the on-chip path (its copies
// are then on the way), else the consumers take it for the slots.  Also
// called as the consumers leave, so the scout never outlives them.
__device__ __forceinline__ bool lookahead_claim(volatile int *flags)
{
    return atomicCAS(const_cast<int *>(flags + kFlagClaim), 0, 2) == 1;
}

}  // namespace sha
