// sha_merge.cuh -- finishing a unit whose key range was split across blocks.
//
// Each block that held part of unit u left a partial state in its slot:
// O_s (G rows x d, unnormalised, fp32), m_s (row maxima, log2 units) and
// l_s (row sums).  The last block to finish merges them with the
// log-sum-exp rule
//     M = max_s m_s,   w_s = 2^(m_s - M) / sum_s 2^(m_s - M) l_s,
//     O = sum_s w_s O_s,
// visiting the parts in block order so the result does not depend on which
// block came last.  Loads are issued so that their latencies overlap: all
// (m_s, l_s) first, staged in shared memory, then the O rows as independent
// 16-byte loads.  The parts are read from the slots, from copies that a
// block brought into its own shared memory ahead of time (sha_lookahead.cuh),
// or, under the clustered cut, from slices of them that the blocks of a
// thread-block cluster stored into each other's shared memory.
#pragma once

#include "sha_device.cuh"
#include "sha_schedule.cuh"

namespace sha {

// Upper bound on the blocks sharing one unit; the host planner keeps every
// call within it.  Bounds the shared staging below (3 * 64 * G floats).
constexpr int kMaxMergeParts = 64;

// Slot of the i-th part of unit u (parts are blocks first, first+1, ...):
// blocks after the first start inside u, so u is their first unit.
__device__ __forceinline__ int merge_slot(int first, int first_slot, int i)
{
    return i == 0 ? first_slot : 2 * (first + i);
}

// Where the parts of a unit are read from.  o(i, e): element e of part i's
// unnormalised O rows (G x D, row-major); m(i, row), l(i, row): its running
// maximum and sum of that row.
// GlobalParts: the blocks' slots in the workspace (read through L2, never a
// stale L1 line), a slot holding O (G x D), then m (G), then l (G).
// SharedParts: copies of slots in this block's shared memory, part i at
// parts + i * stride.
// StagedParts (clustered cut): only elements [e0, e0 + slice) of each part,
// stored by the cluster's blocks into this block's shared memory; part i at
// stage(i), its O elements first, then (m, l) pairs of the rows from offset
// `slice` on.
struct GlobalParts {
    const float *slots;
    int slot_floats, first, first_slot, ml_offset;
    static constexpr bool kShared = false;
    __device__ __forceinline__ const float *base(int i) const
    {
        return slots + (size_t)merge_slot(first, first_slot, i) * slot_floats;
    }
    __device__ __forceinline__ const float *o(int i, int e) const { return base(i) + e; }
    __device__ __forceinline__ const float *m(int i, int row) const
    {
        return base(i) + ml_offset + row;
    }
    __device__ __forceinline__ const float *l(int i, int row, int G) const
    {
        return base(i) + ml_offset + G + row;
    }
};
struct SharedParts {
    const float *parts;
    int stride, ml_offset;
    static constexpr bool kShared = true;
    __device__ __forceinline__ const float *o(int i, int e) const { return parts + i * stride + e; }
    __device__ __forceinline__ const float *m(int i, int row) const
    {
        return parts + i * stride + ml_offset + row;
    }
    __device__ __forceinline__ const float *l(int i, int row, int G) const
    {
        return parts + i * stride + ml_offset + G + row;
    }
};
template <class Stage>
struct StagedParts {
    Stage stage;      // stage(i): part i's staging area in this block
    int e0, slice;
    static constexpr bool kShared = true;
    __device__ __forceinline__ const float *o(int i, int e) const { return stage(i) + (e - e0); }
    __device__ __forceinline__ const float *m(int i, int row) const
    {
        return stage(i) + slice + 2 * row;
    }
    __device__ __forceinline__ const float *l(int i, int row, int) const
    {
        return stage(i) + slice + 2 * row + 1;
    }
};

template <bool kShared>
__device__ __forceinline__ float load_part(const float *p)
{
    if constexpr (kShared) return *p;
    else return __ldcg(p);
}
template <bool kShared>
__device__ __forceinline__ float4 load_part4(const float *p)
{
    if constexpr (kShared) return *reinterpret_cast<const float4 *>(p);
    else return __ldcg(reinterpret_cast<const float4 *>(p));
}

// All NT consumer threads of the merging block call this together.  The
// arithmetic, and its order, is the same wherever the parts are read from, so
// a unit merged from shared-memory copies is bit-identical to one merged from
// the slots.  stage: shared scratch of at least 3 * kMaxMergeParts * G floats,
// free for use.  Only output elements [e_begin, e_end) of the G x D rows are
// written (both multiples of 4; e_end < 0 means all), so several blocks can
// share the work.
template <typename T, int D, int NT, typename Parts>
__device__ __forceinline__ void merge_parts(const Parts &part, int parts, int G,
                                            T *__restrict__ out_rows, float *stage, int tid,
                                            int e_begin = 0, int e_end = -1)
{
    if (e_end < 0) e_end = G * D;
    float *s_m = stage;
    float *s_l = stage + parts * G;
    float *s_w = stage + 2 * parts * G;
    for (int t = tid; t < parts * G; t += NT) {
        const int i = t / G, row = t - i * G;
        s_m[t] = load_part<Parts::kShared>(part.m(i, row));
        s_l[t] = load_part<Parts::kShared>(part.l(i, row, G));
    }
    named_barrier(1, NT);
    for (int row = tid; row < G; row += NT) {
        float M = -INFINITY;
        for (int i = 0; i < parts; ++i) M = fmaxf(M, s_m[i * G + row]);
        float L = 0.f;
        for (int i = 0; i < parts; ++i) L = fmaf(exp2f(s_m[i * G + row] - M), s_l[i * G + row], L);
        const float inv = 1.f / L;
        for (int i = 0; i < parts; ++i) s_w[i * G + row] = exp2f(s_m[i * G + row] - M) * inv;
    }
    named_barrier(1, NT);
    for (int e = e_begin + tid * 4; e < e_end; e += NT * 4) {
        const int row = e / D;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = 0; i < parts; ++i) {
            const float4 x = load_part4<Parts::kShared>(part.o(i, e));
            const float w = s_w[i * G + row];
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        // four elements in one 8-byte store (rows of D 16-bit elements, D % 4 == 0)
        *reinterpret_cast<uint2 *>(out_rows + e) =
            make_uint2(pack2<T>(acc.x, acc.y), pack2<T>(acc.z, acc.w));
    }
    named_barrier(1, NT);   // the staging area is reused by the caller's next unit
}

}  // namespace sha
