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
// 16-byte loads.
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

// All NT consumer threads of the merging block call this together.
// stage: shared scratch of at least 3 * kMaxMergeParts * G floats, free for use.
template <typename T, int D, int NT>
__device__ __forceinline__ void merge_parts(const float *__restrict__ slots, int slot_floats,
                                            int first, int first_slot, int parts, int G,
                                            T *__restrict__ out_rows, float *stage, int tid)
{
    float *s_m = stage;
    float *s_l = stage + parts * G;
    float *s_w = stage + 2 * parts * G;
    for (int t = tid; t < parts * G; t += NT) {
        const int i = t / G, row = t - i * G;
        const float *sl = slots + (size_t)merge_slot(first, first_slot, i) * slot_floats;
        s_m[t] = __ldcg(sl + G * D + row);
        s_l[t] = __ldcg(sl + G * D + G + row);
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
    for (int e = tid * 4; e < G * D; e += NT * 4) {
        const int row = e / D;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
        for (int i = 0; i < parts; ++i) {
            const float *sl = slots + (size_t)merge_slot(first, first_slot, i) * slot_floats;
            const float4 x = __ldcg(reinterpret_cast<const float4 *>(sl + e));
            const float w = s_w[i * G + row];
            acc.x = fmaf(w, x.x, acc.x);
            acc.y = fmaf(w, x.y, acc.y);
            acc.z = fmaf(w, x.z, acc.z);
            acc.w = fmaf(w, x.w, acc.w);
        }
        out_rows[e + 0] = Elem<T>::from_float(acc.x);
        out_rows[e + 1] = Elem<T>::from_float(acc.y);
        out_rows[e + 2] = Elem<T>::from_float(acc.z);
        out_rows[e + 3] = Elem<T>::from_float(acc.w);
    }
    named_barrier(1, NT);   // the staging area is reused by the caller's next unit
}

}  // namespace sha
