// sha_tcgen05.cuh -- sm_100a fifth-generation tensor-core building blocks:
// tensor-memory (TMEM) allocation, shared-memory matrix descriptors for
// 128-byte-swizzled K-major operands, the kind::f16 MMA with an fp32
// accumulator in TMEM, commit-to-mbarrier, TMEM -> register loads, and the
// TMA tiled loads that fill the operands (16-byte cp.async: sha_device.cuh).
//
// Operand layout used throughout: a K-major tile of R rows x 64 elements
// (128 bytes per row) is one "K atom"; 8-row groups of an atom are 1024
// bytes apart and the 16-byte chunks of each row are XOR-swizzled by the row
// index modulo 8 (the TMA 128-byte swizzle, a function of the shared-memory
// address, so every atom starts on a 1024-byte boundary).  An MMA with K = 16
// reads 32 bytes of each row: the descriptor of k-step kk of an atom starts
// 32*kk bytes into it.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "sha_device.cuh"

namespace sha {

// ---- tensor memory -----------------------------------------------------------

// Allocate `cols` TMEM columns (a power of two >= 32) for this CTA; the base
// address is written to shared memory at `dst`.  Executed by one whole warp.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t cols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst)),
                 "r"(cols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

// Free what tmem_alloc returned.  Executed by one whole warp.
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols)
                 : "memory");
}

// Order tcgen05 operations around a thread synchronisation (a barrier or an
// mbarrier wait).
__device__ __forceinline__ void tc_fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- descriptors -------------------------------------------------------------

// Shared-memory matrix descriptor of a K-major, 128-byte-swizzled operand
// starting at shared address `addr`: 8-row groups 1024 bytes apart (stride
// byte offset), leading byte offset unused by swizzled K-major layouts (1),
// descriptor version 1, base offset 0 (atoms are 1024-byte aligned), layout
// type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t umma_desc_k_sw128(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);          // start address, 16-byte units
    d |= (uint64_t)1u << 16;                          // leading byte offset (16 bytes)
    d |= (uint64_t)(1024u >> 4) << 32;                // stride byte offset
    d |= (uint64_t)1u << 46;                          // descriptor version
    d |= (uint64_t)2u << 61;                          // 128-byte swizzle
    return d;
}

// The same for a 64-byte swizzle: 64-byte rows (32 elements), 8-row groups
// 512 bytes apart, layout type 4.
__device__ __forceinline__ uint64_t umma_desc_k_sw64(uint32_t addr)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(512u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)4u << 61;
    return d;
}

// Shared-memory matrix descriptor of an MN-major, 128-byte-swizzled operand:
// 64-element MN blocks `lbo` bytes apart (leading byte offset), 8-row K groups
// `sbo` bytes apart (stride byte offset); each 1024-byte atom holds 8 K rows of
// 64 MN elements, chunks XOR-swizzled by the K row.
__device__ __forceinline__ uint64_t umma_desc_mn_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((addr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::f16 with fp32 accumulation, both operands
// of the same type (fp16, or bf16 when `bf16`), M x N; A and B K-major unless
// `a_mn` / `b_mn` (MN-major).
__host__ __device__ constexpr uint32_t umma_idesc_f16(bool bf16, int M, int N, bool a_mn = false,
                                                      bool b_mn = false)
{
    return (1u << 4)                                  // accumulator format: f32
           | ((bf16 ? 1u : 0u) << 7)                  // A format
           | ((bf16 ? 1u : 0u) << 10)                 // B format
           | ((a_mn ? 1u : 0u) << 15)                 // A major-ness
           | ((b_mn ? 1u : 0u) << 16)                 // B major-ness
           | ((uint32_t)(N >> 3) << 17)               // N / 8
           | ((uint32_t)(M >> 4) << 24);              // M / 16
}

// ---- MMA -----------------------------------------------------------------------

// D[tmem] (+)= A[smem] * B[smem]^T, M x N x 16; `accumulate` = 0 overwrites D.
// Issued by one thread.
__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every MMA this thread has issued so far is done.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

// ---- TMEM -> registers -----------------------------------------------------------

// 16 consecutive 32-bit columns of this thread's TMEM lane (32x32b shape: a
// warp reads lanes 32*(warp%4) .. +31).  Complete with tmem_ld_wait().
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait()
{
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---- TMA loads -----------------------------------------------------------------

// One box of a 2-D tensor map at element coordinates (x, y).
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y,
                                            uint64_t *bar, uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

}  // namespace sha
