// ptx_bs.cuh -- inline-PTX wrappers of the block-scaled MMA path (sm_100a):
// the kind::mxf8f6f4.block_scale instruction and its descriptor, the shared
// memory -> TMEM copy of scale factors (tcgen05.cp) and its descriptor, and a
// register fence for 32-column TMEM loads.  Single instructions,
// as in ptx.cuh; used by gemm_bs_kernel.cuh only.
#pragma once

#include <cstdint>
#include "ptx.cuh"

namespace fp8bs {

// ------------------------------------------------------------------ block-scaled MMA
// kind::mxf8f6f4.block_scale (one scale factor per 32 consecutive K of each
// row of A and of B^T, UE8M0: an 8-bit biased exponent, the value 2^(e-127)).
// The instruction descriptor of this kind has no D-format field (D is F32):
// bits [4,6) the B scale-factor id, [7,10) / [10,13) A / B format (E4M3 = 0),
// 15 / 16 A / B major (K = 0), [17,23) N >> 3, bit 23 the scale type
// (1 = UE8M0), [24,29) M >> 4, [29,31) the A scale-factor id.  The id selects
// the byte of each 32-bit TMEM scale-factor word that this MMA uses.
__host__ __device__ constexpr uint32_t idesc_e4m3_bs(uint32_t M, uint32_t N, uint32_t sf_id)
{
    return (sf_id << 4)
         | (0u << 7) | (0u << 10)
         | (0u << 15) | (0u << 16)
         | ((N >> 3) << 17)
         | (1u << 23)
         | ((M >> 4) << 24)
         | (sf_id << 29);
}

// D[tmem] (+)= (A[smem] . B[smem]^T) with each product scaled by its rows'
// scale factors, read from TMEM at sfa / sfb (the scale-factor byte id is
// carried in bits [30,32) of these addresses as well as in the descriptor).
__device__ __forceinline__ void umma_f8_bs(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                           uint32_t sfa, uint32_t sfb, uint32_t accum)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum), "r"(sfa), "r"(sfb)
        : "memory");
}

// Copies 32 rows x 128 bits from shared memory (described by `sdesc`) into
// TMEM lanes 0..31 of every lane quarter (the same rows in all four), columns
// [col, col+4) of `taddr`.  Issued by one thread; ordered before the same
// thread's later tcgen05.mma (a pipelined pair), and tracked by its
// tcgen05.commit like an MMA.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of the source of tcgen05.cp 32x128b: 32 rows of 16
// bytes stored one after another, i.e. the K-major layout without swizzle
// whose core matrices (8 rows x 16 bytes, 128 contiguous bytes) are 128 bytes
// apart in the row direction (stride byte offset); one core matrix wide, so
// the leading byte offset is unused; descriptor version 1, layout code 0 (no
// swizzle).
__host__ __device__ __forceinline__ uint64_t smem_desc_cp_rows16(uint32_t saddr)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                           // leading byte offset (16 B, unused)
    d |= (uint64_t)(128u >> 4) << 32;                  // stride byte offset
    d |= (uint64_t)1u << 46;                           // version
    return d;
}

// 16-byte shared-memory store.
__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// Makes this thread's generic-proxy writes to shared memory visible to the
// async proxy (TMA, tcgen05) once ordered by a barrier.
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// reg_after_wait for the 32 destination registers of a 32-column load.
__device__ __forceinline__ void reg_after_wait32(uint32_t (&r)[32])
{
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                   "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]),
                   "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31]));
}

}  // namespace fp8bs
