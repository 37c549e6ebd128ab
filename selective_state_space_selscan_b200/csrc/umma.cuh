// umma.cuh -- 5th-generation tensor core (tcgen05 / UMMA) helpers for sm_100a:
// shared-memory matrix descriptors for 128-byte-swizzled bf16 tiles, the
// instruction descriptor for bf16 x bf16 -> fp32, MMA issue and commit, and
// tensor-memory (TMEM) allocation, loads and stores.
//
// Tile conventions (bf16, 128-byte swizzle, base 1024-byte aligned):
//  * K-major tile [R][K]: rows r of 64-element (128 B) slabs; slab s holds
//    k in [64 s, 64 s + 64) for all R rows (R * 128 bytes per slab).  Within
//    a slab, element (r, k) sits at r*128 + ((2k/16) ^ (r%8))*16 + (2k%16).
//    This is exactly what a bulk tensor copy with a {64, R} box and 128-byte
//    swizzle writes.
//  * MN-major tile [K][MN]: K rows, the MN dimension contiguous, split into
//    64-element blocks of K*128 bytes each; element (k, mn) of block b sits
//    at b*K*128 + k*128 + ((2mn'/16) ^ (k%8))*16 + (2mn'%16), mn' = mn - 64b.
#pragma once

#include <cstdint>

#include "ptx.cuh"

namespace selscan {

// byte offset of element (row, col) inside a 128-byte-swizzled tile whose
// rows are 128 bytes (64 bf16) long
__host__ __device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t col_bf16)
{
    const uint32_t byte = col_bf16 * 2u;
    return row * 128u + ((((byte >> 4) ^ (row & 7u))) << 4) + (byte & 15u);
}

// Shared-memory matrix descriptor (sm_100 layout): start address, leading
// and stride byte offsets in 16-byte units, version 1, 128-byte swizzle.
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_byte_addr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= uint64_t((smem_byte_addr >> 4) & 0x3FFFu);
    d |= uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= uint64_t(1) << 46;  // descriptor version for sm_100
    d |= uint64_t(2) << 61;  // SWIZZLE_128B
    return d;
}

// Descriptor of the K-step `kk` (16 bf16 of K) of a K-major tile with R rows.
__device__ __forceinline__ uint64_t umma_desc_kmajor(uint32_t tile_addr, int R, int kk)
{
    const uint32_t k0 = uint32_t(kk) * 16u;
    const uint32_t addr = tile_addr + (k0 >> 6) * uint32_t(R) * 128u + (k0 & 63u) * 2u;
    return umma_desc_sw128(addr, 16u, 1024u);
}

// Descriptor of the K-step `kk` (16 rows) of an MN-major tile with Krows rows.
__device__ __forceinline__ uint64_t umma_desc_mnmajor(uint32_t tile_addr, int Krows, int kk)
{
    const uint32_t addr = tile_addr + uint32_t(kk) * 16u * 128u;
    return umma_desc_sw128(addr, uint32_t(Krows) * 128u, 1024u);
}

// Instruction descriptor: kind::f16 with bf16 A/B, fp32 accumulator.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn_major,
                                                       bool b_mn_major)
{
    return (1u << 4)                          // D format: f32
           | (1u << 7) | (1u << 10)           // A, B format: bf16
           | (uint32_t(a_mn_major) << 15) | (uint32_t(b_mn_major) << 16)
           | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// D[tmem] (+)= A * B^T for one K-step; issued by a single thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate)
{
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "setp.ne.b32 p, %4, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
                 :: "r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
                 : "memory");
}

// Arrive on `bar` once every MMA issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
                 :: "r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void tmem_fence_before_sync()
{
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_fence_after_sync()
{
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Allocation by one full warp; the TMEM base address is written to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_addr(dst)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(taddr), "r"(ncols) : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane
// (warp's lane base + i), columns [col, col+16).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16])
{
    uint32_t r[16];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i)
        v[i] = __uint_as_float(r[i]);
}

// Two 32x32b.x16 loads in flight, one wait: v0 from column address a0, v1
// from a1 (same lane rules as tmem_ld16).
__device__ __forceinline__ void tmem_ld16x2(uint32_t a0, float (&v0)[16], uint32_t a1,
                                            float (&v1)[16])
{
    uint32_t r[32];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32];\n\t"
                 "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
                 "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33];\n\t"
                 "tcgen05.wait::ld.sync.aligned;"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]),
                   "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
                   "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
                   "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]),
                   "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(a0), "r"(a1)
                 : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        v0[i] = __uint_as_float(r[i]);
        v1[i] = __uint_as_float(r[16 + i]);
    }
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16])
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 "
                 "[%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
                 :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])),
                    "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
                    "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                    "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
                    "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])),
                    "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
                    "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
                    "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace selscan
