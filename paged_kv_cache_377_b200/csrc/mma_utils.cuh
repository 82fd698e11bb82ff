// mma_utils.cuh -- shared-memory tiles of the paged pools and the mma.sync
// building blocks shared by the decode and the multi-query kernels.
#pragma once

#include <stdint.h>

namespace pkv {

// Shared address of 16-byte chunk c (0 <= c < D/8) of row t of a K or V tile.
// A tile holds D/64 column halves of [BS rows][128 bytes], each loaded by one
// TMA box with SWIZZLE_128B: the chunk index inside a 128-byte row is XORed
// with the row index mod 8, so 8 consecutive rows at one chunk hit 8 distinct
// bank groups.
template <int BS>
__device__ __forceinline__ uint32_t tile_addr(uint32_t tile, int t, int c) {
    return tile + static_cast<uint32_t>((c >> 3) * (BS * 128) + t * 128) +
           (static_cast<uint32_t>((c & 7) ^ (t & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// d += a (16x16 bf16, row) * b (16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts16(uint32_t addr, uint16_t v) {
    asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

}  // namespace pkv
