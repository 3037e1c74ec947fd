// Warp-level helpers of the two decode kernels (paged_decode.cu and
// paged_decode_balanced.cu).
#pragma once

#include "tv_device.cuh"

namespace tv {

// ---- warp-level bf16 tensor-core products (decode) ---------------------------
// Four 8x8 b16 matrices from shared memory: lane t gives the address of row
// t & 7 of matrix t >> 3; register j receives this lane's two elements of
// matrix j (row lane >> 2, columns 2 (lane & 3), +1), or with .trans those of
// its transpose.  The "memory" clobber keeps them after the generic stores
// (appended rows, zeroed tails) that precede them.
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(addr)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr,
                                              uint32_t (&r)[4]) {
  asm volatile(
      "ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
      : "r"(addr)
      : "memory");
}
// d += A (16x16, row-major fragments) * B (16x8, column fragments), bf16
// inputs, fp32 accumulation.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4],
                                               const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

}  // namespace tv
