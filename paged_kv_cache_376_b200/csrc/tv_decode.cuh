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

// ---- reduce-scatter over the 8 lanes of a decode lane group ----------------
// The decode kernels split a key row over 8 lanes (bits 0-2 of the lane
// index, `chk`) and each lane forms G partial dot products, one per query
// head of the group.  Summing them over the 8 lanes and leaving one head per
// lane takes log2(G) halving steps plus plain all-reduce steps.  A lane keeps
// head (position ^ rs_mask<G>(chk)) at `position`; then at every halving
// step the half it keeps is positions [0, n/2) and the half it sends is
// [n/2, n) on both partners, because the two masks differ by exactly n/2 --
// no lane-dependent selects.  Position 0 ends with the full sum of head
// rs_mask<G>(chk), which equals chk >> log2(8 / G).
template <int G>
__device__ __forceinline__ int rs_mask(int chk) {
  int m = 0, n = G;
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) {
    if (n > 1) {
      if (chk & off) m ^= n / 2;
      n >>= 1;
    }
  }
  return m;
}
template <int G>
__device__ __forceinline__ float reduce_scatter8(float (&part)[G]) {
  int n = G;
#pragma unroll
  for (int off = 4; off >= 1; off >>= 1) {
    if (n > 1) {
#pragma unroll
      for (int h = 0; h < G / 2; ++h)
        if (h < n / 2)
          part[h] += __shfl_xor_sync(0xffffffffu, part[h + n / 2], off);
      n >>= 1;
    } else {
      part[0] += __shfl_xor_sync(0xffffffffu, part[0], off);
    }
  }
  return part[0];
}

}  // namespace tv
