// Lane-group helpers shared by the two decode kernels (paged_decode.cu and
// paged_decode_balanced.cu).
#pragma once

#include "tv_device.cuh"

namespace tv {

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
