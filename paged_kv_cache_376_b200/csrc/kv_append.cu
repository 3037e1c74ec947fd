// KV append: scatter each new token's K and V rows into their page slots.
//
// "tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec. "推理流程：从Prefill到
// Decode": every generated token's K,V are computed and appended to the cache;
// "Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎", sec. "内存池管理": a
// page holds page_size token rows of num_kv_heads x head_dim bf16 values.
// Slot s names row s of the pool viewed as [num_pages * page_size][row]
// (page s / page_size, offset s % page_size).  Negative slots are padding.
//
// The copy is bit-exact: one thread moves one 16-byte vector, so a token row
// of 1 KB (8 heads x 64 x bf16) is 64 fully coalesced vectors per tensor.
// The grid is a multiple of the SM count and strides over the work.  A
// second kernel rotates K by RoPE on the way (tv_kv_append_rope).
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4* __restrict__ k_new,
                     const uint4* __restrict__ v_new,
                     const int32_t* __restrict__ slot_mapping,
                     int64_t num_tokens, uint4* __restrict__ k_pool,
                     uint4* __restrict__ v_pool, int64_t num_slots,
                     int row_vecs, uint32_t* err) {
  const int64_t per_token = 2 * (int64_t)row_vecs;  // K vectors then V
  const int64_t total = num_tokens * per_token;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_token;
    const int r = (int)(i - t * per_token);
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) flag_error(err, DEVERR_BAD_SLOT);
      continue;
    }
    if (r < row_vecs) {
      k_pool[slot * row_vecs + r] = k_new[t * row_vecs + r];
    } else {
      const int c = r - row_vecs;
      v_pool[slot * row_vecs + c] = v_new[t * row_vecs + c];
    }
  }
}

// RoPE variant ("tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec. "Llama
// 3.2 1B架构拆解": the position enters K by a rotation; V is copied as is).
// A head of a K row is 8 vectors of 8 dimensions; vector u < 4 pairs with
// vector u + 4 (dimensions i and i + 32), so one work item moves such a pair
// (rotated) and the 8 V vectors are 8 more items: 12 items per head.
__global__ void __launch_bounds__(256)
    kv_append_rope_kernel(const uint4* __restrict__ k_new,
                          const uint4* __restrict__ v_new,
                          const int32_t* __restrict__ slot_mapping,
                          const int32_t* __restrict__ positions,
                          int64_t num_tokens, uint4* __restrict__ k_pool,
                          uint4* __restrict__ v_pool, int64_t num_slots,
                          int num_kv_heads, const float* __restrict__ cos_sin,
                          int max_position, uint32_t* err) {
  const int row_vecs = num_kv_heads * 8;
  const int64_t per_token = 12 * (int64_t)num_kv_heads;
  const int64_t total = num_tokens * per_token;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = i / per_token;
    const int r = (int)(i - t * per_token);
    const int h = r / 12, u = r - 12 * h;
    const int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    if (slot >= num_slots) {
      if (r == 0) flag_error(err, DEVERR_BAD_SLOT);
      continue;
    }
    const int64_t src = t * row_vecs + h * 8;
    const int64_t dst = slot * row_vecs + h * 8;
    if (u < 4) {
      uint4 lo = k_new[src + u], hi = k_new[src + u + 4];
      const int pos = positions[t];
      if (pos >= 0 && pos < max_position) {
        float c8[8], s8[8];
        rope_load8(cos_sin, pos, 8 * u, c8, s8);
        rope_rotate8(lo, hi, c8, s8);
      } else if (r == 0) {
        flag_error(err, DEVERR_BAD_POSITION);
      }
      k_pool[dst + u] = lo;
      k_pool[dst + u + 4] = hi;
    } else {
      v_pool[dst + u - 4] = v_new[src + u - 4];
    }
  }
}

}  // namespace

cudaError_t launch_kv_append_rope(const void* k_new, const void* v_new,
                                  const int32_t* slot_mapping,
                                  const int32_t* positions, int64_t num_tokens,
                                  void* k_pool, void* v_pool,
                                  int64_t num_slots, int num_kv_heads,
                                  const float* rope_cos_sin,
                                  int rope_max_position, uint32_t* err,
                                  cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int64_t total = num_tokens * 12 * num_kv_heads;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  const int blocks = (int)(want < cap ? want : cap);
  kv_append_rope_kernel<<<blocks, 256, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      slot_mapping, positions, num_tokens, static_cast<uint4*>(k_pool),
      static_cast<uint4*>(v_pool), num_slots, num_kv_heads, rope_cos_sin,
      rope_max_position, err);
  return cudaGetLastError();
}

cudaError_t launch_kv_append(const void* k_new, const void* v_new,
                             const int32_t* slot_mapping, int64_t num_tokens,
                             void* k_pool, void* v_pool, int64_t num_slots,
                             int row_bytes, uint32_t* err,
                             cudaStream_t stream) {
  if (num_tokens == 0) return cudaSuccess;
  const int row_vecs = row_bytes / 16;
  const int64_t total = num_tokens * 2 * row_vecs;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t want = (total + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  const int blocks = (int)(want < cap ? want : cap);
  kv_append_kernel<<<blocks, 256, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new),
      slot_mapping, num_tokens, static_cast<uint4*>(k_pool),
      static_cast<uint4*>(v_pool), num_slots, row_vecs, err);
  return cudaGetLastError();
}

}  // namespace tv
