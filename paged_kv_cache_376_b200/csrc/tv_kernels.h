// Internal launch interface between the C ABI (tv_api.cu) and the kernels.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace tv {

struct DecodeArgs {
  __nv_bfloat16* out;            // [B][Hq][D]            (unsplit)
  float* partial_out;            // [B][Hq][maxP][D]      (split)
  float* partial_lse;            // [B][Hq][maxP]         (split)
  const __nv_bfloat16* q;        // [B][Hq][D]
  const __nv_bfloat16* k_new;    // [B][Hkv][D] (fused append; else null)
  const __nv_bfloat16* v_new;
  __nv_bfloat16* k_pool_w;       // pools, written by the fused append
  __nv_bfloat16* v_pool_w;
  const int32_t* block_tables;   // [B][max_blocks_per_seq]
  const int32_t* context_lens;   // [B]
  // nullable; grown[s] == 0 makes sequence s idle (no append, zero output):
  // the pool's marks of the sequences whose context the step's slot
  // reservation grew (tv_decode_step only)
  const int32_t* grown;
  uint32_t* err;                 // nullable
  // fused append only: RoPE of the new K row at position ctx-1 (nullable)
  const float* rope_cos_sin;     // [rope_max_position][2][32] fp32
  int rope_max_position;
  int max_blocks_per_seq;
  int num_q_heads;
  int num_pages;
  int partition_tokens;
  int max_partitions;
  float scale_log2;              // scale * log2(e)
  int page_shift;                // page_size = 16 << page_shift
  // work-balanced decode only
  int num_seqs;
  int num_kv_heads;
  int32_t* ws_counters;          // [B * Hkv], zero between launches
  float* ws_partials;            // [warps][2][kSlotFloats]
};

// Work-balanced decode (paged_decode_balanced.cu).
constexpr int kMaxBalancedSeqs = 512;    // prefix sums live in shared memory
constexpr int kMinPagesPerWarp = 4;      // smallest range a warp is given
constexpr int kSlotFloats = 16 + 8 * 64; // m[8], l[8], acc[8][64] per segment

int balanced_decode_ctas_per_sm(int group, bool append);
cudaError_t launch_balanced_decode(const DecodeArgs& a, const CUtensorMap& tk,
                                   const CUtensorMap& tv, int group, int ctas,
                                   cudaStream_t stream);

cudaError_t launch_paged_decode(const DecodeArgs& a, const CUtensorMap& tk,
                                const CUtensorMap& tv, int num_kv_heads,
                                int num_seqs, int group, bool split,
                                int parts, cudaStream_t stream);

// Device page pool (page_pool.cu).  Error bits beyond those of tv_device.cuh.
constexpr uint32_t DEVERR_POOL_EMPTY = 1u << 5;  // too few free pages
constexpr uint32_t DEVERR_BAD_SEQ = 1u << 6;     // bad fork / release index
constexpr uint32_t DEVERR_BAD_POSITION = 1u << 7;  // RoPE position off the table
constexpr int kPoolMaxSeqs = 1024;               // one thread per sequence

cudaError_t launch_pool_init(int32_t* state, int num_pages, int page_size,
                             const int32_t* bt, int mb, const int32_t* ctx,
                             int num_seqs, uint32_t* err, cudaStream_t stream);
cudaError_t launch_pool_append(int32_t* state, int num_pages, int page_size,
                               int32_t* bt, int mb, int32_t* ctx,
                               const int32_t* n_new, int num_seqs,
                               int32_t* slot_mapping, void* k_pool,
                               void* v_pool, int row_bytes, uint32_t* err,
                               cudaStream_t stream);
cudaError_t launch_pool_fork(int32_t* state, int num_pages, int32_t* bt,
                             int mb, int32_t* ctx, int num_seqs,
                             const int32_t* src, const int32_t* dst,
                             int num_pairs, uint32_t* err,
                             cudaStream_t stream);
cudaError_t launch_pool_release(int32_t* state, int num_pages, int32_t* bt,
                                int mb, int32_t* ctx, int num_seqs,
                                const int32_t* seqs, int num_release,
                                uint32_t* err, cudaStream_t stream);

// Bounded-wait self-test (selftest.cu).
cudaError_t launch_wait_selftest(uint32_t* err, unsigned long long limit_ns,
                                 unsigned long long* waited_ns,
                                 cudaStream_t stream);

cudaError_t launch_kv_append_rope(const void* k_new, const void* v_new,
                                  const int32_t* slot_mapping,
                                  const int32_t* positions, int64_t num_tokens,
                                  void* k_pool, void* v_pool,
                                  int64_t num_slots, int num_kv_heads,
                                  const float* rope_cos_sin,
                                  int rope_max_position, uint32_t* err,
                                  cudaStream_t stream);

cudaError_t launch_kv_append(const void* k_new, const void* v_new,
                             const int32_t* slot_mapping, int64_t num_tokens,
                             void* k_pool, void* v_pool, int64_t num_slots,
                             int row_bytes, uint32_t* err,
                             cudaStream_t stream);

cudaError_t launch_split_merge(__nv_bfloat16* out, const float* partial_out,
                               const float* partial_lse,
                               const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int partition_tokens,
                               int max_partitions, cudaStream_t stream);

struct PrefillArgs {
  __nv_bfloat16* out;            // [rows][Hq][D]
  const int32_t* query_start_loc;  // [B+1]
  const int32_t* block_tables;
  const int32_t* context_lens;
  uint32_t* err;
  int max_blocks_per_seq;
  int num_seqs;
  int num_q_heads;
  int num_kv_heads;
  int num_pages;
  int max_query_len;
  int64_t num_query_rows;
  float scale_log2;
  int page_shift;                // page_size = 16 << page_shift
  int group;                     // query heads per KV head: 1, 2, 4 or 8
  // Dispatch order: order[i] = seq * prefill_blocks(max_query_len, group) + block of
  // the i-th CTA group (costliest first), written by the ordering kernel
  // into caller workspace; nullptr = grid order.
  int32_t* order;
};

// A prefill CTA owns two MMA tiles of 128 rows = (128 / group) query rows x
// the group's heads, so 256 / group query rows (chunk positions).
constexpr int kPrefillTileRows = 128;
__host__ __device__ inline int prefill_rows_per_cta(int group) {
  return 2 * kPrefillTileRows / group;
}
__host__ __device__ inline int prefill_blocks(int max_query_len, int group) {
  const int rows = prefill_rows_per_cta(group);
  return (max_query_len + rows - 1) / rows;
}

// Launches the ordering kernel first when a.order is set.
cudaError_t launch_paged_prefill(const PrefillArgs& a, const CUtensorMap& tq,
                                 const CUtensorMap& tk, const CUtensorMap& tv,
                                 cudaStream_t stream);

}  // namespace tv
