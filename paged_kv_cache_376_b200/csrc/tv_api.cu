// C ABI of libtv (declared in include/tv.h): argument checks, TMA tensor-map
// encoding and kernel launches.  Nothing here allocates device memory or
// synchronises the host: the pool is the caller's preallocated memory
// ("Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎", sec. "内存池管理":
// preallocate the pool, no cudaMalloc during inference).
#include <cmath>
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tv.h"
#include "tv_kernels.h"

namespace {

thread_local int g_last_cuda_error = 0;

constexpr int kHeadDim = 64;
constexpr int kPageSize = 16;   // the kernels' block: 16 token rows

// Pages of 16 or 32 tokens ([P3] 内存池管理 recommends 16-32); a page is
// 1 << page_shift blocks of 16 rows.
bool page_size_ok(int page_size) { return page_size == 16 || page_size == 32; }
int page_shift(int page_size) { return page_size == 32 ? 1 : 0; }

tv_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return TV_OK;
  g_last_cuda_error = static_cast<int>(e);
  return TV_ERR_CUDA;
}

bool aligned16(const void* p) {
  return (reinterpret_cast<uintptr_t>(p) & 15u) == 0;
}

bool group_ok(int num_q_heads, int num_kv_heads) {
  if (num_q_heads <= 0 || num_kv_heads <= 0) return false;
  if (num_q_heads % num_kv_heads) return false;
  const int g = num_q_heads / num_kv_heads;
  return g == 1 || g == 2 || g == 4 || g == 8;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library needs no link against libcuda.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p,
                                cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// The pool seen as a 2-D bf16 tensor [num_pages * page_size][Hkv * D]; the
// box is one 16-token block of one KV head: 16 rows x 64 elements (128 B)
// (a 32-token page is two boxes).  The 256-byte
// L2 promotion also fetches the neighbouring KV head's row; every decode grid
// reads the KV heads of a page at about the same time, so that row is an L2
// hit for its reader, not a second DRAM read.
tv_status pool_tensor_map(CUtensorMap* map, const void* pool,
                          int64_t num_pages, int page_size, int num_kv_heads,
                          CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return TV_ERR_CUDA;
  const cuuint64_t dims[2] = {(cuuint64_t)num_kv_heads * kHeadDim,
                              (cuuint64_t)num_pages * page_size};
  const cuuint64_t strides[1] = {(cuuint64_t)num_kv_heads * kHeadDim * 2};
  const cuuint32_t box[2] = {kHeadDim, kPageSize};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(pool), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return TV_ERR_CUDA;
  }
  return TV_OK;
}

// q seen as a 3-D bf16 tensor [rows][Hq][D]; the box is rows_per_box rows x
// G heads x 64 elements, i.e. the G query heads of one KV group for 128 / G
// query rows, which land in shared memory as 128 rows of 128 B in (row,
// head) order.
tv_status query_tensor_map(CUtensorMap* map, const void* q, int64_t rows,
                           int num_q_heads, int group, int rows_per_box) {
  auto fn = encode_fn();
  if (!fn) return TV_ERR_CUDA;
  const cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)num_q_heads,
                              (cuuint64_t)(rows > 0 ? rows : 1)};
  const cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2,
                                 (cuuint64_t)num_q_heads * kHeadDim * 2};
  const cuuint32_t box[3] = {kHeadDim, (cuuint32_t)group,
                             (cuuint32_t)rows_per_box};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(q), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    g_last_cuda_error = static_cast<int>(r);
    return TV_ERR_CUDA;
  }
  return TV_OK;
}

tv_status check_attention_shape(int num_q_heads, int num_kv_heads,
                                int head_dim, int page_size) {
  if (head_dim != kHeadDim || !page_size_ok(page_size))
    return TV_ERR_UNSUPPORTED;
  if (!group_ok(num_q_heads, num_kv_heads)) return TV_ERR_UNSUPPORTED;
  return TV_OK;
}

}  // namespace

extern "C" {

const char* tv_status_string(tv_status status) {
  switch (status) {
    case TV_OK: return "TV_OK";
    case TV_ERR_INVALID_ARG: return "TV_ERR_INVALID_ARG";
    case TV_ERR_UNSUPPORTED: return "TV_ERR_UNSUPPORTED";
    case TV_ERR_CUDA: return "TV_ERR_CUDA";
    case TV_ERR_SCRATCH_LIMIT: return "TV_ERR_SCRATCH_LIMIT";
  }
  return "TV_ERR_UNKNOWN";
}

int tv_last_cuda_error(void) { return g_last_cuda_error; }

int tv_version(void) { return 100; }

tv_status tv_kv_append(const void* k_new, const void* v_new,
                       const int32_t* slot_mapping, int64_t num_tokens,
                       void* k_pool, void* v_pool, int64_t num_pages,
                       int num_kv_heads, int head_dim, int page_size,
                       uint32_t* err, void* stream) {
  if (num_tokens < 0 || num_pages <= 0 || num_kv_heads <= 0)
    return TV_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || !page_size_ok(page_size))
    return TV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return TV_OK;
  if (!k_new || !v_new || !slot_mapping || !k_pool || !v_pool)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) ||
      !aligned16(v_pool))
    return TV_ERR_INVALID_ARG;
  const int row_bytes = num_kv_heads * head_dim * 2;
  return cuda_status(tv::launch_kv_append(
      k_new, v_new, slot_mapping, num_tokens, k_pool, v_pool,
      num_pages * page_size, row_bytes, err,
      static_cast<cudaStream_t>(stream)));
}

tv_status tv_kv_append_rope(const void* k_new, const void* v_new,
                            const int32_t* slot_mapping,
                            const int32_t* positions, int64_t num_tokens,
                            void* k_pool, void* v_pool, int64_t num_pages,
                            int num_kv_heads, int head_dim, int page_size,
                            const float* rope_cos_sin, int rope_max_position,
                            uint32_t* err, void* stream) {
  if (num_tokens < 0 || num_pages <= 0 || num_kv_heads <= 0)
    return TV_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || !page_size_ok(page_size))
    return TV_ERR_UNSUPPORTED;
  if (num_tokens == 0) return TV_OK;
  if (!k_new || !v_new || !slot_mapping || !positions || !k_pool ||
      !v_pool || !rope_cos_sin || rope_max_position <= 0)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_pool) ||
      !aligned16(v_pool) || !aligned16(rope_cos_sin))
    return TV_ERR_INVALID_ARG;
  return cuda_status(tv::launch_kv_append_rope(
      k_new, v_new, slot_mapping, positions, num_tokens, k_pool, v_pool,
      num_pages * page_size, num_kv_heads, rope_cos_sin, rope_max_position,
      err, static_cast<cudaStream_t>(stream)));
}

// Device workspace of the work-balanced decode: per-item counters, then two
// partial-result slots per warp of the persistent grid.
struct BalancedWorkspace {
  void* base;
  size_t bytes;
};

static int device_sms() {
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) !=
      cudaSuccess)
    return 0;
  return sms;
}

static size_t counters_bytes(int num_seqs, int num_kv_heads) {
  return ((size_t)num_seqs * num_kv_heads * 4 + 255) / 256 * 256;
}

static int balanced_ctas(int group) {
  const int a = tv::balanced_decode_ctas_per_sm(group, false);
  const int b = tv::balanced_decode_ctas_per_sm(group, true);
  return device_sms() * (a > b ? a : b);
}

static size_t partials_bytes(int ctas) {
  return (size_t)ctas * 4 * 2 * tv::kSlotFloats * sizeof(float);
}

static tv_status decode_common(void* out, float* partial_out,
                               float* partial_lse, const void* q,
                               const void* k_new, const void* v_new,
                               const void* k_pool, const void* v_pool,
                               const int32_t* block_tables,
                               int max_blocks_per_seq,
                               const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int num_kv_heads, int head_dim,
                               int page_size, int64_t num_pages, float scale,
                               int partition_tokens, int max_partitions,
                               bool split, uint32_t* err, void* stream,
                               const BalancedWorkspace* ws = nullptr,
                               const int32_t* grown = nullptr,
                               const float* rope_cos_sin = nullptr,
                               int rope_max_position = 0) {
  tv_status st =
      check_attention_shape(num_q_heads, num_kv_heads, head_dim, page_size);
  if (st != TV_OK) return st;
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_pages <= 0 ||
      !std::isfinite(scale))
    return TV_ERR_INVALID_ARG;
  // the kernels hold token positions (up to max_blocks_per_seq * page_size)
  // and pool rows in 32-bit integers
  if (num_seqs > 65535 || num_pages * page_size > INT32_MAX ||
      (int64_t)max_blocks_per_seq * page_size > INT32_MAX)
    return TV_ERR_UNSUPPORTED;
  if (split && (partition_tokens <= 0 || partition_tokens % page_size ||
                max_partitions <= 0 || max_partitions > 65535))
    return TV_ERR_INVALID_ARG;
  if (num_seqs == 0) return TV_OK;
  if (!q || !k_pool || !v_pool || !block_tables || !context_lens)
    return TV_ERR_INVALID_ARG;
  if (split ? (!partial_out || !partial_lse || !aligned16(partial_out))
            : !out)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k_pool) || !aligned16(v_pool) ||
      (!split && !aligned16(out)))
    return TV_ERR_INVALID_ARG;
  if ((k_new != nullptr) != (v_new != nullptr) || (split && k_new))
    return TV_ERR_INVALID_ARG;
  if (k_new && (!aligned16(k_new) || !aligned16(v_new)))
    return TV_ERR_INVALID_ARG;

  const int shift = page_shift(page_size);
  const bool balanced = ws && num_seqs <= tv::kMaxBalancedSeqs &&
                        max_blocks_per_seq < (1 << 24) &&
                        (num_pages << shift) < (1 << 26) - 1 &&
                        (int64_t)num_seqs * num_kv_heads *
                                (max_blocks_per_seq << shift) < INT32_MAX;
  // both decode kernels read their slices with ldmatrix from 128-byte
  // swizzled boxes
  const CUtensorMapSwizzle swz = CU_TENSOR_MAP_SWIZZLE_128B;
  CUtensorMap tk, tvm;
  st = pool_tensor_map(&tk, k_pool, num_pages, page_size, num_kv_heads, swz);
  if (st != TV_OK) return st;
  st = pool_tensor_map(&tvm, v_pool, num_pages, page_size, num_kv_heads, swz);
  if (st != TV_OK) return st;

  tv::DecodeArgs a{};
  a.out = static_cast<__nv_bfloat16*>(out);
  a.partial_out = partial_out;
  a.partial_lse = partial_lse;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.k_new = static_cast<const __nv_bfloat16*>(k_new);
  a.v_new = static_cast<const __nv_bfloat16*>(v_new);
  a.k_pool_w = static_cast<__nv_bfloat16*>(const_cast<void*>(k_pool));
  a.v_pool_w = static_cast<__nv_bfloat16*>(const_cast<void*>(v_pool));
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.grown = grown;
  a.rope_cos_sin = rope_cos_sin;
  a.rope_max_position = rope_max_position;
  a.err = err;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_q_heads = num_q_heads;
  a.num_pages = static_cast<int>(num_pages);
  a.partition_tokens = split ? partition_tokens : 0;
  a.max_partitions = split ? max_partitions : 1;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.page_shift = shift;
  const int group = num_q_heads / num_kv_heads;
  // The balanced grid needs the prefix sums of every sequence in shared
  // memory, all flattened page positions in int32, page indices in 24 bits
  // and physical page ids in 26 bits (the condition `balanced` above);
  // beyond that the
  // one-CTA-per-(sequence, KV head) kernel serves the call.
  if (balanced) {
    const int cap = balanced_ctas(group);
    if (cap <= 0) return cuda_status(cudaErrorUnknown);
    const size_t cb = counters_bytes(num_seqs, num_kv_heads);
    if (ws->bytes < cb + partials_bytes(cap)) return TV_ERR_INVALID_ARG;
    // groups of num_kv_heads warps, each with >= kMinPagesPerWarp pages
    // (num_seqs * max_blocks_per_seq bounds the page count from above)
    const int64_t groups =
        ((int64_t)num_seqs * (max_blocks_per_seq << shift) +
         tv::kMinPagesPerWarp - 1) / tv::kMinPagesPerWarp;
    const int64_t want = (groups * num_kv_heads + 3) / 4;
    const int64_t least = (num_kv_heads + 3) / 4;   // one whole group
    if (cap < least) return TV_ERR_UNSUPPORTED;
    const int ctas = (int)(want < least ? least : (want < cap ? want : cap));
    a.num_seqs = num_seqs;
    a.num_kv_heads = num_kv_heads;
    a.ws_counters = static_cast<int32_t*>(ws->base);
    a.ws_partials = reinterpret_cast<float*>(static_cast<char*>(ws->base) + cb);
    return cuda_status(tv::launch_balanced_decode(
        a, tk, tvm, group, ctas, static_cast<cudaStream_t>(stream)));
  }
  return cuda_status(tv::launch_paged_decode(
      a, tk, tvm, num_kv_heads, num_seqs, group, split,
      split ? max_partitions : 1, static_cast<cudaStream_t>(stream)));
}

tv_status tv_paged_decode(void* out, const void* q, const void* k_pool,
                          const void* v_pool, const int32_t* block_tables,
                          int max_blocks_per_seq, const int32_t* context_lens,
                          int num_seqs, int num_q_heads, int num_kv_heads,
                          int head_dim, int page_size, int64_t num_pages,
                          float scale, uint32_t* err, void* stream) {
  return decode_common(out, nullptr, nullptr, q, nullptr, nullptr, k_pool,
                       v_pool, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, 0, 1, false, err, stream);
}

tv_status tv_paged_decode_append(void* out, const void* q, const void* k_new,
                                 const void* v_new, void* k_pool, void* v_pool,
                                 const int32_t* block_tables,
                                 int max_blocks_per_seq,
                                 const int32_t* context_lens, int num_seqs,
                                 int num_q_heads, int num_kv_heads,
                                 int head_dim, int page_size,
                                 int64_t num_pages, float scale,
                                 uint32_t* err, void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new)) return TV_ERR_INVALID_ARG;
  return decode_common(out, nullptr, nullptr, q, k_new, v_new, k_pool, v_pool,
                       block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, 0, 1, false, err, stream);
}

tv_status tv_paged_decode_append_rope(
    void* out, const void* q, const void* k_new, const void* v_new,
    void* k_pool, void* v_pool, const int32_t* block_tables,
    int max_blocks_per_seq, const int32_t* context_lens, int num_seqs,
    int num_q_heads, int num_kv_heads, int head_dim, int page_size,
    int64_t num_pages, float scale, const float* rope_cos_sin,
    int rope_max_position, uint32_t* err, void* stream) {
  if (num_seqs > 0 && (!k_new || !v_new || !rope_cos_sin ||
                       !aligned16(rope_cos_sin) || rope_max_position <= 0))
    return TV_ERR_INVALID_ARG;
  return decode_common(out, nullptr, nullptr, q, k_new, v_new, k_pool, v_pool,
                       block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, 0, 1, false, err, stream,
                       nullptr, nullptr, rope_cos_sin, rope_max_position);
}

tv_status tv_decode_workspace_size(int num_seqs, int num_q_heads,
                                   int num_kv_heads, int head_dim,
                                   size_t* bytes) {
  if (!bytes) return TV_ERR_INVALID_ARG;
  tv_status st =
      check_attention_shape(num_q_heads, num_kv_heads, head_dim, kPageSize);
  if (st != TV_OK) return st;
  if (num_seqs < 0) return TV_ERR_INVALID_ARG;
  const int cap = balanced_ctas(num_q_heads / num_kv_heads);
  if (cap <= 0) return cuda_status(cudaErrorUnknown);
  *bytes = counters_bytes(num_seqs, num_kv_heads) + partials_bytes(cap);
  return TV_OK;
}

tv_status tv_paged_decode_balanced(void* out, const void* q,
                                   const void* k_new, const void* v_new,
                                   void* k_pool, void* v_pool,
                                   const int32_t* block_tables,
                                   int max_blocks_per_seq,
                                   const int32_t* context_lens, int num_seqs,
                                   int num_q_heads, int num_kv_heads,
                                   int head_dim, int page_size,
                                   int64_t num_pages, float scale,
                                   void* workspace, size_t workspace_bytes,
                                   uint32_t* err, void* stream) {
  if (num_seqs > 0 && (!workspace || !aligned16(workspace)))
    return TV_ERR_INVALID_ARG;
  const BalancedWorkspace ws{workspace, workspace_bytes};
  return decode_common(out, nullptr, nullptr, q, k_new, v_new, k_pool, v_pool,
                       block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, 0, 1, false, err, stream,
                       &ws);
}

tv_status tv_selftest_wait_timeout(uint32_t* err, int64_t limit_ns,
                                   uint64_t* waited_ns, void* stream) {
  if (!err || limit_ns < 0) return TV_ERR_INVALID_ARG;
  // never longer than the library's own limit
  const int64_t lim = limit_ns < 2000000000 ? limit_ns : 2000000000;
  return cuda_status(tv::launch_wait_selftest(
      err, (unsigned long long)lim,
      reinterpret_cast<unsigned long long*>(waited_ns),
      static_cast<cudaStream_t>(stream)));
}

// ---- device page pool ---------------------------------------------------------

static tv_status pool_common(const int32_t* pool_state, int64_t num_pages,
                             const int32_t* block_tables,
                             int max_blocks_per_seq,
                             const int32_t* context_lens, int num_seqs) {
  if (!pool_state || num_pages <= 0 || num_seqs < 0 ||
      (num_seqs > 0 &&
       (!block_tables || !context_lens || max_blocks_per_seq <= 0)))
    return TV_ERR_INVALID_ARG;
  if (num_pages > (INT32_MAX - 4) / 4 || num_seqs > TV_POOL_MAX_SEQS ||
      (int64_t)max_blocks_per_seq * 32 > INT32_MAX)
    return TV_ERR_UNSUPPORTED;
  return TV_OK;
}

tv_status tv_pool_init(int32_t* pool_state, int64_t num_pages, int page_size,
                       const int32_t* block_tables, int max_blocks_per_seq,
                       const int32_t* context_lens, int num_seqs,
                       uint32_t* err, void* stream) {
  if (!block_tables) num_seqs = 0;
  tv_status st = pool_common(pool_state, num_pages, block_tables,
                             max_blocks_per_seq, context_lens, num_seqs);
  if (st != TV_OK) return st;
  if (!page_size_ok(page_size)) return TV_ERR_UNSUPPORTED;
  return cuda_status(tv::launch_pool_init(
      pool_state, (int)num_pages, page_size, block_tables, max_blocks_per_seq,
      context_lens, num_seqs, err, static_cast<cudaStream_t>(stream)));
}

tv_status tv_pool_append_slots(int32_t* pool_state, int64_t num_pages,
                               int32_t* block_tables, int max_blocks_per_seq,
                               int32_t* context_lens,
                               const int32_t* num_new_tokens, int num_seqs,
                               int32_t* slot_mapping, void* k_pool,
                               void* v_pool, int num_kv_heads, int head_dim,
                               int page_size, uint32_t* err, void* stream) {
  tv_status st = pool_common(pool_state, num_pages, block_tables,
                             max_blocks_per_seq, context_lens, num_seqs);
  if (st != TV_OK) return st;
  if (head_dim != kHeadDim || !page_size_ok(page_size))
    return TV_ERR_UNSUPPORTED;
  if (num_kv_heads <= 0 || !k_pool || !v_pool || !aligned16(k_pool) ||
      !aligned16(v_pool))
    return TV_ERR_INVALID_ARG;
  if (num_seqs == 0) return TV_OK;
  return cuda_status(tv::launch_pool_append(
      pool_state, (int)num_pages, page_size, block_tables, max_blocks_per_seq,
      context_lens, num_new_tokens, num_seqs, slot_mapping, k_pool, v_pool,
      num_kv_heads * head_dim * 2, err, static_cast<cudaStream_t>(stream)));
}

tv_status tv_pool_fork(int32_t* pool_state, int64_t num_pages,
                       int32_t* block_tables, int max_blocks_per_seq,
                       int32_t* context_lens, int num_seqs,
                       const int32_t* src_seqs, const int32_t* dst_seqs,
                       int num_pairs, uint32_t* err, void* stream) {
  tv_status st = pool_common(pool_state, num_pages, block_tables,
                             max_blocks_per_seq, context_lens, num_seqs);
  if (st != TV_OK) return st;
  if (num_pairs < 0 || (num_pairs > 0 && (!src_seqs || !dst_seqs)))
    return TV_ERR_INVALID_ARG;
  if (num_pairs == 0 || num_seqs == 0) return TV_OK;
  return cuda_status(tv::launch_pool_fork(
      pool_state, (int)num_pages, block_tables, max_blocks_per_seq,
      context_lens, num_seqs, src_seqs, dst_seqs, num_pairs, err,
      static_cast<cudaStream_t>(stream)));
}

tv_status tv_pool_release(int32_t* pool_state, int64_t num_pages,
                          int32_t* block_tables, int max_blocks_per_seq,
                          int32_t* context_lens, int num_seqs,
                          const int32_t* seqs, int num_release, uint32_t* err,
                          void* stream) {
  tv_status st = pool_common(pool_state, num_pages, block_tables,
                             max_blocks_per_seq, context_lens, num_seqs);
  if (st != TV_OK) return st;
  if (num_release < 0 || (num_release > 0 && !seqs)) return TV_ERR_INVALID_ARG;
  if (num_release == 0 || num_seqs == 0) return TV_OK;
  return cuda_status(tv::launch_pool_release(
      pool_state, (int)num_pages, block_tables, max_blocks_per_seq,
      context_lens, num_seqs, seqs, num_release, err,
      static_cast<cudaStream_t>(stream)));
}

tv_status tv_decode_step(int32_t* pool_state, int64_t num_pages, void* out,
                         const void* q, const void* k_new, const void* v_new,
                         void* k_pool, void* v_pool, int32_t* block_tables,
                         int max_blocks_per_seq, int32_t* context_lens,
                         int num_seqs, int num_q_heads, int num_kv_heads,
                         int head_dim, int page_size, float scale,
                         void* workspace, size_t workspace_bytes,
                         uint32_t* err, void* stream) {
  tv_status st = check_attention_shape(num_q_heads, num_kv_heads, head_dim,
                                       page_size);
  if (st != TV_OK) return st;
  // check what the attention call checks before the pool is touched, so a
  // rejected step changes nothing
  if (!k_new || !v_new || !out || !q || !aligned16(out) || !aligned16(q) ||
      !aligned16(k_new) || !aligned16(v_new) || !std::isfinite(scale) ||
      num_pages * page_size > INT32_MAX ||
      (workspace && !aligned16(workspace)))
    return TV_ERR_INVALID_ARG;
  st = tv_pool_append_slots(pool_state, num_pages, block_tables,
                            max_blocks_per_seq, context_lens, nullptr,
                            num_seqs, nullptr, k_pool, v_pool, num_kv_heads,
                            head_dim, page_size, err, stream);
  if (st != TV_OK) return st;
  if (num_seqs == 0) return TV_OK;
  // the pool's marks of the sequences that got room for their token: every
  // other sequence is idle in the attention launch (appends nothing, zero
  // output), so a sequence left unserved keeps its cached rows intact
  const int32_t* grown = pool_state + 4 + 4 * num_pages;
  const BalancedWorkspace ws{workspace, workspace_bytes};
  return decode_common(out, nullptr, nullptr, q, k_new, v_new, k_pool, v_pool,
                       block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, 0, 1, false, err, stream,
                       workspace ? &ws : nullptr, grown);
}

tv_status tv_paged_decode_split(float* partial_out, float* partial_lse,
                                const void* q, const void* k_pool,
                                const void* v_pool,
                                const int32_t* block_tables,
                                int max_blocks_per_seq,
                                const int32_t* context_lens, int num_seqs,
                                int num_q_heads, int num_kv_heads,
                                int head_dim, int page_size,
                                int64_t num_pages, float scale,
                                int partition_tokens, int max_partitions,
                                uint32_t* err, void* stream) {
  return decode_common(nullptr, partial_out, partial_lse, q, nullptr, nullptr,
                       k_pool, v_pool, block_tables, max_blocks_per_seq, context_lens,
                       num_seqs, num_q_heads, num_kv_heads, head_dim,
                       page_size, num_pages, scale, partition_tokens,
                       max_partitions, true, err, stream);
}

tv_status tv_split_merge(void* out, const float* partial_out,
                         const float* partial_lse,
                         const int32_t* context_lens, int num_seqs,
                         int num_q_heads, int head_dim, int partition_tokens,
                         int max_partitions, void* stream) {
  if (head_dim != kHeadDim) return TV_ERR_UNSUPPORTED;
  if (num_seqs < 0 || num_q_heads <= 0 || partition_tokens <= 0 ||
      max_partitions <= 0)
    return TV_ERR_INVALID_ARG;
  if (num_seqs > 65535 || num_q_heads > 65535) return TV_ERR_UNSUPPORTED;
  if (num_seqs == 0) return TV_OK;
  if (!out || !partial_out || !partial_lse || !context_lens)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(partial_out)) return TV_ERR_INVALID_ARG;
  return cuda_status(tv::launch_split_merge(
      static_cast<__nv_bfloat16*>(out), partial_out, partial_lse,
      context_lens, num_seqs, num_q_heads, partition_tokens, max_partitions,
      static_cast<cudaStream_t>(stream)));
}

// Items of the ordering list: one per (sequence, block of
// prefill_rows_per_cta(group) rows).  The size query has no group, so it
// answers for the largest group (the most blocks).
static size_t prefill_workspace_bytes(int num_seqs, int max_query_len,
                                      int group = 8) {
  const size_t items =
      (size_t)num_seqs * (size_t)tv::prefill_blocks(max_query_len, group);
  return (items * sizeof(int32_t) + 15) / 16 * 16;
}

tv_status tv_prefill_workspace_size(int num_seqs, int max_query_len,
                                    size_t* bytes) {
  if (!bytes || num_seqs < 0 || max_query_len < 0) return TV_ERR_INVALID_ARG;
  *bytes = prefill_workspace_bytes(num_seqs, max_query_len);
  return TV_OK;
}

tv_status tv_paged_prefill(void* out, const void* q, int64_t num_query_rows,
                           const int32_t* query_start_loc, const void* k_pool,
                           const void* v_pool, const int32_t* block_tables,
                           int max_blocks_per_seq, const int32_t* context_lens,
                           int num_seqs, int max_query_len, int num_q_heads,
                           int num_kv_heads, int head_dim, int page_size,
                           int64_t num_pages, float scale, void* workspace,
                           size_t workspace_bytes, uint32_t* err,
                           void* stream) {
  tv_status st =
      check_attention_shape(num_q_heads, num_kv_heads, head_dim, page_size);
  if (st != TV_OK) return st;
  const int group = num_q_heads / num_kv_heads;   // 1, 2, 4 or 8 (checked)
  // the kernel scales each tile's maximum raw score, which is the maximum
  // of the scaled scores only when the scale is positive
  if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_pages <= 0 ||
      max_query_len < 0 || num_query_rows < 0 || !std::isfinite(scale) ||
      !(scale > 0.f))
    return TV_ERR_INVALID_ARG;
  if (num_seqs > 65535 || num_pages * page_size > INT32_MAX ||
      (int64_t)max_blocks_per_seq * page_size > INT32_MAX)
    return TV_ERR_UNSUPPORTED;
  if (num_seqs == 0 || max_query_len == 0 || num_query_rows == 0)
    return TV_OK;
  if (!out || !q || !query_start_loc || !k_pool || !v_pool || !block_tables ||
      !context_lens)
    return TV_ERR_INVALID_ARG;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_pool) ||
      !aligned16(v_pool))
    return TV_ERR_INVALID_ARG;
  if (workspace &&
      (!aligned16(workspace) ||
       workspace_bytes <
           prefill_workspace_bytes(num_seqs, max_query_len, group)))
    return TV_ERR_INVALID_ARG;
  if (tv::prefill_blocks(max_query_len, group) > 65535) return TV_ERR_UNSUPPORTED;
  // the ordering kernel counts the (sequence, block) items in an int
  if (workspace &&
      (int64_t)num_seqs * tv::prefill_blocks(max_query_len, group) > INT32_MAX)
    return TV_ERR_UNSUPPORTED;

  // Query rows past num_query_rows read as zeros and are never stored.
  CUtensorMap tq, tk, tvm;
  st = query_tensor_map(&tq, q, num_query_rows, num_q_heads, group,
                        tv::kPrefillTileRows / group);
  if (st != TV_OK) return st;
  st = pool_tensor_map(&tk, k_pool, num_pages, page_size, num_kv_heads,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TV_OK) return st;
  st = pool_tensor_map(&tvm, v_pool, num_pages, page_size, num_kv_heads,
                       CU_TENSOR_MAP_SWIZZLE_128B);
  if (st != TV_OK) return st;

  tv::PrefillArgs a{};
  a.out = static_cast<__nv_bfloat16*>(out);
  a.query_start_loc = query_start_loc;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  a.err = err;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_q_heads = num_q_heads;
  a.num_kv_heads = num_kv_heads;
  a.num_pages = static_cast<int>(num_pages);
  a.max_query_len = max_query_len;
  a.num_query_rows = num_query_rows;
  a.scale_log2 = scale * 1.4426950408889634f;
  a.page_shift = page_shift(page_size);
  a.order = static_cast<int32_t*>(workspace);
  a.group = group;
  return cuda_status(tv::launch_paged_prefill(
      a, tq, tk, tvm, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
