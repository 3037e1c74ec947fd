// tv_paged_decode_split_static: split-KV decode plus log-sum-exp merge in one
// call, with the partial results kept in a fixed array that lives inside the
// library, so the caller allocates nothing.
//
// Why it exists.  tv_paged_decode_split needs two caller-owned fp32 buffers
// for its partials.  Some callers cannot provide them on the decode path:
//   * engines that size the KV page pool to (almost) all of device memory at
//     start-up and forbid any further allocation while serving -- a
//     cudaMalloc there either fails or has to take pages from the pool;
//   * latency-critical step loops: cudaMalloc / cudaFree may block and
//     synchronise the device, which stalls every stream mid-step;
//   * plain C hosts that bind only this ABI and have no device allocator.
// For them the partials go to g_tv_split_scratch below instead.
//
// Contract (also stated in include/tv.h):
//   * capacity TV_STATIC_SCRATCH_FLOATS floats (32 MiB) per device, held by
//     every GPU that loads the library until the process exits;
//   * a call needs num_seqs * num_q_heads * max_partitions * (head_dim + 1)
//     floats; a larger call returns TV_ERR_SCRATCH_LIMIT before any launch;
//   * all calls on a device share the one array and it keeps the previous
//     call's contents; nothing in it has to start at zero, because the split
//     kernel writes every partial the merge reads;
//   * calls whose kernels overlap on the GPU (different streams, no ordering
//     between them) race on the array; order them on one stream or with
//     events;
//   * the first call on a device looks up the array's device address with
//     that device current (cudaGetSymbolAddress); make that first call before
//     any stream capture.  The address is remembered together with the
//     identity of the CUDA context it was looked up in; a call that finds
//     another context current (after cudaDeviceReset the runtime makes a new
//     primary context, which loads the library's kernels and the array
//     afresh) looks it up again instead of using an address of the old one.
#include <cstdint>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "tv.h"

namespace {

// The scratch itself.  Host code must not use this name as a pointer: on the
// host it is only a stand-in; the device address comes from
// cudaGetSymbolAddress.
static __device__ __align__(256) float g_tv_split_scratch[TV_STATIC_SCRATCH_FLOATS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};
unsigned long long g_scratch_ctx[kMaxDevices] = {};   // context id, 0 = none

// Unique id of the CUDA context current on this thread (ids are never
// reused within a process), or 0 when none is current or it cannot be read.
// The driver calls come through the runtime's entry-point lookup, so the
// library needs no link against libcuda.
unsigned long long current_context_id() {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault,
                                &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext c = nullptr;
  unsigned long long id = 0;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch on the current device, looked up with that
// device current the first time it is used in the current context (normally
// once per device).  nullptr on failure.
float* scratch_on_current_device() {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_mu);
  const unsigned long long ctx = current_context_id();
  if (!g_scratch_ptr[dev] || ctx == 0 || ctx != g_scratch_ctx[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_tv_split_scratch);
    if (e != cudaSuccess || p == nullptr) {
      g_scratch_ptr[dev] = nullptr;
      return nullptr;
    }
    g_scratch_ptr[dev] = static_cast<float*>(p);
    // the lookup makes the device's primary context current if none was
    g_scratch_ctx[dev] = current_context_id();
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" tv_status tv_paged_decode_split_static(
    void* out, const void* q, const void* k_pool, const void* v_pool,
    const int32_t* block_tables, int max_blocks_per_seq,
    const int32_t* context_lens, int num_seqs, int num_q_heads,
    int num_kv_heads, int head_dim, int page_size, int64_t num_pages,
    float scale, int partition_tokens, int max_partitions, uint32_t* err,
    void* stream) {
  if (num_seqs < 0 || num_q_heads <= 0 || head_dim <= 0 ||
      max_partitions <= 0)
    return TV_ERR_INVALID_ARG;
  if (num_seqs == 0) return TV_OK;
  const uint64_t rows =
      (uint64_t)num_seqs * (uint64_t)num_q_heads * (uint64_t)max_partitions;
  const uint64_t need = rows * (uint64_t)(head_dim + 1);
  if (need > (uint64_t)TV_STATIC_SCRATCH_FLOATS) return TV_ERR_SCRATCH_LIMIT;

  float* scratch = scratch_on_current_device();
  if (!scratch) return TV_ERR_CUDA;
  float* partial_out = scratch;                             // rows x head_dim
  float* partial_lse = scratch + rows * (uint64_t)head_dim; // rows

  tv_status st = tv_paged_decode_split(
      partial_out, partial_lse, q, k_pool, v_pool, block_tables,
      max_blocks_per_seq, context_lens, num_seqs, num_q_heads, num_kv_heads,
      head_dim, page_size, num_pages, scale, partition_tokens, max_partitions,
      err, stream);
  if (st != TV_OK) return st;
  return tv_split_merge(out, partial_out, partial_lse, context_lens, num_seqs,
                        num_q_heads, head_dim, partition_tokens,
                        max_partitions, stream);
}
