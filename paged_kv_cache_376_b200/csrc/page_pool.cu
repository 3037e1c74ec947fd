// KV page pool on the device: free-page stack, per-page reference counts,
// on-demand allocation with copy-on-write of shared pages, fork and release.
//
// What it follows: "Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎",
// sec. 内存池管理 (pages allocated when a request produces a new token,
// returned to the free pool when it ends, shared between requests for prefix
// caching; a free-page list is the pool's core structure), and
// "tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec. PagedAttention (pages
// allocated only when needed; sharing made safe by copy-on-write).
//
// B200 design.  The pool lives in device memory so a decode step (room for
// the new token, then the fused append + attention) runs without the host
// and can be captured in a CUDA graph.  The free list is an array stack
// (constant-time pop/push by index arithmetic instead of a pointer chase).
// The bookkeeping kernels run as one CTA of 1024 threads, one thread per
// sequence (B <= 1024), and take every decision with block-wide scans in a
// fixed order, so the pages a call hands out do not depend on thread timing:
//   * needs are reserved in batch order (exclusive scan), pops take
//     stack[top-1-offset-j];
//   * copy-on-write: a sequence writing into a partly filled page held by
//     r > 1 rows copies it first, except the last writer of that page in
//     batch order when all r holders write this step (that one keeps it);
//     the number of writers per page and the last one are found with
//     atomicAdd / atomicMax on two scratch arrays, both order-independent;
//   * released pages whose count reaches zero are pushed in ascending id
//     order (a scan over the whole pool).
// All of this is integer index work; pages are copied with 16-byte vectors.
#include <cstdint>

#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kThreads = 1024;

struct PoolView {
  int32_t* top;
  int32_t* last_slots;   // slots written by the last append call
  int32_t* page_size;    // tokens per page, set by init (16 or 32)
  int32_t* stack;        // [num_pages]
  int32_t* ref;          // [num_pages]
  int32_t* cnt_app;      // [num_pages], zero between calls
  int32_t* last_app;     // [num_pages], zero between calls
  int32_t* grown;        // [kPoolMaxSeqs]: 1 = got its tokens in the last
                         // append call, 0 = did not (idle, unserved, flagged)
  int num_pages;
};

__host__ __device__ inline PoolView view(int32_t* state, int num_pages) {
  PoolView v;
  v.top = state + 0;
  v.last_slots = state + 2;
  v.page_size = state + 3;
  v.stack = state + 4;
  v.ref = v.stack + num_pages;
  v.cnt_app = v.ref + num_pages;
  v.last_app = v.cnt_app + num_pages;
  v.grown = v.last_app + num_pages;
  v.num_pages = num_pages;
  return v;
}

__device__ __forceinline__ int pages_for(int ctx, int ps) {
  return (ctx + ps - 1) / ps;
}

// Exclusive scan of one int per thread over the threads of the CTA (a
// multiple of 32, at most 1024); *total receives the sum.  `sh` holds 33
// ints.
__device__ int block_exclusive_scan(int v, int* sh, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += t;
  }
  __syncthreads();  // sh may still be read by a previous scan
  if (lane == 31) sh[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = lane < (int)(blockDim.x >> 5) ? sh[lane] : 0;
    int wi = w;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, off);
      if (lane >= off) wi += t;
    }
    sh[lane] = wi - w;                // exclusive prefix of warp totals
    if (lane == 31) sh[32] = wi;      // grand total
  }
  __syncthreads();
  const int res = sh[warp] + incl - v;
  *total = sh[32];
  return res;
}

// ---- init -------------------------------------------------------------------
__global__ void pool_clear_kernel(PoolView p) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < p.num_pages;
       i += gridDim.x * blockDim.x) {
    p.ref[i] = 0;
    p.cnt_app[i] = 0;
    p.last_app[i] = 0;
  }
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < kPoolMaxSeqs;
       i += gridDim.x * blockDim.x)
    p.grown[i] = 0;
}

__global__ void pool_count_refs_kernel(PoolView p, const int32_t* bt, int mb,
                                       const int32_t* ctx, int num_seqs,
                                       int kPS, uint32_t* err) {
  const int64_t total = (int64_t)num_seqs * mb;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int s = (int)(i / mb), b = (int)(i % mb);
    int c = ctx[s];
    if (c < 0 || c > mb * kPS) {
      if (b == 0) flag_error(err, DEVERR_BAD_CONTEXT);
      c = c < 0 ? 0 : mb * kPS;
    }
    if (b >= pages_for(c, kPS)) continue;
    const int page = bt[(size_t)s * mb + b];
    if (page < 0 || page >= p.num_pages) {
      flag_error(err, DEVERR_BAD_PAGE);
      continue;
    }
    atomicAdd(p.ref + page, 1);
  }
}

// stack = unreferenced pages in descending id order (a fresh pool pops 0, 1..)
__global__ void __launch_bounds__(kThreads, 1)
    pool_stack_kernel(PoolView p, int page_size) {
  __shared__ int sh[33];
  int base = 0;
  for (int i0 = 0; i0 < p.num_pages; i0 += kThreads) {
    const int i = i0 + threadIdx.x;
    const int page = p.num_pages - 1 - i;
    const int f = (i < p.num_pages && p.ref[page] == 0) ? 1 : 0;
    int tot;
    const int pos = block_exclusive_scan(f, sh, &tot);
    if (f) p.stack[base + pos] = page;
    base += tot;
  }
  if (threadIdx.x == 0) {
    *p.top = base;
    *p.last_slots = 0;
    *p.page_size = page_size;
  }
}

// ---- append slots -----------------------------------------------------------
// Room for n[s] new tokens at positions ctx .. ctx+n-1 of every sequence.
__global__ void __launch_bounds__(kThreads, 1)
    pool_append_kernel(PoolView p, int32_t* bt, int mb, int32_t* ctx,
                       const int32_t* n_new, int num_seqs,
                       int32_t* slot_mapping, uint8_t* k_pool,
                       uint8_t* v_pool, int row_bytes, int kPS,
                       uint32_t* err) {
  __shared__ int sh[33];
  __shared__ int job_old[kThreads], job_new[kThreads];
  const int s = threadIdx.x;
  const bool live = s < num_seqs;
  // The loads that do not depend on one another go out together (the kernel
  // is a chain of dependent round trips: context -> last page -> its
  // reference count -> free-stack pops); nothing below writes top or ref
  // before the scans.
  const int pool_ps = *p.page_size;
  const int top = *p.top;
  int c = live ? ctx[s] : 0;
  int n = live && n_new ? n_new[s] : 0;
  if (pool_ps != kPS) {   // pools of another page size: touch nothing
    if (threadIdx.x == 0) flag_error(err, DEVERR_BAD_SEQ);
    if (live) p.grown[s] = 0;
    return;
  }
  int part = -1, r = 0;
  if (live) {
    // decode steps (n_new == nullptr) add one token to every live sequence
    if (!n_new) n = c > 0 ? 1 : 0;
    if (n < 0) n = 0;
    if (c < 0 || c + n > mb * kPS) {
      flag_error(err, DEVERR_BAD_CONTEXT);
      n = 0;
    }
    if (n > 0 && c % kPS) {
      part = bt[(size_t)s * mb + c / kPS];
      if (part < 0 || part >= p.num_pages) {
        flag_error(err, DEVERR_BAD_PAGE);
        n = 0;
        part = -1;
      } else {
        atomicAdd(p.cnt_app + part, 1);
        atomicMax(p.last_app + part, s + 1);
        r = p.ref[part];
      }
    }
  }
  __syncthreads();
  // copy-on-write decision (see the file comment) and pages needed; the
  // writer counts are read only for a shared page
  bool cow = false;
  if (part >= 0 && r > 1)
    cow = !(p.cnt_app[part] == r && p.last_app[part] == s + 1);
  const int need =
      n > 0 ? (int)cow + pages_for(c + n, kPS) - pages_for(c, kPS) : 0;
  int total;
  const int off = block_exclusive_scan(need, sh, &total);
  const bool served = live && n > 0 && off + need <= top;
  if (live && n > 0 && !served) flag_error(err, DEVERR_POOL_EMPTY);
  // what a decode step launched next reads: only a sequence whose context
  // grew may append at its last position (any other would overwrite a
  // cached token there)
  if (live) p.grown[s] = served ? 1 : 0;
  int used;
  const int served_need = served ? need : 0;
  (void)block_exclusive_scan(served_need, sh, &used);
  int nslots;
  const int slot_off = block_exclusive_scan(served ? n : 0, sh, &nslots);

  // pops: stack[top-1-off], stack[top-2-off], ... (copy first)
  int job = -1;
  if (served) {
    int k = top - 1 - off;
    if (cow) {
      const int fresh = p.stack[k--];
      bt[(size_t)s * mb + c / kPS] = fresh;
      p.ref[fresh] = 1;
      atomicSub(p.ref + part, 1);
      job_old[s] = part;
      job_new[s] = fresh;
      job = s;
    }
    for (int b = pages_for(c, kPS); b < pages_for(c + n, kPS); ++b) {
      const int fresh = p.stack[k--];
      bt[(size_t)s * mb + b] = fresh;
      p.ref[fresh] = 1;
    }
    if (slot_mapping)
      for (int t = c; t < c + n; ++t)
        slot_mapping[slot_off + (t - c)] =
            bt[(size_t)s * mb + t / kPS] * kPS + t % kPS;
    ctx[s] = c + n;
  }
  // the scratch counters of every written page go back to zero
  __syncthreads();
  if (part >= 0) {
    p.cnt_app[part] = 0;
    p.last_app[part] = 0;
  }
  // copy-on-write copies: each job is one page of K and one of V
  int njobs;
  const int jpos = block_exclusive_scan(job >= 0 ? 1 : 0, sh, &njobs);
  __shared__ int jl_old[kThreads], jl_new[kThreads];
  if (job >= 0) {
    jl_old[jpos] = job_old[job];
    jl_new[jpos] = job_new[job];
  }
  __syncthreads();
  const int page_vec = kPS * row_bytes / 16;   // 16-byte vectors per page
  for (int j = 0; j < njobs; ++j) {
    const size_t src = (size_t)jl_old[j] * kPS * row_bytes;
    const size_t dst = (size_t)jl_new[j] * kPS * row_bytes;
    for (int v = threadIdx.x; v < page_vec; v += blockDim.x) {
      reinterpret_cast<uint4*>(k_pool + dst)[v] =
          reinterpret_cast<const uint4*>(k_pool + src)[v];
      reinterpret_cast<uint4*>(v_pool + dst)[v] =
          reinterpret_cast<const uint4*>(v_pool + src)[v];
    }
  }
  if (threadIdx.x == 0) {
    *p.top = top - used;
    *p.last_slots = nslots;
  }
}

// ---- fork ---------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    pool_fork_kernel(PoolView p, int32_t* bt, int mb, int32_t* ctx,
                     int num_seqs, const int32_t* src, const int32_t* dst,
                     int num_pairs, uint32_t* err) {
  const int kPS = *p.page_size;
  for (int i = 0; i < num_pairs; ++i) {
    const int a = src[i], b = dst[i];
    bool ok = a >= 0 && a < num_seqs && b >= 0 && b < num_seqs && a != b;
    int c = ok ? ctx[a] : 0;
    ok = ok && ctx[b] == 0 && c >= 0 && c <= mb * kPS;
    if (!ok) {
      if (threadIdx.x == 0) flag_error(err, DEVERR_BAD_SEQ);
      __syncthreads();
      continue;
    }
    const int np = pages_for(c, kPS);
    for (int k = threadIdx.x; k < mb; k += kThreads) {
      const int page = k < np ? bt[(size_t)a * mb + k] : -1;
      bt[(size_t)b * mb + k] = page;
      if (page >= 0 && page < p.num_pages) atomicAdd(p.ref + page, 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) ctx[b] = c;
    __syncthreads();
  }
}

// ---- release ------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    pool_release_kernel(PoolView p, int32_t* bt, int mb, int32_t* ctx,
                        int num_seqs, const int32_t* seqs, int num_release,
                        uint32_t* err) {
  constexpr int kList = 8192;   // freed pages sorted in shared memory
  __shared__ int sh[33];
  __shared__ int freed[kList];
  __shared__ int nfreed;
  const int kPS = *p.page_size;
  if (threadIdx.x == 0) nfreed = 0;
  __syncthreads();
  for (int i = 0; i < num_release; ++i) {
    const int s = seqs[i];
    if (s < 0 || s >= num_seqs) {
      if (threadIdx.x == 0) flag_error(err, DEVERR_BAD_SEQ);
      continue;
    }
    int c = ctx[s];
    c = c < 0 ? 0 : (c > mb * kPS ? mb * kPS : c);
    const int np = pages_for(c, kPS);
    for (int k = threadIdx.x; k < mb; k += kThreads) {
      if (k < np) {
        const int page = bt[(size_t)s * mb + k];
        if (page >= 0 && page < p.num_pages &&
            atomicSub(p.ref + page, 1) == 1) {
          p.last_app[page] = 1;   // freed in this call
          const int slot = atomicAdd(&nfreed, 1);
          if (slot < kList) freed[slot] = page;
        }
      }
      bt[(size_t)s * mb + k] = -1;
    }
    __syncthreads();
    if (threadIdx.x == 0) ctx[s] = 0;
    __syncthreads();
  }
  // push the freed pages in ascending id order
  const int top = *p.top;
  const int n = nfreed;
  auto push = [&](int pos, int page) {
    // a consistent pool never overflows; a corrupted one is flagged
    if (top + pos < p.num_pages)
      p.stack[top + pos] = page;
    else
      flag_error(err, DEVERR_BAD_SEQ);
    p.last_app[page] = 0;
  };
  if (n <= kList) {
    // bitonic sort of the list, padded to a power of two
    int m = 1;
    while (m < n) m <<= 1;
    for (int i = n + threadIdx.x; i < m; i += kThreads) freed[i] = INT32_MAX;
    __syncthreads();
    for (int k = 2; k <= m; k <<= 1) {
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = threadIdx.x; i < m; i += kThreads) {
          const int ij = i ^ j;
          if (ij > i) {
            const int x = freed[i], y = freed[ij];
            if (((i & k) == 0) == (x > y)) {
              freed[i] = y;
              freed[ij] = x;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = threadIdx.x; i < n; i += kThreads) push(i, freed[i]);
    if (threadIdx.x == 0) *p.top = min(top + n, p.num_pages);
    return;
  }
  // more than the list holds: scan the whole pool for the flags
  int base = 0;
  for (int i0 = 0; i0 < p.num_pages; i0 += kThreads) {
    const int page = i0 + threadIdx.x;
    const int f = (page < p.num_pages && p.last_app[page]) ? 1 : 0;
    int tot;
    const int pos = block_exclusive_scan(f, sh, &tot);
    if (f) push(base + pos, page);
    base += tot;
  }
  if (threadIdx.x == 0) *p.top = min(top + base, p.num_pages);
}

}  // namespace

cudaError_t launch_pool_init(int32_t* state, int num_pages, int page_size,
                             const int32_t* bt, int mb, const int32_t* ctx,
                             int num_seqs, uint32_t* err,
                             cudaStream_t stream) {
  const PoolView p = view(state, num_pages);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  pool_clear_kernel<<<sms, 256, 0, stream>>>(p);
  if (bt && num_seqs > 0)
    pool_count_refs_kernel<<<sms * 4, 256, 0, stream>>>(
        p, bt, mb, ctx, num_seqs, page_size, err);
  pool_stack_kernel<<<1, kThreads, 0, stream>>>(p, page_size);
  return cudaGetLastError();
}

cudaError_t launch_pool_append(int32_t* state, int num_pages, int page_size,
                               int32_t* bt, int mb, int32_t* ctx,
                               const int32_t* n_new, int num_seqs,
                               int32_t* slot_mapping, void* k_pool,
                               void* v_pool, int row_bytes, uint32_t* err,
                               cudaStream_t stream) {
  // one thread per sequence, whole warps (the scans' barriers are cheaper
  // over fewer warps)
  const int threads = num_seqs < 32 ? 32 : ((num_seqs + 31) / 32) * 32;
  pool_append_kernel<<<1, threads < kThreads ? threads : kThreads, 0, stream>>>(
      view(state, num_pages), bt, mb, ctx, n_new, num_seqs, slot_mapping,
      static_cast<uint8_t*>(k_pool), static_cast<uint8_t*>(v_pool),
      row_bytes, page_size, err);
  return cudaGetLastError();
}

cudaError_t launch_pool_fork(int32_t* state, int num_pages, int32_t* bt,
                             int mb, int32_t* ctx, int num_seqs,
                             const int32_t* src, const int32_t* dst,
                             int num_pairs, uint32_t* err,
                             cudaStream_t stream) {
  pool_fork_kernel<<<1, kThreads, 0, stream>>>(view(state, num_pages), bt, mb,
                                               ctx, num_seqs, src, dst,
                                               num_pairs, err);
  return cudaGetLastError();
}

cudaError_t launch_pool_release(int32_t* state, int num_pages, int32_t* bt,
                                int mb, int32_t* ctx, int num_seqs,
                                const int32_t* seqs, int num_release,
                                uint32_t* err, cudaStream_t stream) {
  pool_release_kernel<<<1, kThreads, 0, stream>>>(view(state, num_pages), bt,
                                                  mb, ctx, num_seqs, seqs,
                                                  num_release, err);
  return cudaGetLastError();
}

}  // namespace tv
