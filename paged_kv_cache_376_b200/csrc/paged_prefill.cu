// Chunked prefill over a paged KV cache on the tcgen05 tensor cores.
//
// What it computes ("tiny-vllm：从零构建高性能LLM推理引擎的完整指南", secs.
// "推理流程：从Prefill到Decode" -- prefill handles the prompt tokens in
// parallel and is compute bound --, "Llama 3.2 1B架构拆解" -- GQA, causal
// mask, softmax, weighted sum of V --, "PagedAttention：从操作系统借来的智慧"
// and "在线Softmax：数值稳定的注意力计算"): sequence s has T new query rows
// whose K,V are already appended; with C keys in its cache, row i (position
// P + i, P = C - T) attends to keys 0 .. P + i.  Tiled attention with an
// online softmax, tile sized to on-chip memory ("Tiny-vLLM 实战：用 C++/CUDA
// 手写高性能 LLM 推理引擎", sec. "算子融合", FlashAttention-like blocking).
//
// B200 design (one CTA per (KV head, block of 256 / G query rows, sequence);
// 12 warps; G = query heads per KV head, 1, 2, 4 or 8):
//  * An MMA tile has M = 128 rows = 128 / G query rows x the G query heads of
//    one KV head (32 x 4 for Llama-3.2-1B), so every K/V tile feeds G heads
//    (GQA reuse).  A CTA owns two such query tiles (A, then B) that share
//    every K/V tile, and the tensor core alternates between them while the
//    other tile's softmax runs.  q arrives by one 3-D TMA box {64 d, G heads,
//    128 / G rows} per tile; MMA row r is query row r / G, head r % G.
//  * Keys come in tiles of 64 = 4 pages; each page of one KV head (16 rows x
//    128 B) is one 2-D TMA box, 128-byte swizzled, so 4 boxes at 2 KB
//    offsets form exactly the canonical K-major SW128 operand.  Pages past
//    the range (or with a bad id) are read at an out-of-range coordinate and
//    arrive as zeros.
//  * P never goes through shared memory: the softmax writes P (bf16) back
//    into the tensor-memory columns its S came from, and P.V is issued with
//    A read from tensor memory, so the tensor core's shared-memory reads are
//    only q, K and V (with P in shared memory the MMAs were starved on
//    shared-memory bandwidth).  S/P is double-buffered per query tile and
//    K/V run through an 8-stage ring, so S_{j+1} is issued while tile j is
//    exponentiated and P_j.V_j while tile j+1 is.
//  * warp 0: TMA producer (q once, K/V ring; the eight page boxes of a key
//    tile go out in one warp instruction, one lane per box).
//    warps 1-3: three MMA-issuing threads.  Warp 3 issues S_t = Q_t K_j^T
//      (M128 N64 K16 x4) for both tiles into one of tile t's two S/P
//      buffers; warp 1 / warp 2 issue O_t += P_t V_j for tile A / B (M128
//      N64 K16 x4, once for P_hi and once for P_lo; V read as an MN-major
//      operand) accumulated in tile t's O.  Issuing a tcgen05.mma takes its
//      thread several times longer than the tensor core needs for one of
//      these small products, so a single issuer left the tensor core idle
//      most of the time; three independent instruction streams keep it fed.
//      Warp 1 also allocates the tensor memory.
//    warps 4-7 / 8-11: softmax of tile A / B.  Thread = one MMA row = one
//      (query, head).  It reads its 64 scores from tensor memory in one load,
//      moves the running maximum only when the tile's maximum exceeds it by
//      more than 2^8 (then O and l are rescaled in place, which is rare, so O
//      stays in tensor memory across key tiles), exponentiates, sums, and
//      stores P_hi / P_lo into the same 64 columns (32 each, two bf16 per
//      column).  After a row's first tile the running maximum is finite, so
//      the warp exponentiates against it and takes the tile maximum in the
//      same pass; only if some row's maximum grew by more than 2^8 does it
//      reload the scores and redo the tile with the rescale (the result is
//      the same either way: the offset rule does not change).  This removes
//      the maximum from the path between the score load and the
//      exponentials, the longest phase of the step after them.  The causal
//      mask is applied only to the tiles that cross the diagonal.
//  * P is split as P_hi = bf16(p), P_lo = bf16(p - P_hi) so the PV product
//    keeps ~16 bits of each weight (fp32-grade accumulation with bf16
//    operands); a single bf16 P carries 8 bits, which is not enough for rows
//    that see few keys.
//  * With a workspace, a one-CTA kernel first lists the (sequence, block)
//    items costliest first (cost = key tiles), and the attention grid
//    takes its work from that list, so that the longest blocks do not start
//    last and hold a few SMs while the rest idle.
//  * Every wait is an mbarrier wait bounded by a 2 s time limit.
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kD = 64;
constexpr int kPS = 16;
constexpr int kQTiles = 2;               // MMA tiles per CTA (A, B)
constexpr int kBM = kPrefillTileRows;    // 128 MMA rows = (128 / G) query rows x G heads
constexpr int kBN = 64;                  // keys per tile
constexpr int kPagesPerTile = kBN / kPS; // 4
constexpr int kST = 8;                   // K/V ring depth
constexpr int kRowBytes = kD * 2;        // 128
constexpr int kTileBytes = kBN * kRowBytes;  // 8 KB
constexpr int kPageBytes = kPS * kRowBytes;  // 2 KB
constexpr int kThreads = 384;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;   // S/P of tile t, buffer b: columns [64(2t+b), +64)
constexpr int kOCol = kQTiles * 2 * kBN;  // O of tile t: [256 + 64t, +64)
constexpr float kRescaleThreshold = 8.f; // log2 units: rescale when max grows > 2^8

constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD, true);

struct PrefillSmem {
  alignas(1024) uint8_t q[kQTiles][kBM * kRowBytes];        // 32 KB
  alignas(1024) uint8_t k[kST][kTileBytes];                 // 64 KB
  alignas(1024) uint8_t v[kST][kTileBytes];                 // 64 KB
  alignas(8) uint64_t q_full;
  uint64_t kv_full[kST], kv_empty[kST];
  uint64_t s_full[kQTiles][2], p_full[kQTiles][2], o_done[kQTiles][2];
  uint64_t drain[3];   // error path: each MMA issuer's own MMAs have finished
  uint32_t tmem_base;
  uint32_t bad_pages[kST];
};

// ---- dispatch order ------------------------------------------------------------
// The cost of a CTA is its number of key tiles, (P + last row + 1) / 64 rounded
// up, so within one launch CTAs differ by up to the longest context / 64 tiles.
// Dispatched in grid order, the costliest can start last and hold a few SMs
// while the rest idle.  This kernel (one CTA) lists the (sequence, block) items
// costliest first by a counting sort: a histogram of the costs in shared memory,
// an exclusive scan in descending cost order, then every item takes the next
// slot of its cost.  Items of equal cost land in an unspecified order; the
// prefill's results do not depend on the order, only its timing does.
constexpr int kOrderThreads = 1024;
constexpr int kCostBuckets = 4096;                // costs above share the top
constexpr int kBucketsPerThread = kCostBuckets / kOrderThreads;

__device__ __forceinline__ int prefill_cost(const PrefillArgs& a, int item,
                                            int nblk) {
  const int seq = item / nblk;
  const int blk = item - seq * nblk;
  const int T = a.query_start_loc[seq + 1] - a.query_start_loc[seq];
  const int ctx = min(a.context_lens[seq],
                      a.max_blocks_per_seq * (kPS << a.page_shift));
  const int rows = prefill_rows_per_cta(a.group);
  const int q0 = blk * rows;
  if (T <= 0 || q0 >= T || T > ctx) return 0;    // no work (or flagged)
  const int tiles =
      (ctx - T + min(q0 + rows, T) + kBN - 1) / kBN;
  return min(tiles, kCostBuckets - 1);
}

__global__ void __launch_bounds__(kOrderThreads, 1)
    prefill_order_kernel(const PrefillArgs a) {
  __shared__ int slot[kCostBuckets];   // histogram, then next free position
  __shared__ int warp_sum[kOrderThreads / 32];
  const int nblk = prefill_blocks(a.max_query_len, a.group);
  const int n = a.num_seqs * nblk;
  for (int i = threadIdx.x; i < kCostBuckets; i += kOrderThreads) slot[i] = 0;
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kOrderThreads)
    atomicAdd(&slot[prefill_cost(a, i, nblk)], 1);
  __syncthreads();
  // thread t owns the buckets of costs kCostBuckets-1-4t down to ...-4t-3
  int own[kBucketsPerThread];
  int sum = 0;
#pragma unroll
  for (int k = 0; k < kBucketsPerThread; ++k) {
    own[k] = slot[kCostBuckets - 1 - (threadIdx.x * kBucketsPerThread + k)];
    sum += own[k];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int w = warp_sum[lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, w, d);
      if (lane >= d) w += v;
    }
    warp_sum[lane] = w;   // inclusive over warps
  }
  __syncthreads();
  int start = incl - sum + (warp > 0 ? warp_sum[warp - 1] : 0);
#pragma unroll
  for (int k = 0; k < kBucketsPerThread; ++k) {
    slot[kCostBuckets - 1 - (threadIdx.x * kBucketsPerThread + k)] = start;
    start += own[k];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += kOrderThreads)
    a.order[atomicAdd(&slot[prefill_cost(a, i, nblk)], 1)] = i;
}

template <int kG>   // query heads per KV head
__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const PrefillArgs a,
                         const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
  constexpr int kQRows = kBM / kG;         // query rows per MMA tile
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  uint8_t* base = smem_dyn + ((1024 - (smem_u32(smem_dyn) & 1023)) & 1023);
  auto& sm = *reinterpret_cast<PrefillSmem*>(base);

  const int kvh = blockIdx.x;
  int blk = gridDim.y - 1 - blockIdx.y;    // heaviest blocks of a sequence first
  int seq = blockIdx.z;
  if (a.order) {                           // costliest (sequence, block) first
    const int item = a.order[blockIdx.y + gridDim.y * blockIdx.z];
    seq = item / gridDim.y;
    blk = item - seq * gridDim.y;
  }
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work of this CTA (uniform across the block) ---------------------------
  const int qs = a.query_start_loc[seq];
  const int T = a.query_start_loc[seq + 1] - qs;
  int ctx = a.context_lens[seq];
  // a page holds 1 << page_shift blocks of 16 tokens, each one TMA box
  const int ctx_cap = a.max_blocks_per_seq * (kPS << a.page_shift);
  const int q0 = blk * kQRows * kQTiles;
  if (q0 >= T) return;
  if (ctx > ctx_cap) {
    if (threadIdx.x == 0) flag_error(a.err, DEVERR_BAD_CONTEXT);
    ctx = ctx_cap;
  }
  if (T < 0 || T > ctx || qs < 0 || qs + T > a.num_query_rows) {
    if (threadIdx.x == 0) flag_error(a.err, DEVERR_BAD_QUERY);
    return;
  }
  const int P = ctx - T;                      // cached prefix length
  // tile t covers query rows [q0 + 32t, q0 + 32t + 32) of the chunk
  int n_tiles_of[kQTiles];
#pragma unroll
  for (int t = 0; t < kQTiles; ++t) {
    const int lo = q0 + t * kQRows;
    const int hi = min(lo + kQRows, T);
    n_tiles_of[t] = hi > lo ? (P + hi + kBN - 1) / kBN : 0;
  }
  const int n_tiles = max(n_tiles_of[0], n_tiles_of[1]);
  const int n_keys = P + min(q0 + kQRows * kQTiles, T);   // keys loaded
  const int n_pages = (n_keys + kPS - 1) / kPS;
  const int32_t* bt = a.block_tables + (size_t)seq * a.max_blocks_per_seq;

  // ---- set-up ------------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int i = 0; i < kST; ++i) {
      mbar_init(smem_u32(&sm.kv_full[i]), 1);
      mbar_init(smem_u32(&sm.kv_empty[i]), 3);   // three issuers
    }
    for (int t = 0; t < kQTiles; ++t) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_u32(&sm.s_full[t][b]), 1);
        mbar_init(smem_u32(&sm.p_full[t][b]), 4);
        mbar_init(smem_u32(&sm.o_done[t][b]), 1);
      }
    }
    for (int i = 0; i < 3; ++i) mbar_init(smem_u32(&sm.drain[i]), 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0) {
    // ======================= TMA producer =====================================
    // Lane 2p + w (p < 4; w = 0: K, 1: V) issues page p's box of K or V, so
    // one warp instruction issues a key tile's eight boxes and one load by
    // lanes 0-3 fetches its four page ids (measured 2 % faster than one
    // thread issuing the eight boxes in turn).
    if (lane == 0) {
      const uint32_t qbar = smem_u32(&sm.q_full);
      mbar_arrive_expect_tx(qbar, kQTiles * kBM * kRowBytes);
#pragma unroll
      for (int t = 0; t < kQTiles; ++t)
        tma_load_3d(smem_u32(sm.q[t]), &tm_q, 0, kvh * kG,
                    qs + q0 + t * kQRows, qbar);
    }
    const int oob_row = (a.num_pages << a.page_shift) * kPS;  // zeros
    const int pp = (lane >> 1) & (kPagesPerTile - 1);
    const bool is_v = lane & 1;
    const bool issuer = lane < 2 * kPagesPerTile;
    const CUtensorMap* tmap = is_v ? &tm_v : &tm_k;
    for (int j = 0; j < n_tiles; ++j) {
      const int st = j % kST;
      if (j >= kST &&
          !__all_sync(0xffffffffu, mbar_wait(smem_u32(&sm.kv_empty[st]),
                                             ((j / kST) + 1) & 1))) {
        if (lane == 0) {
          flag_error(a.err, DEVERR_TIMEOUT);
          // before giving up, let the copies this warp issued land (bounded
          // waits): the last tile of every stage, then q
          for (int jl = j - kST; jl < j; ++jl)
            mbar_wait(smem_u32(&sm.kv_full[jl % kST]), (jl / kST) & 1);
          mbar_wait(smem_u32(&sm.q_full), 0);
        }
        break;
      }
      // lane p < 4 looks up page p of the tile
      int y = oob_row;
      bool badp = false;
      if (lane < kPagesPerTile) {
        const int lp = j * kPagesPerTile + lane;
        if (lp < n_pages) {
          const int pid = __ldg(bt + (lp >> a.page_shift));
          if (pid >= 0 && pid < a.num_pages) {
            y = ((pid << a.page_shift) + (lp & ((1 << a.page_shift) - 1))) * kPS;
          } else {
            badp = true;
          }
        }
      }
      const uint32_t bad = __ballot_sync(0xffffffffu, badp);
      const int row = __shfl_sync(0xffffffffu, y, pp);
      const uint32_t bar = smem_u32(&sm.kv_full[st]);
      if (lane == 0) {
        if (bad) flag_error(a.err, DEVERR_BAD_PAGE);
        sm.bad_pages[st] = bad;
        mbar_arrive_expect_tx(bar, 2 * kTileBytes);
      }
      __syncwarp();
      if (issuer)
        tma_load_2d(smem_u32(is_v ? sm.v[st] : sm.k[st]) + pp * kPageBytes, tmap,
                    kvh * kD, row, bar);
    }
  } else if (warp >= 1 && warp <= 3) {
    // ======================= MMA issuers ======================================
    // warp 3 issues S = Q K^T for both query tiles; warps 1 / 2 issue
    // O += P V for tile A / B.  A tcgen05.mma costs its issuing thread far
    // more time than the tensor core needs for an M128 N64 K16 product, so
    // the three instruction streams run in parallel.  tcgen05.commit tracks
    // only the committing thread's own MMAs, so every issuer signals its own
    // barriers; the K/V stage of tile j is free after all three arrived.
    // Barrier X[t][b] serves the tiles j with j % 2 == b; its (j / 2)-th
    // phase belongs to tile j, so a wait for tile j uses parity (j >> 1) & 1.
    if (lane == 0) {
      bool ok = true;
      if (warp == 3) {
        ok = mbar_wait(smem_u32(&sm.q_full), 0);
        for (int j = 0; ok && j < n_tiles; ++j) {
          if (!mbar_wait(smem_u32(&sm.kv_full[j % kST]), (j / kST) & 1)) {
            ok = false;
            break;
          }
          const int b = j & 1;
          bool any = false;
#pragma unroll
          for (int t = 0; t < kQTiles; ++t) {
            if (j >= n_tiles_of[t]) continue;
            // S/P buffer b holds P of tile j - 2 until its P.V has completed
            if (j >= 2 &&
                !mbar_wait(smem_u32(&sm.o_done[t][b]), ((j - 2) >> 1) & 1)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t q_addr = smem_u32(sm.q[t]);
            const uint32_t k_addr = smem_u32(sm.k[j % kST]);
#pragma unroll
            for (int k = 0; k < kD / 16; ++k) {
              const uint64_t ad = smem_desc_sw128(q_addr + k * 32, 16, 1024);
              const uint64_t bd = smem_desc_sw128(k_addr + k * 32, 16, 1024);
              tc_mma_bf16(tmem + kSCol + (2 * t + b) * kBN, ad, bd, kIdescQK,
                          k > 0);
            }
            tc_commit(smem_u32(&sm.s_full[t][b]));
            any = true;
          }
          if (!ok) break;
          if (any) tc_commit(smem_u32(&sm.kv_empty[j % kST]));
          else mbar_arrive(smem_u32(&sm.kv_empty[j % kST]));
        }
      } else {
        const int t = warp - 1;
        for (int j = 0; ok && j < n_tiles; ++j) {
          const int st = j % kST;
          // every issuer waits for tile j's stage before releasing it, so
          // that no issuer arrives twice in one phase of kv_empty
          if (!mbar_wait(smem_u32(&sm.kv_full[st]), (j / kST) & 1)) {
            ok = false;
            break;
          }
          if (j < n_tiles_of[t]) {
            const int b = j & 1;
            // P of tile j is in tensor memory; where tile A's softmax zeroes
            // stale V rows of this key tile, tile B's P.V also waits for it
            const int key0 = j * kBN;
            const bool zeroed = max(ctx, key0) < min(n_pages * kPS, key0 + kBN);
            if (!mbar_wait(smem_u32(&sm.p_full[t][b]), (j >> 1) & 1) ||
                (t == 1 && zeroed && j < n_tiles_of[0] &&
                 !mbar_wait(smem_u32(&sm.p_full[0][b]), (j >> 1) & 1))) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t v_addr = smem_u32(sm.v[st]);
            const uint32_t p_col = tmem + kSCol + (2 * t + b) * kBN;
#pragma unroll
            for (int part = 0; part < 2; ++part) {          // P_hi, then P_lo
#pragma unroll
              for (int k = 0; k < kBN / 16; ++k) {
                // A = P in tensor memory: keys [16k, 16k+16) = 8 columns
                const uint32_t a_tmem = p_col + part * (kBN / 2) + k * 8;
                // B = V: MN-major (head dim contiguous); 16 keys = 2 x 8 rows
                const uint64_t bd = smem_desc_sw128(v_addr + k * 16 * kRowBytes,
                                                    kTileBytes, 1024);
                tc_mma_bf16_ts(tmem + kOCol + t * kD, a_tmem, bd, kIdescPV,
                               (j | part | k) != 0);
              }
            }
            tc_commit(smem_u32(&sm.o_done[t][b]));
            tc_commit(smem_u32(&sm.kv_empty[st]));
          } else {
            mbar_arrive(smem_u32(&sm.kv_empty[st]));
          }
        }
      }
      if (!ok) {
        flag_error(a.err, DEVERR_TIMEOUT);
        // before giving up, let this thread's MMAs finish (bounded wait), so
        // that none still writes tensor memory when it is freed
        tc_commit(smem_u32(&sm.drain[warp - 1]));
        mbar_wait(smem_u32(&sm.drain[warp - 1]), 0);
      }
    }
  } else if (warp >= 4) {
    // ======================= softmax warpgroups ===============================
    const int t = (warp >> 2) - 1;           // query tile: 0 = A, 1 = B
    const int quarter = warp & 3;            // tensor-memory lane quarter
    const int r = quarter * 32 + lane;       // MMA row
    const int qt0 = q0 + t * kQRows;         // first chunk row of this tile
    const int qi = r / kG;                   // query row within the tile
    const int hh = r % kG;                   // head within the group
    const bool row_real = qt0 + qi < T;
    const int limit = row_real ? P + qt0 + qi : ctx - 1;  // last visible key
    const int my_tiles = n_tiles_of[t];
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const uint32_t s_addr = tmem + lane_base + kSCol + 2 * t * kBN;
    const uint32_t o_addr = tmem + lane_base + kOCol + t * kD;
    const float c = a.scale_log2;

    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < my_tiles; ++j) {
      const int b = j & 1;
      const int st = j % kST;
      const int key0 = j * kBN;
      // every row of the tile sees every key of key tile j?
      const bool full_tile = key0 + kBN - 1 <= P + qt0;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(smem_u32(&sm.s_full[t][b]), (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
      tmem_ld64(s_addr + b * kBN, s);
      const uint32_t bad = sm.bad_pages[st];
      const bool masked = !(full_tile && bad == 0);
      auto apply_mask = [&]() {
#pragma unroll
        for (int x = 0; x < kBN; ++x) {
          const int key = key0 + x;
          const bool vis = key <= limit && !((bad >> (x / kPS)) & 1u);
          s[x] = vis ? s[x] : -INFINITY;
        }
      };
      if (masked) apply_mask();

      // packed fp32x2 arithmetic: one instruction per pair of keys
      float2 lsum2 = make_float2(0.f, 0.f);
      const float2 c2 = make_float2(c, c);
      const float2 neg1 = make_float2(-1.f, -1.f);
      uint32_t hi[kBN / 2], lo[kBN / 2];
      // ---- after a row's first tile the running max is finite: exponentiate
      //      against it while taking the tile maximum in the same pass; only
      //      when a row's maximum grew by more than 2^8 is the tile redone
      //      (S is still in tensor memory) with the rescale below ------------
      bool exact = !__all_sync(0xffffffffu, m_run != -INFINITY);
      if (!exact) {
        float mx = -INFINITY;
        const float2 nm2 = make_float2(-m_run, -m_run);
#pragma unroll
        for (int e = 0; e < kBN / 2; ++e) {
          mx = fmax3(mx, s[2 * e], s[2 * e + 1]);
          const float2 t = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), c2,
                                      nm2);
          const float2 x = make_float2(fast_exp2(t.x), fast_exp2(t.y));
          lsum2 = __fadd2_rn(lsum2, x);
          hi[e] = pack_bf16x2(x.x, x.y);
          const float2 h = make_float2(bf16_lo(hi[e]), bf16_hi(hi[e]));
          const float2 r = __ffma2_rn(h, neg1, x);   // x - hi, exact
          lo[e] = pack_bf16x2(r.x, r.y);
        }
        exact = __any_sync(0xffffffffu, mx * c > m_run + kRescaleThreshold);
        if (exact) {
          tmem_ld64(s_addr + b * kBN, s);
          if (masked) apply_mask();
        }
      }
      if (exact) {
      float mx = -INFINITY;
#pragma unroll
      for (int x = 0; x < kBN; x += 2) mx = fmax3(mx, s[x], s[x + 1]);
      const float m_tile = mx * c;   // scale > 0, so max commutes with it

      // ---- lazy rescale: move the running max only when it grows > 2^8 ----------
      const bool grow = m_tile > m_run + kRescaleThreshold;
      if (__any_sync(0xffffffffu, grow)) {
        const float m_new = grow ? m_tile : m_run;
        const float alpha = fast_exp2(m_run - m_new);   // 0 when m_run = -inf
        l_run *= alpha;
        m_run = m_new;
        if (j >= 1) {   // O holds tiles < j once P.V of tile j-1 is done
          if (!__all_sync(0xffffffffu,
                          mbar_wait(smem_u32(&sm.o_done[t][(j - 1) & 1]),
                                    ((j - 1) >> 1) & 1))) {
            ok = false;
            break;
          }
          tc_fence_after();
          float o[64];
          tmem_ld64(o_addr, o);
#pragma unroll
          for (int d = 0; d < 64; ++d) o[d] *= alpha;
          tmem_st64(o_addr, o);
        }
      }
      const float m_use = m_run == -INFINITY ? 0.f : m_run;

      // ---- exponentials, row sum, P_hi / P_lo back into the S columns ------------
      const float2 nm2 = make_float2(-m_use, -m_use);
      lsum2 = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < kBN / 2; ++e) {
        const float2 t = __ffma2_rn(make_float2(s[2 * e], s[2 * e + 1]), c2,
                                    nm2);
        const float2 x = make_float2(fast_exp2(t.x), fast_exp2(t.y));
        lsum2 = __fadd2_rn(lsum2, x);
        hi[e] = pack_bf16x2(x.x, x.y);
        const float2 h = make_float2(bf16_lo(hi[e]), bf16_hi(hi[e]));
        const float2 r = __ffma2_rn(h, neg1, x);   // x - hi, exact
        lo[e] = pack_bf16x2(r.x, r.y);
      }
      }
      const float lsum = lsum2.x + lsum2.y;
      tmem_st32(s_addr + b * kBN, hi);
      tmem_st32(s_addr + b * kBN + kBN / 2, lo);
      l_run += lsum;

      // ---- keys past the context in a loaded page may hold stale data: zero
      //      their V rows (once per key tile: by tile A where it has this
      //      key tile, else by B; tile B's P.V on a key tile that A zeroes
      //      waits for A's P as well) so that P = 0 cannot meet NaN ----
      if (t == 0 || j >= n_tiles_of[0]) {
        const int z0 = max(ctx, key0);
        const int z1 = min(n_pages * kPS, key0 + kBN);
        const int nz = (z1 - z0) * (kRowBytes / 16);
        for (int i = threadIdx.x - 128 * (t + 1); i < nz; i += 128) {
          const int row = z0 - key0 + i / (kRowBytes / 16);
          const int chn = i % (kRowBytes / 16);
          *reinterpret_cast<uint4*>(&sm.v[st][row * kRowBytes + chn * 16]) =
              make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();   // the zeroed V rows, for the MMA
      tc_fence_before();          // the P stores, for the MMA
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[t][b]));
    }

    // ---- wait for the last P.V, normalise and store --------------------------------
    float o[64];
    if (ok && my_tiles > 0 &&
        __all_sync(0xffffffffu,
                   mbar_wait(smem_u32(&sm.o_done[t][(my_tiles - 1) & 1]),
                             ((my_tiles - 1) >> 1) & 1))) {
      tc_fence_after();
      tmem_ld64(o_addr, o);
    } else {
      if (my_tiles > 0 && lane == 0) flag_error(a.err, DEVERR_TIMEOUT);
#pragma unroll
      for (int d = 0; d < 64; ++d) o[d] = 0.f;
      l_run = 0.f;
    }
    if (row_real && my_tiles > 0) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* dst =
          a.out + ((size_t)(qs + qt0 + qi) * a.num_q_heads + kvh * kG + hh) * kD;
#pragma unroll
      for (int ch = 0; ch < kD / 8; ++ch) {
        uint4 w;
        w.x = pack_bf16x2(o[ch * 8 + 0] * inv, o[ch * 8 + 1] * inv);
        w.y = pack_bf16x2(o[ch * 8 + 2] * inv, o[ch * 8 + 3] * inv);
        w.z = pack_bf16x2(o[ch * 8 + 4] * inv, o[ch * 8 + 5] * inv);
        w.w = pack_bf16x2(o[ch * 8 + 6] * inv, o[ch * 8 + 7] * inv);
        reinterpret_cast<uint4*>(dst)[ch] = w;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem, kTmemCols);
}

}  // namespace

cudaError_t launch_paged_prefill(const PrefillArgs& a, const CUtensorMap& tq,
                                 const CUtensorMap& tk, const CUtensorMap& tv,
                                 cudaStream_t stream) {
  const int smem = sizeof(PrefillSmem) + 1024;
  auto kern = a.group == 1   ? paged_prefill_kernel<1>
              : a.group == 2 ? paged_prefill_kernel<2>
              : a.group == 8 ? paged_prefill_kernel<8>
                             : paged_prefill_kernel<4>;
  if (a.group != 1 && a.group != 2 && a.group != 4 && a.group != 8)
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (a.order) {
    prefill_order_kernel<<<1, kOrderThreads, 0, stream>>>(a);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const int blocks = prefill_blocks(a.max_query_len, a.group);
  dim3 grid(a.num_kv_heads, blocks, a.num_seqs);
  kern<<<grid, kThreads, smem, stream>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace tv
