// Paged decode attention over a block-table KV cache, unsplit and split-KV.
//
// What it computes ("tiny-vllm：从零构建高性能LLM推理引擎的完整指南",
// secs. "PagedAttention：从操作系统借来的智慧", "推理流程：从Prefill到Decode",
// "在线Softmax：数值稳定的注意力计算", "Llama 3.2 1B架构拆解"): for every
// sequence s and query head h, the single new query attends to the keys
// 0 .. context_len-1 of its KV head h / G, found page by page through the
// block table; softmax(scale * q.K) weights the V rows.  Storage is bf16,
// every sum is fp32 ("Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎",
// sec. "CUDA Kernel 优化", item 3).
//
// B200 design.
//  * One CTA per (KV head, sequence[, partition]).  Each K/V page slice it
//    needs is 16 rows x 128 B (one KV head of a [page][16][Hkv][64] page) and
//    is staged in shared memory by one 2-D TMA box per tensor, so the G query
//    heads of the group reuse it from shared memory (GQA reuse).
//  * Four warps per CTA, each with a private ring of kStages page slots and
//    one mbarrier per slot; warp w takes pages w, w+4, w+8, ... so no warp
//    ever waits for another until the final combine.  Block-table entries
//    are prefetched 32 at a time, one per lane, ahead of the TMA issue.
//  * Inside a warp: lane = 8*g + c; lane-group g owns tokens g, g+4, g+8,
//    g+12 of the page, lane c owns head dims [8c, 8c+8).  QK partial dots
//    are summed across the 8 lanes of a group with xor-shuffles; the softmax
//    is online per page in base 2 (q is pre-scaled by scale*log2(e)): one
//    max and one rescale per page, not per token.
//  * The split variant writes the normalised partial output and the natural
//    log-sum-exp of each 512-token (or any multiple of 16) partition; the
//    merge kernel (split_merge.cu) combines them.
//  * The append variant fuses the KV append of the decode step ("推理流程":
//    compute the new token's K,V, append them, then attend): the warp that
//    owns the page holding position context_len-1 writes the new token's row
//    of its KV head into the pool and into its staged copy of that page, so
//    the step is one launch and the new row is never read back from HBM;
//    with a cos/sin table it rotates that K row by RoPE first.
#include "tv_decode.cuh"
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kD = 64;          // head_dim
constexpr int kPS = 16;         // page_size
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRowBytes = kD * 2;                 // one token, one KV head
constexpr int kSliceBytes = kPS * kRowBytes;      // 2 KB
constexpr int kStageBytes = 2 * kSliceBytes;      // K slice + V slice
constexpr float kLazy = 8.f;   // log2 of the growth the running sums allow

template <int kStages>
struct DecodeSmem {
  alignas(128) uint8_t ring[kWarps][kStages][kStageBytes];
  alignas(8) uint64_t full[kWarps][kStages];
};

template <int G>
struct Combine {  // per-warp results handed to the final combine
  float m[kWarps][G];
  float l[kWarps][G];
  float acc[kWarps][G][kD];
};

template <int G, int kStages, bool kSplit, bool kAppend>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 4 : 2)
    paged_decode_kernel(const DecodeArgs a,
                        const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v) {
  static_assert(sizeof(Combine<G>) <= sizeof(DecodeSmem<kStages>::ring),
                "combine buffer must fit in the ring");
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  // 1 KB of slack is requested at launch; align the carve-out by hand.
  uint8_t* smem_raw = smem_dyn + ((1024 - (smem_u32(smem_dyn) & 1023)) & 1023);
  auto& sm = *reinterpret_cast<DecodeSmem<kStages>*>(smem_raw);

  const int kvh = blockIdx.x;
  const int seq = blockIdx.y;
  const int part = kSplit ? blockIdx.z : 0;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 3;   // token sub-group
  const int chk = lane & 7;    // 16-byte chunk of the head dim

  // ---- token range of this CTA --------------------------------------------
  // a decode step (tv_decode_step) treats a sequence whose context did not
  // grow as idle: appending at ctx-1 would overwrite a cached token
  int ctx = (a.grown && a.grown[seq] == 0) ? 0 : a.context_lens[seq];
  // A page holds 1 << page_shift blocks of 16 tokens; the kernel streams
  // blocks, and a block's 16 rows are one TMA box at row (page << shift |
  // sub-block) * 16 of the pool.
  const int ctx_cap = a.max_blocks_per_seq * (kPS << a.page_shift);
  const int num_blocks = a.num_pages << a.page_shift;
  if (ctx < 0 || ctx > ctx_cap) {
    if (threadIdx.x == 0) flag_error(a.err, DEVERR_BAD_CONTEXT);
    ctx = ctx < 0 ? 0 : ctx_cap;
  }
  int tok_begin = 0, tok_end = ctx;
  if (kSplit) {
    tok_begin = part * a.partition_tokens;
    tok_end = min(ctx, tok_begin + a.partition_tokens);
    if (tok_end < tok_begin) tok_end = tok_begin;
  }
  const int first_page = tok_begin / kPS;
  const int n_pages = (tok_end - tok_begin + kPS - 1) / kPS;
  // pages of this warp: first_page + warp + kWarps * i, i < my_n
  const int my_n = n_pages > warp ? (n_pages - warp + kWarps - 1) / kWarps : 0;
  const int32_t* bt = a.block_tables + (size_t)seq * a.max_blocks_per_seq;
  const int sub_mask = (1 << a.page_shift) - 1;

  // ---- fused append: the new token is at position ctx-1 (unsplit kernel) ---
  int app_i = -1;            // local page index of the appended row, this warp
  int app_r = 0;             // its row within the page
  uint4 app_row = make_uint4(0, 0, 0, 0);  // lanes 0-7: K chunk, 8-15: V chunk
  if (kAppend && ctx > 0) {
    const int lp = (ctx - 1) / kPS;
    if (lp % kWarps == warp) {
      app_i = lp / kWarps;
      app_r = (ctx - 1) % kPS;
      if (lane < 16) {
        const __nv_bfloat16* src =
            (lane < 8 ? a.k_new : a.v_new) +
            ((size_t)seq * gridDim.x + kvh) * kD + chk * 8;
        app_row = *reinterpret_cast<const uint4*>(src);
      }
      if (a.rope_cos_sin) {
        // RoPE of the new K row at its position: lane c < 8 holds dimensions
        // 8c .. 8c+7, so lanes c and c ^ 4 hold the two halves of the pairs
        // (i, i + 32); each rotates its pair and keeps its own half
        uint4 other;
        other.x = __shfl_xor_sync(0xffffffffu, app_row.x, 4);
        other.y = __shfl_xor_sync(0xffffffffu, app_row.y, 4);
        other.z = __shfl_xor_sync(0xffffffffu, app_row.z, 4);
        other.w = __shfl_xor_sync(0xffffffffu, app_row.w, 4);
        const int pos = ctx - 1;
        if (lane < 8) {
          if (pos < a.rope_max_position) {
            float c8[8], s8[8];
            rope_load8(a.rope_cos_sin, pos, 8 * (lane & 3), c8, s8);
            uint4 lo = lane < 4 ? app_row : other;
            uint4 hi = lane < 4 ? other : app_row;
            rope_rotate8(lo, hi, c8, s8);
            app_row = lane < 4 ? lo : hi;
          } else if (lane == 0) {
            flag_error(a.err, DEVERR_BAD_POSITION);
          }
        }
      }
    }
  }

  // ---- barriers ------------------------------------------------------------
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&sm.full[warp][s]), 1);
    fence_mbar_init();
  }
  __syncwarp();

  // ---- q for the G heads of this KV head, pre-scaled by scale*log2(e) -----
  // Element pairs (2i, 2i+1) of this lane's 8-element chunk, as float2 so
  // the dot products run on the packed fp32x2 FMA pipe.  Position h holds
  // head h ^ rs_mask (the order reduce_scatter8 expects).
  const int qmask = rs_mask<G>(chk);
  float2 q2[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 v = *reinterpret_cast<const uint4*>(
        a.q + ((size_t)seq * a.num_q_heads + kvh * G + (h ^ qmask)) * kD +
        chk * 8);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i)
      q2[h][i] = make_float2(bf16_lo(w[i]) * a.scale_log2,
                             bf16_hi(w[i]) * a.scale_log2);
  }

  // After the reduce-scatter below, lane chunk c holds the score of head
  // c >> kShift (lanes that share a head hold the same value); head h is
  // read from lane (group, h << kShift).
  constexpr int kShift = G == 8 ? 0 : G == 4 ? 1 : G == 2 ? 2 : 3;
  const int my_head = chk >> kShift;

  float m_run = -INFINITY, l_run = 0.f;   // for head my_head
  float2 acc2[G][4];                      // all heads, this lane's 8 dims
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc2[h][i] = make_float2(0.f, 0.f);

  // Pool blocks of this warp's 16-token blocks, 32 per batch, one per lane
  // (-1 when the block-table entry is not a page of the pool).
  auto load_pids = [&](int batch) -> int {
    const int i = batch * 32 + lane;
    if (i >= my_n) return 0;
    const int b = first_page + warp + kWarps * i;
    const int page = __ldg(bt + (b >> a.page_shift));
    return page >= 0 && page < a.num_pages
               ? (page << a.page_shift) + (b & sub_mask) : -1;
  };
  int pid_cur = load_pids(0);
  int pid_next = load_pids(1);
  const uint64_t policy = l2_policy_evict_first();

  auto issue = [&](int pid, int stage) {
    const bool ok = pid >= 0 && pid < num_blocks;
    if (!ok) flag_error(a.err, DEVERR_BAD_PAGE);
    const int y = (ok ? pid : 0) * kPS;
    const uint32_t bar = smem_u32(&sm.full[warp][stage]);
    const uint32_t dst = smem_u32(&sm.ring[warp][stage][0]);
    mbar_arrive_expect_tx(bar, kStageBytes);
    tma_load_2d_hint(dst, &tm_k, kvh * kD, y, bar, policy);
    tma_load_2d_hint(dst + kSliceBytes, &tm_v, kvh * kD, y, bar, policy);
  };

  // prologue: fill the ring
#pragma unroll
  for (int j = 0; j < kStages; ++j) {
    const int pid = __shfl_sync(0xffffffffu, pid_cur, j);
    if (lane == 0 && j < my_n) issue(pid, j);
  }

  bool failed = false;
  int issued = min(my_n, kStages);
  int i = 0;
  for (; i < my_n; ++i) {
    const int stage = i % kStages;
    const uint32_t parity = (i / kStages) & 1;
    if ((i & 31) == 0 && i > 0) {
      pid_cur = pid_next;
      pid_next = load_pids((i >> 5) + 1);
    }
    const int pid = __shfl_sync(0xffffffffu, pid_cur, i & 31);
    const bool page_ok = pid >= 0 && pid < num_blocks;
    const int page_tok0 = (first_page + warp + kWarps * i) * kPS;
    // warp-uniform: every token of the page is a real key of this range
    const bool full_page = page_ok && page_tok0 + kPS <= tok_end;

    // Every lane observes the barrier (acquire of the TMA bytes); the
    // outcome is made warp-uniform so the warp never diverges on it.
    if (!__all_sync(0xffffffffu,
                    mbar_wait(smem_u32(&sm.full[warp][stage]), parity))) {
      failed = true;
      break;
    }
    uint8_t* kbase = &sm.ring[warp][stage][0];
    uint8_t* vbase = kbase + kSliceBytes;
    if (kAppend && i == app_i) {
      // the staged page now gets the new row; the pool keeps it for later
      if (page_ok && lane < 16) {
        uint8_t* dst = &sm.ring[warp][stage][(lane < 8 ? 0 : kSliceBytes) +
                                             app_r * kRowBytes + chk * 16];
        *reinterpret_cast<uint4*>(dst) = app_row;
        __nv_bfloat16* pool = lane < 8 ? a.k_pool_w : a.v_pool_w;
        *reinterpret_cast<uint4*>(
            pool + (((size_t)pid * kPS + app_r) * gridDim.x + kvh) * kD +
            chk * 8) = app_row;
      }
      __syncwarp();
    }
    if (!full_page) {
      // Rows past the range (or the whole of a bad page) get p = 0; zero
      // their V so that 0 * a stale NaN never reaches the sum.  Each lane
      // clears exactly the rows and chunk it reads below.
#pragma unroll
      for (int r = grp; r < kPS; r += 4)
        if (!(page_ok && page_tok0 + r < tok_end))
          *reinterpret_cast<uint4*>(vbase + r * kRowBytes + chk * 16) =
              make_uint4(0, 0, 0, 0);
    }

    // ---- scores: token it*4+grp, head my_head ---------------------------------
    float s[4];
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int r = it * 4 + grp;
      const uint4 kv =
          *reinterpret_cast<const uint4*>(kbase + r * kRowBytes + chk * 16);
      const uint32_t w[4] = {kv.x, kv.y, kv.z, kv.w};
      float2 k2[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) k2[t] = make_float2(bf16_lo(w[t]), bf16_hi(w[t]));
      float part[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float2 d2 = __fmul2_rn(q2[h][0], k2[0]);
#pragma unroll
        for (int t = 1; t < 4; ++t) d2 = __ffma2_rn(q2[h][t], k2[t], d2);
        part[h] = d2.x + d2.y;
      }
      // reduce-scatter over the 8 lanes of the group (no selects: the q
      // positions are permuted per lane)
      s[it] = reduce_scatter8<G>(part);
      if (!full_page) {
        const bool valid = page_ok && (page_tok0 + r) < tok_end;
        s[it] = valid ? s[it] : -INFINITY;
      }
    }

    // ---- online softmax, once per page, with a lazy offset -----------------------
    // The offset m_run only moves when a page maximum exceeds it by more
    // than 2^kLazy (base 2): exp2(s - m_run) then stays below 2^kLazy, and
    // any offset gives the same acc / l.
    float pm = fmaxf(fmaxf(s[0], s[1]), fmaxf(s[2], s[3]));
    pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 8));
    pm = fmaxf(pm, __shfl_xor_sync(0xffffffffu, pm, 16));
    if (__any_sync(0xffffffffu, pm > m_run + kLazy)) {
      const float m_new = fmaxf(m_run, pm);
      const float alpha = fast_exp2(m_run - (m_new == -INFINITY ? 0.f : m_new));
      m_run = m_new;
      l_run *= alpha;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ah = __shfl_sync(0xffffffffu, alpha, h << kShift);
        const float2 a2 = make_float2(ah, ah);
#pragma unroll
        for (int t = 0; t < 4; ++t) acc2[h][t] = __fmul2_rn(acc2[h][t], a2);
      }
    }
    const float m_use = m_run == -INFINITY ? 0.f : m_run;

    // ---- P.V -------------------------------------------------------------------
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int r = it * 4 + grp;
      const float p = fast_exp2(s[it] - m_use);
      l_run += p;
      const uint4 vv =
          *reinterpret_cast<const uint4*>(vbase + r * kRowBytes + chk * 16);
      const uint32_t w[4] = {vv.x, vv.y, vv.z, vv.w};
      float2 v2[4];
#pragma unroll
      for (int t = 0; t < 4; ++t) v2[t] = make_float2(bf16_lo(w[t]), bf16_hi(w[t]));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float ph = __shfl_sync(0xffffffffu, p, grp * 8 + (h << kShift));
        const float2 p2 = make_float2(ph, ph);
#pragma unroll
        for (int t = 0; t < 4; ++t) acc2[h][t] = __ffma2_rn(p2, v2[t], acc2[h][t]);
      }
    }

    // ---- hand the slot back to the TMA unit ------------------------------------
    fence_proxy_async_smem();
    __syncwarp();
    const int j = i + kStages;
    const int src = ((j >> 5) == (i >> 5)) ? pid_cur : pid_next;
    const int pid_j = __shfl_sync(0xffffffffu, src, j & 31);
    if (j < my_n) {
      if (lane == 0) issue(pid_j, stage);
      ++issued;
    }
  }

  if (failed) {
    // Drain the copies this warp still has in flight (bounded), then wind
    // down with an empty result.
    if (lane == 0) flag_error(a.err, DEVERR_TIMEOUT);
    for (int k = i; k < issued; ++k)
      mbar_wait(smem_u32(&sm.full[warp][k % kStages]), (k / kStages) & 1);
    m_run = -INFINITY;
    l_run = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int t = 0; t < 4; ++t) acc2[h][t] = make_float2(0.f, 0.f);
  }

  // ---- reduce over the 4 lane groups ------------------------------------------
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 8);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 16);
#pragma unroll
  for (int h = 0; h < G; ++h) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      acc2[h][t].x += __shfl_xor_sync(0xffffffffu, acc2[h][t].x, 8);
      acc2[h][t].y += __shfl_xor_sync(0xffffffffu, acc2[h][t].y, 8);
      acc2[h][t].x += __shfl_xor_sync(0xffffffffu, acc2[h][t].x, 16);
      acc2[h][t].y += __shfl_xor_sync(0xffffffffu, acc2[h][t].y, 16);
    }
  }
  __syncthreads();  // every warp is done with its ring
  auto& cb = *reinterpret_cast<Combine<G>*>(smem_raw);
  if (grp == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        cb.acc[warp][h][chk * 8 + 2 * t] = acc2[h][t].x;
        cb.acc[warp][h][chk * 8 + 2 * t + 1] = acc2[h][t].y;
      }
    if ((chk & ((1 << kShift) - 1)) == 0) {
      cb.m[warp][my_head] = m_run;
      cb.l[warp][my_head] = l_run;
    }
  }
  __syncthreads();

  // ---- combine the 4 warps and write ------------------------------------------
  for (int o = threadIdx.x; o < G * kD; o += kThreads) {
    const int h = o / kD;
    const int e = o % kD;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, cb.m[w][h]);
    float L = 0.f, O = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kWarps; ++w) {
        const float f = fast_exp2(cb.m[w][h] - M);
        L = fmaf(cb.l[w][h], f, L);
        O = fmaf(cb.acc[w][h][e], f, O);
      }
    }
    const float out = L > 0.f ? O / L : 0.f;
    const size_t head = (size_t)seq * a.num_q_heads + kvh * G + h;
    if (kSplit) {
      const size_t prow = head * a.max_partitions + part;
      a.partial_out[prow * kD + e] = out;
      if (e == 0)
        a.partial_lse[prow] = L > 0.f ? (M + fast_log2(L)) * kLn2 : -INFINITY;
    } else {
      a.out[head * kD + e] = __float2bfloat16_rn(out);
    }
  }
}

template <int G, int kStages, bool kSplit, bool kAppend>
cudaError_t launch_g(const DecodeArgs& a, const CUtensorMap& tk,
                     const CUtensorMap& tv, int num_kv_heads, int num_seqs,
                     int parts, cudaStream_t stream) {
  auto kern = paged_decode_kernel<G, kStages, kSplit, kAppend>;
  const int smem = sizeof(DecodeSmem<kStages>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(num_kv_heads, num_seqs, parts);
  kern<<<grid, kThreads, smem, stream>>>(a, tk, tv);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_paged_decode(const DecodeArgs& a, const CUtensorMap& tk,
                                const CUtensorMap& tv, int num_kv_heads,
                                int num_seqs, int group, bool split,
                                int parts, cudaStream_t stream) {
  constexpr int S = 3;
  const bool append = a.k_new != nullptr;
  switch (group) {
#define TV_CASE(G)                                                          \
  case G:                                                                   \
    if (split)                                                              \
      return launch_g<G, S, true, false>(a, tk, tv, num_kv_heads, num_seqs, \
                                         parts, stream);                    \
    return append ? launch_g<G, S, false, true>(a, tk, tv, num_kv_heads,    \
                                                num_seqs, 1, stream)        \
                  : launch_g<G, S, false, false>(a, tk, tv, num_kv_heads,   \
                                                 num_seqs, 1, stream);
    TV_CASE(1)
    TV_CASE(2)
    TV_CASE(4)
    TV_CASE(8)
#undef TV_CASE
    default:
      return cudaErrorInvalidValue;
  }
}

}  // namespace tv
