// Work-balanced paged decode: the pages of every (sequence, KV head) pair,
// laid end to end, are cut into equal contiguous ranges, one per warp of a
// persistent grid.
//
// What it computes is the paged decode attention of paged_decode.cu
// ("tiny-vllm：从零构建高性能LLM推理引擎的完整指南", secs. "PagedAttention：
// 从操作系统借来的智慧", "推理流程：从Prefill到Decode", "在线Softmax：数值稳定的
// 注意力计算"), optionally fused with the KV append of the step.  Only the
// distribution of the work differs.
//
// Why.  With one CTA per (sequence, KV head), the grid is a fixed number of
// equal CTAs; whenever that number is not a multiple of (SMs x resident CTAs
// per SM), some SMs hold one CTA more than others and set the kernel time
// (64 sequences x 8 KV heads = 512 CTAs on 148 SMs x 4 slots: 68 SMs carry 4
// CTAs, 80 carry 3).  Mixed context lengths make it worse: the longest
// sequences start wherever the block scheduler puts them and finish last.
// Here the grid is exactly the resident capacity and every warp streams the
// same number of pages (+-1), whatever the length mix.
//
// How.
//  * Sequence s owns n_s = max(1, ceil(ctx_s / 16)) pages; laid end to end
//    they are T = sum_s n_s pages.  The warps form NG groups of Hkv; group
//    g takes pages [g*T/NG, (g+1)*T/NG) and warp h of the group streams KV
//    head h of them, so the Hkv heads of one page -- one contiguous 16 KB
//    block of the pool -- are read at about the same time, as with one CTA
//    per pair.  Item u = s * Hkv + h is the work of one (sequence, KV head)
//    pair.  An empty context keeps one page that is never loaded, so its
//    zero output row is still written.
//  * Every CTA computes the exclusive prefix sum of n_s in shared memory
//    (B <= kMaxBalancedSeqs) and each warp maps its page positions to
//    (s, p), 32 at a time, one per lane, by binary search over it; the
//    lanes then load the block-table entries of those pages.
//  * Each warp runs the same page pipeline as paged_decode.cu (a private
//    ring of kStages TMA-filled page slots, one mbarrier each) straight
//    across item boundaries, so short items cost no pipeline drain.  At the
//    first page of an item it takes the item's q (fetched one item ahead
//    into registers); at the item's last page in its range it finishes the
//    item.  The per-page arithmetic is that of paged_decode.cu: the scores
//    and P.V of the G heads as warp-level bf16 tensor-core products.
//  * An item that lies inside one warp's range is written directly.  An
//    item cut by range boundaries is a set of segments, one per group; each
//    writes (m, l, acc) for its G heads to its workspace slot (slot 0 for
//    the first segment of its range, 1 for the last), fences, and
//    increments the item's counter; the warp that brings the counter to the
//    number of segments merges them with the log-sum-exp rule of the
//    split-KV merge and resets the counter to zero.  Nothing ever waits on
//    another warp, so no spin-wait exists beyond the bounded TMA waits.
//  * Fused append: the page holding position ctx-1 is loaded with the new K
//    and V rows of its KV head (two 128-byte bulk copies into a side slot of
//    the same ring stage, same mbarrier); the warp copies them over the
//    staged row and into the pools.
//  * Online softmax with a lazy maximum: the running offset only moves
//    when a page maximum exceeds it by more than 2^8 (base 2), so a page
//    rarely pays for a rescale; any offset gives the same ratio acc / l.
#include "tv_decode.cuh"
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kD = 64;
constexpr int kPS = 16;
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kStages = 3;
constexpr int kRowBytes = kD * 2;
constexpr int kSliceBytes = kPS * kRowBytes;
constexpr int kStageBytes = 2 * kSliceBytes;
constexpr int kSideBytes = 2 * kRowBytes;        // new K row + new V row
constexpr float kLazy = 8.f;                     // log2 of the allowed growth
constexpr uint32_t kNoPage = (1u << 26) - 1;     // page word: nothing to load

struct BalancedSmem {
  // 1024-byte aligned: the slices are 128-byte-swizzled TMA boxes
  alignas(1024) uint8_t ring[kWarps][kStages][kStageBytes];
  alignas(128) uint8_t side[kWarps][kStages][kSideBytes];
  alignas(8) uint64_t full[kWarps][kStages];
  int32_t warp_total[kWarps];
  int32_t pre[kMaxBalancedSeqs + 1];
  uint8_t last_valid[kMaxBalancedSeqs];  // tokens in each sequence's last page
};

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src,
                                          uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

__device__ __forceinline__ int clamp_ctx(int ctx, int cap) {
  return ctx < 0 ? 0 : (ctx > cap ? cap : ctx);
}

template <int G, bool kAppend>
__global__ void __launch_bounds__(kThreads, G <= 4 ? 4 : 2)
    balanced_decode_kernel(const DecodeArgs a,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  // 1 KB of slack is requested at launch; align the carve-out by hand.
  uint8_t* smem_raw = smem_dyn + ((1024 - (smem_u32(smem_dyn) & 1023)) & 1023);
  auto& sm = *reinterpret_cast<BalancedSmem*>(smem_raw);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grp = lane >> 3;
  const int chk = lane & 7;
  const int B = a.num_seqs;
  const int Hkv = a.num_kv_heads;
  // a page holds 1 << page_shift blocks of 16 tokens; the work unit here is
  // the 16-token block (one TMA box)
  const int ctx_cap = a.max_blocks_per_seq * (kPS << a.page_shift);

  // ---- pages per sequence, exclusive prefix in shared memory ---------------
  for (int s = threadIdx.x; s < B; s += kThreads) {
    // in a decode step, a sequence whose context did not grow is idle
    const int raw = (a.grown && a.grown[s] == 0) ? 0 : a.context_lens[s];
    if ((raw < 0 || raw > ctx_cap) && blockIdx.x == 0)
      flag_error(a.err, DEVERR_BAD_CONTEXT);
    const int ctx = clamp_ctx(raw, ctx_cap);
    sm.pre[s] = ctx > 0 ? (ctx + kPS - 1) / kPS : 1;
    sm.last_valid[s] = (uint8_t)(ctx > 0 ? ctx - (ctx - 1) / kPS * kPS : 0);
  }
  __syncthreads();
  {
    const int per = (B + kThreads - 1) / kThreads;
    const int lo = min(B, (int)threadIdx.x * per);
    const int hi = min(B, lo + per);
    int own = 0;
    for (int s = lo; s < hi; ++s) own += sm.pre[s];
    int incl = own;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += v;
    }
    if (lane == 31) sm.warp_total[warp] = incl;
    __syncthreads();
    int run = incl - own;
    for (int w = 0; w < warp; ++w) run += sm.warp_total[w];
    for (int s = lo; s < hi; ++s) {
      const int n = sm.pre[s];
      sm.pre[s] = run;
      run += n;
    }
    if (threadIdx.x == 0) {
      int tot = 0;
      for (int w = 0; w < kWarps; ++w) tot += sm.warp_total[w];
      sm.pre[B] = tot;
    }
  }
  if (lane == 0) {
    for (int s = 0; s < kStages; ++s) mbar_init(smem_u32(&sm.full[warp][s]), 1);
    fence_mbar_init();
  }
  __syncthreads();  // the last CTA-wide barrier: warps run independently now

  // Work split: T sequence pages (all sequences end to end), NG groups of
  // Hkv warps; group g takes pages [g*T/NG, (g+1)*T/NG) and warp h of the
  // group streams KV head h of them, so the Hkv heads of a page (one 16 KB
  // block of the pool) are read at about the same time.
  const int T = sm.pre[B];
  const int NG = min((int)gridDim.x * kWarps / Hkv,
                     max(1, T / kMinPagesPerWarp));
  const int gw = blockIdx.x * kWarps + warp;
  const int grp_id = gw / Hkv;
  const int head = gw - grp_id * Hkv;
  if (grp_id >= NG) return;
  const int x0 = (int)((int64_t)grp_id * T / NG);
  const int x1 = (int)((int64_t)(grp_id + 1) * T / NG);
  const int n = x1 - x0;  // >= 1 because NG <= T
  // first page of group g's range, and the group whose range holds page x
  auto range_start = [&](int g) { return (int)((int64_t)g * T / NG); };
  auto owner = [&](int x) {
    return (int)(((int64_t)(x + 1) * NG - 1) / T);
  };

  // ---- per-lane page table: positions x0 + 32*batch + lane -----------------
  // One word per 16-token block: bits 0-25 the pool block (kNoPage when nothing is
  // to be loaded: empty context or a bad block-table entry), bit 26 first
  // page of its sequence, bit 27 last page, bits 28-31 valid tokens - 1
  // (15 on every page but the last).  seq0 receives the sequence of the
  // range's first page.
  auto build = [&](int batch, uint32_t& w, int* seq0) {
    const int i = batch * 32 + lane;
    w = kNoPage;
    if (i < n) {
      const int x = x0 + i;
      int lo = 0, hi = B;  // pre[lo] <= x < pre[hi]
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (sm.pre[mid] <= x) lo = mid; else hi = mid;
      }
      const int p = x - sm.pre[lo];
      const bool last = x == sm.pre[lo + 1] - 1;
      const int lv = sm.last_valid[lo];
      uint32_t pid = kNoPage;   // the pool block (16 rows) of this block
      if (lv > 0) {
        const int raw = __ldg(a.block_tables +
                              (size_t)lo * a.max_blocks_per_seq +
                              (p >> a.page_shift));
        if (raw >= 0 && raw < a.num_pages) {
          pid = ((uint32_t)raw << a.page_shift) +
                (uint32_t)(p & ((1 << a.page_shift) - 1));
        } else if (head == 0) {
          flag_error(a.err, DEVERR_BAD_PAGE);
        }
      }
      w = pid | ((uint32_t)(p == 0) << 26) | ((uint32_t)last << 27) |
          ((uint32_t)((last ? lv : kPS) - 1) << 28);
      if (seq0) *seq0 = lo;
    }
  };
  // batches of the issue cursor: the one it is in, and the next
  uint32_t b_w, nb_w;
  int seq0 = 0;
  build(0, b_w, &seq0);
  build(1, nb_w, nullptr);
  seq0 = __shfl_sync(0xffffffffu, seq0, 0);

  const uint64_t policy = l2_policy_evict_first();
  const int kv_x = head * kD;   // TMA x coordinate of this warp's KV head
  auto issue = [&](uint32_t w, int seq, int stage) {
    const uint32_t bar = smem_u32(&sm.full[warp][stage]);
    const uint32_t pid = w & kNoPage;
    if (pid == kNoPage) {  // nothing to load
      mbar_arrive(bar);
      return;
    }
    const int y = (int)pid * kPS;
    const uint32_t dst = smem_u32(&sm.ring[warp][stage][0]);
    // the new token (position ctx-1) is the last valid row of the last page
    const bool app = kAppend && ((w >> 27) & 1);
    mbar_arrive_expect_tx(bar, kStageBytes + (app ? kSideBytes : 0));
    tma_load_2d_hint(dst, &tm_k, kv_x, y, bar, policy);
    tma_load_2d_hint(dst + kSliceBytes, &tm_v, kv_x, y, bar, policy);
    if (app) {
      const size_t row = ((size_t)seq * Hkv + head) * kD;
      const uint32_t side = smem_u32(&sm.side[warp][stage][0]);
      bulk_load(side, a.k_new + row, kRowBytes, bar);
      bulk_load(side + kRowBytes, a.v_new + row, kRowBytes, bar);
    }
  };
  // Page words of the next kStages pages in compute order, taken from the
  // batch when the page is issued (so the compute loop needs no shuffle);
  // seq_issue follows the issue cursor's sequence.
  uint32_t q_w[kStages];
  int seq_issue = seq0;
#pragma unroll
  for (int j = 0; j < kStages; ++j) {
    q_w[j] = __shfl_sync(0xffffffffu, b_w, j);
    if (j > 0 && ((q_w[j] >> 26) & 1)) ++seq_issue;
    if (j < n && lane == 0) issue(q_w[j], seq_issue, j);
  }

  // Warp-level tensor-core layout, as in paged_decode.cu: per page,
  // S^T = K Q^T and O^T += V^T P^T as m16n8k16 bf16 products (fp32
  // accumulation, heads padded to 8 columns).  Lane = 4 g + c holds tokens
  // g, g+8 of the scores and dims 16t + g, +8 of the accumulator, both for
  // heads 2c and 2c+1.
  const int g = lane >> 2;
  const int c = lane & 3;
  const bool hv0 = 2 * c < G, hv1 = 2 * c + 1 < G;
  uint32_t koff[4], voff[4];
  {
    const int mi = lane >> 3, r7 = lane & 7;
    const int kr = r7 + 8 * (mi & 1), vr = r7 + 8 * (mi >> 1);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      koff[k] = kr * kRowBytes + (((2 * k + (mi >> 1)) ^ r7) << 4);
      voff[k] = vr * kRowBytes + (((2 * k + (mi & 1)) ^ r7) << 4);
    }
  }
  const int src_a = 8 * c + (g >> 1), src_b = src_a + 4;
  const uint32_t half_sel = (g & 1) ? 0x7632u : 0x5410u;
  const float sl = a.scale_log2;

  // q fragments (B operand of the scores, head g of the group) of the next
  // item, fetched into registers one item ahead
  uint32_t qn[4][2];
  auto load_q = [&](int sq) {
    const bool ok = sq < B && g < G;
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + ((size_t)(ok ? sq : 0) * a.num_q_heads + head * G +
               (g < G ? g : 0)) * kD);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      qn[k][0] = ok ? __ldg(qrow + 8 * k + c) : 0u;
      qn[k][1] = ok ? __ldg(qrow + 8 * k + c + 4) : 0u;
    }
  };
  load_q(seq0);

  uint32_t qb[4][2];
  float acc[4][4];
  float m0 = INFINITY, m1 = INFINITY, l0 = 0.f, l1 = 0.f;
  bool seg_at_range_start = true;   // the segment began at x0
  bool seg_at_item_start = true;    // the segment began at page 0

  bool failed = false;
  int issued = min(n, kStages);
  int seq = seq0;   // sequence of the page being computed
  int i = 0;
  for (; i < n; ++i) {
    const int stage = i % kStages;
    const uint32_t parity = (i / kStages) & 1;
    const uint32_t w = q_w[0];
    const uint32_t pid = w & kNoPage;
    const bool first_of_item = (w >> 26) & 1;
    const bool last_of_item = (w >> 27) & 1;
    const int valid = (int)(w >> 28) + 1;
    const bool page_ok = pid != kNoPage;
    const bool full_page = page_ok && valid == kPS;

    // ---- a new item starts: take its q, reset the running state ------------
    if (i == 0 || first_of_item) {
      if (i > 0) ++seq;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        qb[k][0] = qn[k][0];
        qb[k][1] = qn[k][1];
      }
#pragma unroll
      for (int t = 0; t < 4; ++t)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
      // padded heads keep +inf: their probabilities are exp2(-inf) = 0
      m0 = hv0 ? -INFINITY : INFINITY;
      m1 = hv1 ? -INFINITY : INFINITY;
      l0 = l1 = 0.f;
      seg_at_range_start = i == 0;
      seg_at_item_start = first_of_item;
      // this warp's next item is the next sequence, same KV head (fetched
      // even when the range ends first: one spare read of G x 128 bytes)
      load_q(seq + 1);
    }

    if (!__all_sync(0xffffffffu,
                    mbar_wait(smem_u32(&sm.full[warp][stage]), parity))) {
      failed = true;
      break;
    }
    uint8_t* kbase = &sm.ring[warp][stage][0];
    uint8_t* vbase = kbase + kSliceBytes;
    if (kAppend && page_ok && last_of_item) {
      // new K/V row of this item: into the staged page and into the pools
      if (lane < 16) {
        const int r = valid - 1;
        const uint4 row = *reinterpret_cast<const uint4*>(
            &sm.side[warp][stage][(lane < 8 ? 0 : kRowBytes) + chk * 16]);
        *reinterpret_cast<uint4*>(kbase + (lane < 8 ? 0 : kSliceBytes) +
                                  r * kRowBytes + ((chk ^ (r & 7)) << 4)) =
            row;
        __nv_bfloat16* pool = lane < 8 ? a.k_pool_w : a.v_pool_w;
        *reinterpret_cast<uint4*>(
            pool + (((size_t)pid * kPS + r) * Hkv + head) * kD + chk * 8) =
            row;
      }
      __syncwarp();
    }

    if (!full_page) {
      // Rows past the context (or the whole of an unloaded page) get p = 0;
      // zero their V so that 0 * a stale NaN never reaches the sum.
#pragma unroll
      for (int e = lane; e < kPS * 8; e += 32) {
        const int r = e >> 3;
        if (!(page_ok && r < valid))
          *reinterpret_cast<uint4*>(vbase + r * kRowBytes + (e & 7) * 16) =
              make_uint4(0, 0, 0, 0);
      }
      __syncwarp();
    }
    const uint32_t kb = smem_u32(kbase), vb = smem_u32(vbase);

    // ---- scores S^T = K Q^T: tokens g, g+8 x heads 2c, 2c+1 ----------------
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t ka[4];
      ldsm_x4(kb + koff[k], ka);
      mma_bf16_16816(s, ka, qb[k][0], qb[k][1]);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) s[e] *= sl;
    if (!full_page) {
      const bool t0 = page_ok && g < valid, t1 = page_ok && g + 8 < valid;
      s[0] = t0 ? s[0] : -INFINITY;
      s[1] = t0 ? s[1] : -INFINITY;
      s[2] = t1 ? s[2] : -INFINITY;
      s[3] = t1 ? s[3] : -INFINITY;
    }

    // ---- online softmax with a lazy offset ----------------------------------
    float pm0 = fmaxf(s[0], s[2]), pm1 = fmaxf(s[1], s[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, off));
      pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, off));
    }
    if (__any_sync(0xffffffffu, pm0 > m0 + kLazy || pm1 > m1 + kLazy)) {
      const float n0 = fmaxf(m0, pm0), n1 = fmaxf(m1, pm1);
      const float a0 = n0 == m0 ? 1.f : fast_exp2(m0 - n0);
      const float a1 = n1 == m1 ? 1.f : fast_exp2(m1 - n1);
      m0 = n0;
      m1 = n1;
      l0 *= a0;
      l1 *= a1;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        acc[t][0] *= a0;
        acc[t][1] *= a1;
        acc[t][2] *= a0;
        acc[t][3] *= a1;
      }
    }
    const float mu0 = m0 == -INFINITY ? 0.f : m0;
    const float mu1 = m1 == -INFINITY ? 0.f : m1;
    const float p0 = fast_exp2(s[0] - mu0), p1 = fast_exp2(s[1] - mu1);
    const float p2 = fast_exp2(s[2] - mu0), p3 = fast_exp2(s[3] - mu1);
    l0 += p0 + p2;
    l1 += p1 + p3;

    // ---- P (bf16 hi + lo) in B layout; O^T += V^T P^T -------------------------
    const uint32_t h01 = pack_bf16x2(p0, p1), h23 = pack_bf16x2(p2, p3);
    const uint32_t r01 = pack_bf16x2(p0 - bf16_lo(h01), p1 - bf16_hi(h01));
    const uint32_t r23 = pack_bf16x2(p2 - bf16_lo(h23), p3 - bf16_hi(h23));
    const uint32_t bh0 = __byte_perm(__shfl_sync(0xffffffffu, h01, src_a),
                                     __shfl_sync(0xffffffffu, h01, src_b),
                                     half_sel);
    const uint32_t bh1 = __byte_perm(__shfl_sync(0xffffffffu, h23, src_a),
                                     __shfl_sync(0xffffffffu, h23, src_b),
                                     half_sel);
    const uint32_t bl0 = __byte_perm(__shfl_sync(0xffffffffu, r01, src_a),
                                     __shfl_sync(0xffffffffu, r01, src_b),
                                     half_sel);
    const uint32_t bl1 = __byte_perm(__shfl_sync(0xffffffffu, r23, src_a),
                                     __shfl_sync(0xffffffffu, r23, src_b),
                                     half_sel);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t va[4];
      ldsm_x4_trans(vb + voff[t], va);
      mma_bf16_16816(acc[t], va, bh0, bh1);
      mma_bf16_16816(acc[t], va, bl0, bl1);
    }

    // ---- hand the slot back, issue the page kStages ahead ------------------------
    fence_proxy_async_smem();
    __syncwarp();
    {
      const int j = i + kStages;
      uint32_t jw = kNoPage;
      if (j < n) {
        if ((j & 31) == 0) {   // the issue cursor enters the next batch
          b_w = nb_w;
          build((j >> 5) + 1, nb_w, nullptr);
        }
        jw = __shfl_sync(0xffffffffu, b_w, j & 31);
        if ((jw >> 26) & 1) ++seq_issue;
        if (lane == 0) issue(jw, seq_issue, stage);
        ++issued;
      }
#pragma unroll
      for (int k = 0; k + 1 < kStages; ++k) q_w[k] = q_w[k + 1];
      q_w[kStages - 1] = jw;
    }

    // ---- the item ends in this range: finish it ---------------------------------
    if (last_of_item || i == n - 1) {
      float L0 = l0, L1 = l1;   // sums over the 8 token lanes of each head
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        L0 += __shfl_xor_sync(0xffffffffu, L0, off);
        L1 += __shfl_xor_sync(0xffffffffu, L1, off);
      }
      const int u = seq * Hkv + head;
      __nv_bfloat16* out_item =
          a.out + ((size_t)seq * a.num_q_heads + head * G) * kD;
      if (seg_at_item_start && last_of_item) {
        // the whole item is in this range
        const float inv0 = L0 > 0.f ? 1.f / L0 : 0.f;
        const float inv1 = L1 > 0.f ? 1.f / L1 : 0.f;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          if (hv0) {
            out_item[2 * c * kD + 16 * t + g] =
                __float2bfloat16_rn(acc[t][0] * inv0);
            out_item[2 * c * kD + 16 * t + g + 8] =
                __float2bfloat16_rn(acc[t][2] * inv0);
          }
          if (hv1) {
            out_item[(2 * c + 1) * kD + 16 * t + g] =
                __float2bfloat16_rn(acc[t][1] * inv1);
            out_item[(2 * c + 1) * kD + 16 * t + g + 8] =
                __float2bfloat16_rn(acc[t][3] * inv1);
          }
        }
      } else {
        // one segment of an item shared with other warps
        float* slot = a.ws_partials +
                      ((size_t)gw * 2 + (seg_at_range_start ? 0 : 1)) *
                          kSlotFloats;
        if (hv0) {
          if (g == 0) {
            slot[2 * c] = m0;
            slot[8 + 2 * c] = L0;
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            slot[16 + 2 * c * kD + 16 * t + g] = acc[t][0];
            slot[16 + 2 * c * kD + 16 * t + g + 8] = acc[t][2];
          }
        }
        if (hv1) {
          if (g == 0) {
            slot[2 * c + 1] = m1;
            slot[8 + 2 * c + 1] = L1;
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            slot[16 + (2 * c + 1) * kD + 16 * t + g] = acc[t][1];
            slot[16 + (2 * c + 1) * kD + 16 * t + g + 8] = acc[t][3];
          }
        }
        __threadfence();
        __syncwarp();
        int old = 0;
        if (lane == 0) old = atomicAdd(a.ws_counters + u, 1);
        old = __shfl_sync(0xffffffffu, old, 0);
        const int item_x = sm.pre[seq];     // first page of sequence seq
        const int g_first = owner(item_x);
        int g_last = grp_id;                // this group holds the last page
        if (!last_of_item)
          g_last = owner(item_x + sm.pre[seq + 1] - sm.pre[seq] - 1);
        if (old == g_last - g_first) {
          // every other segment is in memory: merge them all.  Segment k
          // (k = 0 .. nseg-1) is in warp head of group g_first + k, slot 0
          // except the first one when the item starts inside that group's
          // range.
          __threadfence();
          const int nseg = g_last - g_first + 1;
          const int slot_first = item_x == range_start(g_first) ? 0 : 1;
          auto seg_ptr = [&](int k) {
            return a.ws_partials +
                   ((size_t)((g_first + k) * Hkv + head) * 2 +
                    (k == 0 ? slot_first : 0)) *
                       kSlotFloats;
          };
          // pass 1, one segment per lane: maxima and sums of every head
          float M[G], L[G];
#pragma unroll
          for (int h = 0; h < G; ++h) {
            M[h] = -INFINITY;
            L[h] = 0.f;
          }
          for (int k0 = 0; k0 < nseg; k0 += 32) {
            const int k = k0 + lane;
            float mk[G], lk[G];
#pragma unroll
            for (int h = 0; h < G; ++h) {
              mk[h] = -INFINITY;
              lk[h] = 0.f;
            }
            if (k < nseg) {
              const float* sl = seg_ptr(k);
#pragma unroll
              for (int h = 0; h < G; ++h) {
                mk[h] = __ldcg(sl + h);
                lk[h] = __ldcg(sl + 8 + h);
              }
            }
#pragma unroll
            for (int h = 0; h < G; ++h) {
              float mx = mk[h];
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1)
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
              const float m_new = fmaxf(M[h], mx);
              const float base = m_new == -INFINITY ? 0.f : m_new;
              float sum = lk[h] * fast_exp2(mk[h] - base);
#pragma unroll
              for (int off = 16; off >= 1; off >>= 1)
                sum += __shfl_xor_sync(0xffffffffu, sum, off);
              L[h] = L[h] * fast_exp2(M[h] - base) + sum;
              M[h] = m_new;
            }
          }
          // pass 2: lane (grp, chk) sums head grp (+4), dims 8chk..8chk+7
#pragma unroll
          for (int h0 = 0; h0 < G; h0 += 4) {
            const int h = h0 + grp;
            float Mh = M[0], Lh = L[0];
#pragma unroll
            for (int hh = 1; hh < G; ++hh)
              if (hh == h) {
                Mh = M[hh];
                Lh = L[hh];
              }
            const float base = Mh == -INFINITY ? 0.f : Mh;
            float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
            if (h < G) {
              constexpr int kU = 8;   // partials in flight per lane
              int k = 0;
              for (; k + kU <= nseg; k += kU) {
                float4 v[kU][2];
                float f[kU];
#pragma unroll
                for (int j = 0; j < kU; ++j) {
                  const float* sl = seg_ptr(k + j);
                  const float4* src =
                      reinterpret_cast<const float4*>(sl + 16 + h * kD + chk * 8);
                  v[j][0] = __ldcg(src);
                  v[j][1] = __ldcg(src + 1);
                  f[j] = fast_exp2(__ldcg(sl + h) - base);
                }
#pragma unroll
                for (int j = 0; j < kU; ++j) {
                  o0.x = fmaf(v[j][0].x, f[j], o0.x);
                  o0.y = fmaf(v[j][0].y, f[j], o0.y);
                  o0.z = fmaf(v[j][0].z, f[j], o0.z);
                  o0.w = fmaf(v[j][0].w, f[j], o0.w);
                  o1.x = fmaf(v[j][1].x, f[j], o1.x);
                  o1.y = fmaf(v[j][1].y, f[j], o1.y);
                  o1.z = fmaf(v[j][1].z, f[j], o1.z);
                  o1.w = fmaf(v[j][1].w, f[j], o1.w);
                }
              }
              for (; k < nseg; ++k) {
                const float* sl = seg_ptr(k);
                const float4* src =
                    reinterpret_cast<const float4*>(sl + 16 + h * kD + chk * 8);
                const float4 v0 = __ldcg(src), v1 = __ldcg(src + 1);
                const float f = fast_exp2(__ldcg(sl + h) - base);
                o0.x = fmaf(v0.x, f, o0.x);
                o0.y = fmaf(v0.y, f, o0.y);
                o0.z = fmaf(v0.z, f, o0.z);
                o0.w = fmaf(v0.w, f, o0.w);
                o1.x = fmaf(v1.x, f, o1.x);
                o1.y = fmaf(v1.y, f, o1.y);
                o1.z = fmaf(v1.z, f, o1.z);
                o1.w = fmaf(v1.w, f, o1.w);
              }
              const float inv = Lh > 0.f ? 1.f / Lh : 0.f;
              uint4 o;
              o.x = pack_bf16x2(o0.x * inv, o0.y * inv);
              o.y = pack_bf16x2(o0.z * inv, o0.w * inv);
              o.z = pack_bf16x2(o1.x * inv, o1.y * inv);
              o.w = pack_bf16x2(o1.z * inv, o1.w * inv);
              *reinterpret_cast<uint4*>(out_item + h * kD + chk * 8) = o;
            }
          }
          if (lane == 0) a.ws_counters[u] = 0;
        }
      }
    }
  }

  if (failed) {
    // Drain the copies still in flight (bounded) and give up; outputs of the
    // items this warp did not finish stay unwritten.
    if (lane == 0) flag_error(a.err, DEVERR_TIMEOUT);
    for (int k = i; k < issued; ++k)
      mbar_wait(smem_u32(&sm.full[warp][k % kStages]), (k / kStages) & 1);
  }
}

// Four CTAs of G <= 4 must fit in one SM's 228 KB (1 KB of it reserved per
// CTA) so that 16 warps stream per SM.
static_assert(4 * (sizeof(BalancedSmem) + 1024 + 1024) <= 228 * 1024,
              "shared memory of the balanced decode exceeds 4 CTAs per SM");

template <int G, bool kAppend>
struct BalancedLaunch {
  static constexpr size_t smem_bytes() {
    return sizeof(BalancedSmem) + 1024;
  }
  static int ctas_per_sm() {
    static int occ = -1;  // per process; every B200 gives the same answer
    if (occ < 0) {
      auto kern = balanced_decode_kernel<G, kAppend>;
      if (cudaFuncSetAttribute(kern,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem_bytes()) != cudaSuccess ||
          cudaFuncSetAttribute(kern,
                               cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared) != cudaSuccess)
        return 0;
      int v = 0;
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
              &v, kern, kThreads, smem_bytes()) != cudaSuccess)
        return 0;
      occ = v;
    }
    return occ;
  }
  static cudaError_t run(const DecodeArgs& a, const CUtensorMap& tk,
                         const CUtensorMap& tv, int ctas,
                         cudaStream_t stream) {
    auto kern = balanced_decode_kernel<G, kAppend>;
    cudaError_t e = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(kern,
                               cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    kern<<<ctas, kThreads, smem_bytes(), stream>>>(a, tk, tv);
    return cudaGetLastError();
  }
};

template <int G>
int ctas_per_sm_g(bool append) {
  return append ? BalancedLaunch<G, true>::ctas_per_sm()
                : BalancedLaunch<G, false>::ctas_per_sm();
}

}  // namespace

int balanced_decode_ctas_per_sm(int group, bool append) {
  switch (group) {
    case 1: return ctas_per_sm_g<1>(append);
    case 2: return ctas_per_sm_g<2>(append);
    case 4: return ctas_per_sm_g<4>(append);
    case 8: return ctas_per_sm_g<8>(append);
    default: return 0;
  }
}

cudaError_t launch_balanced_decode(const DecodeArgs& a, const CUtensorMap& tk,
                                   const CUtensorMap& tv, int group, int ctas,
                                   cudaStream_t stream) {
  const bool append = a.k_new != nullptr;
  switch (group) {
#define TV_CASE(G)                                                        \
  case G:                                                                 \
    return append ? BalancedLaunch<G, true>::run(a, tk, tv, ctas, stream) \
                  : BalancedLaunch<G, false>::run(a, tk, tv, ctas, stream);
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
