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
//  * Per page the G query heads need S^T = K Q^T and O^T += V^T P^T: dense
//    products over 64 dims and 16 tokens, which each warp runs on the tensor
//    cores as m16n8k16 bf16 products with fp32 accumulation (4 for the
//    scores, 8 for P.V with P split into two bf16 terms), the page slices
//    read by ldmatrix from the 128-byte-swizzled TMA boxes.  Unpacking bf16
//    to fp32 and reducing dot products across lanes, which made up most of
//    the instructions of an fp32 FMA formulation, disappear.  The softmax is
//    online per page in base 2: one max and (lazily) one rescale per page.
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
  alignas(1024) uint8_t ring[kWarps][kStages][kStageBytes];
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
  const int chk = lane & 7;    // 16-byte chunk of the appended row

  // Block-table entries of this warp's first 64 blocks, loaded before and
  // independently of the context length (bounded by the table row; entries
  // past the context are loaded but never used), so the two loads overlap.
  const int32_t* bt = a.block_tables + (size_t)seq * a.max_blocks_per_seq;
  const int sub_mask = (1 << a.page_shift) - 1;
  const int first_page = kSplit ? part * a.partition_tokens / kPS : 0;
  auto table_pid = [&](int i) -> int {
    const int b = first_page + warp + kWarps * i;
    if ((b >> a.page_shift) >= a.max_blocks_per_seq) return -1;
    const int page = __ldg(bt + (b >> a.page_shift));
    return page >= 0 && page < a.num_pages
               ? (page << a.page_shift) + (b & sub_mask) : -1;
  };
  int pid_cur = table_pid(lane);
  int pid_next = table_pid(32 + lane);

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
  const int n_pages = (tok_end - tok_begin + kPS - 1) / kPS;
  // pages of this warp: first_page + warp + kWarps * i, i < my_n
  const int my_n = n_pages > warp ? (n_pages - warp + kWarps - 1) / kWarps : 0;

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

  // ---- warp-level tensor-core layout ---------------------------------------
  // Per page and KV head the work is two small dense products for the G
  // query heads of the group: S^T = K Q^T (16 tokens x G heads, contraction
  // over the 64 dims) and O^T += V^T P^T (64 dims x G heads, contraction over
  // the 16 tokens), each as m16n8k16 bf16 products with fp32 accumulation,
  // heads padded to the 8 columns of the product.  Lane = 4 * g + c:
  //  * S^T fragment: tokens g and g + 8, heads 2c and 2c + 1;
  //  * O^T fragment of dim tile t: dims 16t + g and 16t + g + 8, the same
  //    heads 2c, 2c + 1, so the running max / sum of a lane's heads (and
  //    their rescaling of O) never leave the lane.
  const int g = lane >> 2;
  const int c = lane & 3;
  const bool hv0 = 2 * c < G, hv1 = 2 * c + 1 < G;   // real heads of the lane

  // q of head g as the B operand of S^T = K Q^T: dims 16k + 2c, +1 (b0) and
  // 16k + 2c + 8, +9 (b1), unscaled bf16; padded heads are zero.
  uint32_t qb[4][2];
  {
    const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
        a.q + ((size_t)seq * a.num_q_heads + kvh * G + (g < G ? g : 0)) * kD);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      qb[k][0] = g < G ? __ldg(qrow + 8 * k + c) : 0u;
      qb[k][1] = g < G ? __ldg(qrow + 8 * k + c + 4) : 0u;
    }
  }
  // ldmatrix row addresses inside a 2 KB page slice stored with the 128-byte
  // swizzle (16-byte chunk j of row r at chunk j ^ (r & 7)).  K: matrices
  // (rows 0-7 | 8-15) x (chunk 2k | 2k+1) in A-fragment order; V, loaded
  // transposed: (chunk 2t | 2t+1) x (rows 0-7 | 8-15).
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
  // P^T as the B operand of the P.V product: lane (g, c) needs P of tokens
  // 2c, 2c+1 (and + 8) for head g, held by lanes 8c + g/2 and 8c + 4 + g/2
  // as the (head 2c', 2c'+1) halves of a bf16 pair; the byte permutation
  // picks half g & 1 of each.
  const int src_a = 8 * c + (g >> 1), src_b = src_a + 4;
  const uint32_t half_sel = (g & 1) ? 0x7632u : 0x5410u;

  // running max (base 2, scaled) / sum per head of the lane; padded heads
  // start at +inf so their probabilities are exp2(-inf) = 0
  float m0 = hv0 ? -INFINITY : INFINITY, m1 = hv1 ? -INFINITY : INFINITY;
  float l0 = 0.f, l1 = 0.f;
  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
  const float sl = a.scale_log2;

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
        const int ch = lane & 7;
        uint8_t* dst = (lane < 8 ? kbase : vbase) + app_r * kRowBytes +
                       ((ch ^ (app_r & 7)) << 4);
        *reinterpret_cast<uint4*>(dst) = app_row;
        __nv_bfloat16* pool = lane < 8 ? a.k_pool_w : a.v_pool_w;
        *reinterpret_cast<uint4*>(
            pool + (((size_t)pid * kPS + app_r) * gridDim.x + kvh) * kD +
            ch * 8) = app_row;
      }
      __syncwarp();
    }
    if (!full_page) {
      // Rows past the range (or the whole of a bad page) get p = 0; zero
      // their V so that 0 * a stale NaN never reaches the sum.
#pragma unroll
      for (int e = lane; e < kPS * 8; e += 32) {
        const int r = e >> 3;
        if (!(page_ok && page_tok0 + r < tok_end))
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
      const bool t0 = page_ok && page_tok0 + g < tok_end;
      const bool t1 = page_ok && page_tok0 + g + 8 < tok_end;
      s[0] = t0 ? s[0] : -INFINITY;
      s[1] = t0 ? s[1] : -INFINITY;
      s[2] = t1 ? s[2] : -INFINITY;
      s[3] = t1 ? s[3] : -INFINITY;
    }

    // ---- online softmax, once per page, with a lazy offset -----------------
    // The offset only moves when a page maximum exceeds it by more than
    // 2^kLazy (base 2): exp2(s - m) then stays below 2^kLazy, and any offset
    // gives the same acc / l.
    float pm0 = fmaxf(s[0], s[2]), pm1 = fmaxf(s[1], s[3]);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      pm0 = fmaxf(pm0, __shfl_xor_sync(0xffffffffu, pm0, off));
      pm1 = fmaxf(pm1, __shfl_xor_sync(0xffffffffu, pm1, off));
    }
    if (__any_sync(0xffffffffu, pm0 > m0 + kLazy || pm1 > m1 + kLazy)) {
      const float n0 = fmaxf(m0, pm0), n1 = fmaxf(m1, pm1);
      // equal offsets (both -inf, or a padded head's +inf) keep the sums
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

    // ---- P as two bf16 terms (hi + lo, ~16 significant bits) in B layout ---
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

    // ---- O^T += V^T P^T ------------------------------------------------------
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint32_t va[4];
      ldsm_x4_trans(vb + voff[t], va);
      mma_bf16_16816(acc[t], va, bh0, bh1);
      mma_bf16_16816(acc[t], va, bl0, bl1);
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
    m0 = hv0 ? -INFINITY : INFINITY;
    m1 = hv1 ? -INFINITY : INFINITY;
    l0 = l1 = 0.f;
#pragma unroll
    for (int t = 0; t < 4; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
  }

  // ---- sums over the 8 token lanes (g) of each head -----------------------
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  __syncthreads();  // every warp is done with its ring
  auto& cb = *reinterpret_cast<Combine<G>*>(smem_raw);
  if (hv0) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      cb.acc[warp][2 * c][16 * t + g] = acc[t][0];
      cb.acc[warp][2 * c][16 * t + g + 8] = acc[t][2];
    }
    if (g == 0) {
      cb.m[warp][2 * c] = m0;
      cb.l[warp][2 * c] = l0;
    }
  }
  if (hv1) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      cb.acc[warp][2 * c + 1][16 * t + g] = acc[t][1];
      cb.acc[warp][2 * c + 1][16 * t + g + 8] = acc[t][3];
    }
    if (g == 0) {
      cb.m[warp][2 * c + 1] = m1;
      cb.l[warp][2 * c + 1] = l1;
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
