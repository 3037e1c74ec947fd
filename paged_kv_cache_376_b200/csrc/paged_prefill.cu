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
// B200 design (one CTA per (KV head, 32-query tile, sequence); 6 warps):
//  * M = 128 MMA rows = 32 query rows x the 4 query heads of one KV head, so
//    every K/V tile feeds 4 heads (GQA reuse) and one tcgen05.mma of M = 128
//    covers them.  q arrives by one 3-D TMA box {64 d, 4 heads, 32 rows}.
//  * Keys come in tiles of 128 = 8 pages; each page of one KV head (16 rows x
//    128 B) is one 2-D TMA box, 128-byte swizzled, so 8 boxes at 2 KB
//    offsets form exactly the canonical K-major SW128 operand.  Pages past
//    the range (or with a bad id) are read at an out-of-range coordinate and
//    arrive as zeros.
//  * warp 0: TMA producer (q once, K/V through a 3-stage ring).
//    warp 1: tensor-memory allocation and the single MMA-issuing thread:
//      S_j = Q K_j^T (M128 N128 K16 x4) into one of two S buffers in tensor
//      memory, then O_{j-1} = P_{j-1} V_{j-1} (M128 N64 K16 x8, twice: once
//      for P_hi and once for P_lo; V read as an MN-major operand) into one of
//      two O buffers.
//  * P is split as P_hi = bf16(p), P_lo = bf16(p - P_hi) so the PV product
//    keeps ~16 bits of each weight (fp32-grade accumulation with bf16
//    operands); a single bf16 P carries 8 bits, which is not enough for rows
//    that see few keys.
//    warps 2-5: softmax.  Thread = one MMA row = one (query, head).  It reads
//      its 128 scores with tcgen05.ld, masks causally, updates the running
//      max/sum in base 2 (no cross-thread reduction at all), writes P as bf16
//      into the swizzled K-major layout the MMA reads, and folds the previous
//      tile's O into fp32 registers (o = o * alpha + O).
//  * Every wait is an mbarrier wait bounded by a 2 s time limit.
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kD = 64;
constexpr int kPS = 16;
constexpr int kG = 4;                    // query heads per KV head
constexpr int kQRows = 32;               // query rows per CTA
constexpr int kBM = kQRows * kG;         // 128 MMA rows
constexpr int kBN = 128;                 // keys per tile
constexpr int kPagesPerTile = kBN / kPS; // 8
constexpr int kST = 2;                   // K/V ring depth
constexpr int kRowBytes = kD * 2;        // 128
constexpr int kTileBytes = kBN * kRowBytes;  // 16 KB
constexpr int kPageBytes = kPS * kRowBytes;  // 2 KB
constexpr int kThreads = 192;
constexpr int kTmemCols = 512;
constexpr int kSCol = 0;                 // S buffers: columns [0, 256)
constexpr int kOCol = 2 * kBN;           // O buffers: columns [256, 384)

constexpr uint32_t kIdescQK = idesc_bf16_f32(kBM, kBN, false);
constexpr uint32_t kIdescPV = idesc_bf16_f32(kBM, kD, true);

struct PrefillSmem {
  alignas(1024) uint8_t q[kBM * kRowBytes];          // 16 KB
  alignas(1024) uint8_t k[kST][kTileBytes];          // 32 KB
  alignas(1024) uint8_t v[kST][kTileBytes];          // 32 KB
  // P = P_hi + P_lo, both bf16: [buffer][hi/lo][key half][128 rows x 128 B]
  alignas(1024) uint8_t p[2][2][2][kBM * kRowBytes];  // 128 KB
  alignas(8) uint64_t q_full;
  uint64_t kv_full[kST], kv_empty[kST];
  uint64_t s_full[2], s_free[2], p_full[2], o_full[2], o_free[2];
  uint32_t tmem_base;
  uint32_t bad_pages[kST];
};

__global__ void __launch_bounds__(kThreads, 1)
    paged_prefill_kernel(const PrefillArgs a,
                         const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
  extern __shared__ __align__(1024) uint8_t smem_dyn[];
  uint8_t* base = smem_dyn + ((1024 - (smem_u32(smem_dyn) & 1023)) & 1023);
  auto& sm = *reinterpret_cast<PrefillSmem*>(base);

  const int kvh = blockIdx.x;
  const int tile = gridDim.y - 1 - blockIdx.y;   // heaviest tiles first
  const int seq = blockIdx.z;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- work of this CTA (uniform across the block) ---------------------------
  const int qs = a.query_start_loc[seq];
  const int T = a.query_start_loc[seq + 1] - qs;
  int ctx = a.context_lens[seq];
  const int ctx_cap = a.max_blocks_per_seq * kPS;
  const int q0 = tile * kQRows;
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
  const int q_hi = min(q0 + kQRows, T);       // rows [q0, q_hi) are real
  const int n_keys = P + q_hi;                // keys [0, n_keys) are needed
  const int n_tiles = (n_keys + kBN - 1) / kBN;
  const int n_pages = (n_keys + kPS - 1) / kPS;
  const int32_t* bt = a.block_tables + (size_t)seq * a.max_blocks_per_seq;

  // ---- set-up ------------------------------------------------------------------
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&sm.q_full), 1);
    for (int i = 0; i < kST; ++i) {
      mbar_init(smem_u32(&sm.kv_full[i]), 1);
      mbar_init(smem_u32(&sm.kv_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&sm.s_full[i]), 1);
      mbar_init(smem_u32(&sm.s_free[i]), 4);
      mbar_init(smem_u32(&sm.p_full[i]), 4);
      mbar_init(smem_u32(&sm.o_full[i]), 1);
      mbar_init(smem_u32(&sm.o_free[i]), 4);
    }
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
    if (lane == 0) {
      const uint32_t qbar = smem_u32(&sm.q_full);
      mbar_arrive_expect_tx(qbar, kBM * kRowBytes);
      tma_load_3d(smem_u32(sm.q), &tm_q, 0, kvh * kG, qs + q0, qbar);
      const int oob_row = a.num_pages * kPS;   // reads as zeros
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j % kST;
        if (j >= kST &&
            !mbar_wait(smem_u32(&sm.kv_empty[st]), ((j / kST) + 1) & 1)) {
          flag_error(a.err, DEVERR_TIMEOUT);
          break;
        }
        uint32_t bad = 0;
        int rows[kPagesPerTile];
#pragma unroll
        for (int p = 0; p < kPagesPerTile; ++p) {
          const int lp = j * kPagesPerTile + p;
          int y = oob_row;
          if (lp < n_pages) {
            const int pid = __ldg(bt + lp);
            if (pid >= 0 && pid < a.num_pages) {
              y = pid * kPS;
            } else {
              bad |= 1u << p;
            }
          }
          rows[p] = y;
        }
        if (bad) flag_error(a.err, DEVERR_BAD_PAGE);
        sm.bad_pages[st] = bad;
        const uint32_t bar = smem_u32(&sm.kv_full[st]);
        mbar_arrive_expect_tx(bar, 2 * kTileBytes);
#pragma unroll
        for (int p = 0; p < kPagesPerTile; ++p) {
          tma_load_2d(smem_u32(sm.k[st]) + p * kPageBytes, &tm_k, kvh * kD,
                      rows[p], bar);
          tma_load_2d(smem_u32(sm.v[st]) + p * kPageBytes, &tm_v, kvh * kD,
                      rows[p], bar);
        }
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================================
    if (lane == 0) {
      bool ok = mbar_wait(smem_u32(&sm.q_full), 0);
      const uint32_t q_addr = smem_u32(sm.q);
      auto issue_pv = [&](int t) -> bool {
        const int b = t & 1;
        const int st = t % kST;
        if (!mbar_wait(smem_u32(&sm.p_full[b]), (t >> 1) & 1)) return false;
        if (t >= 2 &&
            !mbar_wait(smem_u32(&sm.o_free[b]), ((t >> 1) + 1) & 1))
          return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sm.v[st]);
#pragma unroll
        for (int part = 0; part < 2; ++part) {          // P_hi, then P_lo
          const uint32_t p_addr = smem_u32(sm.p[b][part][0]);
#pragma unroll
          for (int k = 0; k < kBN / 16; ++k) {
            // A = P: K-major; keys [16k, 16k+16) sit in half k/4, byte 32*(k%4)
            const uint64_t ad = smem_desc_sw128(
                p_addr + (k >> 2) * (kBM * kRowBytes) + (k & 3) * 32, 16,
                1024);
            // B = V: MN-major (head dim contiguous); 16 keys = 2 x 8 rows
            const uint64_t bd =
                smem_desc_sw128(v_addr + k * 16 * kRowBytes, kTileBytes, 1024);
            tc_mma_bf16(tmem + kOCol + b * kD, ad, bd, kIdescPV,
                        (part | k) != 0);
          }
        }
        tc_commit(smem_u32(&sm.o_full[b]));
        tc_commit(smem_u32(&sm.kv_empty[st]));
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int st = j % kST;
        const int b = j & 1;
        if (!mbar_wait(smem_u32(&sm.kv_full[st]), (j / kST) & 1) ||
            (j >= 2 &&
             !mbar_wait(smem_u32(&sm.s_free[b]), ((j >> 1) + 1) & 1))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sm.k[st]);
#pragma unroll
        for (int k = 0; k < kD / 16; ++k) {
          const uint64_t ad = smem_desc_sw128(q_addr + k * 32, 16, 1024);
          const uint64_t bd = smem_desc_sw128(k_addr + k * 32, 16, 1024);
          tc_mma_bf16(tmem + kSCol + b * kBN, ad, bd, kIdescQK, k > 0);
        }
        tc_commit(smem_u32(&sm.s_full[b]));
        if (j >= 1 && !issue_pv(j - 1)) {
          ok = false;
          break;
        }
      }
      if (ok && !issue_pv(n_tiles - 1)) ok = false;
      if (!ok) flag_error(a.err, DEVERR_TIMEOUT);
    }
  } else {
    // ======================= softmax warps ====================================
    const int quarter = warp & 3;            // tensor-memory lane quarter
    const int r = quarter * 32 + lane;       // MMA row
    const int qi = r >> 2;                   // query row within the tile
    const int hh = r & 3;                    // head within the group
    const bool row_real = q0 + qi < T;
    const int limit = row_real ? P + q0 + qi : ctx - 1;  // last visible key
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const float c = a.scale_log2;

    float o[kD];
#pragma unroll
    for (int d = 0; d < kD; ++d) o[d] = 0.f;
    float m_run = -INFINITY, l_run = 0.f, alpha_prev = 1.f;
    bool ok = true;

    auto fold_o = [&](int t, float alpha) -> bool {
      const int b = t & 1;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(smem_u32(&sm.o_full[b]), (t >> 1) & 1)))
        return false;
      tc_fence_after();
      float ov[32];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        tmem_ld32(tmem + lane_base + kOCol + b * kD + h2 * 32, ov);
#pragma unroll
        for (int d = 0; d < 32; ++d)
          o[h2 * 32 + d] = fmaf(o[h2 * 32 + d], alpha, ov[d]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.o_free[b]));
      return true;
    };

    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      const int st = j % kST;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(smem_u32(&sm.s_full[b]), (j >> 1) & 1))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[kBN];
#pragma unroll
      for (int cq = 0; cq < kBN / 32; ++cq) {
        float tmp[32];
        tmem_ld32(tmem + lane_base + kSCol + b * kBN + cq * 32, tmp);
#pragma unroll
        for (int x = 0; x < 32; ++x) s[cq * 32 + x] = tmp[x];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.s_free[b]));

      // ---- mask, running max, exponentials --------------------------------
      const int key0 = j * kBN;
      const uint32_t bad = sm.bad_pages[st];
      float tmax = -INFINITY;
#pragma unroll
      for (int x = 0; x < kBN; ++x) {
        const int key = key0 + x;
        const bool vis = key <= limit && !((bad >> (x / kPS)) & 1u);
        s[x] = vis ? s[x] * c : -INFINITY;
        tmax = fmaxf(tmax, s[x]);
      }
      const float m_new = fmaxf(m_run, tmax);
      const float m_use = m_new == -INFINITY ? 0.f : m_new;
      const float alpha = fast_exp2(m_run - m_use);
      float lsum = 0.f;
#pragma unroll
      for (int x = 0; x < kBN; ++x) {
        s[x] = fast_exp2(s[x] - m_use);
        lsum += s[x];
      }
      l_run = fmaf(l_run, alpha, lsum);
      m_run = m_new;

      // ---- keys past the context in a loaded page may hold stale data:
      //      zero their V rows so that P = 0 cannot meet NaN in the MMA -----
      {
        const int z0 = max(ctx, key0);
        const int z1 = min(((n_keys + kPS - 1) / kPS) * kPS, key0 + kBN);
        const int nz = (z1 - z0) * (kRowBytes / 16);
        for (int t = threadIdx.x - 64; t < nz; t += 128) {
          const int row = z0 - key0 + t / (kRowBytes / 16);
          const int ch = t % (kRowBytes / 16);
          *reinterpret_cast<uint4*>(&sm.v[st][row * kRowBytes + ch * 16]) =
              make_uint4(0, 0, 0, 0);
        }
      }

      // ---- P_hi, P_lo (bf16) into the swizzled K-major layout -------------------
      {
        uint8_t* phi = sm.p[b][0][0] + r * kRowBytes;
        uint8_t* plo = sm.p[b][1][0] + r * kRowBytes;
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int x = half * 64 + ch * 8;
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              hi[e] = pack_bf16x2(s[x + 2 * e], s[x + 2 * e + 1]);
              lo[e] = pack_bf16x2(s[x + 2 * e] - bf16_lo(hi[e]),
                                  s[x + 2 * e + 1] - bf16_hi(hi[e]));
            }
            const int off = half * (kBM * kRowBytes) + ((ch ^ (r & 7)) * 16);
            *reinterpret_cast<uint4*>(phi + off) =
                make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(plo + off) =
                make_uint4(lo[0], lo[1], lo[2], lo[3]);
          }
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[b]));

      // ---- fold the previous tile's P.V ------------------------------------------
      if (j >= 1 && !fold_o(j - 1, alpha_prev)) {
        ok = false;
        break;
      }
      alpha_prev = alpha;
    }
    if (ok && !fold_o(n_tiles - 1, alpha_prev)) ok = false;
    if (!ok) {
      if (lane == 0) flag_error(a.err, DEVERR_TIMEOUT);
#pragma unroll
      for (int d = 0; d < kD; ++d) o[d] = 0.f;
      l_run = 0.f;
    }

    // ---- normalise and store ---------------------------------------------------
    if (row_real) {
      const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
      __nv_bfloat16* dst =
          a.out + ((size_t)(qs + q0 + qi) * a.num_q_heads + kvh * kG + hh) * kD;
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
  cudaError_t e = cudaFuncSetAttribute(
      paged_prefill_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int tiles = (a.max_query_len + kQRows - 1) / kQRows;
  dim3 grid(a.num_kv_heads, tiles, a.num_seqs);
  paged_prefill_kernel<<<grid, kThreads, smem, stream>>>(a, tq, tk, tv);
  return cudaGetLastError();
}

}  // namespace tv
