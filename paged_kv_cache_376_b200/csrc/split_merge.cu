// Log-sum-exp merge of split-KV partials.
//
// A long context is cut into logical partitions of partition_tokens keys;
// paged_decode.cu writes, per (sequence, head, partition p), the normalised
// partial output o_p and lse_p = ln(sum of exp(scaled scores)) over that
// partition.  Softmax over the whole context is then the blockwise form of
// the online softmax ("tiny-vllm：从零构建高性能LLM推理引擎的完整指南", sec.
// "在线Softmax：数值稳定的注意力计算"; "Tiny-vLLM 实战：用 C++/CUDA 手写高性能
// LLM 推理引擎", sec. "算子融合" on tiled attention):
//   M = max_p lse_p,  out = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M).
//
// One CTA of 128 threads per (head, sequence): the lse row is reduced in
// shared memory, then 8 partition lanes x 16 lanes of float4 stream the
// partials (each partition row is 256 contiguous bytes).
#include "tv_device.cuh"
#include "tv_kernels.h"

namespace tv {
namespace {

constexpr int kD = 64;
constexpr int kThreads = 128;
constexpr int kPartLanes = kThreads / (kD / 4);  // 8

__global__ void __launch_bounds__(kThreads)
    split_merge_kernel(__nv_bfloat16* __restrict__ out,
                       const float* __restrict__ partial_out,
                       const float* __restrict__ partial_lse,
                       const int32_t* __restrict__ context_lens,
                       int num_q_heads, int partition_tokens,
                       int max_partitions) {
  __shared__ float red[kThreads];
  __shared__ float4 accs[kPartLanes][kD / 4];
  const int h = blockIdx.x;
  const int seq = blockIdx.y;
  const int tid = threadIdx.x;
  const size_t row = (size_t)seq * num_q_heads + h;
  const float* lse = partial_lse + row * max_partitions;
  const float* po = partial_out + row * max_partitions * kD;

  int ctx = context_lens[seq];
  if (ctx < 0) ctx = 0;
  int nparts = (ctx + partition_tokens - 1) / partition_tokens;
  if (nparts > max_partitions) nparts = max_partitions;

  // M = max lse
  float m = -INFINITY;
  for (int p = tid; p < nparts; p += kThreads) m = fmaxf(m, lse[p]);
  red[tid] = m;
  __syncthreads();
  for (int s = kThreads / 2; s > 0; s >>= 1) {
    if (tid < s) red[tid] = fmaxf(red[tid], red[tid + s]);
    __syncthreads();
  }
  const float M = red[0];
  __syncthreads();

  // weighted sums
  const int pl = tid / (kD / 4);   // partition lane
  const int dq = tid % (kD / 4);   // float4 of the head dim
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float wsum = 0.f;
  if (M != -INFINITY) {
    // four partitions per lane in flight: the loads of a group are issued
    // before any of them is used (the merge is bound by their latency)
    constexpr int kU = 4;
    int p = pl;
    for (; p + (kU - 1) * kPartLanes < nparts; p += kU * kPartLanes) {
      float l[kU];
      float4 v[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        l[u] = lse[p + u * kPartLanes];
        v[u] = reinterpret_cast<const float4*>(
            po + (size_t)(p + u * kPartLanes) * kD)[dq];
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const float w =
            l[u] == -INFINITY ? 0.f : fast_exp2((l[u] - M) * kLog2e);
        acc.x = fmaf(w, v[u].x, acc.x);
        acc.y = fmaf(w, v[u].y, acc.y);
        acc.z = fmaf(w, v[u].z, acc.z);
        acc.w = fmaf(w, v[u].w, acc.w);
        wsum += w;
      }
    }
    for (; p < nparts; p += kPartLanes) {
      const float l = lse[p];
      const float w = l == -INFINITY ? 0.f : fast_exp2((l - M) * kLog2e);
      const float4 v = reinterpret_cast<const float4*>(po + (size_t)p * kD)[dq];
      acc.x = fmaf(w, v.x, acc.x);
      acc.y = fmaf(w, v.y, acc.y);
      acc.z = fmaf(w, v.z, acc.z);
      acc.w = fmaf(w, v.w, acc.w);
      wsum += w;
    }
  }
  accs[pl][dq] = acc;
  red[tid] = wsum;   // identical across dq lanes of one partition lane
  __syncthreads();
  if (tid < kD / 4) {
    float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
    float W = 0.f;
#pragma unroll
    for (int k = 0; k < kPartLanes; ++k) {
      const float4 v = accs[k][tid];
      t.x += v.x;
      t.y += v.y;
      t.z += v.z;
      t.w += v.w;
      W += red[k * (kD / 4)];
    }
    const float inv = W > 0.f ? 1.f / W : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(t.x * inv, t.y * inv);
    packed.y = pack_bf16x2(t.z * inv, t.w * inv);
    reinterpret_cast<uint2*>(out + row * kD)[tid] = packed;
  }
}

}  // namespace

cudaError_t launch_split_merge(__nv_bfloat16* out, const float* partial_out,
                               const float* partial_lse,
                               const int32_t* context_lens, int num_seqs,
                               int num_q_heads, int partition_tokens,
                               int max_partitions, cudaStream_t stream) {
  if (num_seqs == 0) return cudaSuccess;
  dim3 grid(num_q_heads, num_seqs);
  split_merge_kernel<<<grid, kThreads, 0, stream>>>(
      out, partial_out, partial_lse, context_lens, num_q_heads,
      partition_tokens, max_partitions);
  return cudaGetLastError();
}

}  // namespace tv
