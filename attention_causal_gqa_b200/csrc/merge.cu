// LSE merge of split-KV partial results.
//
// The online-softmax recurrence of the "attention study note" (section
// "online-softmax 分块计算原理"), applied to whole splits: with normalised partial
// outputs o_s and log-sum-exps lse_s of disjoint key sets,
//   M = max_s lse_s,  w_s = exp(lse_s - M),
//   lse = M + ln(sum_s w_s),  o = sum_s w_s o_s / sum_s w_s.
// Splits are combined in index order, so the result is deterministic.
#include <cuda_bf16.h>

#include "kernels.h"

namespace attn {

// One warp per (b, head); lanes own interleaved 4-column groups.
__global__ void merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                             const int32_t* __restrict__ seq_lens, __nv_bfloat16* __restrict__ out,
                             float* __restrict__ lse, int B, int H, int D, int n_splits, int tokens_per_split) {
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= B * H) return;
  const int b = gw / H, h = gw % H;
  const int L = max(0, __ldg(seq_lens + b));
  int ns = (L + tokens_per_split - 1) / tokens_per_split;
  ns = min(ns, n_splits);
  __nv_bfloat16* orow = out + static_cast<size_t>(gw) * D;
  if (ns == 0) {
    for (int d = lane * 4; d < D; d += 128) {
      reinterpret_cast<uint2*>(orow + d)[0] = make_uint2(0u, 0u);
    }
    if (lane == 0) lse[gw] = -INFINITY;
    return;
  }
  const float* pl = part_lse + static_cast<size_t>(b) * n_splits * H + h;
  float M = -INFINITY;
  for (int s = lane; s < ns; s += 32) M = fmaxf(M, pl[static_cast<size_t>(s) * H]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float w = __expf(pl[static_cast<size_t>(s) * H] - M);
    wsum += w;
    const float* po = part_o + ((static_cast<size_t>(b) * n_splits + s) * H + h) * D;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int d = lane * 4 + i * 128;
      if (d < D) {
        const float4 v = *reinterpret_cast<const float4*>(po + d);
        acc[4 * i] += w * v.x;
        acc[4 * i + 1] += w * v.y;
        acc[4 * i + 2] += w * v.z;
        acc[4 * i + 3] += w * v.w;
      }
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int d = lane * 4 + i * 128;
    if (d < D) {
      const __nv_bfloat162 a = __floats2bfloat162_rn(acc[4 * i] * inv, acc[4 * i + 1] * inv);
      const __nv_bfloat162 c = __floats2bfloat162_rn(acc[4 * i + 2] * inv, acc[4 * i + 3] * inv);
      uint2 u;
      u.x = *reinterpret_cast<const uint32_t*>(&a);
      u.y = *reinterpret_cast<const uint32_t*>(&c);
      *reinterpret_cast<uint2*>(orow + d) = u;
    }
  }
  if (lane == 0) lse[gw] = M + logf(wsum);
}

cudaError_t launch_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out, float* lse,
                         int B, int H, int D, int n_splits, int tokens_per_split, cudaStream_t stream) {
  const long long warps = static_cast<long long>(B) * H;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  merge_kernel<<<static_cast<int>(blocks), threads, 0, stream>>>(part_o, part_lse, seq_lens,
                                                                 static_cast<__nv_bfloat16*>(out), lse, B, H, D,
                                                                 n_splits, tokens_per_split);
  return cudaGetLastError();
}

}  // namespace attn
