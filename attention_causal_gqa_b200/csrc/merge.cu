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
#include "sm100.cuh"

namespace attn {

// One CTA per (sequence b, group of kMergeHeads heads); the partials of split s of b
// are one contiguous [H, D] fp32 block, so a CTA reads a contiguous kMergeHeads x D slab
// per split (every thread 4 consecutive columns, all splits' loads in flight in batches).
// The split weights w = e^(lse_s - max) and their sums are formed once per head in
// shared memory; the result is o = sum_s w_s o_s / sum_s w_s in split order
// (deterministic), lse = max + ln sum_s w_s.
constexpr int kMergeHeads = 8;
constexpr int kMergeMaxSplits = 256;  // splits whose weights fit the CTA's table; the rest in a second pass

__global__ void __launch_bounds__(256) merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                                    const int32_t* __restrict__ seq_lens, __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse, int B, int H, int D, int n_splits,
                                                    int tokens_per_split) {
  griddep_wait();  // launched as a dependent of the kernel that wrote the partials
  __shared__ float s_w[kMergeMaxSplits][kMergeHeads];
  __shared__ float s_m[kMergeHeads], s_sum[kMergeHeads];
  const int groups = (H + kMergeHeads - 1) / kMergeHeads;
  const int b = blockIdx.x / groups, h0 = (blockIdx.x % groups) * kMergeHeads;
  const int nh = min(kMergeHeads, H - h0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = max(0, __ldg(seq_lens + b));
  const int ns = min((L + tokens_per_split - 1) / tokens_per_split, n_splits);
  // this thread's 4 columns of the slab: head h0 + hh, column d
  const int per_head = D / 4;  // 4-column groups per head
  const int hh = tid / per_head, d = (tid % per_head) * 4;
  const bool active = hh < nh && tid < kMergeHeads * per_head;
  if (ns == 0) {
    if (active) *reinterpret_cast<uint2*>(out + (static_cast<size_t>(b) * H + h0 + hh) * D + d) = make_uint2(0u, 0u);
    if (tid < nh) lse[static_cast<size_t>(b) * H + h0 + tid] = -INFINITY;
    return;
  }
  const float* pl = part_lse + static_cast<size_t>(b) * n_splits * H + h0;
  // warp w < nh: the maximum and the weights of head h0 + w over the splits
  if (warp < nh) {
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, __ldg(pl + static_cast<size_t>(s) * H + warp));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float sum = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float w = __expf(__ldg(pl + static_cast<size_t>(s) * H + warp) - M);
      if (s < kMergeMaxSplits) s_w[s][warp] = w;
      sum += w;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if (lane == 0) {
      s_m[warp] = M;
      s_sum[warp] = sum;
    }
  }
  __syncthreads();
  if (!active) return;
  const float* po = part_o + (static_cast<size_t>(b) * n_splits * H + h0 + hh) * D + d;
  const size_t stride = static_cast<size_t>(H) * D;  // from one split's block to the next
  const float Mh = s_m[hh];
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int kBatch = 8;
  for (int s0 = 0; s0 < ns; s0 += kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u)
      if (s0 + u < ns) v[u] = *reinterpret_cast<const float4*>(po + (s0 + u) * stride);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int s = s0 + u;
      if (s < ns) {
        const float w = s < kMergeMaxSplits ? s_w[s][hh] : __expf(__ldg(pl + static_cast<size_t>(s) * H + hh) - Mh);
        acc.x += w * v[u].x;
        acc.y += w * v[u].y;
        acc.z += w * v[u].z;
        acc.w += w * v[u].w;
      }
    }
  }
  const float inv = 1.f / s_sum[hh];
  const __nv_bfloat162 a = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 c = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&c);
  *reinterpret_cast<uint2*>(out + (static_cast<size_t>(b) * H + h0 + hh) * D + d) = u;
  if (d == 0) lse[static_cast<size_t>(b) * H + h0 + hh] = Mh + logf(s_sum[hh]);
}

cudaError_t launch_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out, float* lse,
                         int B, int H, int D, int n_splits, int tokens_per_split, cudaStream_t stream) {
  if (D % 4 != 0 || kMergeHeads * (D / 4) > 256) return cudaErrorInvalidValue;
  const long long blocks = static_cast<long long>(B) * ((H + kMergeHeads - 1) / kMergeHeads);
  return launch_pdl(merge_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream, part_o, part_lse,
                    seq_lens, static_cast<__nv_bfloat16*>(out), lse, B, H, D, n_splits, tokens_per_split);
}

// ------------------------------------------------------------ parts merge
// Partial results of the same query rows over disjoint key sets, one per part (the
// slices of every sequence's cache that different GPUs hold): bf16 outputs
// [n_parts, rows, D] and fp32 LSEs [n_parts, rows], combined in part order. One warp
// per row; lane l owns the column pairs 2l + 64 i.
template <int D>
__global__ void parts_merge_kernel(const __nv_bfloat16* __restrict__ o_parts, const float* __restrict__ lse_parts,
                                   int n_parts, long long rows, __nv_bfloat16* __restrict__ out,
                                   float* __restrict__ lse) {
  constexpr int NP = D / 64;  // column pairs per lane
  const long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float M = -INFINITY;
  for (int s = lane; s < n_parts; s += 32) M = fmaxf(M, lse_parts[static_cast<size_t>(s) * rows + r]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  __nv_bfloat162* orow = reinterpret_cast<__nv_bfloat162*>(out + r * D);
  if (!(M > -INFINITY)) {  // every part empty: no key at all
#pragma unroll
    for (int i = 0; i < NP; ++i) orow[lane + 32 * i] = __floats2bfloat162_rn(0.f, 0.f);
    if (lane == 0) lse[r] = -INFINITY;
    return;
  }
  float2 acc[NP];
#pragma unroll
  for (int i = 0; i < NP; ++i) acc[i] = make_float2(0.f, 0.f);
  float wsum = 0.f;
  for (int s = 0; s < n_parts; ++s) {
    const float ls = lse_parts[static_cast<size_t>(s) * rows + r];
    if (!(ls > -INFINITY)) continue;  // an empty part carries no weight (its output is not read)
    const float w = __expf(ls - M);
    wsum += w;
    const __nv_bfloat162* po = reinterpret_cast<const __nv_bfloat162*>(o_parts + (static_cast<size_t>(s) * rows + r) * D);
#pragma unroll
    for (int i = 0; i < NP; ++i) {
      const float2 v = __bfloat1622float2(po[lane + 32 * i]);
      acc[i].x += w * v.x;
      acc[i].y += w * v.y;
    }
  }
  const float inv = 1.f / wsum;
#pragma unroll
  for (int i = 0; i < NP; ++i) orow[lane + 32 * i] = __floats2bfloat162_rn(acc[i].x * inv, acc[i].y * inv);
  if (lane == 0) lse[r] = M + logf(wsum);
}

cudaError_t launch_parts_merge(const void* o_parts, const float* lse_parts, int n_parts, long long rows, int D,
                               void* out, float* lse, cudaStream_t stream) {
  const int threads = 256;
  const long long blocks = (rows * 32 + threads - 1) / threads;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  const auto* op = static_cast<const __nv_bfloat16*>(o_parts);
  auto* o = static_cast<__nv_bfloat16*>(out);
  switch (D) {
    case 64: parts_merge_kernel<64><<<static_cast<int>(blocks), threads, 0, stream>>>(op, lse_parts, n_parts, rows, o, lse); break;
    case 128: parts_merge_kernel<128><<<static_cast<int>(blocks), threads, 0, stream>>>(op, lse_parts, n_parts, rows, o, lse); break;
    case 256: parts_merge_kernel<256><<<static_cast<int>(blocks), threads, 0, stream>>>(op, lse_parts, n_parts, rows, o, lse); break;
    case 512: parts_merge_kernel<512><<<static_cast<int>(blocks), threads, 0, stream>>>(op, lse_parts, n_parts, rows, o, lse); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

// ------------------------------------------------------------ range merge
template <int UNIT>
__device__ __forceinline__ int units_of(const int32_t* lens, int b, int T_max) {
  const int L = min(max(__ldg(lens + b), 0), T_max);
  return (L + UNIT - 1) / UNIT;
}

// One warp per (b, head). The partial-result kernels that balance work by ranges
// (the MLA decode with 64-token tiles as units, the FP8 paged decode with 16-token
// pages) lay the units of all sequences out in one position space, a non-empty
// sequence of n units taking SEG + n positions (its unit u at position SEG + u; SEG
// weighs the fixed cost of a segment), and cut its N positions into n_ranges contiguous
// ranges [N c / n_ranges, N (c + 1) / n_ranges); range c writes one partial result per
// sequence it meets, at slot c + b. The ranges meeting sequence b (units at positions
// [f_b, e_b)) are those from the one holding position f_b to the one holding e_b - 1:
// range c holds position x iff floor(N c / P) <= x < floor(N (c + 1) / P), i.e.
// c = floor(((x + 1) P - 1) / N). They are combined in range order (deterministic).
template <int DIM, int UNIT, int SEG>
__global__ void range_merge_kernel(const float* __restrict__ part_o, const float* __restrict__ part_lse,
                                   const int32_t* __restrict__ seq_lens, __nv_bfloat16* __restrict__ out,
                                   float* __restrict__ lse, int B, int H, int T_max, int n_ranges) {
  griddep_wait();  // launched as a dependent of the kernel that wrote the partials
  constexpr int VEC = DIM / 32;  // contiguous columns per lane
  static_assert(VEC == 2 || VEC % 4 == 0, "whole float2 or float4 columns per lane");
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= B * H) return;
  const int b = gw / H, h = gw % H;
  long long N = 0, s_b = 0;
  for (int i = lane; i < B; i += 32) {
    const int n = units_of<UNIT>(seq_lens, i, T_max);
    const int u = n > 0 ? n + SEG : 0;
    N += u;
    if (i < b) s_b += u;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    N += __shfl_xor_sync(0xffffffffu, N, o);
    s_b += __shfl_xor_sync(0xffffffffu, s_b, o);
  }
  const int n_b = units_of<UNIT>(seq_lens, b, T_max);
  const long long f_b = s_b + SEG, e_b = f_b + n_b;
  const long long P = n_ranges;
  int c0 = 0, c1 = -1;  // contributing ranges (none for an empty sequence)
  if (n_b > 0) {
    c0 = static_cast<int>(((f_b + 1) * P - 1) / N);
    c1 = static_cast<int>((e_b * P - 1) / N);
  }
  __nv_bfloat16* orow = out + static_cast<size_t>(gw) * DIM + lane * VEC;
  float M = -INFINITY;
  for (int c = c0; c <= c1; ++c)
    if (N * (c + 1) / P > N * c / P) M = fmaxf(M, part_lse[static_cast<size_t>(c + b) * H + h]);
  uint32_t packed[VEC / 2];
  if (!(M > -INFINITY)) {
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) packed[i] = 0u;
    if (lane == 0) lse[gw] = -INFINITY;
  } else {
    float acc[VEC];
#pragma unroll
    for (int i = 0; i < VEC; ++i) acc[i] = 0.f;
    float wsum = 0.f;
#pragma unroll 2
    for (int c = c0; c <= c1; ++c) {
      if (!(N * (c + 1) / P > N * c / P)) continue;  // an empty range writes nothing
      const size_t slot = static_cast<size_t>(c + b);
      const float w = __expf(part_lse[slot * H + h] - M);
      wsum += w;
      const float* po = part_o + (slot * H + h) * DIM + lane * VEC;
      if constexpr (VEC == 2) {
        const float2 v = *reinterpret_cast<const float2*>(po);
        acc[0] += w * v.x;
        acc[1] += w * v.y;
      } else {
#pragma unroll
        for (int q = 0; q < VEC / 4; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(po + 4 * q);
          acc[4 * q] += w * v.x;
          acc[4 * q + 1] += w * v.y;
          acc[4 * q + 2] += w * v.z;
          acc[4 * q + 3] += w * v.w;
        }
      }
    }
    const float inv = 1.f / wsum;
#pragma unroll
    for (int i = 0; i < VEC / 2; ++i) {
      const __nv_bfloat162 t = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
      packed[i] = *reinterpret_cast<const uint32_t*>(&t);
    }
    if (lane == 0) lse[gw] = M + logf(wsum);
  }
  if constexpr (VEC % 8 == 0) {
#pragma unroll
    for (int i = 0; i < VEC / 8; ++i)
      reinterpret_cast<uint4*>(orow)[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
  } else if constexpr (VEC == 4) {
    reinterpret_cast<uint2*>(orow)[0] = make_uint2(packed[0], packed[1]);
  } else {
    reinterpret_cast<uint32_t*>(orow)[0] = packed[0];
  }
}

template <int DIM, int UNIT, int SEG>
static cudaError_t launch_range_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out,
                                      float* lse, int B, int H, int T_max, int n_ranges, cudaStream_t stream) {
  const long long warps = static_cast<long long>(B) * H;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  return launch_pdl(range_merge_kernel<DIM, UNIT, SEG>, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0, stream,
                    part_o, part_lse, seq_lens, static_cast<__nv_bfloat16*>(out), lse, B, H, T_max, n_ranges);
}

cudaError_t launch_mla_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out,
                             float* lse, int B, int H, int T_max, int n_pairs, cudaStream_t stream) {
  return launch_range_merge<512, kMlaTile, kMlaSegCost>(part_o, part_lse, seq_lens, out, lse, B, H, T_max, n_pairs, stream);
}

cudaError_t launch_decode_range_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out,
                                      float* lse, int B, int H, int D, int T_max, int n_ranges, cudaStream_t stream) {
  if (D == 64) return launch_range_merge<64, 16, 0>(part_o, part_lse, seq_lens, out, lse, B, H, T_max, n_ranges, stream);
  if (D == 128) return launch_range_merge<128, 16, 0>(part_o, part_lse, seq_lens, out, lse, B, H, T_max, n_ranges, stream);
  return cudaErrorInvalidValue;
}

}  // namespace attn
