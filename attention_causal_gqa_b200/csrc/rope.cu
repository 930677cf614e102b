// RoPE prologue ("From 32K to 256K: DeepSeek long-context", section 2.1 for the
// rotation, section 2.5 for the cos/sin cache [max_len, head_dim/2, 2]).
//
// The table stores cos and sin of pos * theta^(-2i/D) for every integer position
// and pair; each angle is formed in fp64 straight from the integer position (no
// running phase), then rounded to fp32. Pairs are adjacent elements (2i, 2i+1):
//   y[2i]   = x[2i] cos - x[2i+1] sin
//   y[2i+1] = x[2i] sin + x[2i+1] cos
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"

namespace attn {

__global__ void rope_table_kernel(float2* __restrict__ cs, int S, int D, double theta) {
  const int half = D / 2;
  const long long n = static_cast<long long>(S) * half;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int pos = static_cast<int>(idx / half);
    const int i = static_cast<int>(idx % half);
    const double inv_freq = pow(theta, -2.0 * i / D);
    double s, c;
    sincos(static_cast<double>(pos) * inv_freq, &s, &c);
    cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// bf16 K [rows, D] (row r at position r % S) -> rotated fp16 K. One thread per
// 8 elements. Values beyond the fp16 range set the range flag of the status word.
__global__ void rope_k_f16_kernel(const uint4* __restrict__ x, uint4* __restrict__ y,
                                  const float2* __restrict__ cs, long long rows, int S, int D,
                                  int* __restrict__ status) {
  const int cpr = D / 8;
  const long long n = rows * cpr;
  bool in_range = true;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = idx / cpr;
    const int c = static_cast<int>(idx % cpr);
    const int pos = static_cast<int>(r % S);
    const uint4 raw = x[idx];
    const float2* t = cs + static_cast<long long>(pos) * (D / 2) + c * 4;
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t ow[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = __uint_as_float(w[e] << 16);
      const float x1 = __uint_as_float(w[e] & 0xFFFF0000u);
      const float2 a = t[e];
      const float y0 = x0 * a.x - x1 * a.y, y1 = x0 * a.y + x1 * a.x;
      in_range = in_range && fabsf(y0) <= 65504.f && fabsf(y1) <= 65504.f;
      const __half2 v = __floats2half2_rn(y0, y1);
      ow[e] = *reinterpret_cast<const uint32_t*>(&v);
    }
    y[idx] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
  if (!in_range) atomicOr(status, 8);
}

// fp32 X [rows, D] -> hi = bf16(x) in out[0, rows), lo = bf16(x - hi) in out[rows, 2 rows),
// rotating first (row r at position r % S) when cs is non-null. One thread per 8 elements.
__global__ void split_f32_kernel(const float4* __restrict__ x, uint4* __restrict__ out,
                                 const float2* __restrict__ cs, long long rows, int S, int D) {
  const int cpr = D / 8;
  const long long n = rows * cpr;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float4 a = x[2 * idx], b = x[2 * idx + 1];
    float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    if (cs) {
      const long long r = idx / cpr;
      const int c = static_cast<int>(idx % cpr);
      const float2* t = cs + static_cast<long long>(r % S) * (D / 2) + c * 4;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 cz = t[e];
        const float x0 = f[2 * e], x1 = f[2 * e + 1];
        f[2 * e] = x0 * cz.x - x1 * cz.y;
        f[2 * e + 1] = x0 * cz.y + x1 * cz.x;
      }
    }
    uint32_t hw[4], lw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
      const float2 hf = __bfloat1622float2(h);
      const __nv_bfloat162 l = __floats2bfloat162_rn(f[2 * e] - hf.x, f[2 * e + 1] - hf.y);
      hw[e] = *reinterpret_cast<const uint32_t*>(&h);
      lw[e] = *reinterpret_cast<const uint32_t*>(&l);
    }
    out[idx] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
    out[idx + n] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
  }
}

static int grid_for(long long n, int threads) {
  long long g = (n + threads - 1) / threads;
  const long long cap = 148LL * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

cudaError_t launch_rope_table(float2* cs, int S, int D, double theta, cudaStream_t stream) {
  const long long n = static_cast<long long>(S) * (D / 2);
  rope_table_kernel<<<grid_for(n, 256), 256, 0, stream>>>(cs, S, D, theta);
  return cudaGetLastError();
}

cudaError_t launch_rope_k_f16(const void* k, void* k_f16, const float2* cs, long long rows, int S, int D,
                              int* status, cudaStream_t stream) {
  const long long n = rows * (D / 8);
  rope_k_f16_kernel<<<grid_for(n, 256), 256, 0, stream>>>(static_cast<const uint4*>(k), static_cast<uint4*>(k_f16),
                                                          cs, rows, S, D, status);
  return cudaGetLastError();
}

cudaError_t launch_split_f32(const float* x, void* out, const float2* cs, long long rows, int S, int D,
                             cudaStream_t stream) {
  const long long n = rows * (D / 8);
  split_f32_kernel<<<grid_for(n, 256), 256, 0, stream>>>(reinterpret_cast<const float4*>(x),
                                                         static_cast<uint4*>(out), cs, rows, S, D);
  return cudaGetLastError();
}

}  // namespace attn
