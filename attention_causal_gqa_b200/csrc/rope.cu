// RoPE prologue ("From 32K to 256K: DeepSeek long-context", section 2.1 for the
// rotation, section 2.5 for the cos/sin cache [max_len, head_dim/2, 2]).
//
// The table stores cos and sin of pos * theta^(-2i/D) for every integer position
// and pair; each angle is formed in fp64 straight from the integer position (no
// running phase), then rounded to fp32. Pairs are adjacent elements (2i, 2i+1):
//   y[2i]   = x[2i] cos - x[2i+1] sin
//   y[2i+1] = x[2i] sin + x[2i+1] cos
#include <cmath>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "prologue.h"

namespace attn {

// theta^(-2i/D) for every pair i, computed once on the host in fp64.
struct RopeFreqs {
  double inv[64];
};

__global__ void rope_table_kernel(float2* __restrict__ cs, int S, int half, const __grid_constant__ RopeFreqs f) {
  const long long n = static_cast<long long>(S) * half;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int pos = static_cast<int>(idx / half);
    const int i = static_cast<int>(idx - static_cast<long long>(pos) * half);
    double s, c;
    sincos(static_cast<double>(pos) * f.inv[i], &s, &c);
    cs[idx] = make_float2(static_cast<float>(c), static_cast<float>(s));
  }
}

// The two operand-preparation kernels share one layout: a block of 256 threads
// covers 256 / CPR consecutive positions (CPR = D / 8 chunks of 8 elements per
// row), and blockIdx.y strides over the heads. Each thread loads the cos/sin of
// its chunk once and reuses them for every head it visits, and all index
// arithmetic is 32-bit except the final element offset.
template <int CPR>
__device__ __forceinline__ bool chunk_position(int S, int& pos, int& c) {
  constexpr int RPB = 256 / CPR;
  c = threadIdx.x % CPR;
  pos = blockIdx.x * RPB + threadIdx.x / CPR;
  return pos < S;
}

template <int CPR>
__device__ __forceinline__ void load_cs4(const float2* __restrict__ cs, int pos, int c, float2 (&a)[4]) {
  const float4* t = reinterpret_cast<const float4*>(cs + static_cast<size_t>(pos) * (CPR * 4) + c * 4);
  const float4 t0 = __ldg(t), t1 = __ldg(t + 1);
  a[0] = make_float2(t0.x, t0.y);
  a[1] = make_float2(t0.z, t0.w);
  a[2] = make_float2(t1.x, t1.y);
  a[3] = make_float2(t1.z, t1.w);
}

// bf16 X [heads, S, D] -> rotated fp16 X (used for K and for Q). Values beyond
// the fp16 range set the range flag of the status word.
template <int CPR>
__global__ void __launch_bounds__(256) rope_f16_kernel(const uint4* __restrict__ x, uint4* __restrict__ y,
                                                       const float2* __restrict__ cs, int heads, int S,
                                                       int* __restrict__ status) {
  int pos, c;
  if (!chunk_position<CPR>(S, pos, c)) return;
  float2 a[4];
  load_cs4<CPR>(cs, pos, c, a);
  bool in_range = true;
  for (int hd = blockIdx.y; hd < heads; hd += gridDim.y) {
    const size_t idx = (static_cast<size_t>(hd) * S + pos) * CPR + c;
    const uint4 raw = x[idx];
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t ow[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float x0 = __uint_as_float(w[e] << 16);
      const float x1 = __uint_as_float(w[e] & 0xFFFF0000u);
      const float y0 = x0 * a[e].x - x1 * a[e].y, y1 = x0 * a[e].y + x1 * a[e].x;
      in_range = in_range && fabsf(y0) <= 65504.f && fabsf(y1) <= 65504.f;
      const __half2 v = __floats2half2_rn(y0, y1);
      ow[e] = *reinterpret_cast<const uint32_t*>(&v);
    }
    y[idx] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  }
  if (!in_range) atomicOr(status, 8);
}

// fp32 X [heads, S, D] -> hi = bf16(x) in out[0, heads), lo = bf16(x - hi) in
// out[heads, 2 heads), rotating first when cs is non-null.
template <int CPR>
__global__ void __launch_bounds__(256) split_f32_kernel(const float4* __restrict__ x, uint4* __restrict__ out,
                                                        const float2* __restrict__ cs, int heads, int S) {
  int pos, c;
  if (!chunk_position<CPR>(S, pos, c)) return;
  float2 a[4];
  if (cs) load_cs4<CPR>(cs, pos, c, a);
  const size_t n = static_cast<size_t>(heads) * S * CPR;
  for (int hd = blockIdx.y; hd < heads; hd += gridDim.y) {
    const size_t idx = (static_cast<size_t>(hd) * S + pos) * CPR + c;
    const float4 u = x[2 * idx], v = x[2 * idx + 1];
    float f[8] = {u.x, u.y, u.z, u.w, v.x, v.y, v.z, v.w};
    if (cs) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float x0 = f[2 * e], x1 = f[2 * e + 1];
        f[2 * e] = x0 * a[e].x - x1 * a[e].y;
        f[2 * e + 1] = x0 * a[e].y + x1 * a[e].x;
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

// Grid of the operand-preparation kernels: position blocks in x, enough head
// slices in y for about 32 blocks per SM.
static dim3 operand_grid(int heads, int S, int cpr) {
  const int rpb = 256 / cpr;
  const int gx = (S + rpb - 1) / rpb;
  int gy = (148 * 32) / gx;
  if (gy < 1) gy = 1;
  if (gy > heads) gy = heads;
  if (gy > 65535) gy = 65535;
  return dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy));
}

static int grid_for(long long n, int threads) {
  long long g = (n + threads - 1) / threads;
  const long long cap = 148LL * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return static_cast<int>(g);
}

cudaError_t launch_rope_table(float2* cs, int S, int D, double theta, cudaStream_t stream) {
  const int half = D / 2;
  if (half < 1 || half > 64) return cudaErrorInvalidValue;
  RopeFreqs f{};
  for (int i = 0; i < half; ++i) f.inv[i] = std::pow(theta, -2.0 * i / D);
  const long long n = static_cast<long long>(S) * half;
  rope_table_kernel<<<grid_for(n, 256), 256, 0, stream>>>(cs, S, half, f);
  return cudaGetLastError();
}

cudaError_t launch_rope_k_f16(const void* k, void* k_f16, const float2* cs, long long rows, int S, int D,
                              int* status, cudaStream_t stream) {
  const long long heads = rows / S;
  if (heads * S != rows || heads > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid = operand_grid(static_cast<int>(heads), S, D / 8);
  const uint4* x = static_cast<const uint4*>(k);
  uint4* y = static_cast<uint4*>(k_f16);
  if (D == 128) rope_f16_kernel<16><<<grid, 256, 0, stream>>>(x, y, cs, static_cast<int>(heads), S, status);
  else if (D == 64) rope_f16_kernel<8><<<grid, 256, 0, stream>>>(x, y, cs, static_cast<int>(heads), S, status);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

cudaError_t launch_split_f32(const float* x, void* out, const float2* cs, long long rows, int S, int D,
                             cudaStream_t stream) {
  const long long heads = rows / S;
  if (heads * S != rows || heads > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid = operand_grid(static_cast<int>(heads), S, D / 8);
  const float4* xx = reinterpret_cast<const float4*>(x);
  uint4* o = static_cast<uint4*>(out);
  if (D == 64) split_f32_kernel<8><<<grid, 256, 0, stream>>>(xx, o, cs, static_cast<int>(heads), S);
  else if (D == 128) split_f32_kernel<16><<<grid, 256, 0, stream>>>(xx, o, cs, static_cast<int>(heads), S);
  else return cudaErrorInvalidValue;
  return cudaGetLastError();
}

}  // namespace attn
