// RoPE prologue ("From 32K to 256K: DeepSeek long-context", section 2.1 for the
// rotation, section 2.5 for the cos/sin cache [max_len, head_dim/2, 2]).
//
// The angle of pair i at position pos is pos * f * theta^(-2i/D) (f: a frequency scale,
// 1 for plain RoPE; section 2.2 scales the frequencies by a factor, section 2.4 rescales
// the base theta, which callers pass as theta), always formed in fp64 straight from the
// integer position (no running phase). The table (for the fp32-input and chunked paths)
// stores its cos and sin rounded to fp32; the bf16 prefill prologue reduces the fp64
// angle to [-pi, pi] and takes cos and sin in fp32 inside the rotation kernel, so Q and K
// are rotated by one launch with no table pass. Pairs are adjacent elements (2i, 2i+1)
// by default:
//   y[2i]   = x[2i] cos - x[2i+1] sin
//   y[2i+1] = x[2i] sin + x[2i+1] cos
// and (i, i + D/2) in the half-split layout (the concatenated-halves form of section 2.4).
#include <cmath>

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "prologue.h"
#include "sm100.cuh"

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

// The operand-preparation kernels share one layout: a block of 256 threads covers
// 256 / CPR consecutive positions (CPR = D / 8 chunks of 8 elements per row), and
// blockIdx.y strides over the heads. Each thread obtains the cos/sin of its chunk
// once (computed, or from the table) and reuses them for every head it visits, and
// all index arithmetic is 32-bit except the final element offset.
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

// Two 16-bit values of a rotated operand: fp16 (flags values beyond its range) or bf16.
template <bool BF16>
__device__ __forceinline__ uint32_t pack_operand(float a, float b, bool& in_range) {
  if (BF16) {
    const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<const uint32_t*>(&v);
  }
  in_range = in_range && fabsf(a) <= 65504.f && fabsf(b) <= 65504.f;
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// The cos/sin of pairs 8c .. 8c+7 (half-split layout: chunk c of the first half).
template <int CPR>
__device__ __forceinline__ void load_cs8(const float2* __restrict__ cs, int pos, int c, float2 (&a)[8]) {
  const float4* t = reinterpret_cast<const float4*>(cs + static_cast<size_t>(pos) * (CPR * 4) + c * 8);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float4 u = __ldg(t + k);
    a[2 * k] = make_float2(u.x, u.y);
    a[2 * k + 1] = make_float2(u.z, u.w);
  }
}

template <int CPR, bool HALF>
__global__ void __launch_bounds__(256) split_f32_kernel(const float4* __restrict__ x, uint4* __restrict__ out,
                                                        const float2* __restrict__ cs, int heads, int S) {
  griddep_wait();  // launched as a dependent of the cos/sin table
  int pos, c;
  if (!chunk_position<CPR>(S, pos, c)) return;
  if (HALF && c >= CPR / 2) return;
  constexpr int NC = HALF ? 2 : 1;  // chunks per thread
  float2 a[8];
  if (cs) {
    if constexpr (HALF) {
      load_cs8<CPR>(cs, pos, c, a);
    } else {
      float2 a4[4];
      load_cs4<CPR>(cs, pos, c, a4);
#pragma unroll
      for (int e = 0; e < 4; ++e) a[e] = a4[e];
    }
  }
  const size_t n = static_cast<size_t>(heads) * S * CPR;
  for (int hd = blockIdx.y; hd < heads; hd += gridDim.y) {
    const size_t idx = (static_cast<size_t>(hd) * S + pos) * CPR + c;
    float f[NC][8];
#pragma unroll
    for (int q = 0; q < NC; ++q) {
      const size_t ix = idx + q * (CPR / 2);
      const float4 u = x[2 * ix], v = x[2 * ix + 1];
      f[q][0] = u.x; f[q][1] = u.y; f[q][2] = u.z; f[q][3] = u.w;
      f[q][4] = v.x; f[q][5] = v.y; f[q][6] = v.z; f[q][7] = v.w;
    }
    if (cs) {
      if constexpr (HALF) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float x0 = f[0][e], x1 = f[NC - 1][e];
          f[0][e] = x0 * a[e].x - x1 * a[e].y;
          f[NC - 1][e] = x0 * a[e].y + x1 * a[e].x;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = f[0][2 * e], x1 = f[0][2 * e + 1];
          f[0][2 * e] = x0 * a[e].x - x1 * a[e].y;
          f[0][2 * e + 1] = x0 * a[e].y + x1 * a[e].x;
        }
      }
    }
#pragma unroll
    for (int q = 0; q < NC; ++q) {
      uint32_t hw[4], lw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __nv_bfloat162 h = __floats2bfloat162_rn(f[q][2 * e], f[q][2 * e + 1]);
        const float2 hf = __bfloat1622float2(h);
        const __nv_bfloat162 l = __floats2bfloat162_rn(f[q][2 * e] - hf.x, f[q][2 * e + 1] - hf.y);
        hw[e] = *reinterpret_cast<const uint32_t*>(&h);
        lw[e] = *reinterpret_cast<const uint32_t*>(&l);
      }
      const size_t ix = idx + q * (CPR / 2);
      out[ix] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
      out[ix + n] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
    }
  }
}

// Grid of the operand-preparation kernels: position blocks in x, enough head
// slices in y for about 32 blocks per SM.
// cos/sin of pos * inv[i]: the angle is formed and reduced to [-pi, pi] in fp64 (no
// running phase, exact to ~1e-12 rad however large pos * inv[i] grows), then its cosine
// and sine come from the fp32 routine (about 1e-7 absolute error, a thousand times below
// the 16-bit rounding of the rotated operand).
__device__ __forceinline__ float2 cos_sin_of(int pos, double inv) {
  constexpr double kTwoPi = 6.283185307179586476925286766559;
  const double th = static_cast<double>(pos) * inv;
  const double r = th - kTwoPi * rint(th / kTwoPi);
  float sn, cs;
  sincosf(static_cast<float>(r), &sn, &cs);
  return make_float2(cs, sn);
}

// One launch for both operands of a bf16 prefill: rotates Q rows [0, hq) and K rows
// [0, hk) of [heads, S, D] into 16-bit operands (fp16, or bf16 for BF16), computing the
// cos/sin of its own pairs instead of reading a table (so no table kernel runs first).
// Interleaved pairs (2i, 2i+1), or the half-split layout (HALF: element d with d + D/2,
// handled by the threads of the first half's chunks). fp16 values beyond its range set
// the range flag of the status word.
template <int CPR, bool HALF, bool BF16>
__global__ void __launch_bounds__(256) rope_qk_kernel(const uint4* __restrict__ q, uint4* __restrict__ qo, int hq,
                                                      const uint4* __restrict__ k, uint4* __restrict__ ko, int hk,
                                                      int S, const __grid_constant__ RopeFreqs f,
                                                      int* __restrict__ status) {
  int pos, c;
  if (!chunk_position<CPR>(S, pos, c)) return;
  if (HALF && c >= CPR / 2) return;
  constexpr int NPAIR = HALF ? 8 : 4;  // pairs whose cos/sin this thread needs
  float2 a[NPAIR];
#pragma unroll
  for (int e = 0; e < NPAIR; ++e) a[e] = cos_sin_of(pos, f.inv[NPAIR * c + e]);
  bool in_range = true;
  // kUnroll heads per step, all loads issued before any store, so each thread keeps
  // kUnroll (x2 for HALF) 16-byte loads in flight
  constexpr int kUnroll = 4;
  const int H = hq + hk;
  for (int hd0 = blockIdx.y; hd0 < H; hd0 += kUnroll * gridDim.y) {
    uint4 rl[kUnroll], rh[kUnroll];
    size_t ix[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int hd = hd0 + u * gridDim.y;
      if (hd >= H) continue;
      const bool isq = hd < hq;
      ix[u] = (static_cast<size_t>(isq ? hd : hd - hq) * S + pos) * CPR + c;
      const uint4* x = isq ? q : k;
      rl[u] = x[ix[u]];
      if (HALF) rh[u] = x[ix[u] + CPR / 2];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int hd = hd0 + u * gridDim.y;
      if (hd >= H) continue;
      uint4* y = hd < hq ? qo : ko;
      if (!HALF) {
        const uint32_t w[4] = {rl[u].x, rl[u].y, rl[u].z, rl[u].w};
        uint32_t ow[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = __uint_as_float(w[e] << 16), x1 = __uint_as_float(w[e] & 0xFFFF0000u);
          ow[e] = pack_operand<BF16>(x0 * a[e].x - x1 * a[e].y, x0 * a[e].y + x1 * a[e].x, in_range);
        }
        y[ix[u]] = make_uint4(ow[0], ow[1], ow[2], ow[3]);
      } else {
        const uint32_t wl[4] = {rl[u].x, rl[u].y, rl[u].z, rl[u].w}, wh[4] = {rh[u].x, rh[u].y, rh[u].z, rh[u].w};
        uint32_t ol[4], oh[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float l0 = __uint_as_float(wl[e] << 16), l1 = __uint_as_float(wl[e] & 0xFFFF0000u);
          const float h0 = __uint_as_float(wh[e] << 16), h1 = __uint_as_float(wh[e] & 0xFFFF0000u);
          const float2 c0 = a[2 * e], c1 = a[2 * e + 1];
          ol[e] = pack_operand<BF16>(l0 * c0.x - h0 * c0.y, l1 * c1.x - h1 * c1.y, in_range);
          oh[e] = pack_operand<BF16>(l0 * c0.y + h0 * c0.x, l1 * c1.y + h1 * c1.x, in_range);
        }
        y[ix[u]] = make_uint4(ol[0], ol[1], ol[2], ol[3]);
        y[ix[u] + CPR / 2] = make_uint4(oh[0], oh[1], oh[2], oh[3]);
      }
    }
  }
  if (!in_range) atomicOr(status, 8);
}

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

cudaError_t launch_rope_table(float2* cs, int S, int D, double theta, double freq_scale, cudaStream_t stream) {
  const int half = D / 2;
  if (half < 1 || half > 64) return cudaErrorInvalidValue;
  RopeFreqs f{};
  for (int i = 0; i < half; ++i) f.inv[i] = freq_scale * std::pow(theta, -2.0 * i / D);
  const long long n = static_cast<long long>(S) * half;
  rope_table_kernel<<<grid_for(n, 256), 256, 0, stream>>>(cs, S, half, f);
  return cudaGetLastError();
}

cudaError_t launch_rope_qk(const void* q, void* q_op, long long q_heads, const void* k, void* k_op, long long k_heads,
                           int S, int D, double theta, double freq_scale, bool half_split, int* status,
                           cudaStream_t stream, bool bf16_out) {
  const int half = D / 2;
  if (half < 1 || half > 64 || q_heads + k_heads > 0x7fffffffLL) return cudaErrorInvalidValue;
  RopeFreqs f{};
  for (int i = 0; i < half; ++i) f.inv[i] = freq_scale * std::pow(theta, -2.0 * i / D);
  const int hq = static_cast<int>(q_heads), hk = static_cast<int>(k_heads);
  // every thread rotates up to four heads of its chunk in one step
  const int rpb = 256 / (D / 8);
  const dim3 grid(static_cast<unsigned>((S + rpb - 1) / rpb), static_cast<unsigned>(std::min(65535, (hq + hk + 3) / 4)));
  const auto* xq = static_cast<const uint4*>(q);
  const auto* xk = static_cast<const uint4*>(k);
  auto* yq = static_cast<uint4*>(q_op);
  auto* yk = static_cast<uint4*>(k_op);
#define ATTN_ROPE_QK(CPR, HALF, BF)                                                                      \
  rope_qk_kernel<CPR, HALF, BF><<<grid, 256, 0, stream>>>(xq, yq, hq, xk, yk, hk, S, f, status)
  if (D == 128) {
    if (half_split) { if (bf16_out) ATTN_ROPE_QK(16, true, true); else ATTN_ROPE_QK(16, true, false); }
    else { if (bf16_out) ATTN_ROPE_QK(16, false, true); else ATTN_ROPE_QK(16, false, false); }
  } else if (D == 64) {
    if (half_split) { if (bf16_out) ATTN_ROPE_QK(8, true, true); else ATTN_ROPE_QK(8, true, false); }
    else { if (bf16_out) ATTN_ROPE_QK(8, false, true); else ATTN_ROPE_QK(8, false, false); }
  } else {
    return cudaErrorInvalidValue;
  }
#undef ATTN_ROPE_QK
  return cudaGetLastError();
}

cudaError_t launch_split_f32(const float* x, void* out, const float2* cs, long long rows, int S, int D,
                             bool half_split, cudaStream_t stream) {
  const long long heads = rows / S;
  if (heads * S != rows || heads > 0x7fffffffLL) return cudaErrorInvalidValue;
  const dim3 grid = operand_grid(static_cast<int>(heads), S, D / 8);
  const float4* xx = reinterpret_cast<const float4*>(x);
  uint4* o = static_cast<uint4*>(out);
  const int h = static_cast<int>(heads);
  if (D == 64 && half_split) return launch_pdl(split_f32_kernel<8, true>, grid, dim3(256), 0, stream, xx, o, cs, h, S);
  if (D == 64) return launch_pdl(split_f32_kernel<8, false>, grid, dim3(256), 0, stream, xx, o, cs, h, S);
  if (D == 128 && half_split) return launch_pdl(split_f32_kernel<16, true>, grid, dim3(256), 0, stream, xx, o, cs, h, S);
  if (D == 128) return launch_pdl(split_f32_kernel<16, false>, grid, dim3(256), 0, stream, xx, o, cs, h, S);
  return cudaErrorInvalidValue;
}

}  // namespace attn
