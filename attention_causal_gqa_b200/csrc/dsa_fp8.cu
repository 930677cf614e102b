// FP8 (E4M3) latent cache for the DeepSeek sparse attention path: the gather of the
// selected latent rows dequantises them for the MLA decode kernel.
//
// "7 anti-patterns of DeepSeek attention optimisation", section 3.3: E4M3 codes (largest
// value 448) times scale factors; here one fp32 scale per token and 128-wide latent block.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dsa.h"
#include "dsa_fp8.h"

namespace attn {

namespace {

// FP8 latent cache: the selected latent rows are E4M3 codes with one fp32 scale per 128-wide
// block; each lane dequantises 16 codes (one block has 8 lanes) into bf16, which is what the
// MLA decode kernel reads. The rotary rows are copied as they are.
__global__ void __launch_bounds__(256, 4) dsa_gather_fp8_kernel(const uint8_t* __restrict__ kv,
                                                                const float* __restrict__ kv_scale,
                                                                const __nv_bfloat16* __restrict__ pe,
                                                                const int32_t* __restrict__ idx,
                                                                const int32_t* __restrict__ seq_lens,
                                                                __nv_bfloat16* __restrict__ kv_sel,
                                                                __nv_bfloat16* __restrict__ pe_sel,
                                                                int32_t* __restrict__ n_sel, int B, int T_max,
                                                                int top_k, int Dr, int* status) {
  constexpr int Dc = 512, kBlk = 128;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(B) * top_k) return;
  const int b = static_cast<int>(gw / top_k), i = static_cast<int>(gw % top_k);
  const int L = min(max(__ldg(seq_lens + b), 0), T_max);
  const int n = min(L, top_k);
  if (i == 0 && lane == 0) n_sel[b] = n;
  if (i >= n) return;
  int t = __ldg(idx + static_cast<size_t>(b) * top_k + i);
  if (t < 0 || t >= L) {
    if (lane == 0) atomicOr(status, kDevErrBadIndex);
    t = 0;
  }
  const size_t row = static_cast<size_t>(b) * T_max + t;
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(kv + row * Dc) + lane);  // codes 16 lane .. 16 lane + 15
  const float sc = __ldg(kv_scale + row * (Dc / kBlk) + (16 * lane) / kBlk);
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  uint32_t o[8];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint32_t h2[2];
    asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %2;\ncvt.rn.f16x2.e4m3x2 %0, lo;\ncvt.rn.f16x2.e4m3x2 %1, hi;\n}"
        : "=r"(h2[0]), "=r"(h2[1])
        : "r"(words[k]));
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&h2[e]));
      const __nv_bfloat162 v = __floats2bfloat162_rn(f.x * sc, f.y * sc);
      o[2 * k + e] = *reinterpret_cast<const uint32_t*>(&v);
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(kv_sel + (static_cast<size_t>(b) * top_k + i) * Dc + 16 * lane);
  dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
  dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  if (lane < Dr / 8)
    reinterpret_cast<uint4*>(pe_sel + (static_cast<size_t>(b) * top_k + i) * Dr)[lane] =
        __ldg(reinterpret_cast<const uint4*>(pe + row * Dr) + lane);
}

}  // namespace

cudaError_t launch_dsa_gather_fp8(const void* kv_codes, const float* kv_scale, const void* pe, const int32_t* idx,
                                  const int32_t* seq_lens, void* kv_sel, void* pe_sel, int32_t* n_sel, int B,
                                  int T_max, int top_k, int Dc, int Dr, int* status, cudaStream_t stream) {
  if (Dc != 512 || Dr % 8 != 0 || Dr > 8 * 32) return cudaErrorInvalidValue;
  const long long warps = static_cast<long long>(B) * top_k;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  dsa_gather_fp8_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const uint8_t*>(kv_codes), kv_scale, static_cast<const __nv_bfloat16*>(pe), idx, seq_lens,
      static_cast<__nv_bfloat16*>(kv_sel), static_cast<__nv_bfloat16*>(pe_sel), n_sel, B, T_max, top_k, Dr, status);
  return cudaGetLastError();
}

}  // namespace attn
