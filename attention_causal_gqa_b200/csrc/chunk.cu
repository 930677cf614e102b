// Chunked prefill into the paged KV cache: the operand preparation around the
// prefill kernel.
//
// "From 32K to 256K: DeepSeek long-context", chapter 1 (a streaming KV cache for
// incremental processing; long sequences cut into chunks; a PagedAttention
// variant) and "attention study note", section "Page Attention" (pages reached
// through a per-sequence block table). New token i of sequence b sits at position
// cache_lens[b] + i:
//   kv_append_kernel     rotates the new keys at their positions (RoPE from the
//                        fp64-angle table) and writes them and the values, in
//                        bf16, into their 16-token pages;
//   kv_gather_kernel     copies each sequence's cache (old and new tokens) into a
//                        contiguous operand: keys as fp16 (exact for bf16 values
//                        in range), values as bf16, zeros past the sequence;
//   rope_rows_f16_kernel rotates the new queries at their positions into fp16.
// The prefill kernel then runs on those operands with each sequence's query
// offset, so query i sees keys t <= cache_lens[b] + i. Chunks may differ in length
// (new_lens[b] <= S_new, padded to S_new): only the first new_lens[b] tokens of a
// sequence are appended and attend; its other rows come out as zeros with LSE -inf.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "prologue.h"
#include "sm100.cuh"

namespace attn {

namespace {

__device__ __forceinline__ int clamp_len(const int32_t* lens, int b, int max_len, int* status) {
  const int L = __ldg(lens + b);
  if (L < 0 || L > max_len) {
    atomicOr(status, kDevErrBadLength);
    return L < 0 ? 0 : max_len;
  }
  return L;
}

// Rotate the 8 values of chunk c of a row at position pos (cs == nullptr: no rotation).
// Half-split layout: chunk c < D/16 (elements 8c .. 8c+7) pairs element by element with
// chunk c + D/16; pair 8c + e turns by the table's angle 8c + e.
__device__ __forceinline__ void rotate16_half(const uint4 lo_raw, const uint4 hi_raw, const float2* __restrict__ cs,
                                              int pos, int c, int D, float (&lo)[8], float (&hi)[8]) {
  const uint32_t wl[4] = {lo_raw.x, lo_raw.y, lo_raw.z, lo_raw.w}, wh[4] = {hi_raw.x, hi_raw.y, hi_raw.z, hi_raw.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float x0 = __uint_as_float((e & 1) ? (wl[e >> 1] & 0xFFFF0000u) : (wl[e >> 1] << 16));
    const float x1 = __uint_as_float((e & 1) ? (wh[e >> 1] & 0xFFFF0000u) : (wh[e >> 1] << 16));
    const float2 a = __ldg(cs + static_cast<size_t>(pos) * (D / 2) + c * 8 + e);
    lo[e] = x0 * a.x - x1 * a.y;
    hi[e] = x0 * a.y + x1 * a.x;
  }
}

__device__ __forceinline__ void rotate8(const uint4 raw, const float2* __restrict__ cs, int pos, int c, int D,
                                        float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float x0 = __uint_as_float(w[e] << 16);
    const float x1 = __uint_as_float(w[e] & 0xFFFF0000u);
    if (cs) {
      const float2 a = __ldg(cs + static_cast<size_t>(pos) * (D / 2) + c * 4 + e);
      f[2 * e] = x0 * a.x - x1 * a.y;
      f[2 * e + 1] = x0 * a.y + x1 * a.x;
    } else {
      f[2 * e] = x0;
      f[2 * e + 1] = x1;
    }
  }
}

__device__ __forceinline__ uint4 pack8_bf16_rn(const float (&f)[8]) {
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
    o[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ uint4 pack8_f16_checked(const float (&f)[8], bool& in_range) {
  uint32_t o[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    in_range = in_range && fabsf(f[2 * e]) <= 65504.f && fabsf(f[2 * e + 1]) <= 65504.f;
    const __half2 h = __floats2half2_rn(f[2 * e], f[2 * e + 1]);
    o[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// New tokens of sequence b (all S_new unless chunks differ in length).
__device__ __forceinline__ int new_len(const ChunkGeometry& g, int b, int* status) {
  return g.new_lens ? clamp_len(g.new_lens, b, g.S_new, status) : g.S_new;
}

// Physical page of logical page lp of sequence b, or -1 (flagged) when the table
// has no valid entry for it.
__device__ __forceinline__ int page_of(const int32_t* __restrict__ table, int b, int lp, int max_pages, int num_pages,
                                       int* status) {
  if (lp >= max_pages) {
    atomicOr(status, kDevErrBadLength);
    return -1;
  }
  const int page = __ldg(table + static_cast<size_t>(b) * max_pages + lp);
  if (page < 0 || page >= num_pages) {
    atomicOr(status, kDevErrBadPage);
    return -1;
  }
  return page;
}

// One thread per 8-element chunk of a (sequence, kv head, new token) row of k_new / v_new.
__global__ void kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                 uint4* __restrict__ k_pages, uint4* __restrict__ v_pages, const float2* __restrict__ cs,
                                 ChunkGeometry g, int* __restrict__ status) {
  const int cpr = g.D / 8;
  const int n = g.B * g.Hkv * g.S_new * cpr;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += gridDim.x * blockDim.x) {
    const int c = idx % cpr, r = idx / cpr;
    const int i = r % g.S_new, kvh = (r / g.S_new) % g.Hkv, b = r / (g.S_new * g.Hkv);
    if (i >= new_len(g, b, status)) continue;  // past this sequence's chunk
    const int pos = clamp_len(g.cache_lens, b, g.max_cache_len, status) + i;
    const int page = page_of(g.block_table, b, pos / g.page_size, g.max_pages, g.num_pages, status);
    if (page < 0) continue;
    const size_t dst = ((static_cast<size_t>(page) * g.page_size + pos % g.page_size) * g.Hkv + kvh) * cpr + c;
    if (g.half_split && cs) {  // the thread of chunk c < cpr/2 writes chunks c and c + cpr/2
      if (c >= cpr / 2) continue;
      float lo[8], hi[8];
      rotate16_half(k_new[idx], k_new[idx + cpr / 2], cs, pos, c, g.D, lo, hi);
      k_pages[dst] = pack8_bf16_rn(lo);
      k_pages[dst + cpr / 2] = pack8_bf16_rn(hi);
      v_pages[dst] = v_new[idx];
      v_pages[dst + cpr / 2] = v_new[idx + cpr / 2];
      continue;
    }
    float f[8];
    rotate8(k_new[idx], cs, pos, c, g.D, f);
    k_pages[dst] = pack8_bf16_rn(f);
    v_pages[dst] = v_new[idx];
  }
}

constexpr int kChunkKeyBlock = 128;  // key rows per block of the prefill kernel in the chunk path

// One thread per 8-element chunk of the contiguous operands [B * Hkv, Sk_max, D]; rows of a
// sequence past its last 128-key block are left as they are (the prefill kernel never
// loads them), rows between its length and that block's end become zeros.
__global__ void kv_gather_kernel(const uint4* __restrict__ k_pages, const uint4* __restrict__ v_pages,
                                 uint4* __restrict__ k_op, uint4* __restrict__ v_op, ChunkGeometry g, int Sk_max,
                                 int* __restrict__ status) {
  griddep_wait();  // launched as a dependent of the cache append
  const int cpr = g.D / 8;
  const long long n = static_cast<long long>(g.B) * g.Hkv * Sk_max * cpr;
  bool in_range = true;
  // four chunks per step, all page loads issued before any store (more bytes in flight)
  constexpr int kUnroll = 4;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long base = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; base < n;
       base += kUnroll * stride) {
    uint4 kr[kUnroll], vr[kUnroll];
    bool have[kUnroll], wr[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long idx = base + u * stride;
      have[u] = wr[u] = false;
      if (idx >= n) continue;
      const int c = static_cast<int>(idx % cpr);
      const long long r = idx / cpr;
      const int j = static_cast<int>(r % Sk_max);
      const int z = static_cast<int>(r / Sk_max), b = z / g.Hkv, kvh = z % g.Hkv;
      const int Sk_b = clamp_len(g.cache_lens, b, g.max_cache_len, status) + new_len(g, b, status);
      // rows past the sequence's last 128-key block are never loaded by the prefill kernel
      wr[u] = j < ((Sk_b + kChunkKeyBlock - 1) / kChunkKeyBlock) * kChunkKeyBlock;
      if (j < Sk_b) {
        const int page = page_of(g.block_table, b, j / g.page_size, g.max_pages, g.num_pages, status);
        if (page >= 0) {
          const size_t src = ((static_cast<size_t>(page) * g.page_size + j % g.page_size) * g.Hkv + kvh) * cpr + c;
          kr[u] = k_pages[src];
          vr[u] = v_pages[src];
          have[u] = true;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long idx = base + u * stride;
      if (!wr[u]) continue;
      uint4 kq = make_uint4(0, 0, 0, 0), vq = make_uint4(0, 0, 0, 0);
      if (have[u]) {
        float f[8];
        rotate8(kr[u], nullptr, 0, static_cast<int>(idx % cpr), g.D, f);
        kq = pack8_f16_checked(f, in_range);
        vq = vr[u];
      }
      k_op[idx] = kq;
      v_op[idx] = vq;
    }
  }
  if (!in_range) atomicOr(status, kDevErrRange);
}

// Rows [B * Hq, S_new, D] of new queries, rotated at cache_lens[b] + i into fp16.
__global__ void rope_rows_f16_kernel(const uint4* __restrict__ x, uint4* __restrict__ y, const float2* __restrict__ cs,
                                     ChunkGeometry g, int Hq, float* __restrict__ lse, int* __restrict__ status) {
  griddep_wait();  // launched as a dependent of the cache gather
  const int cpr = g.D / 8;
  const int n = g.B * Hq * g.S_new * cpr;
  bool in_range = true;
  for (int idx = blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += gridDim.x * blockDim.x) {
    const int c = idx % cpr, r = idx / cpr;
    const int i = r % g.S_new, b = r / (g.S_new * Hq);
    if (i >= new_len(g, b, status)) {  // a row past this sequence's chunk: its final output
      y[idx] = make_uint4(0, 0, 0, 0);
      if (c == 0) lse[r] = -INFINITY;
      continue;
    }
    const int pos = clamp_len(g.cache_lens, b, g.max_cache_len, status) + i;
    if (g.half_split && cs) {  // the thread of chunk c < cpr/2 writes chunks c and c + cpr/2
      if (c >= cpr / 2) continue;
      float lo[8], hi[8];
      rotate16_half(x[idx], x[idx + cpr / 2], cs, pos, c, g.D, lo, hi);
      y[idx] = pack8_f16_checked(lo, in_range);
      y[idx + cpr / 2] = pack8_f16_checked(hi, in_range);
      continue;
    }
    float f[8];
    rotate8(x[idx], cs, pos, c, g.D, f);
    y[idx] = pack8_f16_checked(f, in_range);
  }
  if (!in_range) atomicOr(status, kDevErrRange);
}

int grid_for(long long n, int threads) {
  long long b = (n + threads - 1) / threads;
  const long long cap = 148LL * 16;
  return static_cast<int>(b < 1 ? 1 : (b > cap ? cap : b));
}

}  // namespace

cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages, const float2* cs,
                             const ChunkGeometry& g, int* status, cudaStream_t stream) {
  const long long n = static_cast<long long>(g.B) * g.Hkv * g.S_new * (g.D / 8);
  kv_append_kernel<<<grid_for(n, 256), 256, 0, stream>>>(static_cast<const uint4*>(k_new),
                                                         static_cast<const uint4*>(v_new), static_cast<uint4*>(k_pages),
                                                         static_cast<uint4*>(v_pages), cs, g, status);
  return cudaGetLastError();
}

cudaError_t launch_kv_gather(const void* k_pages, const void* v_pages, void* k_op, void* v_op, const ChunkGeometry& g,
                             int Sk_max, int* status, cudaStream_t stream) {
  const long long n = static_cast<long long>(g.B) * g.Hkv * Sk_max * (g.D / 8);
  return launch_pdl(kv_gather_kernel, dim3(grid_for(n, 256)), dim3(256), 0, stream, static_cast<const uint4*>(k_pages),
                    static_cast<const uint4*>(v_pages), static_cast<uint4*>(k_op), static_cast<uint4*>(v_op), g, Sk_max,
                    status);
}

cudaError_t launch_rope_rows_f16(const void* q, void* q_f16, const float2* cs, const ChunkGeometry& g, int Hq,
                                 float* lse, int* status, cudaStream_t stream) {
  const long long n = static_cast<long long>(g.B) * Hq * g.S_new * (g.D / 8);
  return launch_pdl(rope_rows_f16_kernel, dim3(grid_for(n, 256)), dim3(256), 0, stream, static_cast<const uint4*>(q),
                    static_cast<uint4*>(q_f16), cs, g, Hq, lse, status);
}

}  // namespace attn
