// DeepSeek sparse attention: lightning indexer, top-k selection and the gather of the
// selected tokens.
//
// "attention study note", section "Lighting Indexer": each cached token s gets an index
// score sum_j w_j * ReLU(q_j . k_s) over the indexer heads j (queries q_j, one key k_s per
// token shared by the heads); only the best-scoring tokens are attended. Here the
// attention over them is the absorbed MLA decode (mla.cu), run on the gathered rows.
//
// * dsa_index_kernel: one CTA per 64 tokens of one sequence. The 64 x 128 bf16 key block
//   is staged in shared memory (16-byte chunks XOR-swizzled by row, so ldmatrix reads are
//   conflict free); warp w owns indexer heads 16w .. 16w+15 and runs S = Q K^T as
//   mma.sync m16n8k16 (fp32 accumulation), then ReLU, the head weights and the sum over
//   its 16 heads in registers and shuffles; the four warps' partial sums meet in shared
//   memory. HBM-bound on the keys (256 B per token, 64 flop per byte).
// * dsa_topk_kernel: one CTA per sequence. Radix selection on order-preserving 32-bit
//   keys (four 8-bit digit passes with shared-memory histograms) finds the k-th largest
//   score; a final pass keeps every score above it and, of the scores equal to it, the
//   ones with the smallest token indices, writing the selection in ascending token order
//   (block-wide ballot prefix sums).
// * dsa_gather_kernel: one warp per selected token copies its latent row (Dc) and rotary
//   row (Dr) into contiguous [B, top_k, .] buffers that the MLA decode reads as caches.
#include <cuda_bf16.h>

#include "dsa.h"

namespace attn {

namespace {

constexpr int kIdxTokens = 64;   // tokens per indexer CTA
constexpr int kIdxThreads = 128;  // four warps: 16 indexer heads each
constexpr int kTopkThreads = 1024;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Order-preserving map of a float onto an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kIdxThreads) dsa_index_kernel(const DsaIndexParams p) {
  constexpr int D = kDsaIndexDim;
  __shared__ __align__(128) uint8_t kblk[kIdxTokens * D * 2];  // [token][16 chunks of 16 B], chunk ^ (token & 7)
  __shared__ float red[kIdxThreads / 32][kIdxTokens];
  const int b = blockIdx.y, t0 = blockIdx.x * kIdxTokens;
  const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* srow = p.scores + static_cast<size_t>(b) * p.T_max;
  if (t0 >= L) {  // the whole block lies past the sequence
    if (tid < kIdxTokens && t0 + tid < p.T_max) srow[t0 + tid] = -INFINITY;
    return;
  }
  // stage the key block; rows past the sequence are zeros
  const uint8_t* kb = static_cast<const uint8_t*>(p.k) + (static_cast<size_t>(b) * p.T_max + t0) * (D * 2);
#pragma unroll
  for (int i = tid; i < kIdxTokens * 16; i += kIdxThreads) {
    const int r = i >> 4, ch = i & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t0 + r < L) v = __ldg(reinterpret_cast<const uint4*>(kb + static_cast<size_t>(r) * (D * 2) + ch * 16));
    *reinterpret_cast<uint4*>(kblk + r * (D * 2) + ((ch ^ (r & 7)) << 4)) = v;
  }
  // this warp's 16 heads: A fragments of Q (rows = heads) and the two head weights of the lane
  const int g = lane >> 2, c = lane & 3;
  const int h0 = 16 * warp;
  const bool active = h0 < p.HI;
  uint32_t qa[D / 16][4];
  float w0 = 0.f, w1 = 0.f;
  if (active) {
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q) + (static_cast<size_t>(b) * p.HI + h0) * D;
#pragma unroll
    for (int kt = 0; kt < D / 16; ++kt) {
      const int d0 = kt * 16 + 2 * c;
      qa[kt][0] = *reinterpret_cast<const uint32_t*>(qb + g * D + d0);
      qa[kt][1] = *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d0);
      qa[kt][2] = *reinterpret_cast<const uint32_t*>(qb + g * D + d0 + 8);
      qa[kt][3] = *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d0 + 8);
    }
    w0 = __ldg(p.w + static_cast<size_t>(b) * p.HI + h0 + g);
    w1 = __ldg(p.w + static_cast<size_t>(b) * p.HI + h0 + g + 8);
  }
  __syncthreads();
  if (active) {
    const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(kblk));
    const int mi = lane >> 3, r8 = lane & 7;  // ldmatrix: matrix index and row within it
#pragma unroll
    for (int np = 0; np < kIdxTokens / 16; ++np) {  // 16 tokens: two n-tiles of 8
      float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kt = 0; kt < D / 16; ++kt) {
        // matrices: (tokens 0-7, dims lo), (tokens 0-7, dims hi), (tokens 8-15, lo), (8-15, hi)
        const int tok = 16 * np + (mi >> 1) * 8 + r8;
        const int ch = 2 * kt + (mi & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(base + tok * (D * 2) + ((ch ^ (tok & 7)) << 4), b0, b1, b2, b3);
        mma_bf16_16816(acc0, qa[kt], b0, b1);
        mma_bf16_16816(acc1, qa[kt], b2, b3);
      }
      // ReLU, head weights, sum over this lane's two heads, then over the 8 row groups
      float v[4];
      v[0] = w0 * fmaxf(acc0[0], 0.f) + w1 * fmaxf(acc0[2], 0.f);  // token 16np + 2c
      v[1] = w0 * fmaxf(acc0[1], 0.f) + w1 * fmaxf(acc0[3], 0.f);  // token 16np + 2c + 1
      v[2] = w0 * fmaxf(acc1[0], 0.f) + w1 * fmaxf(acc1[2], 0.f);  // token 16np + 8 + 2c
      v[3] = w0 * fmaxf(acc1[1], 0.f) + w1 * fmaxf(acc1[3], 0.f);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) v[e] += __shfl_xor_sync(0xffffffffu, v[e], sh);
      }
      if (g == 0) {
        red[warp][16 * np + 2 * c] = v[0];
        red[warp][16 * np + 2 * c + 1] = v[1];
        red[warp][16 * np + 8 + 2 * c] = v[2];
        red[warp][16 * np + 8 + 2 * c + 1] = v[3];
      }
    }
  } else {
    for (int i = lane; i < kIdxTokens; i += 32) red[warp][i] = 0.f;
  }
  __syncthreads();
  if (tid < kIdxTokens && t0 + tid < p.T_max) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kIdxThreads / 32; ++w) s += red[w][tid];
    srow[t0 + tid] = t0 + tid < L ? s : -INFINITY;
  }
}

__global__ void __launch_bounds__(kTopkThreads) dsa_topk_kernel(const float* __restrict__ scores,
                                                                const int32_t* __restrict__ seq_lens,
                                                                int32_t* __restrict__ idx, int T_max, int top_k) {
  __shared__ unsigned hist[256];
  __shared__ unsigned wcnt[2][kTopkThreads / 32];
  __shared__ uint32_t sh_prefix;
  __shared__ unsigned sh_need;
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int L = min(max(__ldg(seq_lens + b), 0), T_max);
  const float* s = scores + static_cast<size_t>(b) * T_max;
  int32_t* out = idx + static_cast<size_t>(b) * top_k;
  const int n = min(L, top_k);
  for (int i = n + tid; i < top_k; i += kTopkThreads) out[i] = -1;
  if (n == 0) return;
  if (L <= top_k) {  // every token is kept
    for (int i = tid; i < L; i += kTopkThreads) out[i] = i;
    return;
  }
  // radix selection of the top_k-th largest key, most significant digit first:
  // `need` counts how many keys still to take from the band that matches `prefix`
  uint32_t prefix = 0u, mask = 0u;
  unsigned need = static_cast<unsigned>(top_k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    for (int i = tid; i < L; i += kTopkThreads) {
      const uint32_t key = order_key(s[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8l down to 248 - 8l; counts accumulate from the top digit
      unsigned c8[8], tot = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c8[j] = hist[255 - 8 * lane - j];
        tot += c8[j];
      }
      unsigned incl = tot;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      const unsigned excl = incl - tot;
      if (excl < need && need <= incl) {  // exactly one lane: the band that holds the need-th key
        unsigned run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c8[j] >= need) {
            sh_prefix = prefix | (static_cast<uint32_t>(255 - 8 * lane - j) << shift);
            sh_need = need - run;
            break;
          }
          run += c8[j];
        }
      }
    }
    __syncthreads();
    prefix = sh_prefix;
    need = sh_need;
    mask |= 0xFFu << shift;
  }
  // prefix is now the key of the top_k-th largest score: keep every key above it and the
  // first `need` keys equal to it in token order; write positions by ballot prefix sums
  const uint32_t tau = prefix;
  const unsigned lt = (1u << lane) - 1u;
  unsigned eq_base = 0u, out_base = 0u;
  for (int base = 0; base < L; base += kTopkThreads) {
    const int i = base + tid;
    bool gt = false, eq = false;
    if (i < L) {
      const uint32_t key = order_key(s[i]);
      gt = key > tau;
      eq = key == tau;
    }
    const unsigned be = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wcnt[0][warp] = __popc(be);
    __syncthreads();
    unsigned eq_pre = 0u, eq_tot = 0u;
    for (int w = 0; w < kTopkThreads / 32; ++w) {
      const unsigned v = wcnt[0][w];
      eq_pre += w < warp ? v : 0u;
      eq_tot += v;
    }
    const bool sel = gt || (eq && eq_base + eq_pre + __popc(be & lt) < need);
    const unsigned bs = __ballot_sync(0xffffffffu, sel);
    if (lane == 0) wcnt[1][warp] = __popc(bs);
    __syncthreads();
    unsigned s_pre = 0u, s_tot = 0u;
    for (int w = 0; w < kTopkThreads / 32; ++w) {
      const unsigned v = wcnt[1][w];
      s_pre += w < warp ? v : 0u;
      s_tot += v;
    }
    const unsigned pos = out_base + s_pre + __popc(bs & lt);
    if (sel && pos < static_cast<unsigned>(top_k)) out[pos] = i;
    eq_base += eq_tot;
    out_base += s_tot;
    __syncthreads();  // wcnt is rewritten by the next tile
  }
}

__global__ void dsa_gather_kernel(const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ pe,
                                  const int32_t* __restrict__ idx, const int32_t* __restrict__ seq_lens,
                                  __nv_bfloat16* __restrict__ kv_sel, __nv_bfloat16* __restrict__ pe_sel,
                                  int32_t* __restrict__ n_sel, int B, int T_max, int top_k, int Dc, int Dr,
                                  int* status) {
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
  const uint4* src = reinterpret_cast<const uint4*>(kv + (static_cast<size_t>(b) * T_max + t) * Dc);
  uint4* dst = reinterpret_cast<uint4*>(kv_sel + (static_cast<size_t>(b) * top_k + i) * Dc);
  for (int j = lane; j < Dc / 8; j += 32) dst[j] = __ldg(src + j);
  const uint4* psrc = reinterpret_cast<const uint4*>(pe + (static_cast<size_t>(b) * T_max + t) * Dr);
  uint4* pdst = reinterpret_cast<uint4*>(pe_sel + (static_cast<size_t>(b) * top_k + i) * Dr);
  for (int j = lane; j < Dr / 8; j += 32) pdst[j] = __ldg(psrc + j);
}

}  // namespace

cudaError_t launch_dsa_index(const DsaIndexParams& p, cudaStream_t stream) {
  if (p.HI < 16 || p.HI > kDsaMaxIndexHeads || p.HI % 16 != 0) return cudaErrorInvalidValue;
  const dim3 grid((p.T_max + kIdxTokens - 1) / kIdxTokens, p.B);
  dsa_index_kernel<<<grid, kIdxThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const float* scores, const int32_t* seq_lens, int32_t* idx, int B, int T_max, int top_k,
                            cudaStream_t stream) {
  dsa_topk_kernel<<<B, kTopkThreads, 0, stream>>>(scores, seq_lens, idx, T_max, top_k);
  return cudaGetLastError();
}

cudaError_t launch_dsa_gather(const void* kv, const void* pe, const int32_t* idx, const int32_t* seq_lens,
                              void* kv_sel, void* pe_sel, int32_t* n_sel, int B, int T_max, int top_k, int Dc,
                              int Dr, int* status, cudaStream_t stream) {
  if (Dc % 8 != 0 || Dr % 8 != 0) return cudaErrorInvalidValue;
  const long long warps = static_cast<long long>(B) * top_k;
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  dsa_gather_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(kv), static_cast<const __nv_bfloat16*>(pe), idx, seq_lens,
      static_cast<__nv_bfloat16*>(kv_sel), static_cast<__nv_bfloat16*>(pe_sel), n_sel, B, T_max, top_k, Dc, Dr,
      status);
  return cudaGetLastError();
}

}  // namespace attn
