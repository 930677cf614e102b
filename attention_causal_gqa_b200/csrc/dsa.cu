// DeepSeek sparse attention: lightning indexer, top-k selection and the gather of the
// selected tokens.
//
// "attention study note", section "Lighting Indexer": each cached token s gets an index
// score sum_j w_j * ReLU(q_j . k_s) over the indexer heads j (queries q_j, one key k_s per
// token shared by the heads); only the best-scoring tokens are attended. Here the
// attention over them is the absorbed MLA decode (mla.cu), run on the gathered rows.
//
// * dsa_index_kernel: one CTA per 256 tokens of one sequence, in four 64 x 128 bf16 key
//   tiles staged in shared memory by cp.async, the next while the current is used
//   (16-byte chunks XOR-swizzled by row, so ldmatrix reads are conflict free); warp w owns indexer heads 16w .. 16w+15 and runs S = Q K^T as
//   mma.sync m16n8k16 (fp32 accumulation), then ReLU, the head weights and the sum over
//   its 16 heads in registers and shuffles; the four warps' partial sums meet in shared
//   memory. HBM-bound on the keys (256 B per token, 64 flop per byte).
// * dsa_topk_kernel: one CTA per sequence. Radix selection on order-preserving 32-bit
//   keys (four 8-bit digit passes with shared-memory histograms, over the keys staged in
//   shared memory once; warp w owns a contiguous segment of them) finds the k-th largest
//   score; a final pass keeps every score above it and, of the scores equal to it, the ones
//   with the smallest token indices, writing the selection in ascending token order (warp
//   ballots within a segment, one warp's scan across segments: two block barriers).
// * dsa_gather_kernel: one warp per two selected tokens copies their latent rows (Dc) and
//   rotary rows (Dr), all loads in flight first, into contiguous [B, top_k, .] buffers that
//   the MLA decode reads as caches.
#include <cuda_bf16.h>

#include "dsa.h"

namespace attn {

namespace {

constexpr int kIdxTokens = 64;   // tokens per indexer block (one key tile in shared memory)
constexpr int kIdxBlocks = 4;    // blocks per indexer CTA: Q loaded once, the next tile copied during the current
constexpr int kIdxThreads = 128;  // four warps: 16 indexer heads each
constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 48 * 1024;  // sequences up to this many tokens keep their keys in shared memory
constexpr int kGatherRows = 2;            // selected rows per gather warp

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

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kIdxThreads) dsa_index_kernel(const DsaIndexParams p) {
  constexpr int D = kDsaIndexDim;
  constexpr int TILE = kIdxTokens * D * 2;  // bytes of one key tile
  // two key tiles [token][16 chunks of 16 B], chunk ^ (token & 7), copied while the other is used
  __shared__ __align__(128) uint8_t kblk[2][TILE];
  __shared__ float red[kIdxThreads / 32][kIdxTokens];
  const int b = blockIdx.y, c0 = blockIdx.x * (kIdxTokens * kIdxBlocks);
  const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* srow = p.scores + static_cast<size_t>(b) * p.T_max;
  const int c1 = min(c0 + kIdxTokens * kIdxBlocks, p.T_max);
  if (c0 >= L) {  // the whole range lies past the sequence
    for (int t = c0 + tid; t < c1; t += kIdxThreads) srow[t] = -INFINITY;
    return;
  }
  const int nblk = (min(c1, L) - c0 + kIdxTokens - 1) / kIdxTokens;  // tiles holding tokens of the sequence
  const uint8_t* kbase = static_cast<const uint8_t*>(p.k) + static_cast<size_t>(b) * p.T_max * (D * 2);
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(&kblk[0][0]));
  auto copy_tile = [&](int j) {  // key rows c0 + 64 j ..; rows past the sequence become zeros
    const int t0 = c0 + j * kIdxTokens;
#pragma unroll
    for (int i = tid; i < kIdxTokens * 16; i += kIdxThreads) {
      const int r = i >> 4, ch = i & 15;
      const bool in = t0 + r < L;
      const uint8_t* src = kbase + static_cast<size_t>(in ? t0 + r : 0) * (D * 2) + ch * 16;
      cp_async16(sbase + (j & 1) * TILE + r * (D * 2) + ((ch ^ (r & 7)) << 4), src, in ? 16 : 0);
    }
    cp_async_commit();
  };
  copy_tile(0);
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
  const int mi = lane >> 3, r8 = lane & 7;  // ldmatrix: matrix index and row within it
  for (int j = 0; j < nblk; ++j) {
    if (j + 1 < nblk) {
      copy_tile(j + 1);
      cp_async_wait<1>();  // tile j has landed (tile j + 1 may still be in flight)
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();  // tile j visible to every warp; red free again
    if (active) {
      const uint32_t base = sbase + (j & 1) * TILE;
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
        // ReLU, head weights, sum over this lane's two heads, then over the 8 row groups.
        // The rounding steps are spelled out (no free contraction into fused multiply-adds)
        // so every token takes the same ones: equal keys give bit-equal scores.
        float v[4];
        v[0] = __fmaf_rn(w1, fmaxf(acc0[2], 0.f), __fmul_rn(w0, fmaxf(acc0[0], 0.f)));  // token 16np + 2c
        v[1] = __fmaf_rn(w1, fmaxf(acc0[3], 0.f), __fmul_rn(w0, fmaxf(acc0[1], 0.f)));  // token 16np + 2c + 1
        v[2] = __fmaf_rn(w1, fmaxf(acc1[2], 0.f), __fmul_rn(w0, fmaxf(acc1[0], 0.f)));  // token 16np + 8 + 2c
        v[3] = __fmaf_rn(w1, fmaxf(acc1[3], 0.f), __fmul_rn(w0, fmaxf(acc1[1], 0.f)));
#pragma unroll
        for (int e = 0; e < 4; ++e) {
#pragma unroll
          for (int sh = 4; sh < 32; sh <<= 1) v[e] = __fadd_rn(v[e], __shfl_xor_sync(0xffffffffu, v[e], sh));
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
    __syncthreads();  // red complete; tile j no longer read (the copy into it is issued next round)
    const int t = c0 + j * kIdxTokens + tid;
    if (tid < kIdxTokens && t < p.T_max) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < kIdxThreads / 32; ++w) sum = __fadd_rn(sum, red[w][tid]);
      srow[t] = t < L ? sum : -INFINITY;
    }
  }
  // slots of this CTA's range past the sequence's last tile
  for (int t = c0 + nblk * kIdxTokens + tid; t < c1; t += kIdxThreads) srow[t] = -INFINITY;
}

// SMEM: the sequence's keys are converted once into shared memory (T_max <= kTopkSmemKeys)
// and every pass reads them there; otherwise each pass re-reads the scores (L2).
template <bool SMEM>
__global__ void __launch_bounds__(kTopkThreads) dsa_topk_kernel(const float* __restrict__ scores,
                                                                const int32_t* __restrict__ seq_lens,
                                                                int32_t* __restrict__ idx, int T_max, int top_k) {
  extern __shared__ uint32_t skeys[];
  __shared__ unsigned whist[kTopkThreads / 32][256];  // one histogram per warp, summed into hist
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
  if constexpr (SMEM) {
#pragma unroll 8
    for (int i = tid; i < L; i += kTopkThreads) skeys[i] = order_key(s[i]);
    __syncthreads();
  }
  auto key_at = [&](int i) -> uint32_t {
    if constexpr (SMEM) return skeys[i];
    else return order_key(s[i]);
  };
  // warp w owns the contiguous keys [seg0, seg1)
  const int seg = (L + kTopkThreads / 32 - 1) / (kTopkThreads / 32);
  const int seg0 = min(L, warp * seg), seg1 = min(L, seg0 + seg);
  // radix selection of the top_k-th largest key, most significant digit first:
  // `need` counts how many keys still to take from the band that matches `prefix`
  uint32_t prefix = 0u, mask = 0u;
  unsigned need = static_cast<unsigned>(top_k);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < (kTopkThreads / 32) * 256; i += kTopkThreads) (&whist[0][0])[i] = 0u;
    __syncthreads();
    // the digits are few and repeated (the top digit is sign and exponent): each thread
    // counts a run of equal digits in a register and adds it with one atomic when it ends
    unsigned cur = 256u, cnt = 0u;
    for (int i = seg0 + lane; i < seg1; i += 32) {
      const uint32_t key = key_at(i);
      if ((key & mask) != prefix) continue;
      const unsigned dg = (key >> shift) & 0xFFu;
      if (dg != cur) {
        if (cnt) atomicAdd(&whist[warp][cur], cnt);
        cur = dg;
        cnt = 0u;
      }
      ++cnt;
    }
    if (cnt) atomicAdd(&whist[warp][cur], cnt);
    __syncthreads();
    if (tid < 256) {
      unsigned t = 0u;
#pragma unroll 8
      for (int w = 0; w < kTopkThreads / 32; ++w) t += whist[w][tid];
      hist[tid] = t;
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
  // (a) per warp: how many of its keys are above tau and equal to it
  unsigned n_gt = 0u, n_eq = 0u;
  for (int i0 = seg0; i0 < seg1; i0 += 32) {
    const int i = i0 + lane;
    uint32_t key = 0u;
    if (i < seg1) key = key_at(i);
    n_gt += __popc(__ballot_sync(0xffffffffu, i < seg1 && key > tau));
    n_eq += __popc(__ballot_sync(0xffffffffu, i < seg1 && key == tau));
  }
  if (lane == 0) {
    wcnt[0][warp] = n_eq;
    wcnt[1][warp] = n_gt;
  }
  __syncthreads();
  // (b) one warp: equal keys before each warp, then each warp's share and output offset
  if (warp == 0) {
    const unsigned eq = wcnt[0][lane], gtc = wcnt[1][lane];
    unsigned incl = eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned eq_pre = incl - eq;
    const unsigned take = eq_pre >= need ? 0u : min(eq, need - eq_pre);
    const unsigned mine = gtc + take;
    unsigned oin = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, oin, o);
      if (lane >= o) oin += t;
    }
    wcnt[0][lane] = eq_pre;
    wcnt[1][lane] = oin - mine;
  }
  __syncthreads();
  // (c) per warp, in token order: keys above tau, and equal ones while their rank < need
  const unsigned eq_pre = wcnt[0][warp];
  unsigned eq_seen = 0u, out_off = wcnt[1][warp];
  for (int i0 = seg0; i0 < seg1; i0 += 32) {
    const int i = i0 + lane;
    uint32_t key = 0u;
    if (i < seg1) key = key_at(i);
    const bool gt = i < seg1 && key > tau, eq = i < seg1 && key == tau;
    const unsigned be = __ballot_sync(0xffffffffu, eq);
    const bool sel = gt || (eq && eq_pre + eq_seen + __popc(be & lt) < need);
    const unsigned bs = __ballot_sync(0xffffffffu, sel);
    const unsigned pos = out_off + __popc(bs & lt);
    if (sel && pos < static_cast<unsigned>(top_k)) out[pos] = i;
    eq_seen += __popc(be);
    out_off += __popc(bs);
  }
}

__global__ void __launch_bounds__(256, 4) dsa_gather_kernel(const __nv_bfloat16* __restrict__ kv, const __nv_bfloat16* __restrict__ pe,
                                  const int32_t* __restrict__ idx, const int32_t* __restrict__ seq_lens,
                                  __nv_bfloat16* __restrict__ kv_sel, __nv_bfloat16* __restrict__ pe_sel,
                                  int32_t* __restrict__ n_sel, int B, int T_max, int top_k, int Dc, int Dr,
                                  int* status) {
  // warp gw copies the selected rows i0 .. i0 + kGatherRows - 1 of sequence b, all loads first
  const int rows_per_b = (top_k + kGatherRows - 1) / kGatherRows;
  const long long gw = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= static_cast<long long>(B) * rows_per_b) return;
  const int b = static_cast<int>(gw / rows_per_b), i0 = static_cast<int>(gw % rows_per_b) * kGatherRows;
  const int L = min(max(__ldg(seq_lens + b), 0), T_max);
  const int n = min(L, top_k);
  if (i0 == 0 && lane == 0) n_sel[b] = n;
  if (i0 >= n) return;
  int t[kGatherRows];
#pragma unroll
  for (int r = 0; r < kGatherRows; ++r) {
    t[r] = i0 + r < n ? __ldg(idx + static_cast<size_t>(b) * top_k + i0 + r) : -2;
    if (t[r] != -2 && (t[r] < 0 || t[r] >= L)) {
      if (lane == 0) atomicOr(status, kDevErrBadIndex);
      t[r] = 0;
    }
  }
  constexpr int kMaxChunks = 4;  // 16-byte chunks of a latent row per lane (Dc <= 512)
  const int kv_chunks = Dc / 8, pe_chunks = Dr / 8;
  uint4 v[kGatherRows][kMaxChunks];
  uint4 w[kGatherRows];
#pragma unroll
  for (int r = 0; r < kGatherRows; ++r) {
    if (t[r] < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(kv + (static_cast<size_t>(b) * T_max + t[r]) * Dc);
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j)
      if (lane + 32 * j < kv_chunks) v[r][j] = __ldg(src + lane + 32 * j);
    if (lane < pe_chunks) w[r] = __ldg(reinterpret_cast<const uint4*>(pe + (static_cast<size_t>(b) * T_max + t[r]) * Dr) + lane);
  }
#pragma unroll
  for (int r = 0; r < kGatherRows; ++r) {
    if (t[r] < 0) continue;
    uint4* dst = reinterpret_cast<uint4*>(kv_sel + (static_cast<size_t>(b) * top_k + i0 + r) * Dc);
#pragma unroll
    for (int j = 0; j < kMaxChunks; ++j)
      if (lane + 32 * j < kv_chunks) dst[lane + 32 * j] = v[r][j];
    if (lane < pe_chunks) reinterpret_cast<uint4*>(pe_sel + (static_cast<size_t>(b) * top_k + i0 + r) * Dr)[lane] = w[r];
  }
}

}  // namespace

cudaError_t launch_dsa_index(const DsaIndexParams& p, cudaStream_t stream) {
  if (p.HI < 16 || p.HI > kDsaMaxIndexHeads || p.HI % 16 != 0) return cudaErrorInvalidValue;
  const dim3 grid((p.T_max + kIdxTokens * kIdxBlocks - 1) / (kIdxTokens * kIdxBlocks), p.B);
  dsa_index_kernel<<<grid, kIdxThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const float* scores, const int32_t* seq_lens, int32_t* idx, int B, int T_max, int top_k,
                            cudaStream_t stream) {
  if (T_max <= kTopkSmemKeys) {
    const int smem = T_max * static_cast<int>(sizeof(uint32_t));
    cudaError_t e = cudaFuncSetAttribute(dsa_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    dsa_topk_kernel<true><<<B, kTopkThreads, smem, stream>>>(scores, seq_lens, idx, T_max, top_k);
  } else {
    dsa_topk_kernel<false><<<B, kTopkThreads, 0, stream>>>(scores, seq_lens, idx, T_max, top_k);
  }
  return cudaGetLastError();
}

cudaError_t launch_dsa_gather(const void* kv, const void* pe, const int32_t* idx, const int32_t* seq_lens,
                              void* kv_sel, void* pe_sel, int32_t* n_sel, int B, int T_max, int top_k, int Dc,
                              int Dr, int* status, cudaStream_t stream) {
  if (Dc % 8 != 0 || Dr % 8 != 0 || Dc > 8 * 32 * 4 || Dr > 8 * 32) return cudaErrorInvalidValue;
  const long long warps = static_cast<long long>(B) * ((top_k + kGatherRows - 1) / kGatherRows);
  const int threads = 256;
  const long long blocks = (warps * 32 + threads - 1) / threads;
  dsa_gather_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(kv), static_cast<const __nv_bfloat16*>(pe), idx, seq_lens,
      static_cast<__nv_bfloat16*>(kv_sel), static_cast<__nv_bfloat16*>(pe_sel), n_sel, B, T_max, top_k, Dc, Dr,
      status);
  return cudaGetLastError();
}

}  // namespace attn
