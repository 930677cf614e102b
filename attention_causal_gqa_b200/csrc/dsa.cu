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
#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kTopkSmemKeys = 48 * 1024;  // sequences up to this many tokens keep their keys in shared memory
constexpr int kGatherRows = 2;            // selected rows per gather warp

// Order-preserving map of a float onto an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTcTok = 128;    // tokens per tile: the M of the score MMA
constexpr int kTcTiles = 16;   // tiles per CTA
constexpr int kTcThreads = 128;
constexpr int kTcQBox = 64 * 128;          // bytes of one 64-column block of Q (64 head rows)
constexpr int kTcKBox = kTcTok * 128;      // bytes of one 64-column block of a key tile
constexpr int kTcQBytes = 2 * kTcQBox;     // Q: 64 heads x 128 dims
constexpr int kTcKBytes = 2 * kTcKBox;     // key tile: 128 tokens x 128 dims
constexpr int kTcSmem = 1024 + kTcQBytes + 2 * kTcKBytes + 1024;

// Scores on the 5th-generation tensor cores: S^T = K Q^T with the tile's 128 tokens as M,
// the (up to) 64 indexer heads as N and d = 128 as K, accumulated in TMEM (two 64-column
// accumulators, so tile j + 1's MMAs run while tile j is read back). Q (64 x 128) and each
// key tile (128 x 128) arrive by TMA with 128-byte swizzle; one warp issues the MMAs. In the
// epilogue each thread owns one token (its TMEM lane): ReLU, head weights and the sum over
// heads in a fixed order from two tcgen05.ld of 32 columns.
__global__ void __launch_bounds__(kTcThreads, 1)
    dsa_index_kernel(const DsaIndexParams p, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + kTcQBytes;  // two stages
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kTcQBytes + 2 * kTcKBytes);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;    // [2]
  uint64_t* mma_done = bars + 3;  // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_w = reinterpret_cast<float*>(tmem_slot + 2);  // 64 head weights (0 past HI)

  const int b = blockIdx.y, c0 = blockIdx.x * (kTcTok * kTcTiles);
  const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
  const int tid = threadIdx.x, warp = tid >> 5;
  float* srow = p.scores + static_cast<size_t>(b) * p.T_max;
  const int c1 = min(c0 + kTcTok * kTcTiles, p.T_max);
  if (c0 >= L) {  // the whole range lies past the sequence
    for (int t = c0 + tid; t < c1; t += kTcThreads) srow[t] = -INFINITY;
    return;
  }
  const int ntiles = (min(c1, L) - c0 + kTcTok - 1) / kTcTok;
  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&mma_done[s], 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (tid < 64) s_w[tid] = tid < p.HI ? __ldg(p.w + static_cast<size_t>(b) * p.HI + tid) : 0.f;
  if (warp == 0) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto load_tile = [&](int j) {  // key rows c0 + 128 j .. into stage j & 1
    uint8_t* dst = sK + (j & 1) * kTcKBytes;
    mbar_arrive_expect_tx(&k_full[j & 1], kTcKBytes);
    tma_load_3d(dst, &tmK, &k_full[j & 1], 0, c0 + j * kTcTok, b);
    tma_load_3d(dst + kTcKBox, &tmK, &k_full[j & 1], 64, c0 + j * kTcTok, b);
  };
  if (tid == 0) {
    prefetch_tmap(&tmQ);
    prefetch_tmap(&tmK);
    mbar_arrive_expect_tx(q_full, kTcQBytes);
    tma_load_3d(sQ, &tmQ, q_full, 0, 0, b);
    tma_load_3d(sQ + kTcQBox, &tmQ, q_full, 64, 0, b);
    load_tile(0);
    if (ntiles > 1) load_tile(1);
  }
  constexpr uint32_t idesc = idesc_f32acc(1, kTcTok, 64, false, false);  // bf16 x bf16 -> f32, K-major both
  constexpr uint32_t HI = sdesc_hi_sw128(1024);
  const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
  const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16);
  bool ok = true;
  auto issue = [&](int j) {  // warp 0: the 8 k-steps of tile j into accumulator j & 1
    ok = ok && mbar_wait_warp(&k_full[j & 1], (j >> 1) & 1, abort_flag, p.status);
    if (j == 0) ok = ok && mbar_wait_warp(q_full, 0, abort_flag, p.status);
    if (!ok) return;
    tc_fence_after();
    const uint32_t a0 = k_lo + (((j & 1) * kTcKBytes) >> 4);
    const uint32_t d = tmem + (j & 1) * 64;
#pragma unroll
    for (int kb = 0; kb < 8; ++kb) {
      const uint32_t ao = ((kb >> 2) * kTcKBox + (kb & 3) * 32) >> 4;
      const uint32_t bo = ((kb >> 2) * kTcQBox + (kb & 3) * 32) >> 4;
      umma_f16_lohi_warp(d, a0 + ao, HI, q_lo + bo, HI, idesc, kb > 0 ? 1u : 0u);
    }
    umma_commit_warp(&mma_done[j & 1]);
  };
  if (warp == 0) issue(0);
  for (int j = 0; j < ntiles; ++j) {
    if (warp == 0 && j + 1 < ntiles) issue(j + 1);
    ok = ok && mbar_wait(&mma_done[j & 1], (j >> 1) & 1, abort_flag, p.status);
    if (__syncthreads_or(!ok)) break;
    tc_fence_after();
    // stage j & 1 is free once its MMAs are done: bring in tile j + 2
    if (tid == 0 && j + 2 < ntiles) load_tile(j + 2);
    // epilogue: this thread's token is row 32 warp + lane of the accumulator
    float score = 0.f;
    {
      uint32_t v[32];
      const uint32_t base = tmem + (static_cast<uint32_t>(32 * warp) << 16) + (j & 1) * 64;
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        tmem_ld32(base + 32 * half, v);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 32; ++h) score = __fmaf_rn(s_w[32 * half + h], fmaxf(__uint_as_float(v[h]), 0.f), score);
      }
    }
    const int t = c0 + j * kTcTok + tid;
    if (t < p.T_max) srow[t] = t < L ? score : -INFINITY;
    tc_fence_before();
    __syncthreads();  // accumulator j & 1 read by every warp before tile j + 2's MMAs reuse it
  }
  // slots of this CTA's range past the sequence's last tile
  for (int t = c0 + ntiles * kTcTok + tid; t < c1; t += kTcThreads) srow[t] = -INFINITY;
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
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

cudaError_t launch_dsa_index(const DsaIndexParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             cudaStream_t stream) {
  if (p.HI < 1 || p.HI > kDsaMaxIndexHeads) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(dsa_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTcSmem);
  if (e != cudaSuccess) return e;
  const dim3 grid((p.T_max + kTcTok * kTcTiles - 1) / (kTcTok * kTcTiles), p.B);
  dsa_index_kernel<<<grid, kTcThreads, kTcSmem, stream>>>(p, tmQ, tmK);
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
