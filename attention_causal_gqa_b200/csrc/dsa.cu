// DeepSeek sparse attention: lightning indexer, top-k selection and the gather of the
// selected tokens.
//
// "attention study note", section "Lighting Indexer": each cached token s gets an index
// score sum_j w_j * ReLU(q_j . k_s) over the indexer heads j (queries q_j, one key k_s per
// token shared by the heads); only the best-scoring tokens are attended. Here the
// attention over them is the absorbed MLA decode (mla.cu), run on the gathered rows.
//
// * dsa_index_kernel: persistent, one CTA per SM over an even split of the flattened
//   128-token key tiles of all sequences. A TMA producer streams the tiles through a
//   4-stage ring (and each sequence's Q, double-buffered); one warp issues S^T = K Q^T on
//   the tensor cores (tokens as M = 128, indexer heads as N = 64) into two TMEM
//   accumulators; four epilogue warps apply ReLU, the head weights and the sum over heads
//   per token. HBM-bound on the keys (256 B per token read, 4 B written).
// * dsa_topk_kernel: a cluster of four CTAs per sequence, each owning a quarter of its
//   tokens. Radix selection on order-preserving 32-bit keys (four 8-bit digit passes; the
//   CTAs' shared-memory histograms are added through distributed shared memory) finds the
//   k-th largest score; a final pass keeps every score above it and, of the scores equal
//   to it, the ones with the smallest token indices, writing the selection in ascending
//   token order (counts of the earlier slices come from the other CTAs of the cluster).
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
constexpr int kTopkCluster = 4;           // CTAs per sequence in the top-k selection
constexpr int kTopkSmemKeys = 47 * 1024;  // slices up to this many tokens keep their keys in shared memory
                                          // (with the kernel's 36 KB of static shared memory)
constexpr int kGatherRows = 2;            // selected rows per gather warp

// Order-preserving map of a float onto an unsigned key (larger float, larger key).
__device__ __forceinline__ uint32_t order_key(float x) {
  const uint32_t u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kTcTok = 128;          // tokens per tile: the M of the score MMA
constexpr int kIdxStages = 4;        // key tiles in flight per CTA
constexpr int kIdxThreads = 192;     // producer warp, MMA warp, four epilogue warps
constexpr int kTcQBox = 64 * 128;    // bytes of one 64-column block of Q (64 head rows)
constexpr int kTcKBox = kTcTok * 128;  // bytes of one 64-column block of a key tile
constexpr int kTcQBytes = 2 * kTcQBox;  // Q: 64 heads x 128 dims
constexpr int kTcKBytes = 2 * kTcKBox;  // key tile: 128 tokens x 128 dims
constexpr int kIdxBars = 2 * kIdxStages + 8;
constexpr int kIdxSmem = 1024 + 2 * kTcQBytes + kIdxStages * kTcKBytes + kIdxBars * 8 + 16 + 4 * 2 * 64 * 4;

__device__ __forceinline__ int idx_tiles_of(const int32_t* lens, int b, int T_max) {
  const int L = min(max(__ldg(lens + b), 0), T_max);
  return (L + kTcTok - 1) / kTcTok;
}

// Calls fn(b, first_tile, end_tile, global_tile_offset_before) for every piece (segment)
// of CTA c's share of the flattened 128-token tiles of all sequences: the N tiles are
// cut into G contiguous ranges [N c / G, N (c + 1) / G). Whole warps call this (32
// sequences per step of the scan); every role enumerates the same segments.
template <typename F>
__device__ __forceinline__ void for_each_index_segment(const DsaIndexParams& p, int c, int G, F&& fn) {
  const int lane = threadIdx.x & 31;
  constexpr unsigned kAll = 0xffffffffu;
  long long N = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32)
    N += __reduce_add_sync(kAll, static_cast<unsigned>(b0 + lane < p.B ? idx_tiles_of(p.seq_lens, b0 + lane, p.T_max) : 0));
  const long long lo = N * c / G, hi = N * (c + 1) / G;
  long long cs = 0;
  int cb = 0, done = 0;
  while (cb < p.B && cs < hi) {
    const int n = cb + lane < p.B ? idx_tiles_of(p.seq_lens, cb + lane, p.T_max) : 0;
    int incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += t;
    }
    const long long first = cs + (incl - n);
    const int a = static_cast<int>(lo > first ? lo - first : 0);
    const int e = static_cast<int>(hi - first < n ? hi - first : n);
    const unsigned m = __ballot_sync(kAll, e > a);
    if (!m) {
      cs += __shfl_sync(kAll, incl, 31);
      cb += 32;
      continue;
    }
    const int j = __ffs(m) - 1;
    const int t0 = __shfl_sync(kAll, a, j), t1 = __shfl_sync(kAll, e, j);
    cs += __shfl_sync(kAll, incl, j);
    cb += j + 1;
    fn(cb - 1, t0, t1, done);
    done += t1 - t0;
  }
}

// Scores on the 5th-generation tensor cores: S^T = K Q^T with a tile's 128 tokens as M,
// the (up to) 64 indexer heads as N and d = 128 as K, accumulated in TMEM. Persistent:
// CTA c walks its contiguous share of the flattened tiles. Roles (192 threads):
//   warp 0     TMA producer: the sequence's Q (64 x 128, double-buffered per segment) and
//              the key tiles (128 x 128) into a kIdxStages ring, 128-byte swizzle
//   warp 1     TMEM (two 64-column accumulators) and the 8 MMAs of each tile
//   warps 2-5  epilogue: each thread owns one token (its TMEM lane), reads the tile's 64
//              head scores, frees the accumulator and sums ReLU x head weight in a fixed
//              order; tokens past the sequence score -inf
// Scores of tokens past each sequence's last tile are set to -inf by the epilogue warps
// (sequences b = c mod G). Every wait is bounded.
__global__ void __launch_bounds__(kIdxThreads, 1)
    dsa_index_kernel(const DsaIndexParams p, const __grid_constant__ CUtensorMap tmQ,
                     const __grid_constant__ CUtensorMap tmK) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                   // [2 segment slots]
  uint8_t* sK = smem + 2 * kTcQBytes;   // [kIdxStages]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sK + kIdxStages * kTcKBytes);
  uint64_t* k_full = bars;                      // [stages]
  uint64_t* k_empty = k_full + kIdxStages;      // [stages] the tile's MMAs are done
  uint64_t* q_full = k_empty + kIdxStages;      // [2]
  uint64_t* q_empty = q_full + 2;               // [2] the segment's MMAs are done
  uint64_t* acc_full = q_empty + 2;             // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2] the epilogue read the accumulator
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_w = reinterpret_cast<float*>(tmem_slot + 4);  // [4 epilogue warps][2 segment slots][64] head weights

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int c = blockIdx.x, G = gridDim.x;
  if (tid == 0) {
    for (int i = 0; i < kIdxStages; ++i) {
      mbar_init(&k_full[i], 1);
      mbar_init(&k_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 1);
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
    }
    bool ok = true;
    int seg = 0;
    for_each_index_segment(p, c, G, [&](int b, int t0, int t1, int g0) {
      if (lane == 0 && ok) {
        const int qs = seg & 1;
        ok = mbar_wait(&q_empty[qs], ((seg >> 1) & 1) ^ 1, abort_flag, p.status);
        if (ok) {
          mbar_arrive_expect_tx(&q_full[qs], kTcQBytes);
          tma_load_3d(sQ + qs * kTcQBytes, &tmQ, &q_full[qs], 0, 0, b);
          tma_load_3d(sQ + qs * kTcQBytes + kTcQBox, &tmQ, &q_full[qs], 64, 0, b);
        }
        for (int t = t0; ok && t < t1; ++t) {
          const int g = g0 + t - t0, st = g % kIdxStages;
          ok = mbar_wait(&k_empty[st], ((g / kIdxStages) & 1) ^ 1, abort_flag, p.status);
          if (!ok) break;
          uint8_t* dst = sK + st * kTcKBytes;
          mbar_arrive_expect_tx(&k_full[st], kTcKBytes);
          tma_load_3d(dst, &tmK, &k_full[st], 0, t * kTcTok, b);
          tma_load_3d(dst + kTcKBox, &tmK, &k_full[st], 64, t * kTcTok, b);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      ++seg;
    });
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_f32acc(1, kTcTok, 64, false, false);  // bf16 x bf16 -> f32, K-major both
    constexpr uint32_t HI = sdesc_hi_sw128(1024);
    const uint32_t q_lo = sdesc_lo(smem_u32(sQ), 16);
    const uint32_t k_lo = sdesc_lo(smem_u32(sK), 16);
    bool ok = true;
    int seg = 0;
    for_each_index_segment(p, c, G, [&](int, int t0, int t1, int g0) {
      const int qs = seg & 1;
      ok = ok && mbar_wait_warp(&q_full[qs], (seg >> 1) & 1, abort_flag, p.status);
      for (int i = 0; ok && i < t1 - t0; ++i) {
        const int g = g0 + i, st = g % kIdxStages;
        if (!(ok = mbar_wait_warp(&k_full[st], (g / kIdxStages) & 1, abort_flag, p.status))) break;
        if (!(ok = mbar_wait_warp(&acc_empty[g & 1], ((g >> 1) & 1) ^ 1, abort_flag, p.status))) break;
        tc_fence_after();
        const uint32_t a0 = k_lo + ((st * kTcKBytes) >> 4);
        const uint32_t b0 = q_lo + ((qs * kTcQBytes) >> 4);
        const uint32_t d = tmem + (g & 1) * 64;
#pragma unroll
        for (int kb = 0; kb < 8; ++kb) {
          const uint32_t ao = ((kb >> 2) * kTcKBox + (kb & 3) * 32) >> 4;
          const uint32_t bo = ((kb >> 2) * kTcQBox + (kb & 3) * 32) >> 4;
          umma_f16_lohi_warp(d, a0 + ao, HI, b0 + bo, HI, idesc, kb > 0 ? 1u : 0u);
        }
        umma_commit_warp(&acc_full[g & 1]);
        umma_commit_warp(&k_empty[st]);
      }
      if (ok) umma_commit_warp(&q_empty[qs]);  // Q of this segment is free once its MMAs are done
      ++seg;
    });
  } else {
    // -------------------------------------------------------------- epilogue
    const int et = tid - 64;                 // 0 .. 127
    const int quarter = warp & 3;            // TMEM lanes this warp may read
    const int row = 32 * quarter + lane;     // token of the tile
    // scores of tokens past each sequence's last tile
    for (int b = c; b < p.B; b += G) {
      const int from = idx_tiles_of(p.seq_lens, b, p.T_max) * kTcTok;
      float* srow = p.scores + static_cast<size_t>(b) * p.T_max;
      for (int t = from + et; t < p.T_max; t += 128) srow[t] = -INFINITY;
    }
    bool ok = true;
    int seg = 0;
    for_each_index_segment(p, c, G, [&](int b, int t0, int t1, int g0) {
      if (!ok) return;
      // this warp's copy of the sequence's head weights (0 past HI)
      float* w = s_w + ((warp - 2) * 2 + (seg & 1)) * 64;
#pragma unroll
      for (int hh = lane; hh < 64; hh += 32) w[hh] = hh < p.HI ? __ldg(p.w + static_cast<size_t>(b) * p.HI + hh) : 0.f;
      __syncwarp();
      const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
      float* srow = p.scores + static_cast<size_t>(b) * p.T_max;
      for (int i = 0; i < t1 - t0; ++i) {
        const int g = g0 + i;
        if (__any_sync(0xffffffffu, !mbar_wait(&acc_full[g & 1], (g >> 1) & 1, abort_flag, p.status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t v0[32], v1[32];
        const uint32_t base = tmem + (static_cast<uint32_t>(32 * quarter) << 16) + (g & 1) * 64;
        tmem_ld32(base, v0);
        tmem_ld32(base + 32, v1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&acc_empty[g & 1]);
        float score = 0.f;
#pragma unroll
        for (int h = 0; h < 32; ++h) score = __fmaf_rn(w[h], fmaxf(__uint_as_float(v0[h]), 0.f), score);
#pragma unroll
        for (int h = 0; h < 32; ++h) score = __fmaf_rn(w[32 + h], fmaxf(__uint_as_float(v1[h]), 0.f), score);
        const int t = (t0 + i) * kTcTok + row;
        if (t < p.T_max) srow[t] = t < L ? score : -INFINITY;
      }
      ++seg;
    });
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

// One cluster of kTopkCluster CTAs per sequence; CTA r owns the keys of tokens
// [L r / C, L (r + 1) / C). Radix selection of the top_k-th largest key, most significant
// 8-bit digit first: each CTA counts the digits of its keys that still match the selected
// prefix (per-warp histograms summed in shared memory), the cluster's histograms are
// added through distributed shared memory in rank order, and every CTA picks the same
// digit. Then every key above the threshold and, of the keys equal to it, the first
// `need` in token order are written in ascending token order: each CTA learns from the
// others how many keys above / equal to the threshold precede its slice.
// SMEM: the slice's keys are converted once into shared memory; otherwise each pass
// re-reads the scores (L2).
template <bool SMEM>
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    dsa_topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int32_t* __restrict__ idx,
                    int T_max, int top_k) {
  griddep_wait();  // launched as a dependent of the indexer
  extern __shared__ uint32_t skeys[];
  __shared__ unsigned whist[kTopkThreads / 32][256];  // one histogram per warp, summed into hist
  __shared__ unsigned hist[2][256];                   // this CTA's histogram of a pass (pass parity), read by the cluster
  __shared__ unsigned ghist[256];                     // the cluster's histogram of the pass
  __shared__ unsigned wcnt[2][kTopkThreads / 32];
  __shared__ unsigned ccnt[2];                        // this CTA's (equal, above) counts, read by the cluster
  __shared__ unsigned sh_base[2];                     // equal keys before this slice, output offset of this slice
  __shared__ uint32_t sh_prefix;
  __shared__ unsigned sh_need;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = cluster_ctarank();
  const int b = blockIdx.x / kTopkCluster;
  const int L = min(max(__ldg(seq_lens + b), 0), T_max);
  const float* s = scores + static_cast<size_t>(b) * T_max;
  int32_t* out = idx + static_cast<size_t>(b) * top_k;
  const int n = min(L, top_k);
  const int lo = static_cast<int>(static_cast<long long>(L) * rank / kTopkCluster);
  const int hi = static_cast<int>(static_cast<long long>(L) * (rank + 1) / kTopkCluster);
  // the -1 tail of the index list, split over the cluster
  {
    const int t0 = n + static_cast<int>(static_cast<long long>(top_k - n) * rank / kTopkCluster);
    const int t1 = n + static_cast<int>(static_cast<long long>(top_k - n) * (rank + 1) / kTopkCluster);
    for (int i = t0 + tid; i < t1; i += kTopkThreads) out[i] = -1;
  }
  // both exits depend on the sequence only: the whole cluster takes them together
  if (n == 0) return;
  if (L <= top_k) {  // every token is kept
    for (int i = lo + tid; i < hi; i += kTopkThreads) out[i] = i;
    return;
  }
  if constexpr (SMEM) {
#pragma unroll 8
    for (int i = lo + tid; i < hi; i += kTopkThreads) skeys[i - lo] = order_key(s[i]);
  }
  auto key_at = [&](int i) -> uint32_t {
    if constexpr (SMEM) return skeys[i - lo];
    else return order_key(s[i]);
  };
  // warp w owns the contiguous keys [seg0, seg1) of the slice
  const int seg = (hi - lo + kTopkThreads / 32 - 1) / (kTopkThreads / 32);
  const int seg0 = min(hi, lo + warp * seg), seg1 = min(hi, seg0 + seg);
  uint32_t prefix = 0u, mask = 0u;
  unsigned need = static_cast<unsigned>(top_k);  // keys still to take from the band that matches prefix
  for (int pass = 0, shift = 24; shift >= 0; ++pass, shift -= 8) {
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
      hist[pass & 1][tid] = t;
    }
    // the cluster's histograms of this pass are complete (and every CTA has finished
    // reading the previous use of this parity's buffer, two passes back)
    cluster_sync_all();
    if (tid < 256) {
      const uint32_t a = smem_u32(&hist[pass & 1][tid]);
      unsigned t = 0u;
#pragma unroll
      for (int r = 0; r < kTopkCluster; ++r) t += ld_dsmem_u32(mapa_peer(a, r));
      ghist[tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds digits 255 - 8l down to 248 - 8l; counts accumulate from the top digit
      unsigned c8[8], tot = 0u;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c8[j] = ghist[255 - 8 * lane - j];
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
  // first `need` keys equal to it in token order
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
  if (warp == 0) {
    const unsigned eq = wcnt[0][lane], gt = wcnt[1][lane];
    const unsigned eq_all = __reduce_add_sync(0xffffffffu, eq), gt_all = __reduce_add_sync(0xffffffffu, gt);
    if (lane == 0) {
      ccnt[0] = eq_all;
      ccnt[1] = gt_all;
    }
  }
  cluster_sync_all();
  if (warp == 0) {
    // lane r < C reads CTA r's counts; the slices before this one give its bases
    unsigned eq_r = 0u, gt_r = 0u;
    if (lane < kTopkCluster) {
      eq_r = ld_dsmem_u32(mapa_peer(smem_u32(&ccnt[0]), lane));
      gt_r = ld_dsmem_u32(mapa_peer(smem_u32(&ccnt[1]), lane));
    }
    unsigned eq_incl = eq_r;
#pragma unroll
    for (int o = 1; o < kTopkCluster; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, eq_incl, o);
      if (lane >= o) eq_incl += t;
    }
    const unsigned eq_pre = eq_incl - eq_r;
    const unsigned take = eq_pre >= need ? 0u : min(eq_r, need - eq_pre);
    const unsigned mine = lane < kTopkCluster ? gt_r + take : 0u;
    unsigned o_incl = mine;
#pragma unroll
    for (int o = 1; o < kTopkCluster; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, o_incl, o);
      if (lane >= o) o_incl += t;
    }
    const unsigned eq_base = __shfl_sync(0xffffffffu, eq_pre, rank);
    const unsigned out_base = __shfl_sync(0xffffffffu, o_incl - mine, rank);
    // (b) equal keys before each warp, then each warp's share and output offset
    const unsigned eq = wcnt[0][lane], gtc = wcnt[1][lane];
    unsigned incl = eq;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const unsigned w_eq_pre = eq_base + incl - eq;
    const unsigned w_take = w_eq_pre >= need ? 0u : min(eq, need - w_eq_pre);
    const unsigned w_mine = gtc + w_take;
    unsigned oin = w_mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned t = __shfl_up_sync(0xffffffffu, oin, o);
      if (lane >= o) oin += t;
    }
    wcnt[0][lane] = w_eq_pre;
    wcnt[1][lane] = out_base + oin - w_mine;
  }
  // no CTA leaves while another may still read its counts
  cluster_sync_all();
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
  cudaError_t e = cudaFuncSetAttribute(dsa_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kIdxSmem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  dsa_index_kernel<<<sms, kIdxThreads, kIdxSmem, stream>>>(p, tmQ, tmK);
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const float* scores, const int32_t* seq_lens, int32_t* idx, int B, int T_max, int top_k,
                            cudaStream_t stream) {
  const int slice = (T_max + kTopkCluster - 1) / kTopkCluster + 1;  // largest slice of a sequence
  const dim3 grid(static_cast<unsigned>(B) * kTopkCluster);
  if (slice <= kTopkSmemKeys) {
    const int smem = slice * static_cast<int>(sizeof(uint32_t));
    cudaError_t e = cudaFuncSetAttribute(dsa_topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    return launch_pdl(dsa_topk_kernel<true>, grid, dim3(kTopkThreads), smem, stream, scores, seq_lens, idx, T_max, top_k);
  }
  return launch_pdl(dsa_topk_kernel<false>, grid, dim3(kTopkThreads), 0, stream, scores, seq_lens, idx, T_max, top_k);
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
