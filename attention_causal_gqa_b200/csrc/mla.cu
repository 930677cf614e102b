// DeepSeek MLA absorbed decode on tcgen05 tensor cores (sm_100a).
//
// "DeepSeek-V3 attention: einsum vs hand-optimised" (absorbed form):
//   scores[h, t] = (q_nope[h] . kv_cache[t] + q_pe[h] . pe_cache[t]) * scale
//   out[h]       = softmax_t(scores[h]) . kv_cache
// The two score terms are one product over the concatenated 576-wide operand
// [q_nope | q_pe] . [kv_cache | pe_cache]^T ("attention study note", MLA
// decoupled-RoPE section: the rotary part is concatenated to the content part).
//
// Work split. O (128 heads x 512 fp32) fills a whole SM's tensor memory, so a
// cluster of two CTAs shares every 64-token tile: rank r owns kv columns
// [256 r, 256 r + 256) and rotary columns [32 r, 32 r + 32) -- 288 of the 576
// reduction columns each, 18 MMAs per tile on both SMs. Each CTA
//   * loads only its own columns of each tile (no byte is loaded twice),
//   * computes its partial score block S_r = Q_r . K_r^T (M = 128 heads, N = 64
//     tokens, Q_r kept in tensor memory as the A operand),
//   * sends S_r to its peer through distributed shared memory and adds the peer's
//     part (rank-0 part + rank-1 part in both CTAs: identical bits, hence the same
//     running max and sum on both sides),
//   * accumulates O[:, its 256 kv columns] += P . V with P in tensor memory.
// The exchange runs on its own warps: four sender warps read each partial score
// tile out of TMEM as soon as it is computed, stage it and copy it to the peer,
// while the softmax warps work on the previous tile.
// Scheduling is persistent: the flattened sequence of 64-token tiles of all
// sequences is cut into one contiguous range per cluster; each maximal piece of
// a range inside one sequence (a segment) produces one normalised partial result
// and its LSE, merged per sequence by the range merge (merge.cu).
//
// Roles per CTA (480 threads). A warp reaches only its TMEM lane quarter
// q = warp % 4, i.e. heads [32 q, 32 q + 32), one thread per head.
//   * Softmax warps 0-7: warpgroup w (warps 4w .. 4w + 3) handles tokens
//     [32 w, 32 w + 32) of every tile. Warps q and q + 4 share the heads and
//     combine their half-tile maxima through shared memory; each keeps the running
//     sum of its own tokens. They add the staged own part and the peer's part,
//     run the online softmax and write P into TMEM.
//   * Sender warps 11-14 (quarter warp % 4): read the 64 partial scores of their
//     heads out of TMEM (freeing the S buffer for the next tile), stage them in
//     shared memory and send them to the same sender's receive block on the peer
//     with one bulk copy that completes on the peer's barrier.
//   * Warp 8 is the TMA producer, warp 9 allocates TMEM and issues Q K^T, warp 10
//     issues P V.
// Every wait is bounded; no named barrier is used, so a role that gives up
// cannot strand the others.
// TMEM columns: O [0, 256), Q_r [256, 400), S [416, 480), P [480, 512).
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kH = 128, kDc = 512, kDr = 64;
constexpr int TN = kMlaTile;              // tokens per tile
constexpr int HALF = TN / 2;              // tokens per softmax warpgroup
constexpr int KV_BOX = TN * 128;          // one 64-column kv block of a tile (TN rows of 128 bytes)
constexpr int PE_BOX = TN * 64;           // this CTA's 32 rotary columns (TN rows of 64 bytes)
constexpr int STAGE = 4 * KV_BOX + PE_BOX;
constexpr int NST = 4;                    // ring depth
constexpr int XCHUNK = 32 * TN * 4;       // one quarter's block of partial scores: 32 heads x 64 tokens fp32
constexpr int XBUF = 4 * XCHUNK;
constexpr int O_COL = 0, Q_COL = 256, S_COL = 416, P_COL = 480;
constexpr int TMEM_COLS = 512;
constexpr int kMlaThreads = 480;
constexpr int kNumBars = 2 * NST + 4 + 12 + 8 + 3;
constexpr int SMEM_BYTES = 1024 + NST * STAGE + 2 * XBUF + 2 * (2 * 2 * kH * 4) + kNumBars * 8 + 16;
static_assert(TN == 64, "the exchange and P layout assume 64-token tiles");
static_assert(Q_COL + 144 <= S_COL && S_COL + TN <= P_COL && P_COL + TN / 2 <= TMEM_COLS, "TMEM budget");
static_assert(STAGE % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

// One bulk copy of a staged block from this CTA's shared memory into the peer's,
// completing its bytes on the peer's mbarrier.
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                                  uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src_cta), "r"(bytes), "r"(bar_cluster)
               : "memory");
}
// Remote arrive that says "these bytes were read". It is relaxed (a release at cluster
// scope measured 25-40% slower per launch); callers issue it only under a branch on a
// value computed from every lane's loaded data, so the reads have returned before the
// peer can learn that the block may be overwritten.
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}

__device__ __forceinline__ int tiles_of(const int32_t* lens, int b, int T_max) {
  const int L = min(max(__ldg(lens + b), 0), T_max);
  return (L + TN - 1) / TN;
}

// Calls fn(b, first_tile, end_tile, global_tile_offset_before, b_next) for every segment
// of cluster `pair` in order; b_next is b + 1 when the cluster's range reaches past this
// segment (a hint for prefetching), else -1. The ranges are cut in a position space where
// a non-empty sequence of n tiles takes kMlaSegCost + n positions, its tile t at position
// kMlaSegCost + t; the cluster holding a tile's position computes it. The host keeps the
// position count below 2^31. Whole warps call this (the scan takes 32 sequences per
// step); every role enumerates the same segments.
template <typename F>
__device__ __forceinline__ void for_each_segment(const MlaParams& p, int pair, F&& fn) {
  const int lane = threadIdx.x & 31;
  constexpr unsigned kAll = 0xffffffffu;
  unsigned N = 0;
  for (int b0 = 0; b0 < p.B; b0 += 32) {
    const int n = b0 + lane < p.B ? tiles_of(p.seq_lens, b0 + lane, p.T_max) : 0;
    N += __reduce_add_sync(kAll, static_cast<unsigned>(n > 0 ? n + kMlaSegCost : 0));
  }
  const int lo = static_cast<int>(static_cast<long long>(N) * pair / p.n_pairs);
  const int hi = static_cast<int>(static_cast<long long>(N) * (pair + 1) / p.n_pairs);
  // cursor: next sequence to examine (cb) and its first position (cs); only these and
  // the tile count stay live while a segment runs
  int cb = 0, cs = 0, done = 0;
  while (cb < p.B && cs < hi) {
    const int n = cb + lane < p.B ? tiles_of(p.seq_lens, cb + lane, p.T_max) : 0;
    const int u = n > 0 ? n + kMlaSegCost : 0;
    int incl = u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(kAll, incl, o);
      if (lane >= o) incl += t;
    }
    const int first = cs + (incl - u) + kMlaSegCost;  // position of this lane's tile 0
    const int a = max(lo - first, 0), e = min(hi - first, n);
    const unsigned m = __ballot_sync(kAll, n > 0 && e > a);
    if (!m) {  // nothing of this range among these 32 sequences
      cs += __shfl_sync(kAll, incl, 31);
      cb += 32;
      continue;
    }
    const int j = __ffs(m) - 1;
    const int t0 = __shfl_sync(kAll, a, j), t1 = __shfl_sync(kAll, e, j);
    const int more = __shfl_sync(kAll, static_cast<int>(hi > first + e), j);
    const int b = cb + j;
    cs += __shfl_sync(kAll, incl, j);
    cb = b + 1;
    fn(b, t0, t1, done, more && cb < p.B ? cb : -1);
    done += t1 - t0;
  }
}

// 32 consecutive bf16 pairs (128 bytes) of a row into registers.
__device__ __forceinline__ void load_row32(const uint32_t* src, uint32_t (&r)[32]) {
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src + e));
    r[e] = v.x;
    r[e + 1] = v.y;
    r[e + 2] = v.z;
    r[e + 3] = v.w;
  }
}

__device__ __forceinline__ void mla_body(const MlaParams& p, const CUtensorMap* tmKV, const CUtensorMap* tmPE,
                                         uint8_t* smem, const int R) {
  const uint32_t PEER = 1 - R;
  uint8_t* sKV = smem;
  // partial-score blocks [4 quarters][2 token halves][32 heads][32 tokens]: from the peer / own, staged
  float* xrecv = reinterpret_cast<float*>(smem + NST * STAGE);
  float* xsend = xrecv + XBUF / 4;
  float* mx_sh = xsend + XBUF / 4;                                // [2 parity][2 wg][kH] half-tile maxima
  float* l_sh = mx_sh + 2 * 2 * kH;                               // [2 parity][2 wg][kH] half sums at a segment end
  uint64_t* bars = reinterpret_cast<uint64_t*>(l_sh + 2 * 2 * kH);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_full = kv_empty + NST;  // S(k) computed
  uint64_t* s_free = s_full + 1;      // the sender warps have read S(k) out of TMEM
  uint64_t* p_full = s_free + 1;      // P(k) written (and any O rescale done)
  uint64_t* o_done = p_full + 1;      // P(k) V(k) completed
  uint64_t* x_full = o_done + 1;      // [4] the peer's block for quarter q landed in xrecv
  uint64_t* x_empty = x_full + 4;     // [4] the peer's softmax warps of quarter q consumed what was sent
  uint64_t* own_free = x_empty + 4;   // [4] this CTA's softmax warps of quarter q consumed the staged block
  uint64_t* mx_bar = own_free + 4;    // [4] warps q and q + 4 published their half maxima
  uint64_t* l_bar = mx_bar + 4;       // [4] warps q and q + 4 published their half sums
  uint64_t* q_ready = l_bar + 4;      // Q_r of the segment is in TMEM
  uint64_t* o_free = q_ready + 1;     // the segment's partial result has been read out of O
  uint64_t* mma_done = o_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_free, 128);
    mbar_init(p_full, 256);
    mbar_init(o_done, 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(&x_full[i], 1);    // the sender's expect_tx arrive + the bytes of the peer's bulk copy
      mbar_init(&x_empty[i], 2);   // remote arrives from the peer's two softmax warps of quarter i
      mbar_init(&own_free[i], 2);  // this CTA's two softmax warps of quarter i
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&mx_bar[i], 64);
      mbar_init(&l_bar[i], 64);
    }
    mbar_init(q_ready, 256);
    mbar_init(o_free, 256);
    mbar_init(mma_done, 2);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_sync_all();  // the peer's barriers exist (and are armed) before any remote access
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    // --------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(tmKV);
      prefetch_tmap(tmPE);
    }
    int g = 0;
    bool ok = true;
    for_each_segment(p, pair, [&](int b, int t0, int t1, int, int) {
      for (int t = t0; t < t1 && ok; ++t, ++g) {
        if (lane == 0) {
          const int s = g % NST;
          if (!mbar_wait(&kv_empty[s], ((g / NST) & 1) ^ 1, abort_flag, p.status)) {
            ok = false;
          } else {
            uint8_t* dst = sKV + s * STAGE;
            mbar_arrive_expect_tx(&kv_full[s], STAGE);
#pragma unroll
            for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * KV_BOX, tmKV, &kv_full[s], R * 256 + c * 64, t * TN, b);
            tma_load_3d(dst + 4 * KV_BOX, tmPE, &kv_full[s], R * 32, t * TN, b);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    });
  } else if (warp == 9 || warp == 10) {
    // ------------------------------ MMA issuers (whole warps): 9 = scores, 10 = P V
    constexpr uint32_t HI128 = sdesc_hi_sw128(1024);
    bool ok = true;
    int seg = 0;
    if (warp == 9) {
      constexpr uint32_t HI64 = sdesc_hi_sw64(512);
      constexpr uint32_t idesc_s = idesc_f32acc(1, 128, TN, false, false);
      const uint32_t kv_lo_k = sdesc_lo(smem_u32(sKV), 16);
      for_each_segment(p, pair, [&](int, int t0, int t1, int g0, int) {
        if (!ok) return;
        if (!(ok = mbar_wait_warp(q_ready, seg & 1, abort_flag, p.status))) return;
        ++seg;
        tc_fence_after();
        for (int i = 0; ok && i < t1 - t0; ++i) {
          const int k = g0 + i;
          // single S buffer: S(k - 1) must have been read out by the sender warps
          if (k >= 1 && !(ok = mbar_wait_warp(s_free, (k - 1) & 1, abort_flag, p.status))) break;
          if (!(ok = mbar_wait_warp(&kv_full[k % NST], (k / NST) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t b0 = kv_lo_k + (((k % NST) * STAGE) >> 4);
          const uint32_t d = tmem_base + S_COL;
#pragma unroll 1
          for (int bx = 0; bx < 4; ++bx)
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
              umma_f16_ts_warp(d, tmem_base + Q_COL + (bx * 4 + kq) * 8, b0 + ((bx * KV_BOX + kq * 32) >> 4), HI128,
                               idesc_s, (bx > 0 || kq > 0) ? 1u : 0u);
#pragma unroll
          for (int kq = 0; kq < 2; ++kq)  // the 32 rotary columns: 64-byte rows, 64-byte swizzle
            umma_f16_ts_warp(d, tmem_base + Q_COL + 128 + kq * 8, b0 + ((4 * KV_BOX + kq * 32) >> 4), HI64, idesc_s,
                             1u);
          umma_commit_warp(s_full);
        }
      });
    } else {
      constexpr uint32_t idesc_o = idesc_f32acc(1, 128, 256, false, true);
      const uint32_t kv_lo_v = sdesc_lo(smem_u32(sKV), KV_BOX);  // MN-major: 64-column blocks KV_BOX apart
      for_each_segment(p, pair, [&](int, int t0, int t1, int g0, int) {
        if (!ok) return;
        for (int i = 0; ok && i < t1 - t0; ++i) {
          const int k = g0 + i;
          if (!(ok = mbar_wait_warp(p_full, k & 1, abort_flag, p.status))) break;
          // the first P V of a segment overwrites O: the previous segment's result must be out
          if (i == 0 && seg > 0 && !(ok = mbar_wait_warp(o_free, (seg - 1) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t b0 = kv_lo_v + (((k % NST) * STAGE) >> 4);
          const uint32_t a0 = tmem_base + P_COL;
#pragma unroll
          for (int kb = 0; kb < TN / 16; ++kb)
            umma_f16_ts_warp(tmem_base + O_COL, a0 + kb * 8, b0 + ((kb * 16 * 128) >> 4), HI128, idesc_o,
                             (i > 0 || kb > 0) ? 1u : 0u);
          umma_commit_warp(o_done);
          umma_commit_warp(&kv_empty[k % NST]);  // S(k) was complete before P(k) existed
        }
        ++seg;
      });
    }
    umma_commit_warp(mma_done);
    mbar_wait_warp(mma_done, 0, abort_flag, p.status);
  } else if (warp >= 11) {
    // ------------------------------------------ sender warps: quarter q = warp % 4
    const int q = warp & 3;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float* stage = xsend + (q * 2 * 32 + lane) * HALF;  // this lane's row of token half 0 (half 1: 32 rows on)
    const uint32_t peer_recv = mapa_peer(smem_u32(xrecv + q * 2 * 32 * HALF), PEER);
    const uint32_t peer_full = mapa_peer(smem_u32(&x_full[q]), PEER);
    const uint32_t send_src = smem_u32(xsend + q * 2 * 32 * HALF);
    bool ok = true;
    for_each_segment(p, pair, [&](int, int t0, int t1, int g0, int) {
      for (int i = 0; ok && i < t1 - t0; ++i) {
        const int k = g0 + i;
        // S(k) out of TMEM; the buffer may then take S(k + 1)
        if (!(ok = mbar_wait_warp(s_full, k & 1, abort_flag, p.status))) break;
        tc_fence_after();
        uint32_t r0[32], r1[32];
        tmem_ld32(t_lane + S_COL, r0);
        tmem_ld32(t_lane + S_COL + HALF, r1);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(s_free);
        // the staged block of tile k - 1 has been read here, and the peer has consumed
        // what it received of tile k - 1 (its copy had landed, so the staging block was read)
        if (!(ok = mbar_wait_warp(&own_free[q], (k & 1) ^ 1, abort_flag, p.status))) break;
        if (!(ok = mbar_wait_warp(&x_empty[q], (k & 1) ^ 1, abort_flag, p.status))) break;
#pragma unroll
        for (int c = 0; c < HALF / 4; ++c) {
          const int cc = 4 * ((c + lane) & (HALF / 4 - 1));
          *reinterpret_cast<uint4*>(stage + cc) = make_uint4(r0[4 * c], r0[4 * c + 1], r0[4 * c + 2], r0[4 * c + 3]);
          *reinterpret_cast<uint4*>(stage + 32 * HALF + cc) =
              make_uint4(r1[4 * c], r1[4 * c + 1], r1[4 * c + 2], r1[4 * c + 3]);
        }
        fence_proxy_async_smem();  // the bulk copy reads the staged block through the async proxy
        __threadfence_block();     // and this CTA's softmax warps read it once x_full completes
        __syncwarp();
        if (lane == 0) {
          // x_full(k) completes on this arrive and the peer's bytes, in either order; the
          // arrive comes after the own block is staged, since the softmax warps read both
          // parts as soon as the phase completes
          mbar_arrive_expect_tx(&x_full[q], XCHUNK);
          bulk_copy_to_peer(peer_recv, send_src, XCHUNK, peer_full);
        }
      }
    });
  } else {
    // ------------------------------------------------- softmax warpgroups
    const int w = warp >> 2;               // token half
    const int q = warp & 3;                // lane quarter
    const int h = q * 32 + lane;           // head == TMEM lane
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const float sl2 = p.scale_log2;
    const int row = ((q * 2 + w) * 32 + lane) * HALF;
    const float* my_recv = xrecv + row;
    const float* my_own = xsend + row;
    const uint32_t peer_empty = mapa_peer(smem_u32(&x_empty[q]), PEER);
    bool alive = true;
    auto fail = [&](bool ok) -> bool {
      if (__any_sync(0xffffffffu, !ok)) alive = false;
      return !alive;
    };
    int seg = 0;
    for_each_segment(p, pair, [&](int b, int t0, int t1, int g0, int b_next) {
      if (!alive) return;
      const int n = t1 - t0;
      // Q_r of sequence b into TMEM (bf16 pairs are already in the operand layout). Every
      // S MMA of the previous segment has completed: its last score tile was staged.
      {
        const uint32_t* qn = reinterpret_cast<const uint32_t*>(
            reinterpret_cast<const __nv_bfloat16*>(p.q_nope) + (static_cast<size_t>(b) * kH + h) * kDc + R * 256 +
            w * 128);
        uint32_t r[32];
        load_row32(qn, r);
        tmem_st32(t_lane + Q_COL + w * 64, r);
        load_row32(qn + 32, r);
        tmem_st32(t_lane + Q_COL + w * 64 + 32, r);
        if (w == 1) {
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(
              reinterpret_cast<const __nv_bfloat16*>(p.q_pe) + (static_cast<size_t>(b) * kH + h) * kDr + R * 32);
          uint32_t r16[16];
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(qp + e));
            r16[e] = v.x;
            r16[e + 1] = v.y;
            r16[e + 2] = v.z;
            r16[e + 3] = v.w;
          }
          tmem_st16(t_lane + Q_COL + 128, r16);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(q_ready);
        if (b_next >= 0) {  // the next segment's Q rows into L2 while this one runs
          const char* nx = reinterpret_cast<const char*>(reinterpret_cast<const __nv_bfloat16*>(p.q_nope) +
                                                         (static_cast<size_t>(b_next) * kH + h) * kDc + R * 256 + w * 128);
          prefetch_l2(nx);
          prefetch_l2(nx + 128);
          if (w == 1)
            prefetch_l2(reinterpret_cast<const __nv_bfloat16*>(p.q_pe) + (static_cast<size_t>(b_next) * kH + h) * kDr +
                        R * 32);
        }
      }
      const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
      float m_run = -INFINITY, l_run = 0.f;
      for (int i = 0; i < n; ++i) {
        const int k = g0 + i;
        // own staged part + the peer's part of tile k: rank-0 part + rank-1 part in both CTAs
        if (fail(mbar_wait(&x_full[q], k & 1, abort_flag, p.status))) return;
        float s[HALF];
#pragma unroll
        for (int c = 0; c < HALF / 4; ++c) {
          const int cc = 4 * ((c + lane) & (HALF / 4 - 1));
          const float4 v = *reinterpret_cast<const float4*>(my_recv + cc);
          const float4 o = *reinterpret_cast<const float4*>(my_own + cc);
          s[4 * c + 0] = R == 0 ? o.x + v.x : v.x + o.x;
          s[4 * c + 1] = R == 0 ? o.y + v.y : v.y + o.y;
          s[4 * c + 2] = R == 0 ? o.z + v.z : v.z + o.z;
          s[4 * c + 3] = R == 0 ? o.w + v.w : v.w + o.w;
        }
        const int valid = L - (t0 + i) * TN - w * HALF;  // tokens of this half inside the sequence
        if (valid < HALF) {
#pragma unroll
          for (int c = 0; c < HALF; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        float mx0 = fmax3f(s[0], s[1], s[2]), mx1 = fmax3f(s[3], s[4], s[5]);
#pragma unroll
        for (int c = 6; c + 3 < HALF; c += 4) {
          mx0 = fmax3f(mx0, s[c], s[c + 1]);
          mx1 = fmax3f(mx1, s[c + 2], s[c + 3]);
        }
        mx0 = fmaxf(mx0, s[HALF - 2]);
        mx1 = fmaxf(mx1, s[HALF - 1]);
        const float mxh = fmaxf(mx0, mx1);
        // The half maximum depends on every value this lane read from both blocks, and the
        // ballot on it on every lane's: past it, the whole warp's reads have returned and
        // both blocks may be given back (the predicate is always true: fmaxf never yields
        // that NaN payload).
        if (__ballot_sync(0xffffffffu, __float_as_uint(mxh) != 0x7fc00001u) != 0u && lane == 0) {
          mbar_arrive(&own_free[q]);
          mbar_arrive_remote_relaxed(peer_empty);
        }
        // the other half's maximum (warp q + 4 or q - 4 holds the same heads)
        float* mslot = mx_sh + (k & 1) * 2 * kH;
        mslot[w * kH + h] = mxh;
        mbar_arrive(&mx_bar[q]);
        if (fail(mbar_wait(&mx_bar[q], k & 1, abort_flag, p.status))) return;
        const float m_tile = fmaxf(mslot[h], mslot[kH + h]) * sl2;
        bool rescale = false;
        float alpha = 1.f;
        if (i == 0) {
          m_run = m_tile;
        } else if (__any_sync(0xffffffffu, m_tile > m_run + 8.0f)) {
          rescale = true;
          const float m_new = fmaxf(m_run, m_tile);
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
        }
        // P = 2^(s * scale * log2 e - m); in a half without masked tokens 1 of every 4
        // pairs takes the FMA-pipe exp2, which relieves the MUFU (shared by two warps)
        uint32_t pp[HALF / 2];
        float2 lsum = make_float2(0.f, 0.f);
        const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_run, -m_run);
        const bool soft = valid >= HALF;
#pragma unroll
        for (int c = 0; c < HALF; c += 2) {
          const float2 z = ffma2(make_float2(s[c], s[c + 1]), sc2, nm2);
          float2 e;
          if (soft && (c & 6) == 6) {
            e = exp2_fma2(z);
          } else {
            e.x = ex2_approx(z.x);
            e.y = ex2_approx(z.y);
          }
          lsum = fadd2(lsum, e);
          pp[c / 2] = pack_bf16x2(e.x, e.y);
        }
        // one P buffer: P(k - 1) V(k - 1) must be complete before P(k) replaces it
        // (and before O is rescaled)
        if (k >= 1) {
          if (fail(mbar_wait(o_done, (k - 1) & 1, abort_flag, p.status))) return;
          tc_fence_after();
        }
        if (rescale) {
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            tmem_ld32(t_lane + O_COL + w * 128 + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(t_lane + O_COL + w * 128 + c * 32, r);
          }
        }
        tmem_st16(t_lane + P_COL + w * (HALF / 2), pp);
        if (valid < HALF) {
          // cached rows past the sequence end may hold anything: zero this CTA's value
          // columns for them so that 0 * garbage cannot reach O
          uint8_t* st = sKV + (k % NST) * STAGE;
          const int r0 = w * HALF + max(valid, 0), nbad = (w + 1) * HALF - r0;
          for (int idx = q * 32 + lane; idx < 4 * nbad * 8; idx += 128) {
            const int bxx = idx / (nbad * 8), r = r0 + (idx / 8) % nbad, ch = idx % 8;
            *reinterpret_cast<uint4*>(st + bxx * KV_BOX + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(p_full);
        l_run = l_run * alpha + (lsum.x + lsum.y);
      }
      // segment epilogue: O / l for this CTA's 256 columns (128 per warpgroup) and the
      // LSE (rank 0). P V of the segment's last tile completes after all earlier ones.
      const int k_last = g0 + n - 1;
      if (fail(mbar_wait(o_done, k_last & 1, abort_flag, p.status))) return;
      tc_fence_after();
      float* lslot = l_sh + (seg & 1) * 2 * kH;
      lslot[w * kH + h] = l_run;
      mbar_arrive(&l_bar[q]);
      if (fail(mbar_wait(&l_bar[q], seg & 1, abort_flag, p.status))) return;
      const float l_tot = lslot[h] + lslot[kH + h];
      const int slot = pair + b;
      const float inv_l = 1.f / l_tot;
      // O / l leaves through this warp's 4 KB block of the staging area, transposed so that
      // each store instruction writes four whole 128-byte row pieces. The block is idle
      // from here to the next segment's first score tile, once the peer has consumed the
      // last tile (the copy out of it has completed).
      if (fail(mbar_wait(&x_empty[q], k_last & 1, abort_flag, p.status))) return;
      float* stg = xsend + (q * 2 + w) * 32 * HALF;
      float* obase = p.part_o + (static_cast<size_t>(slot) * kH + q * 32) * kDc + R * 256 + w * 128;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + O_COL + w * 128 + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 8; ++j)  // row `lane`, 16-byte chunk j at slot j ^ (lane & 7)
          *reinterpret_cast<float4*>(stg + lane * 32 + 4 * (j ^ (lane & 7))) =
              make_float4(__uint_as_float(r[4 * j]) * inv_l, __uint_as_float(r[4 * j + 1]) * inv_l,
                          __uint_as_float(r[4 * j + 2]) * inv_l, __uint_as_float(r[4 * j + 3]) * inv_l);
        __syncwarp();
#pragma unroll 1
        for (int i = 0; i < 8; ++i) {  // rows 4i .. 4i + 3, eight lanes per row
          const int rr = 4 * i + (lane >> 3), j = lane & 7;
          *reinterpret_cast<float4*>(obase + static_cast<size_t>(rr) * kDc + c * 32 + 4 * j) =
              *reinterpret_cast<const float4*>(stg + rr * 32 + 4 * (j ^ (rr & 7)));
        }
        __syncwarp();
      }
      if (R == 0 && w == 0) p.part_lse[static_cast<size_t>(slot) * kH + h] = (m_run + log2f(l_tot)) * 0.69314718055994531f;
      tc_fence_before();  // O reads are complete before the next segment's P V overwrites O
      mbar_arrive(o_free);
      ++seg;
    });
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no remote access to this CTA's shared memory is still pending
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMlaThreads, 1)
    mla_kernel(const __grid_constant__ MlaParams p, const __grid_constant__ CUtensorMap tmKV,
               const __grid_constant__ CUtensorMap tmPE) {
  griddep_wait();  // (a dependent of the row gather in the sparse form)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  mla_body(p, &tmKV, &tmPE, smem, static_cast<int>(cluster_ctarank()));
}

int mla_pairs_for_device() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int pairs = sms / 2;
  return pairs < kMlaMaxPairs ? pairs : kMlaMaxPairs;
}

cudaError_t launch_mla(const MlaParams& p, const CUtensorMap& tmKV, const CUtensorMap& tmPE, cudaStream_t stream) {
  cudaError_t e = cudaFuncSetAttribute(mla_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(mla_kernel, dim3(2 * p.n_pairs), dim3(kMlaThreads), SMEM_BYTES, stream, p, tmKV, tmPE);
}

}  // namespace attn
