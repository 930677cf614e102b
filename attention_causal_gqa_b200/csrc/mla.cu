// DeepSeek MLA absorbed decode on tcgen05 tensor cores (sm_100a).
//
// "DeepSeek-V3 attention: einsum vs hand-optimised" (absorbed form):
//   scores[h, t] = (q_nope[h] . kv_cache[t] + q_pe[h] . pe_cache[t]) * scale
//   out[h]       = softmax_t(scores[h]) . kv_cache
// The two score terms are one product over the concatenated 576-wide operand
// [q_nope | q_pe] . [kv_cache | pe_cache]^T ("attention study note", MLA
// decoupled-RoPE section: the rotary part is concatenated to the content part).
//
// Work split. A cluster of two CTAs (two SMs) shares every token tile and splits
// the 576 reduction columns: rank 0 owns kv columns 0-255, rank 1 owns kv columns
// 256-511 plus the 64 rotary columns. Each CTA
//   * loads only its own columns of each kv/pe tile (no byte is loaded twice),
//   * computes its partial score block S_r = Q_r . KV_r^T (Q_r kept in TMEM),
//   * sends S_r to its peer through distributed shared memory (staged, then one
//     bulk copy per warp) and adds the peer's part (rank-0 part + rank-1 part in
//     both CTAs: identical bits),
//   * runs the online softmax on the full scores (both CTAs, same m and l),
//   * accumulates O[:, its 256 columns] += P . KV[:, its 256 columns], with P
//     written into TMEM and used as the MMA A operand.
// Scheduling is persistent: the flattened sequence of 32-token tiles of all
// sequences is cut into one contiguous range per cluster; each maximal piece of
// a range inside one sequence (a segment) produces one normalised partial result
// and its LSE, merged per sequence by mla_merge_kernel (merge.cu).
//
// Roles per CTA (352 threads): warpgroups 0 and 1 take the tiles in turn (tile k
// goes to warpgroup k % 2, one thread per head): each reads its partial score tile
// out of TMEM, sends it to the peer, adds the peer's part, and runs the online
// softmax on it, writing P. Only the running max (early in a tile) and the running
// sum (late in a tile) pass from one warpgroup to the other, through shared memory,
// so two tiles are in flight at once. The owner of a segment's first tile loads
// Q_r into TMEM; the owner of its last tile writes the partial result. Warp 8 is
// the TMA producer, warp 9 allocates TMEM and issues Q K^T, warp 10 issues P V.
// TMEM columns: O [0,256), Q_r [256, 416), S double buffer [416, 480) (tile k in
// buffer k % 2), P double buffer [480, 512).
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kH = 128, kDc = 512, kDr = 64;
constexpr int TN = kMlaTile;              // tokens per tile
constexpr int KV_BOX = TN * 128;          // one 64-column block of a tile (TN rows of 128 bytes)
constexpr int NST = 7;                    // kv ring depth
constexpr int STAGE = 5 * KV_BOX;         // room for the larger (rank-1) share
constexpr int XBUF = kH * TN * 4;         // one fp32 exchange buffer (one per tile parity)
constexpr int O_COL = 0, Q_COL = 256, S_COL = 416, P_COL = 480;  // S: 2 x TN fp32, P: 2 x TN/2 bf16 pairs
constexpr int TMEM_COLS = 512;
constexpr int kMlaThreads = 352;
constexpr int SMEM_BYTES = 1024 + NST * STAGE + 4 * XBUF + 4 * kH * 4 + 512;
static_assert(S_COL + 2 * TN <= P_COL && P_COL + TN <= TMEM_COLS, "TMEM budget");
static_assert(SMEM_BYTES <= 232448, "shared memory budget");

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t mapa_peer(uint32_t saddr, uint32_t peer) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(peer));
  return r;
}
// One bulk copy of a staged block from this CTA's shared memory into the peer's,
// completing its bytes on the peer's mbarrier (the copy engine moves the block:
// far fewer transactions than per-thread remote stores).
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst_cluster, uint32_t src_cta, uint32_t bytes,
                                                  uint32_t bar_cluster) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   dst_cluster),
               "r"(src_cta), "r"(bytes), "r"(bar_cluster)
               : "memory");
}
// Remote arrive without release semantics: used only to say "these bytes were read",
// where the reads have already returned their values (no write needs publishing).
__device__ __forceinline__ void mbar_arrive_remote_relaxed(uint32_t bar_cluster_addr) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ int tiles_of(const int32_t* lens, int b, int T_max) {
  const int L = min(max(__ldg(lens + b), 0), T_max);
  return (L + TN - 1) / TN;
}

// Calls fn(b, first_tile, end_tile, global_tile_offset_before) for every segment of
// cluster `pair` in order. Every role enumerates the same segments.
template <typename F>
__device__ __forceinline__ void for_each_segment(const MlaParams& p, int pair, F&& fn) {
  long long N = 0;
  for (int b = 0; b < p.B; ++b) N += tiles_of(p.seq_lens, b, p.T_max);
  const long long lo = N * pair / p.n_pairs, hi = N * (pair + 1) / p.n_pairs;
  long long s = 0;
  int done = 0;
  for (int b = 0; b < p.B && s < hi; ++b) {
    const int n = tiles_of(p.seq_lens, b, p.T_max);
    const long long e = s + n;
    const long long a0 = s > lo ? s : lo, a1 = e < hi ? e : hi;
    if (a1 > a0) {
      fn(b, static_cast<int>(a0 - s), static_cast<int>(a1 - s), done);
      done += static_cast<int>(a1 - a0);
    }
    s = e;
  }
}

// One body for both ranks (a runtime rank keeps the code small enough for the
// instruction cache; both ranks differ only in loop bounds and column offsets).
__device__ __forceinline__ void mla_body(const MlaParams& p, const CUtensorMap* tmKV, const CUtensorMap* tmPE,
                                         uint8_t* smem, const int R) {
  const int NKB = R == 0 ? 4 : 5;  // 64-column blocks of the score reduction owned by this CTA
  const int STAGE_BYTES = NKB * KV_BOX;
  const uint32_t PEER = 1 - R;
  uint8_t* sKV = smem;
  float* xbuf = reinterpret_cast<float*>(smem + NST * STAGE);               // [2][kH][TN] from the peer
  float* sbuf = xbuf + 2 * kH * TN;                                         // [2][kH][TN] own, staged for the copy
  float* m_sh = reinterpret_cast<float*>(smem + NST * STAGE + 4 * XBUF);    // [2][kH] running max after tile k
  float* l_sh = m_sh + 2 * kH;                                              // [2][kH] running sum after tile k
  uint64_t* bars = reinterpret_cast<uint64_t*>(l_sh + 2 * kH);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = kv_full + NST;
  uint64_t* s_full = kv_empty + NST;   // [2] S(k) computed into S buffer k % 2
  uint64_t* s_free = s_full + 2;       // [2] S(k) has been read out of TMEM
  uint64_t* p_full = s_free + 2;       // [2] P(k) written into P buffer k % 2
  uint64_t* o_done = p_full + 2;       // [2] P(k) V(k) completed
  uint64_t* x_full = o_done + 2;       // [2] the peer's partial scores of tile k landed in xbuf[k % 2]
  uint64_t* x_empty = x_full + 2;      // [2] the peer has consumed what this CTA sent for tile k
  uint64_t* m_ready = x_empty + 2;     // [2] running max after tile k is in m_sh[k % 2]
  uint64_t* l_ready = m_ready + 2;     // [2] running sum after tile k is in l_sh[k % 2]
  uint64_t* q_ready = l_ready + 2;     // Q_r of the segment is in TMEM
  uint64_t* o_free = q_ready + 1;      // the segment's partial result has been read out of O
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
    for (int u = 0; u < 2; ++u) {
      mbar_init(&s_full[u], 1);
      mbar_init(&s_free[u], 128);
      mbar_init(&p_full[u], 128);
      mbar_init(&o_done[u], 1);
      mbar_init(&x_full[u], 1);   // one expect_tx arrive per phase + the bytes of the peer's bulk copies
      mbar_init(&x_empty[u], 1);  // one remote arrive from the peer
      mbar_init(&m_ready[u], 128);
      mbar_init(&l_ready[u], 128);
    }
    mbar_init(q_ready, 128);
    mbar_init(o_free, 128);
    mbar_init(mma_done, 2);
    *abort_flag = 0;
    fence_mbar_init();
    // arm the receive buffers for the first two tiles
    for (int u = 0; u < 2; ++u) mbar_arrive_expect_tx(&x_full[u], XBUF);
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
      if (R == 1) prefetch_tmap(tmPE);
      int g = 0;
      bool ok = true;
      for_each_segment(p, pair, [&](int b, int t0, int t1, int) {
        for (int t = t0; t < t1 && ok; ++t, ++g) {
          const int s = g % NST;
          if (!mbar_wait(&kv_empty[s], ((g / NST) & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
          uint8_t* dst = sKV + s * STAGE;
          mbar_arrive_expect_tx(&kv_full[s], STAGE_BYTES);
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(dst + c * KV_BOX, tmKV, &kv_full[s], R * 256 + c * 64, t * TN, b);
          if (R == 1) tma_load_3d(dst + 4 * KV_BOX, tmPE, &kv_full[s], 0, t * TN, b);
        }
      });
    }
  } else if (warp >= 9) {
    // ------------------------------ MMA issuers (whole warps): 9 = scores, 10 = P V
    constexpr uint32_t HI = sdesc_hi_sw128(1024);
    bool ok = true;
    int seg = 0;
    if (warp == 9) {
      constexpr uint32_t idesc_s = idesc_f32acc(1, 128, TN, false, false);
      const uint32_t kv_lo_k = sdesc_lo(smem_u32(sKV), 16);
      for_each_segment(p, pair, [&](int, int t0, int t1, int g0) {
        if (!ok) return;
        if (!(ok = mbar_wait_warp(q_ready, seg & 1, abort_flag, p.status))) return;
        ++seg;
        tc_fence_after();
        for (int i = 0; ok && i < t1 - t0; ++i) {
          const int k = g0 + i;
          if (k >= 2 && !(ok = mbar_wait_warp(&s_free[k & 1], ((k - 2) >> 1) & 1, abort_flag, p.status))) break;
          if (!(ok = mbar_wait_warp(&kv_full[k % NST], (k / NST) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t b0 = kv_lo_k + (((k % NST) * STAGE) >> 4);
          const uint32_t d = tmem_base + S_COL + (k & 1) * TN;
#pragma unroll 1
          for (int bx = 0; bx < NKB; ++bx)
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
              umma_f16_ts_warp(d, tmem_base + Q_COL + (bx * 4 + kq) * 8, b0 + ((bx * KV_BOX + kq * 32) >> 4), HI,
                               idesc_s, (bx > 0 || kq > 0) ? 1u : 0u);
          umma_commit_warp(&s_full[k & 1]);
        }
      });
    } else {
      constexpr uint32_t idesc_o = idesc_f32acc(1, 128, 256, false, true);
      const uint32_t kv_lo_v = sdesc_lo(smem_u32(sKV), KV_BOX);  // MN-major: 64-column blocks KV_BOX apart
      for_each_segment(p, pair, [&](int, int t0, int t1, int g0) {
        if (!ok) return;
        for (int i = 0; ok && i < t1 - t0; ++i) {
          const int k = g0 + i;
          if (!(ok = mbar_wait_warp(&p_full[k & 1], (k >> 1) & 1, abort_flag, p.status))) break;
          // the first P V of a segment overwrites O: the previous segment's result must be out
          if (i == 0 && seg > 0 && !(ok = mbar_wait_warp(o_free, (seg - 1) & 1, abort_flag, p.status))) break;
          tc_fence_after();
          const uint32_t b0 = kv_lo_v + (((k % NST) * STAGE) >> 4);
          const uint32_t a0 = tmem_base + P_COL + (k & 1) * (TN / 2);
#pragma unroll
          for (int kb = 0; kb < TN / 16; ++kb)
            umma_f16_ts_warp(tmem_base + O_COL, a0 + kb * 8, b0 + ((kb * 16 * 128) >> 4), HI, idesc_o,
                             (i > 0 || kb > 0) ? 1u : 0u);
          umma_commit_warp(&o_done[k & 1]);
          umma_commit_warp(&kv_empty[k % NST]);  // S(k) is complete too: P(k) was computed from it
        }
        ++seg;
      });
    }
    umma_commit_warp(mma_done);
    mbar_wait_warp(mma_done, 0, abort_flag, p.status);
  } else {
    // ----------------------------- softmax warpgroups: tile k is handled by warpgroup k % 2
    const int a = warp >> 2;
    const int h = (warp & 3) * 32 + lane;  // head == TMEM lane
    const int th = threadIdx.x - 128 * a;
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint32_t peer_xbuf = mapa_peer(smem_u32(xbuf), PEER);
    const uint32_t peer_xfull = mapa_peer(smem_u32(x_full), PEER);
    const uint32_t peer_xempty = mapa_peer(smem_u32(x_empty), PEER);
    float* my_x = xbuf + (a * kH + h) * TN;
    bool alive = true;
    auto fail = [&](bool ok) -> bool {
      if (__any_sync(0xffffffffu, !ok)) alive = false;
      return !alive;
    };
    for_each_segment(p, pair, [&](int b, int t0, int t1, int g0) {
      if (!alive) return;
      const int n = t1 - t0;
      // Q_r row of head h into TMEM (bf16 pairs are already in the operand layout), by
      // the owner of the segment's first tile, once the last score tile of the previous
      // segment has been read (then every earlier Q K^T has completed).
      if ((g0 & 1) == a) {
        if (g0 > 0 && fail(mbar_wait(&m_ready[a ^ 1], ((g0 - 1) >> 1) & 1, abort_flag, p.status))) return;
        const uint32_t* qn = reinterpret_cast<const uint32_t*>(
            reinterpret_cast<const __nv_bfloat16*>(p.q_nope) + (static_cast<size_t>(b) * kH + h) * kDc + R * 256);
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {  // 4 x 32 columns = 256 bf16
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(qn + c * 32 + e));
            r[e] = v.x; r[e + 1] = v.y; r[e + 2] = v.z; r[e + 3] = v.w;
          }
          tmem_st32(t_lane + Q_COL + c * 32, r);
        }
        if (R == 1) {
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(
              reinterpret_cast<const __nv_bfloat16*>(p.q_pe) + (static_cast<size_t>(b) * kH + h) * kDr);
          uint32_t r[32];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const uint4 v = __ldg(reinterpret_cast<const uint4*>(qp + e));
            r[e] = v.x; r[e + 1] = v.y; r[e + 2] = v.z; r[e + 3] = v.w;
          }
          tmem_st32(t_lane + Q_COL + 128, r);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(q_ready);
      }
      const int L = min(max(__ldg(p.seq_lens + b), 0), p.T_max);
      float m_k = -INFINITY, l_k = 0.f;
      for (int i = (g0 & 1) == a ? 0 : 1; i < n; i += 2) {
        const int k = g0 + i;
        const uint32_t ph = (k >> 1) & 1;
        // partial scores of tile k out of TMEM; the buffer is free for S(k + 2) at once
        if (fail(mbar_wait(&s_full[a], ph, abort_flag, p.status))) return;
        tc_fence_after();
        uint32_t cur[TN];
        tmem_ld32(t_lane + S_COL + a * TN, cur);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&s_free[a]);
        // send them to the peer (chunk c of a row at slot (c + h) mod 8): stage the tile,
        // then one thread copies all of it. The staging buffer and the peer's receive
        // buffer are both free once the peer has consumed tile k - 2 (its copy had landed).
        if (fail(mbar_wait(&x_empty[a], ph ^ 1, abort_flag, p.status))) return;  // carries no data: plain wait
        {
          float* mine = sbuf + (a * kH + h) * TN;
#pragma unroll
          for (int c = 0; c < TN / 4; ++c)
            *reinterpret_cast<uint4*>(mine + 4 * ((c + h) & (TN / 4 - 1))) =
                make_uint4(cur[4 * c], cur[4 * c + 1], cur[4 * c + 2], cur[4 * c + 3]);
          fence_proxy_async_smem();
          __syncwarp();
          // each warp sends its own 32 rows as soon as they are staged
          const int row0 = (warp & 3) * 32;
          if (lane == 0)
            bulk_copy_to_peer(peer_xbuf + a * XBUF + row0 * (TN * 4), smem_u32(sbuf + (a * kH + row0) * TN),
                              XBUF / 4, peer_xfull + a * 8);
        }
        // add the peer's part: rank-0 part + rank-1 part in both CTAs (identical bits). The
        // peer's copied bytes complete on this local barrier, which makes them visible
        // to a plain wait (same rule as a TMA load).
        if (fail(mbar_wait(&x_full[a], ph, abort_flag, p.status))) return;
        float s[TN];
#pragma unroll
        for (int c = 0; c < TN / 4; ++c) {
          const float4 v = *reinterpret_cast<const float4*>(my_x + 4 * ((c + h) & (TN / 4 - 1)));
          const float w0 = __uint_as_float(cur[4 * c]), w1 = __uint_as_float(cur[4 * c + 1]);
          const float w2 = __uint_as_float(cur[4 * c + 2]), w3 = __uint_as_float(cur[4 * c + 3]);
          s[4 * c + 0] = R == 0 ? w0 + v.x : v.x + w0;
          s[4 * c + 1] = R == 0 ? w1 + v.y : v.y + w1;
          s[4 * c + 2] = R == 0 ? w2 + v.z : v.z + w2;
          s[4 * c + 3] = R == 0 ? w3 + v.w : v.w + w3;
        }
        named_bar_sync(1 + a, 128);  // every row of xbuf[a] has been read
        if (th == 0) {
          mbar_arrive_remote_relaxed(peer_xempty + a * 8);
          mbar_arrive_expect_tx(&x_full[a], XBUF);  // re-arm for tile k + 2
        }
        const int valid = L - (t0 + i) * TN;  // tokens of this tile inside the sequence
        if (valid < TN) {
#pragma unroll
          for (int c = 0; c < TN; ++c)
            if (c >= valid) s[c] = -INFINITY;
        }
        float mx0 = fmax3f(s[0], s[1], s[2]), mx1 = fmax3f(s[3], s[4], s[5]);
#pragma unroll
        for (int c = 6; c + 3 < TN; c += 4) {
          mx0 = fmax3f(mx0, s[c], s[c + 1]);
          mx1 = fmax3f(mx1, s[c + 2], s[c + 3]);
        }
        mx0 = fmaxf(mx0, s[TN - 2]);
        mx1 = fmaxf(mx1, s[TN - 1]);
        const float m_tile = fmaxf(mx0, mx1) * sl2;
        // running max after tile k - 1 (from the other warpgroup; ignored at a segment start)
        float m_prev = -INFINITY;
        if (k > 0) {
          if (fail(mbar_wait(&m_ready[a ^ 1], ((k - 1) >> 1) & 1, abort_flag, p.status))) return;
          if (i > 0) m_prev = m_sh[(a ^ 1) * kH + h];
        }
        bool rescale = false;
        if (i == 0) {
          m_k = m_tile;
        } else {
          rescale = __any_sync(0xffffffffu, m_tile > m_prev + 8.0f);
          m_k = rescale ? fmaxf(m_prev, m_tile) : m_prev;
        }
        m_sh[a * kH + h] = m_k;
        mbar_arrive(&m_ready[a]);
        const float alpha = rescale ? ex2_approx(m_prev - m_k) : 1.f;
        if (rescale) {
          // O must hold P V of tile k - 1 before it is scaled
          if (fail(mbar_wait(&o_done[a ^ 1], ((k - 1) >> 1) & 1, abort_flag, p.status))) return;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 8; ++c) {
            uint32_t r[32];
            tmem_ld32(t_lane + O_COL + c * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(t_lane + O_COL + c * 32, r);
          }
        }
        uint32_t pp[TN / 2];
        float la = 0.f, lb = 0.f;
#pragma unroll
        for (int c = 0; c < TN; c += 2) {
          const float e0 = ex2_approx(fmaf(s[c], sl2, -m_k));
          const float e1 = ex2_approx(fmaf(s[c + 1], sl2, -m_k));
          la += e0;
          lb += e1;
          pp[c / 2] = pack_bf16x2(e0, e1);
        }
        // P buffer a last held P(k - 2): its P V must be complete before it is overwritten
        if (k >= 2) {
          if (fail(mbar_wait(&o_done[a], ((k - 2) >> 1) & 1, abort_flag, p.status))) return;
          tc_fence_after();
        }
        tmem_st16(t_lane + P_COL + a * (TN / 2), pp);
        if (valid < TN) {
          // cached rows past the sequence end may hold anything: zero this CTA's
          // value columns for them so that 0 * garbage cannot reach O
          uint8_t* st = sKV + (k % NST) * STAGE;
          const int nbad = TN - valid;
          for (int idx = th; idx < 4 * nbad * 8; idx += 128) {
            const int bxx = idx / (nbad * 8), r = valid + (idx / 8) % nbad, ch = idx % 8;
            *reinterpret_cast<uint4*>(st + bxx * KV_BOX + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          named_bar_sync(1 + a, 128);  // every zero row is written before any thread signals P
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&p_full[a]);
        // running sum after tile k (from the other warpgroup's sum after tile k - 1)
        float l_prev = 0.f;
        if (k > 0) {
          if (fail(mbar_wait(&l_ready[a ^ 1], ((k - 1) >> 1) & 1, abort_flag, p.status))) return;
          if (i > 0) l_prev = l_sh[(a ^ 1) * kH + h];
        }
        l_k = l_prev * alpha + (la + lb);
        l_sh[a * kH + h] = l_k;
        mbar_arrive(&l_ready[a]);
      }
      // segment epilogue by the owner of the last tile: O / l for this CTA's 256
      // columns, and the LSE (rank 0). P V of the segment's earlier tiles completed
      // before P V of its last one.
      const int k_last = g0 + n - 1;
      if ((k_last & 1) == a) {
        if (fail(mbar_wait(&o_done[a], (k_last >> 1) & 1, abort_flag, p.status))) return;
        tc_fence_after();
        const int slot = pair + b;
        const float inv_l = 1.f / l_k;
        float* orow = p.part_o + (static_cast<size_t>(slot) * kH + h) * kDc + R * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + O_COL + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + c * 32 + e) =
                make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                            __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
        }
        if (R == 0) p.part_lse[static_cast<size_t>(slot) * kH + h] = (m_k + log2f(l_k)) * 0.69314718055994531f;
        tc_fence_before();  // O reads are complete before the next segment's P V overwrites O
        mbar_arrive(o_free);
      }
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
  mla_kernel<<<2 * p.n_pairs, kMlaThreads, SMEM_BYTES, stream>>>(p, tmKV, tmPE);
  return cudaGetLastError();
}

}  // namespace attn
