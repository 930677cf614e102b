// Causal GQA prefill on tcgen05 tensor cores (sm_100a).
//
// Computes O = softmax(scale * rope(Q) rope(K)^T [causal mask]) V and the
// natural-log LSE of every row, tile by tile with the online-softmax recurrence
// ("attention study note", sections "FlashAttention的改进" and
// "online-softmax 分块计算原理": running max m, running sum l, and the matching
// rescale of the output accumulator). Query head h reads KV head h / (Hq/Hkv)
// (same page, GQA worked table).
//
// A work item is two 128-row query tiles that share one KV head: two heads of
// the same group over the same rows when the group size is even, otherwise two
// consecutive row blocks of one head. The grid is persistent (one CTA per SM):
// each CTA walks its share of the items, heaviest first, and the next item's Q
// and K/V loads and first Q K^T overlap the current item's last blocks and
// epilogue. Roles (320 threads):
//   warps 0-3  softmax warpgroup of tile 0 (one thread per query row)
//   warps 4-7  softmax warpgroup of tile 1
//   warp  8    TMA producer: both Q tiles, then K/V tiles into a shared-memory ring
//   warp  9    TMEM allocator and tcgen05.mma issuer (elected lane of the warp)
// TMEM holds S_0, S_1 (BN fp32 columns each) and O_0, O_1 (D columns each).
// Q and K arrive by TMA already in operand form: rotated (RoPE, cos/sin table
// with fp64 angles) and rounded by the prologue kernels, so a CTA starts its
// first Q K^T as soon as the two tiles land. P (16-bit) is written back into
// the columns of S_t and feeds O += P V as the A operand straight from TMEM, so
// shared-memory bandwidth is spent on Q, K and V only. Per tile the tensor pipe runs P_t V_j before Q_t K_{j+1}^T,
// which both keeps P_t intact until it is consumed and guarantees that O_t is
// final for step j when S_t(j+1) is reported ready.
//
// Operand precision (every shared-memory tile is 16-bit):
//   kModeBF16   bf16 input, no RoPE: Q K^T and P V in bf16 (exact inputs).
//   kModeF16QK  bf16 input with RoPE: the rotated Q and K are rounded to fp16
//               (11-bit significand, same tensor-core rate as bf16) so the
//               rotation costs 8x less rounding than a bf16 round trip; P V in bf16.
//   kModeSplit  fp32 input: every operand x is carried as hi = bf16(x) plus
//               lo = bf16(x - hi), and each product uses the three terms
//               hi*hi + hi*lo + lo*hi (about 16 significant bits per operand).
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include <type_traits>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

enum { kModeBF16 = 0, kModeF16QK = 1, kModeSplit = 2 };

template <int D, int BN, int MODE>
struct PrefillShape {
  static constexpr int BM = 128;
  static constexpr bool SPLIT = MODE == kModeSplit;
  static constexpr int NPART = SPLIT ? 2 : 1;  // hi (and lo) parts of each operand tile
  static constexpr int Q_BOX = BM * 128;       // bytes of one 64-column block of a Q tile
  static constexpr int Q_PART = BM * D * 2;
  static constexpr int KV_BOX = BN * 128;
  static constexpr int KV_PART = BN * D * 2;
  static constexpr int KV_SLOT = NPART * KV_PART;
  static constexpr int P_COLS = BN / 2;      // TMEM columns of one 16-bit P part
  static constexpr int FIXED = 2 * NPART * Q_PART;
  static constexpr int NST_RAW = (232448 - 1024 - 256 - FIXED) / KV_SLOT;
  static constexpr int NST = NST_RAW > 8 ? 8 : NST_RAW;
  static constexpr int SMEM_BYTES = 1024 /*align slack*/ + FIXED + NST * KV_SLOT + 256 /*barriers*/;
  static constexpr int TMEM_NEEDED = 2 * BN + 2 * D;
  static constexpr int TMEM_COLS = TMEM_NEEDED <= 256 ? 256 : 512;
  static constexpr int S_COL0 = 0;
  static constexpr int O_COL0 = 2 * BN;
  static constexpr uint32_t QK_FMT = MODE == kModeF16QK ? 0u : 1u;  // f16 : bf16
  static_assert(NST >= 2, "K/V ring needs at least two slots");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
  static_assert(TMEM_NEEDED <= 512, "TMEM budget");
  static_assert(D % 64 == 0 && BN % 64 == 0, "tiles are whole 128-byte swizzle rows");
  static_assert(NPART * P_COLS <= BN, "P parts fit in the columns of S");
};

constexpr float kRescaleThreshold = 8.0f;  // log2 domain: rescale O only when the max grows by > 2^8

// 8 consecutive values -> one 16-byte chunk of bf16 elements.
__device__ __forceinline__ uint4 pack8_bf16(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

template <typename TIn>
__device__ __forceinline__ void store32(TIn* dst, const float* f);
template <>
__device__ __forceinline__ void store32<__nv_bfloat16>(__nv_bfloat16* dst, const float* f) {
#pragma unroll
  for (int i = 0; i < 4; ++i) reinterpret_cast<uint4*>(dst)[i] = pack8_bf16(f + 8 * i);
}
template <>
__device__ __forceinline__ void store32<float>(float* dst, const float* f) {
#pragma unroll
  for (int i = 0; i < 8; ++i)
    reinterpret_cast<float4*>(dst)[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
}

// Pairs out of every 8 of a softmax row that take the FMA-pipe exp2 (blocks without masking).
constexpr int kPolyPer8 = 2;

// A work item: two 128-row query tiles that share one KV head.
struct PrefillItem {
  int b, h0, h1, r0_0, r0_1, n_kv0, n_kv1;
  int off;  // position of query row 0 among the keys (0 for a plain prefill)
  int len;  // valid query rows of the sequence (S unless chunks differ in length)
};

// Item w of the list ordered heaviest (last row blocks) first.
template <int BN>
__device__ __forceinline__ PrefillItem prefill_item(const PrefillParams& p, int w) {
  constexpr int BM = 128;
  PrefillItem it;
  if (p.pair_heads) {
    const int units = p.B * (p.Hq / 2);
    const int rb = p.n_row_blocks - 1 - w / units;
    const int bh = w % units;
    it.b = bh / (p.Hq / 2);
    it.h0 = 2 * (bh % (p.Hq / 2));
    it.h1 = it.h0 + 1;
    it.r0_0 = it.r0_1 = rb * BM;
  } else {
    const int units = p.B * p.Hq;
    const int n_rp = (p.n_row_blocks + 1) / 2;
    const int rp = n_rp - 1 - w / units;
    const int bh = w % units;
    it.b = bh / p.Hq;
    it.h0 = it.h1 = bh % p.Hq;
    it.r0_0 = 2 * rp * BM;
    it.r0_1 = it.r0_0 + BM;
  }
  it.off = 0;
  if (p.q_off) {
    const int o = __ldg(p.q_off + it.b);
    it.off = o < 0 ? 0 : (o > p.max_off ? p.max_off : o);
  }
  it.len = p.S;
  if (p.q_len) {
    const int n = __ldg(p.q_len + it.b);
    it.len = n < 0 ? 0 : (n > p.S ? p.S : n);
  }
  // keys 0 .. off + len - 1; with the causal mask query row r sees keys <= off + r
  auto n_kv_for = [&](int r0) -> int {
    if (r0 >= it.len) return 0;
    if (!p.causal) return (it.off + it.len + BN - 1) / BN;
    return (it.off + min(it.len, r0 + BM) - 1) / BN + 1;
  };
  it.n_kv0 = n_kv_for(it.r0_0);
  it.n_kv1 = n_kv_for(it.r0_1);
  return it;
}

// The persistent grid walks the heaviest-first list in snake order: in round r,
// CTA c takes item r * G + c (r even) or r * G + G - 1 - c (r odd), so every CTA
// gets a similar mix of long and short items.
__device__ __forceinline__ int prefill_item_index(int r, int c, int G) {
  return r * G + ((r & 1) ? (G - 1 - c) : c);
}

template <int D, int BN, int MODE>
__global__ void __launch_bounds__(320, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap tmQ,
                   const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV) {
  griddep_wait();  // launched as a dependent of the operand prologue
  using Sh = PrefillShape<D, BN, MODE>;
  using TIn = typename std::conditional<MODE == kModeSplit, float, __nv_bfloat16>::type;
  constexpr int NP = Sh::NPART;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                           // [2 tiles][NP parts][Q_PART]
  uint8_t* sKV = sQ + 2 * NP * Sh::Q_PART;      // [NST][NP parts][KV_PART]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + Sh::NST * Sh::KV_SLOT);
  uint64_t* kv_full = bars;                     // [NST]
  uint64_t* kv_empty = bars + Sh::NST;          // [NST]
  uint64_t* q_full = bars + 2 * Sh::NST;        // [1] the item's Q tiles landed
  uint64_t* q_empty = q_full + 1;               // [1] every Q K^T of the item has completed
  uint64_t* s_full = q_empty + 1;               // [2]
  uint64_t* p_full = s_full + 2;                // [2]
  uint64_t* o_done = p_full + 2;                // [2]
  uint64_t* o_free = o_done + 2;                // [2] the item's O_t has been read out
  uint64_t* mma_done = o_free + 2;              // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const int G = gridDim.x;
  const int n_rounds = (p.n_items + G - 1) / G;
  // Calls fn(item) for this CTA's items in order; every role walks the same list. An
  // item whose two tiles have no rows to compute (past the end of a shorter chunk) is
  // skipped by every role alike.
  auto for_each_item = [&](auto&& fn) {
    for (int r = 0; r < n_rounds; ++r) {
      const int w = prefill_item_index(r, blockIdx.x, G);
      if (w >= p.n_items) continue;
      const PrefillItem it = prefill_item<BN>(p, w);
      if (it.n_kv0 == 0 && it.n_kv1 == 0) continue;
      if (!fn(it)) return;
    }
  };

  // -------------------------------------------------------------------- setup
  if (threadIdx.x == 0) {
    for (int i = 0; i < Sh::NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&s_full[t], 1);
      mbar_init(&p_full[t], 128);
      mbar_init(&o_done[t], 1);
      mbar_init(&o_free[t], 128);
    }
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, Sh::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 8) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&tmQ);
      prefetch_tmap(&tmK);
      prefetch_tmap(&tmV);
      const int zlo = p.B * p.Hkv;  // the lo parts follow the hi parts in the split layout
      int kv_i = 0, nq = 0;           // position in the K/V ring sequence; items so far
      for_each_item([&](const PrefillItem& it) -> bool {
        // Both Q tiles (rows past S arrive as zeros), already in operand form, once the
        // previous item's Q K^T products have all completed.
        if (nq > 0 && !mbar_wait(q_empty, (nq - 1) & 1, abort_flag, p.status)) return false;
        ++nq;
        mbar_arrive_expect_tx(q_full, 2 * NP * Sh::Q_PART);
        for (int t = 0; t < 2; ++t) {
          const int zq = it.b * p.Hq + (t ? it.h1 : it.h0), r0 = t ? it.r0_1 : it.r0_0;
#pragma unroll
          for (int u = 0; u < NP; ++u)
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(sQ + (t * NP + u) * Sh::Q_PART + c * Sh::Q_BOX, &tmQ, q_full, c * 64, r0,
                          zq + u * p.B * p.Hq);
        }
        const int zc = it.b * p.Hkv + it.h0 / p.G;
        const int n_max = max(it.n_kv0, it.n_kv1);
        for (int i = 0; i < 2 * n_max; ++i, ++kv_i) {  // K_j at 2j, V_j at 2j + 1
          const int j = i >> 1;
          const int s = kv_i % Sh::NST;
          const uint32_t ph = (kv_i / Sh::NST) & 1;
          if (!mbar_wait(&kv_empty[s], ph ^ 1, abort_flag, p.status)) return false;
          uint8_t* dst = sKV + s * Sh::KV_SLOT;
          mbar_arrive_expect_tx(&kv_full[s], Sh::KV_SLOT);
          const CUtensorMap* map = (i & 1) ? &tmV : &tmK;
#pragma unroll
          for (int u = 0; u < NP; ++u)
#pragma unroll
            for (int c = 0; c < D / 64; ++c)
              tma_load_3d(dst + u * Sh::KV_PART + c * Sh::KV_BOX, map, &kv_full[s], c * 64, j * BN, zc + u * zlo);
        }
        return true;
      });
    }
  } else if (warp == 9) {
    // -------------------------------------------------- MMA issuer (whole warp)
    {
      constexpr uint32_t idesc_qk = idesc_f32acc(Sh::QK_FMT, 128, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_f32acc(1, 128, D, false, true);
      // (A part, B part) products: hi*hi, plus hi*lo and lo*hi for split operands
      constexpr int NPROD = Sh::SPLIT ? 3 : 1;
      bool ok = true;
      // Descriptor words: the high word is shared by every operand; the low word
      // carries the start address (>> 4), advanced by compile-time offsets below.
      constexpr uint32_t HI = sdesc_hi_sw128(1024);
      constexpr uint32_t LBO_K = 16;            // unused for K-major swizzled operands
      const uint32_t q_lo = sdesc_lo(smem_u32(sQ), LBO_K);
      const uint32_t kv_lo_k = sdesc_lo(smem_u32(sKV), LBO_K);
      const uint32_t kv_lo_v = sdesc_lo(smem_u32(sKV), Sh::KV_BOX);  // MN-major V: LBO = 64-column block stride
      auto issue_qk = [&](int t, int slot) {
        const uint32_t a0 = q_lo + ((t * NP * Sh::Q_PART) >> 4);
        const uint32_t b0 = kv_lo_k + ((slot * Sh::KV_SLOT) >> 4);
        const uint32_t d = tmem_base + Sh::S_COL0 + t * BN;
#pragma unroll
        for (int kb = 0; kb < D / 16; ++kb) {
#pragma unroll
          for (int x = 0; x < NPROD; ++x) {
            const int pa = x == 2 ? 1 : 0, pb = x == 1 ? 1 : 0;
            const uint32_t ao = (pa * Sh::Q_PART + (kb >> 2) * Sh::Q_BOX + (kb & 3) * 32) >> 4;
            const uint32_t bo = (pb * Sh::KV_PART + (kb >> 2) * Sh::KV_BOX + (kb & 3) * 32) >> 4;
            umma_f16_lohi_warp(d, a0 + ao, HI, b0 + bo, HI, idesc_qk, (kb > 0 || x > 0) ? 1u : 0u);
          }
        }
      };
      auto issue_pv = [&](int t, int slot, bool acc) {
        const uint32_t a0 = tmem_base + Sh::S_COL0 + t * BN;  // P_t lives in the columns of S_t
        const uint32_t b0 = kv_lo_v + ((slot * Sh::KV_SLOT) >> 4);
        const uint32_t d = tmem_base + Sh::O_COL0 + t * D;
#pragma unroll
        for (int kb = 0; kb < BN / 16; ++kb) {
#pragma unroll
          for (int x = 0; x < NPROD; ++x) {
            const int pa = x == 2 ? 1 : 0, pb = x == 1 ? 1 : 0;
            const uint32_t bo = (pb * Sh::KV_PART + kb * 16 * 128) >> 4;
            umma_f16_ts_warp(d, a0 + pa * Sh::P_COLS + kb * 8, b0 + bo, HI, idesc_pv, (acc || kb > 0 || x > 0) ? 1u : 0u);
          }
        }
      };
      int kv_i = 0, nq = 0;    // position in the K/V ring sequence; items so far
      int g[2] = {0, 0};       // blocks of tile t processed in earlier items (barrier phases)
      int ne[2] = {0, 0};      // earlier items with work for tile t (o_free phases)
      for_each_item([&](const PrefillItem& it) -> bool {
        const int n_kv[2] = {it.n_kv0, it.n_kv1};
        const int n_max = max(n_kv[0], n_kv[1]);
        if (!(ok = mbar_wait_warp(q_full, nq & 1, abort_flag, p.status))) return false;
        ++nq;
        auto slot_of = [&](int i) { return (kv_i + i) % Sh::NST; };
        auto par_of = [&](int i) -> uint32_t { return ((kv_i + i) / Sh::NST) & 1; };
        // K_0; S_t(0) overwrites the columns that held P_t of the previous item, whose
        // P V was issued earlier on the same in-order pipe.
        if (!(ok = mbar_wait_warp(&kv_full[slot_of(0)], par_of(0), abort_flag, p.status))) return false;
        tc_fence_after();
        for (int t = 0; t < 2; ++t)
          if (n_kv[t] > 0) {
            issue_qk(t, slot_of(0));
            umma_commit_warp(&s_full[t]);
          }
        umma_commit_warp(&kv_empty[slot_of(0)]);
        for (int j = 0; ok && j < n_max; ++j) {
          const int sV = slot_of(2 * j + 1), sK = slot_of(2 * j + 2);
          if (!(ok = mbar_wait_warp(&kv_full[sV], par_of(2 * j + 1), abort_flag, p.status))) break;
          bool k_ready = false;
          for (int t = 0; t < 2 && ok; ++t) {
            if (j >= n_kv[t]) continue;
            if (!(ok = mbar_wait_warp(&p_full[t], (g[t] + j) & 1, abort_flag, p.status))) break;
            // the item's first P V overwrites O_t: the previous item's result must be out
            if (j == 0 && ne[t] > 0 && !(ok = mbar_wait_warp(&o_free[t], (ne[t] - 1) & 1, abort_flag, p.status)))
              break;
            tc_fence_after();
            // P_t V_j first: it reads P_t from the columns that Q_t K_{j+1}^T overwrites.
            issue_pv(t, sV, j > 0);
            umma_commit_warp(&o_done[t]);
            if (j + 1 < n_kv[t]) {
              if (!k_ready) {
                if (!(ok = mbar_wait_warp(&kv_full[sK], par_of(2 * j + 2), abort_flag, p.status))) break;
                tc_fence_after();
                k_ready = true;
              }
              issue_qk(t, sK);
              umma_commit_warp(&s_full[t]);
            }
          }
          if (!ok) break;
          umma_commit_warp(&kv_empty[sV]);
          if (k_ready) umma_commit_warp(&kv_empty[sK]);
        }
        if (!ok) return false;
        umma_commit_warp(q_empty);  // every Q K^T of the item has been issued
        for (int t = 0; t < 2; ++t) {
          g[t] += n_kv[t];
          ne[t] += n_kv[t] > 0;
        }
        kv_i += 2 * n_max;
        return true;
      });
      // drain: every MMA issued above has completed once this barrier flips
      umma_commit_warp(mma_done);
      mbar_wait_warp(mma_done, 0, abort_flag, p.status);
    }
  } else {
    // ------------------------------------------------------- softmax warpgroups
    const int t = warp >> 2;
    const int wr = warp & 3;
    const int row = wr * 32 + lane;  // TMEM lane == query row within the tile
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(wr * 32) << 16);
    const float sl2 = p.scale_log2;
    bool alive = true;
    int g = 0;  // blocks of this tile processed in earlier items (barrier phases)
    for_each_item([&](const PrefillItem& it) -> bool {
    const int h = t ? it.h1 : it.h0;
    const int r0 = t ? it.r0_1 : it.r0_0;
    const int n_kv = t ? it.n_kv1 : it.n_kv0;
    const int b = it.b;
    if (n_kv == 0) return true;
    const int grow = r0 + row;
    const bool row_valid = grow < it.len;
    float m_run = -INFINITY;
    float l_run = 0.f;
    const int limit = it.off + (p.causal ? min(grow, it.len - 1) : it.len - 1);  // last key this row may see

    for (int j = 0; j < n_kv && alive; ++j) {
      bool ok = mbar_wait(&s_full[t], (g + j) & 1, abort_flag, p.status);
      if (__any_sync(0xffffffffu, !ok)) { alive = false; break; }
      tc_fence_after();
      // The whole S row comes to registers with back-to-back TMEM loads and one wait.
      constexpr int NCH = BN / 32;
      const int thr = limit - j * BN;  // columns > thr are masked
      const bool need_mask = __any_sync(0xffffffffu, thr < BN - 1);  // diagonal or ragged tile
      uint32_t sr[NCH][32];
#pragma unroll
      for (int c = 0; c < NCH; ++c) tmem_ld32(t_lane + Sh::S_COL0 + t * BN + c * 32, sr[c]);
      tmem_ld_wait();
      if (need_mask) {
#pragma unroll
        for (int c = 0; c < NCH; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e > thr) sr[c][e] = __float_as_uint(-INFINITY);
      }
      float mxa = -INFINITY, mxb = -INFINITY, mxc = -INFINITY, mxd = -INFINITY;
#pragma unroll
      for (int c = 0; c < NCH; ++c)
#pragma unroll
        for (int e = 0; e < 32; e += 8) {  // four independent max chains
          mxa = fmax3f(mxa, __uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1]));
          mxb = fmax3f(mxb, __uint_as_float(sr[c][e + 2]), __uint_as_float(sr[c][e + 3]));
          mxc = fmax3f(mxc, __uint_as_float(sr[c][e + 4]), __uint_as_float(sr[c][e + 5]));
          mxd = fmax3f(mxd, __uint_as_float(sr[c][e + 6]), __uint_as_float(sr[c][e + 7]));
        }
      const float mx = fmaxf(fmaxf(mxa, mxb), fmaxf(mxc, mxd));
      const float m_tile = mx * sl2;
      const float m_new = fmaxf(m_run, m_tile);

      // S_t(j) being ready implies P_t V_{j-1} has completed (same in-order tensor
      // pipe, and the commit covers every earlier MMA), so O_t may be rescaled now.
      float alpha = 1.f;
      bool rescale = false;
      if (j > 0) {
        rescale = __any_sync(0xffffffffu, m_new > m_run + kRescaleThreshold);
        if (rescale) {
          alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
          l_run *= alpha;
        }
      } else {
        m_run = m_new;
      }

      // P = exp2(s * scale * log2(e) - m) as 16-bit pairs into the columns of S_t, and the row sum.
      // In blocks without masked columns, kPolyPer8 of every 8 pairs take the FMA-pipe
      // exp2 so the MUFU and FMA pipes share the work.
      const float2 sl2x2 = make_float2(sl2, sl2);
      const float2 nmx2 = make_float2(-m_run, -m_run);
      const uint32_t p_col = t_lane + Sh::S_COL0 + t * BN;
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      auto exp_rows = [&](auto poly_tag) {
        constexpr bool kPoly = decltype(poly_tag)::value;
        auto ex = [&](float2 z, int q) -> float2 {
          if (kPoly && (q * kPolyPer8) % 8 < kPolyPer8) return exp2_fma2(z);
          return make_float2(ex2_approx(z.x), ex2_approx(z.y));
        };
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t ph[16];
          uint32_t pl[Sh::SPLIT ? 16 : 1];
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float2 z0 = ffma2(make_float2(__uint_as_float(sr[c][e]), __uint_as_float(sr[c][e + 1])), sl2x2, nmx2);
            const float2 z1 = ffma2(make_float2(__uint_as_float(sr[c][e + 2]), __uint_as_float(sr[c][e + 3])), sl2x2, nmx2);
            const float2 p0 = ex(z0, e >> 1);
            const float2 p1 = ex(z1, (e >> 1) + 1);
            acc[(e >> 1) & 3] = fadd2(acc[(e >> 1) & 3], p0);
            acc[((e >> 1) + 1) & 3] = fadd2(acc[((e >> 1) + 1) & 3], p1);
            if constexpr (Sh::SPLIT) {
              const float h0 = __bfloat162float(__float2bfloat16_rn(p0.x)), h1 = __bfloat162float(__float2bfloat16_rn(p0.y));
              const float h2 = __bfloat162float(__float2bfloat16_rn(p1.x)), h3 = __bfloat162float(__float2bfloat16_rn(p1.y));
              ph[e >> 1] = pack_bf16x2(h0, h1);
              ph[(e >> 1) + 1] = pack_bf16x2(h2, h3);
              pl[e >> 1] = pack_bf16x2(p0.x - h0, p0.y - h1);
              pl[(e >> 1) + 1] = pack_bf16x2(p1.x - h2, p1.y - h3);
            } else {
              ph[e >> 1] = pack_bf16x2(p0.x, p0.y);
              ph[(e >> 1) + 1] = pack_bf16x2(p1.x, p1.y);
            }
          }
          tmem_st16(p_col + c * 16, ph);
          if constexpr (Sh::SPLIT) tmem_st16(p_col + Sh::P_COLS + c * 16, pl);
        }
      };
      if (Sh::SPLIT || need_mask)
        exp_rows(std::false_type{});
      else
        exp_rows(std::true_type{});
      const float2 acc01 = fadd2(acc[0], acc[1]), acc23 = fadd2(acc[2], acc[3]);
      const float lsum = (acc01.x + acc01.y) + (acc23.x + acc23.y);
      // O *= alpha (warp-uniform decision; exact because P and l use the same m)
      if (rescale) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          const uint32_t ta = t_lane + Sh::O_COL0 + t * D + c * 32;
          tmem_ld32(ta, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(ta, r);
        }
      }
      tmem_st_wait();  // P (and a rescaled O) are in TMEM before the MMA may read them
      l_run += lsum;
      tc_fence_before();
      mbar_arrive(&p_full[t]);
    }

    // Epilogue: O / l and LSE = (m + log2 l) * ln 2; then O_t is free for the next item.
    if (alive) {
      bool ok = mbar_wait(&o_done[t], (g + n_kv - 1) & 1, abort_flag, p.status);
      if (__any_sync(0xffffffffu, !ok)) alive = false;
      if (alive) {
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        TIn* orow = reinterpret_cast<TIn*>(p.out) + ((static_cast<size_t>(b) * p.Hq + h) * p.S + grow) * D;
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + Sh::O_COL0 + t * D + c * 32, r);
          tmem_ld_wait();
          if (row_valid) {
            float f[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(r[e]) * inv_l;
            store32<TIn>(orow + c * 32, f);
          }
        }
        if (row_valid)
          p.lse[(static_cast<size_t>(b) * p.Hq + h) * p.S + grow] = (m_run + log2f(l_run)) * 0.69314718055994531f;
        tc_fence_before();
        mbar_arrive(&o_free[t]);
      }
    }
    g += n_kv;
    return alive;
    });
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem_base, Sh::TMEM_COLS);
  }
}

template <int D, int BN, int MODE>
static cudaError_t launch_prefill_t(const PrefillParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                                    const CUtensorMap& tmV,
                                    int grid, cudaStream_t stream) {
  using Sh = PrefillShape<D, BN, MODE>;
  auto kern = prefill_kernel<D, BN, MODE>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Sh::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_pdl(kern, dim3(grid), dim3(320), Sh::SMEM_BYTES, stream, p, tmQ, tmK, tmV);
}

int prefill_block_n(int D, bool f32) {
  (void)D;
  return f32 ? 64 : 128;
}

cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           int D, bool f32,
                           bool rope, int grid, cudaStream_t stream) {
  if (f32) {
    if (D == 64) return launch_prefill_t<64, 64, kModeSplit>(p, tmQ, tmK, tmV, grid, stream);
    return cudaErrorInvalidValue;
  }
  if (rope) {
    // (the chunk path leaves its operand rows past a sequence's last 128-key block unwritten)
    if (D == 128) return launch_prefill_t<128, 128, kModeF16QK>(p, tmQ, tmK, tmV, grid, stream);
    if (D == 64) return launch_prefill_t<64, 128, kModeF16QK>(p, tmQ, tmK, tmV, grid, stream);
  } else {
    if (D == 128) return launch_prefill_t<128, 128, kModeBF16>(p, tmQ, tmK, tmV, grid, stream);
    if (D == 64) return launch_prefill_t<64, 128, kModeBF16>(p, tmQ, tmK, tmV, grid, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace attn
