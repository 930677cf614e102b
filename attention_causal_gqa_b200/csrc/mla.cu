// DeepSeek MLA absorbed decode on tcgen05 tensor cores (sm_100a).
//
// "DeepSeek-V3 attention: einsum vs hand-optimised" (absorbed form):
//   scores[h, t] = (q_nope[h] . kv_cache[t] + q_pe[h] . pe_cache[t]) * scale
//   out[h]       = softmax_t(scores[h]) . kv_cache
// The two score terms are one product over the concatenated 576-wide operand
// [q_nope | q_pe] . [kv_cache | pe_cache]^T ("attention study note", MLA
// decoupled-RoPE section: the rotary part is concatenated to the content part).
//
// Work unit: one split of 512 cached tokens of one sequence and one half of the
// 512 latent output columns (a CTA pair shares a split; each recomputes S, so
// the output accumulator of 128 heads x 256 fp32 fits TMEM next to S).
// Roles (192 threads):
//   warps 0-3  softmax warpgroup, one thread per head; epilogue
//   warp  4    TMA producer (Q once, then kv/pe tiles of TN tokens)
//   warp  5    TMEM allocator and single-thread tcgen05.mma issuer
// TMEM: S double buffer (2 x TN fp32 columns) and O (256 fp32 columns).
// Q stays resident in shared memory (9 swizzled 128-byte column blocks).
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kMlaH = 128, kMlaDc = 512, kMlaDr = 64;
constexpr int kMlaKB = (kMlaDc + kMlaDr) / 64;    // 9 column blocks of 64
constexpr int kMlaQBox = 128 * 128;                // one 64-column block of Q: 16 KB
constexpr int kMlaQBytes = kMlaKB * kMlaQBox;      // 147456
constexpr int kMlaHalf = kMlaDc / 2;               // output columns per CTA
constexpr int kMlaSplitTokens = kMlaTokensPerTile * kMlaTilesPerSplit;

// SWIZZLE_NONE K-major descriptor: 8x16-byte core matrices, LBO along K, SBO along M/N.
__device__ __forceinline__ uint64_t sdesc_interleave(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  return d;  // layout type 0
}

}  // namespace

template <int TN, int NST>
__global__ void __launch_bounds__(192, 1)
    mla_kernel(const __grid_constant__ MlaParams p, const __grid_constant__ CUtensorMap tmQn,
               const __grid_constant__ CUtensorMap tmQp, const __grid_constant__ CUtensorMap tmKV,
               const __grid_constant__ CUtensorMap tmPE) {
  constexpr int KV_BOX = TN * 128;             // one 64-column block of a kv/pe tile
  constexpr int STAGE = kMlaKB * KV_BOX;
  constexpr int P_BYTES = 128 * TN * 2;
  constexpr int TMEM_COLS = 512;
  constexpr int O_COL = 256;
  static_assert(2 * TN <= O_COL, "S buffers fit below O");
  static_assert(TN % 32 == 0, "one 32-column TMEM load per tile");

  const int half = blockIdx.x & 1;
  const int rest = blockIdx.x >> 1;
  const int split = rest % p.n_splits;
  const int b = rest / p.n_splits;
  int L = __ldg(p.seq_lens + b);
  if (L > p.T_max) {
    if (threadIdx.x == 0) atomicOr(p.status, kDevErrBadLength);
    L = p.T_max;
  }
  const int t0 = split * kMlaSplitTokens;
  if (t0 >= L) return;  // uniform for the whole CTA
  const int ntok = min(kMlaSplitTokens, L - t0);
  const int n_tiles = (ntok + TN - 1) / TN;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = sQ + kMlaQBytes;
  uint8_t* sP = sKV + NST * STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + P_BYTES);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + NST;
  uint64_t* q_full = bars + 2 * NST;
  uint64_t* s_full = q_full + 1;   // [2]
  uint64_t* p_full = s_full + 2;
  uint64_t* o_done = p_full + 1;
  uint64_t* mma_done = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < NST; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4) {
    // --------------------------------------------------------------- producer
    if (lane == 0) {
      prefetch_tmap(&tmQn);
      prefetch_tmap(&tmQp);
      prefetch_tmap(&tmKV);
      prefetch_tmap(&tmPE);
      mbar_arrive_expect_tx(q_full, kMlaQBytes);
#pragma unroll
      for (int c = 0; c < kMlaDc / 64; ++c) tma_load_3d(sQ + c * kMlaQBox, &tmQn, q_full, c * 64, 0, b);
      tma_load_3d(sQ + (kMlaDc / 64) * kMlaQBox, &tmQp, q_full, 0, 0, b);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % NST;
        if (!mbar_wait(&kv_empty[s], ((j / NST) & 1) ^ 1, abort_flag, p.status)) break;
        uint8_t* dst = sKV + s * STAGE;
        mbar_arrive_expect_tx(&kv_full[s], STAGE);
        const int tok = t0 + j * TN;
#pragma unroll
        for (int c = 0; c < kMlaDc / 64; ++c) tma_load_3d(dst + c * KV_BOX, &tmKV, &kv_full[s], c * 64, tok, b);
        tma_load_3d(dst + (kMlaDc / 64) * KV_BOX, &tmPE, &kv_full[s], 0, tok, b);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_f32acc(1, 128, TN, false, false);
      constexpr uint32_t idesc_o = idesc_f32acc(1, 128, kMlaHalf, false, true);
      auto issue_s = [&](int j) {
        const uint32_t a0 = smem_u32(sQ);
        const uint32_t b0 = smem_u32(sKV + (j % NST) * STAGE);
        const uint32_t d = tmem_base + (j & 1) * TN;
#pragma unroll
        for (int kb = 0; kb < kMlaKB * 4; ++kb) {
          const uint64_t ad = sdesc_sw128(a0 + (kb >> 2) * kMlaQBox + (kb & 3) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(b0 + (kb >> 2) * KV_BOX + (kb & 3) * 32, 16, 1024);
          umma_ss<false>(d, ad, bd, idesc_s, kb > 0 ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int j) {
        const uint32_t a0 = smem_u32(sP);
        const uint32_t b0 = smem_u32(sKV + (j % NST) * STAGE) + half * 4 * KV_BOX;
        const uint32_t d = tmem_base + O_COL;
#pragma unroll
        for (int kb = 0; kb < TN / 16; ++kb) {
          const uint64_t ad = sdesc_interleave(a0 + kb * 2 * 128, 128, TN * 16);
          const uint64_t bd = sdesc_sw128(b0 + kb * 16 * 128, KV_BOX, 1024);
          umma_ss<false>(d, ad, bd, idesc_o, (j > 0 || kb > 0) ? 1u : 0u);
        }
      };
      bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
      for (int j = 0; ok && j < 2 && j < n_tiles; ++j) {
        ok = mbar_wait(&kv_full[j % NST], (j / NST) & 1, abort_flag, p.status);
        if (!ok) break;
        tc_fence_after();
        issue_s(j);
        umma_commit(&s_full[j & 1]);
      }
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (!mbar_wait(p_full, j & 1, abort_flag, p.status)) break;
        tc_fence_after();
        issue_pv(j);
        umma_commit(o_done);
        umma_commit(&kv_empty[j % NST]);
        const int jn = j + 2;
        if (jn < n_tiles) {
          if (!mbar_wait(&kv_full[jn % NST], (jn / NST) & 1, abort_flag, p.status)) break;
          tc_fence_after();
          issue_s(jn);
          umma_commit(&s_full[jn & 1]);
        }
      }
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, p.status);
    }
  } else {
    // -------------------------------------------------------- softmax warpgroup
    const int row = warp * 32 + lane;  // head
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY, l_run = 0.f;
    bool alive = true;
    for (int j = 0; j < n_tiles && alive; ++j) {
      bool ok = mbar_wait(&s_full[j & 1], (j >> 1) & 1, abort_flag, p.status);
      if (__any_sync(0xffffffffu, !ok)) { alive = false; break; }
      tc_fence_after();
      float s[TN];
#pragma unroll
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_lane + (j & 1) * TN + c * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[e]);
      }
      const int rem = ntok - j * TN;  // valid tokens in this tile
      if (rem < TN) {
#pragma unroll
        for (int c = 0; c < TN; ++c)
          if (c >= rem) s[c] = -INFINITY;
      }
      float mx = s[0];
#pragma unroll
      for (int c = 1; c < TN; ++c) mx = fmaxf(mx, s[c]);
      const float m_new = fmaxf(m_run, mx * sl2);
      if (j > 0) {
        ok = mbar_wait(o_done, (j - 1) & 1, abort_flag, p.status);
        if (__any_sync(0xffffffffu, !ok)) { alive = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, m_new > m_run + 8.0f)) {
          const float alpha = ex2_approx(m_run - m_new);
          m_run = m_new;
          l_run *= alpha;
#pragma unroll
          for (int c = 0; c < kMlaHalf / 32; ++c) {
            uint32_t r[32];
            const uint32_t ta = t_lane + O_COL + c * 32;
            tmem_ld32(ta, r);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
            tmem_st32(ta, r);
          }
          tmem_st_wait();
        }
      } else {
        m_run = m_new;
      }
      if (rem < TN) {
        // cached rows past the sequence end may hold anything: zero this half's
        // value columns for them so that 0 * garbage cannot reach O
        uint8_t* st = sKV + (j % NST) * STAGE + half * 4 * KV_BOX;
        const int nbad = TN - rem;
        for (int idx = threadIdx.x; idx < 4 * nbad * 8; idx += 128) {
          const int bx = idx / (nbad * 8), r = rem + (idx / 8) % nbad, ch = idx % 8;
          *reinterpret_cast<uint4*>(st + bx * KV_BOX + r * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      // P (bf16) in the SWIZZLE_NONE K-major layout: core matrix (row/8, key/8) at
      // (row/8) * TN*16 + (key/8) * 128, rows 16 bytes apart inside it.
      const float neg_m = -m_run;
      float lsum = 0.f;
#pragma unroll
      for (int c = 0; c < TN / 8; ++c) {
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          f[e] = ex2_approx(fmaf(s[c * 8 + e], sl2, neg_m));
          lsum += f[e];
        }
        const uint4 v = make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                                   pack_bf16x2(f[6], f[7]));
        *reinterpret_cast<uint4*>(sP + (row >> 3) * (TN * 16) + c * 128 + (row & 7) * 16) = v;
      }
      l_run += lsum;
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full);
    }
    if (alive) {
      bool ok = mbar_wait(o_done, (n_tiles - 1) & 1, abort_flag, p.status);
      if (!__any_sync(0xffffffffu, !ok)) {
        tc_fence_after();
        const float inv_l = 1.f / l_run;
        float* orow = p.part_o + ((static_cast<size_t>(b) * p.n_splits + split) * kMlaH + row) * kMlaDc + half * kMlaHalf;
#pragma unroll
        for (int c = 0; c < kMlaHalf / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_lane + O_COL + c * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 4)
            *reinterpret_cast<float4*>(orow + c * 32 + e) =
                make_float4(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l,
                            __uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
        }
        if (half == 0)
          p.part_lse[(static_cast<size_t>(b) * p.n_splits + split) * kMlaH + row] =
              (m_run + log2f(l_run)) * 0.69314718055994531f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

cudaError_t launch_mla(const MlaParams& p, const CUtensorMap& tmQn, const CUtensorMap& tmQp,
                       const CUtensorMap& tmKV, const CUtensorMap& tmPE, cudaStream_t stream) {
  constexpr int TN = kMlaTokensPerTile, NST = 2;
  constexpr int smem = 1024 + kMlaQBytes + NST * kMlaKB * TN * 128 + 128 * TN * 2 + 128;
  static_assert(smem <= 232448, "shared memory budget");
  auto kern = mla_kernel<TN, NST>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = 2 * p.n_splits * p.B;
  kern<<<grid, 192, smem, stream>>>(p, tmQn, tmQp, tmKV, tmPE);
  return cudaGetLastError();
}

}  // namespace attn
