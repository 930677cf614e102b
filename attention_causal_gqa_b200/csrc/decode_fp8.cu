// Paged GQA decode over an FP8 (E4M3) cache.
//
// "7 anti-patterns of DeepSeek attention optimisation", section 3.3: cached values
// are E4M3 codes (largest magnitude 448) times a scale; here one fp32 scale per
// (page, kv head). The attention is the paged decode of decode.cu ("attention study
// note", sections "Page Attention" and the online-softmax sections); each CTA covers
// one contiguous range of the pages of all sequences and writes a normalised partial
// output and its LSE per sequence it meets, which merge.cu combines.
//
// The cache is half the bytes of the bf16 one, so the time per page halves too.
// Two things would then limit, and the design removes both:
//   * shared memory: staging converted fp16 tiles in shared memory and reading them
//     back with ldmatrix costs about four times the page's own bytes in wavefronts.
//     Here no lane writes shared memory: each loads the codes its mma fragments need
//     straight from the page's TMA image and converts them in registers.
//   * tensor issue: with G = 4 query heads per KV head, m16 tiles over heads waste
//     three quarters of every mma. Both products run transposed instead, tokens and
//     dims on the m side: S^T = K Q^T (m = the page's 16 tokens, n = 8 query heads)
//     and O^T = V^T P^T (m = 16 dims, n = 8 heads). movmatrix turns the P^T
//     accumulator tile into the B fragment of the second product.
// Fragment orders chosen so every lane's loads are 16 contiguous bytes:
//   * S^T: the dot product over d is order-free, so k-slot 2c+e of k-step kt stands
//     for d = 32c + 4kt + e and slot 2c+8+e for d = 32c + 4kt + 2 + e; lane (g, c)
//     reads 32 code bytes of tokens g and g + 8, and Q is loaded in the same order;
//   * O^T: m-row g of m-tile t stands for d = 16g + t and row g + 8 for d = 16g + 8 + t;
//     lane (g, c) reads 16 code bytes (d = 16g .. 16g+15) of tokens 2c, 2c+1, 2c+8,
//     2c+9 and ends up holding d = 16g .. 16g+15 of heads 2c and 2c+1.
// Under the 128-byte swizzle each of these loads is bank-conflict free.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kF8Warps = 8;  // compute warps, one per KV head (Hkv <= 8)
constexpr int kF8Threads = (kF8Warps + 1) * 32;
constexpr int kF8Stages = 6;  // 32 KB per stage at Hkv = 8, D = 128

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// The two E4M3 codes in the low (cvt_e4m3x2_lo) or high (cvt_e4m3x2_hi) 16 bits of w
// as an fp16 pair, the lower byte in the lower half. Every E4M3 value (largest 448,
// subnormals down to 2^-9) is exact in fp16.
__device__ __forceinline__ uint32_t cvt_e4m3x2_lo(uint32_t w) {
  uint32_t d;
  asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %1;\ncvt.rn.f16x2.e4m3x2 %0, lo;\n}" : "=r"(d) : "r"(w));
  return d;
}
__device__ __forceinline__ uint32_t cvt_e4m3x2_hi(uint32_t w) {
  uint32_t d;
  asm("{\n.reg .b16 lo, hi;\nmov.b32 {lo, hi}, %1;\ncvt.rn.f16x2.e4m3x2 %0, hi;\n}" : "=r"(d) : "r"(w));
  return d;
}
__device__ __forceinline__ uint32_t word_of(const uint4& v, int i) {
  return i == 0 ? v.x : i == 1 ? v.y : i == 2 ? v.z : v.w;
}

__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t w, bool& in_range) {
  const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xFFFF0000u);
  in_range = in_range && fabsf(lo) <= 65504.f && fabsf(hi) <= 65504.f;
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// The transpose of an 8 x 8 b16 tile held as an mma accumulator fragment (lane (g, c):
// row g, columns 2c and 2c + 1), in the same fragment form.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

}  // namespace

// What the producer tells the consumers about the page in a stage.
struct F8StageMeta {
  int b;       // sequence
  int pg;      // page index within the sequence
  int flags;   // kF8First: first page of this CTA's range in b; kF8Last: its last; kF8End: no page
  int L;       // the sequence's length (clamped to max_pages * 16)
  float ks[kF8Warps];  // key scale of each kv head
  float vs[kF8Warps];  // 2^8 * value scale of each kv head
};
constexpr int kF8First = 1, kF8Last = 2, kF8End = 4;

__device__ __forceinline__ int f8_pages_of(const DecodeParams& p, int b) {
  const int L = min(max(__ldg(p.seq_lens + b), 0), p.max_pages * 16);
  return (L + 15) >> 4;
}

// The TMA image of a stage is K then V, each [head][token][D bytes] with 128-byte
// swizzle. Products run in fp16 with fp32 accumulation: the codes convert exactly to
// their values, Q converts exactly from bf16 within the fp16 range. The key scale
// multiplies the scores in fp32; 2^8 * the value scale multiplies P before it is
// rounded to fp16 (the same fp16 range for P as values held at 2^-8 would give), l
// sums the unscaled P, and the 2^-8 returns in the final normalisation.
//
// Work balance: the per-CTA rate is bounded by the consumers' arithmetic, not by a
// shared HBM rate, so a CTA that runs out of work early is lost time. The pages of
// all sequences (N in total, in sequence order) are cut into gridDim.x contiguous
// ranges [N c / P, N (c + 1) / P): every CTA streams the same number of pages (+-1),
// whatever the length mix. The producer walks its range and hands each page's
// sequence, position and scales to the consumers with the page itself.
// D = 128: one 128-byte swizzle row per token and head (the fragment orders above);
// D = 64: 64-byte rows under the 64-byte swizzle (chunk x of token t stored at chunk
// x ^ ((t >> 1) & 3)), the same orders with d = 16c + 4kt + e for the scores (one 16-byte
// chunk per lane and token) and m-row g of m-tile t standing for d = 8g + t, row g + 8 for
// d = 8g + 4 + t (8 code bytes per lane and token) for the output.
template <int NH, int D>  // 8-head column tiles: G <= 8 * NH
__global__ void __launch_bounds__(kF8Threads, 1)
    decode_fp8_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                      const __grid_constant__ CUtensorMap tmV) {
  static_assert(D == 64 || D == 128, "code rows of 64 or 128 bytes");
  constexpr int KT = D / 16;  // k-steps of the score product
  constexpr int MT = D / 16;  // m-tiles of the output product
  constexpr int QU = D / 32;  // 16-byte pieces of a lane's share of a query row
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int page_bytes = 16 * p.Hkv * D;  // one page of K (or V) codes, all heads
  const int stage_bytes = 2 * page_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kF8Stages * stage_bytes);
  uint64_t* empty = full + kF8Stages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kF8Stages);
  F8StageMeta* meta = reinterpret_cast<F8StageMeta*>(smem + kF8Stages * stage_bytes + 256);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kF8Stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kF8Warps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kF8Warps) {
    // ---------------------------------------------------------------- producer
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    // pages per sequence: lane l sums the contiguous block [l * per, (l + 1) * per)
    const int per = (p.B + 31) / 32;
    const int bl0 = min(lane * per, p.B), bl1 = min(bl0 + per, p.B);
    long long sum = 0;
    for (int b = bl0; b < bl1; ++b) sum += f8_pages_of(p, b);
    long long incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    const long long N = __shfl_sync(0xffffffffu, incl, 31);
    const long long P = gridDim.x;
    const long long u0 = N * blockIdx.x / P, u1 = N * (blockIdx.x + 1) / P;
    int it = 0;  // ring position
    if (u1 > u0) {
      // the sequence holding page u0: found in the one lane block that contains it
      const long long excl = incl - sum;
      const unsigned hold = __ballot_sync(0xffffffffu, excl <= u0 && u0 < incl);
      const int src = __ffs(hold) - 1;
      int b = 0;
      long long s_b = 0;
      if (lane == src) {
        b = bl0;
        s_b = excl;
        for (int n = f8_pages_of(p, b); s_b + n <= u0; n = f8_pages_of(p, b)) {
          s_b += n;
          ++b;
        }
      }
      b = __shfl_sync(0xffffffffu, b, src);
      s_b = __shfl_sync(0xffffffffu, s_b, src);
      for (; s_b < u1 && b < p.B; ++b) {  // the sequences meeting [u0, u1), in order
        int L = __ldg(p.seq_lens + b);
        if (L > p.max_pages * 16) {
          if (lane == 0) atomicOr(p.status, kDevErrBadLength);
          L = p.max_pages * 16;
        }
        L = max(L, 0);
        const int np = (L + 15) >> 4;
        const int a = static_cast<int>(max(0LL, u0 - s_b)), e = static_cast<int>(min(static_cast<long long>(np), u1 - s_b));
        for (int c0 = a; c0 < e; c0 += 32) {
          // chunk of up to 32 pages: lane j owns page c0 + j (its id and scales) and hands it over
          const int cn = min(32, e - c0);
          int phys = 0;
          float ks[kF8Warps], vs[kF8Warps];
          if (lane < cn) {
            phys = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + c0 + lane);
            if (phys < 0 || phys >= p.num_pages) {
              atomicOr(p.status, kDevErrBadPage);
              phys = 0;
            }
#pragma unroll
            for (int hh = 0; hh < kF8Warps; ++hh) {
              ks[hh] = hh < p.Hkv ? __ldg(p.k_scale + static_cast<size_t>(phys) * p.Hkv + hh) : 0.f;
              vs[hh] = hh < p.Hkv ? 256.f * __ldg(p.v_scale + static_cast<size_t>(phys) * p.Hkv + hh) : 0.f;
            }
          }
          for (int j = 0; j < cn; ++j, ++it) {
            const int s = it % kF8Stages;
            bool ok = true;
            if (lane == j) {  // one lane waits for the slot, writes its metadata and starts the copies
              ok = mbar_wait(&empty[s], ((it / kF8Stages) & 1) ^ 1, abort_flag, p.status);
              if (ok) {
                F8StageMeta& m = meta[s];
                m.b = b;
                m.pg = c0 + j;
                m.flags = (c0 + j == a ? kF8First : 0) | (c0 + j == e - 1 ? kF8Last : 0);
                m.L = L;
#pragma unroll
                for (int hh = 0; hh < kF8Warps; ++hh) {
                  m.ks[hh] = ks[hh];
                  m.vs[hh] = vs[hh];
                }
                uint8_t* dst = smem + s * stage_bytes;
                mbar_arrive_expect_tx(&full[s], stage_bytes);
                tma_load_4d(dst, &tmK, &full[s], 0, 0, 0, phys);
                tma_load_4d(dst + page_bytes, &tmV, &full[s], 0, 0, 0, phys);
              }
            }
            if (!__shfl_sync(0xffffffffu, ok, j)) return;
          }
        }
        s_b += np;
      }
    }
    // end of the range: a stage with no page
    if (lane == 0) {
      const int s = it % kF8Stages;
      if (mbar_wait(&empty[s], ((it / kF8Stages) & 1) ^ 1, abort_flag, p.status)) {
        meta[s].flags = kF8End;
        mbar_arrive(&full[s]);
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  const int h = warp;  // KV head of this warp
  const bool busy = h < p.Hkv;
  const int G = p.G;
  const float sl2 = p.scale_log2;
  uint32_t qf[NH][KT][2];  // Q^T (B operand of S^T) of the current sequence
  float o[NH][MT][4];      // O^T: rows d = (D/8)g + t (elements 0, 1) and (D/8)g + D/16 + t (2, 3),
                           // columns heads 8j + 2c (elements 0, 2) and 8j + 2c + 1 (1, 3)
  float m[NH][2], l[NH][2];  // heads 8j + 2c + x; l sums this lane's tokens only
  for (int it = 0;; ++it) {
    const int s = it % kF8Stages;
    const bool ok = mbar_wait(&full[s], (it / kF8Stages) & 1, abort_flag, p.status);
    if (__any_sync(0xffffffffu, !ok)) return;
    const int flags = meta[s].flags;
    if (flags & kF8End) return;
    if (!busy) {
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      continue;
    }
    const int b = meta[s].b, pg = meta[s].pg, L = meta[s].L;
    const float ks = meta[s].ks[h], vs = meta[s].vs[h];
    if (flags & kF8First) {
      // Q^T as the B operand of S^T (n = query head): for head tile j lane (g, c) holds
      // d = 32c .. 32c+31 of query head 8j + g of this KV head's group (0 past G).
      bool in_range = true;
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        const int row = 8 * j + g;
        const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                                  (static_cast<size_t>(b) * p.Hq + h * G + row) * D + (D / 4) * c;
        uint4 r[QU];
#pragma unroll
        for (int i = 0; i < QU; ++i)
          r[i] = row < G ? *reinterpret_cast<const uint4*>(qb + 8 * i) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int kt = 0; kt < KT; ++kt) {  // words 2kt, 2kt + 1: d = 32c + 4kt + {0,1} and {2,3}
          qf[j][kt][0] = bf16x2_to_f16x2(word_of(r[kt >> 1], (2 * kt) & 3), in_range);
          qf[j][kt][1] = bf16x2_to_f16x2(word_of(r[kt >> 1], (2 * kt + 1) & 3), in_range);
        }
      }
      if (!in_range) atomicOr(p.status, kDevErrRange);
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        m[j][0] = m[j][1] = -INFINITY;
        l[j][0] = l[j][1] = 0.f;
#pragma unroll
        for (int t = 0; t < MT; ++t) o[j][t][0] = o[j][t][1] = o[j][t][2] = o[j][t][3] = 0.f;
      }
    }
    const int rem = L - pg * 16;  // valid tokens in this page (>= 1)
    const uint8_t* kpg = smem + s * stage_bytes + h * 16 * D;  // this head's 16 token rows
    const int g7 = g & 7;
    uint4 kc[4];
    if constexpr (D == 128) {
      // keys: d = 32c .. 32c+31 (logical 16-byte chunks 2c, 2c+1) of tokens g and g + 8
      kc[0] = *reinterpret_cast<const uint4*>(kpg + g * D + (((2 * c) ^ g7) << 4));
      kc[1] = *reinterpret_cast<const uint4*>(kpg + g * D + (((2 * c + 1) ^ g7) << 4));
      kc[2] = *reinterpret_cast<const uint4*>(kpg + (g + 8) * D + (((2 * c) ^ g7) << 4));
      kc[3] = *reinterpret_cast<const uint4*>(kpg + (g + 8) * D + (((2 * c + 1) ^ g7) << 4));
    } else {
      // keys: d = 16c .. 16c+15 (logical chunk c) of tokens g and g + 8 (the same swizzle
      // phase: (g + 8) >> 1 and g >> 1 agree in their low two bits)
      const int sw = (g >> 1) & 3;
      kc[0] = *reinterpret_cast<const uint4*>(kpg + g * D + ((c ^ sw) << 4));
      kc[2] = *reinterpret_cast<const uint4*>(kpg + (g + 8) * D + ((c ^ sw) << 4));
      kc[1] = kc[3] = make_uint4(0, 0, 0, 0);
    }

    // S^T = K Q^T: rows g, g + 8 = tokens; columns 2c, 2c + 1 = heads 8j + 2c + x
    float sc[NH][4];
#pragma unroll
    for (int j = 0; j < NH; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
    for (int kt = 0; kt < KT; ++kt) {
      const uint32_t w0 = word_of(kc[kt >> 2], kt & 3), w1 = word_of(kc[2 + (kt >> 2)], kt & 3);
      const uint32_t a[4] = {cvt_e4m3x2_lo(w0), cvt_e4m3x2_lo(w1), cvt_e4m3x2_hi(w0), cvt_e4m3x2_hi(w1)};
#pragma unroll
      for (int j = 0; j < NH; ++j) mma_f16_16816(sc[j], a, qf[j][kt][0], qf[j][kt][1]);
    }
    // mask tokens past the end, scale into the log2 domain, online softmax per head
    const bool ok0 = g < rem, ok1 = g + 8 < rem;
    uint32_t pb[NH][2];  // P^T -> B fragments of O^T: P[head 8j + g][tokens 2c.., 8 + 2c..]
    bool rescale = false;
    float al[NH][2];
#pragma unroll
    for (int j = 0; j < NH; ++j) {
      const float f = sl2 * ks;
      const float v0 = ok0 ? sc[j][0] * f : -INFINITY, v1 = ok0 ? sc[j][1] * f : -INFINITY;
      const float v2 = ok1 ? sc[j][2] * f : -INFINITY, v3 = ok1 ? sc[j][3] * f : -INFINITY;
      float mx0 = fmaxf(v0, v2), mx1 = fmaxf(v1, v3);
#pragma unroll
      for (int sh = 4; sh < 32; sh <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
      }
      const float n0 = fmaxf(m[j][0], mx0), n1 = fmaxf(m[j][1], mx1);
      al[j][0] = ex2_approx(m[j][0] - n0);  // exp2(-inf) = 0 on the first page
      al[j][1] = ex2_approx(m[j][1] - n1);
      m[j][0] = n0;
      m[j][1] = n1;
      const float p0 = ex2_approx(v0 - n0), p1 = ex2_approx(v1 - n1);
      const float p2 = ex2_approx(v2 - n0), p3 = ex2_approx(v3 - n1);
      l[j][0] = l[j][0] * al[j][0] + p0 + p2;
      l[j][1] = l[j][1] * al[j][1] + p1 + p3;
      rescale = rescale || al[j][0] != 1.f || al[j][1] != 1.f;
      pb[j][0] = movmatrix_trans(pack_f16x2(p0 * vs, p1 * vs));  // tokens 0-7
      pb[j][1] = movmatrix_trans(pack_f16x2(p2 * vs, p3 * vs));  // tokens 8-15
    }
    if (__any_sync(0xffffffffu, rescale)) {  // once the maxima settle O needs no rescale
#pragma unroll
      for (int j = 0; j < NH; ++j)
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          o[j][t][0] *= al[j][0];
          o[j][t][1] *= al[j][1];
          o[j][t][2] *= al[j][0];
          o[j][t][3] *= al[j][1];
        }
    }
    // values: d = 16g .. 16g+15 (D = 128: logical chunk g) or 8g .. 8g+7 (D = 64: half
    // g & 1 of chunk g >> 1) of tokens 2c, 2c+1, 2c+8, 2c+9; tokens past the end become
    // zeros so 0 * garbage cannot poison O
    uint4 vc[4];
    {
      const uint8_t* vpg = kpg + page_bytes;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int t = 2 * c + (i & 1) + 8 * (i >> 1);
        if constexpr (D == 128) {
          vc[i] = t < rem ? *reinterpret_cast<const uint4*>(vpg + t * D + ((g ^ (t & 7)) << 4))
                          : make_uint4(0, 0, 0, 0);
        } else {
          const uint2 w = t < rem ? *reinterpret_cast<const uint2*>(vpg + t * D + (((g >> 1) ^ ((t >> 1) & 3)) << 4) +
                                                                    (g & 1) * 8)
                                  : make_uint2(0, 0);
          vc[i] = make_uint4(w.x, w.y, 0, 0);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);  // the codes are in registers: the stage may be refilled
    // O^T += V^T P^T; A of m-tile t: byte t (row g) and byte 8 + t (row g + 8) of the
    // token pairs (2c, 2c+1) and (2c+8, 2c+9)
#pragma unroll
    for (int t = 0; t < MT; t += 2) {
      // bytes t, t + 1 of the two tokens interleaved: the low half pairs d = 16g + t,
      // the high half d = 16g + t + 1 (and + 8 for rows g + 8)
      const uint32_t sel = (t & 3) | ((4 + (t & 3)) << 4) | ((1 + (t & 3)) << 8) | ((5 + (t & 3)) << 12);
      const int wl = t >> 2, wh = (D == 128 ? 2 : 1) + (t >> 2);  // words of rows g and g + 8
      const uint32_t u0 = __byte_perm(word_of(vc[0], wl), word_of(vc[1], wl), sel);
      const uint32_t u1 = __byte_perm(word_of(vc[0], wh), word_of(vc[1], wh), sel);
      const uint32_t u2 = __byte_perm(word_of(vc[2], wl), word_of(vc[3], wl), sel);
      const uint32_t u3 = __byte_perm(word_of(vc[2], wh), word_of(vc[3], wh), sel);
      const uint32_t a0[4] = {cvt_e4m3x2_lo(u0), cvt_e4m3x2_lo(u1), cvt_e4m3x2_lo(u2), cvt_e4m3x2_lo(u3)};
      const uint32_t a1[4] = {cvt_e4m3x2_hi(u0), cvt_e4m3x2_hi(u1), cvt_e4m3x2_hi(u2), cvt_e4m3x2_hi(u3)};
#pragma unroll
      for (int j = 0; j < NH; ++j) {
        mma_f16_16816(o[j][t], a0, pb[j][0], pb[j][1]);
        mma_f16_16816(o[j][t + 1], a1, pb[j][0], pb[j][1]);
      }
    }
    if (flags & kF8Last) {
      const size_t base = (static_cast<size_t>(blockIdx.x) + b) * p.Hq + h * G;  // slot range + b
#pragma unroll
      for (int j = 0; j < NH; ++j)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          float lx = l[j][x];
#pragma unroll
          for (int sh = 4; sh < 32; sh <<= 1) lx += __shfl_xor_sync(0xffffffffu, lx, sh);
          const int head = 8 * j + 2 * c + x;
          if (head >= G) continue;
          const float inv = 0.00390625f / lx;
          float* r = p.part_o + (base + head) * D + (D / 8) * g;  // rows g: d = (D/8)g + t; rows g + 8: + D/16
#pragma unroll
          for (int q4 = 0; q4 < MT / 4; ++q4) {
            const int t = 4 * q4;
            *reinterpret_cast<float4*>(r + t) = make_float4(o[j][t][x] * inv, o[j][t + 1][x] * inv,
                                                            o[j][t + 2][x] * inv, o[j][t + 3][x] * inv);
            *reinterpret_cast<float4*>(r + D / 16 + t) =
                make_float4(o[j][t][2 + x] * inv, o[j][t + 1][2 + x] * inv, o[j][t + 2][2 + x] * inv,
                            o[j][t + 3][2 + x] * inv);
          }
          if (g == 0) p.part_lse[base + head] = (m[j][x] + log2f(lx)) * 0.69314718055994531f;
        }
    }
  }
}

cudaError_t launch_decode_fp8(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int* n_ranges,
                              cudaStream_t stream) {
  if ((p.D != 128 && p.D != 64) || p.Hkv > kF8Warps || p.Hkv < 1 || p.G < 1 || p.G > 16)
    return cudaErrorInvalidValue;
  const int smem = 1024 + kF8Stages * 2 * 16 * p.Hkv * p.D + 256 + kF8Stages * static_cast<int>(sizeof(F8StageMeta));
  auto kern = p.D == 128 ? (p.G <= 8 ? decode_fp8_kernel<1, 128> : decode_fp8_kernel<2, 128>)
                         : (p.G <= 8 ? decode_fp8_kernel<1, 64> : decode_fp8_kernel<2, 64>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148, per_sm = 1;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // D = 64 with one head tile fits two CTAs per SM (half the stage bytes, fewer registers):
  // twice the warps to hide the per-page softmax and hand-off latency
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kF8Threads, smem);
  if (e != cudaSuccess) return e;
  per_sm = per_sm < 1 ? 1 : (per_sm > 2 ? 2 : per_sm);
  const int grid = sms * per_sm < kDecodeFp8MaxRanges ? sms * per_sm : kDecodeFp8MaxRanges;
  *n_ranges = grid;
  kern<<<grid, kF8Threads, smem, stream>>>(p, tmK, tmV);
  return cudaGetLastError();
}

}  // namespace attn
