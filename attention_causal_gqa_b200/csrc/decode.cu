// Paged split-KV GQA decode (one query token per sequence).
//
// "attention study note", section "Page Attention": keys and values live in
// fixed-size pages (16 tokens here) reached through a per-sequence block table.
// Each split of a sequence (kDecodePagesPerSplit pages) produces a normalised
// partial output and its LSE; merge.cu combines the splits with the block-level
// form of the online-softmax recurrence (section "online-softmax 分块计算原理").
//
// Data movement is the bound: 4 flop per byte. A persistent CTA per SM streams
// whole pages (all KV heads of 16 tokens: 32 KB of K plus 32 KB of V at Hkv=8,
// D=128) with one TMA per page and tensor into a shared-memory ring. The tensor
// map is 5-D so the shared-memory image is [head][d/64][token][64] with 128-byte
// swizzle, i.e. tokens on consecutive rows, which makes the ldmatrix reads below
// bank-conflict free. Warp w handles KV head w of the page's head group and up to
// 16 of its query heads (one m16 row tile); the two tiny products (16 x 16 tokens
// x D) run as warp-level mma.sync m16n8k16 with fp32 accumulation so instruction
// issue stays far below the HBM rate.
// A work item is (sequence, split, head group, query tile): KV heads are taken 8 at
// a time (one TMA box of up to 8 heads per page), so any Hkv is served without
// reading a page twice; a group size G > 16 takes ceil(G / 16) query tiles, each of
// which reads the pages again (GQA shapes with G <= 16 read every byte once).
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace attn {

namespace {

constexpr int kDecWarps = 8;           // compute warps, one per KV head of a head group
constexpr int kDecThreads = (kDecWarps + 1) * 32;
constexpr int kDecStages = 3;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}


}  // namespace

template <int D>
__global__ void __launch_bounds__(kDecThreads, 1)
    decode_kernel(const __grid_constant__ DecodeParams p, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV) {
  constexpr int DH = D / 64;                 // 128-byte column blocks per row
  constexpr int KT = D / 16;                 // k-steps of the score product
  constexpr int NT = D / 8;                  // n-tiles of the output product
  constexpr int PPS = kDecodePagesPerSplit;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int page_bytes = 16 * p.HG * D * 2;  // one page of K (or V), the heads of one group
  const int stage_bytes = 2 * page_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kDecStages * stage_bytes);
  uint64_t* empty = full + kDecStages;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kDecStages);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kDecWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  // item k: sequence k % B; then query tile, head group and split (outermost)
  const int n_items = p.B * p.n_qt * p.n_hg * p.n_splits;

  if (warp == kDecWarps) {
    // ---------------------------------------------------------------- producer
    prefetch_tmap(&tmK);
    prefetch_tmap(&tmV);
    int it = 0;  // ring position
    for (int k = blockIdx.x; k < n_items; k += gridDim.x) {
      const int b = k % p.B, hg = (k / (p.B * p.n_qt)) % p.n_hg, split = k / (p.B * p.n_qt * p.n_hg);
      int L = __ldg(p.seq_lens + b);
      if (L > p.max_pages * 16) {
        if (lane == 0) atomicOr(p.status, kDevErrBadLength);
        L = p.max_pages * 16;
      }
      const int npages = (L + 15) >> 4;
      const int pg0 = split * PPS;
      if (pg0 >= npages) continue;
      const int pg1 = min(npages, pg0 + PPS);
      // the split's page ids, one per lane
      int my_page = 0;
      if (lane < pg1 - pg0) {
        my_page = __ldg(p.block_table + static_cast<size_t>(b) * p.max_pages + pg0 + lane);
        if (my_page < 0 || my_page >= p.num_pages) {
          atomicOr(p.status, kDevErrBadPage);
          my_page = 0;
        }
      }
      for (int pg = pg0; pg < pg1; ++pg, ++it) {
        const int phys = __shfl_sync(0xffffffffu, my_page, pg - pg0);
        const int s = it % kDecStages;
        const uint32_t ph = (it / kDecStages) & 1;
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, p.status);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) return;
        if (lane == 0) {
          uint8_t* dst = smem + s * stage_bytes;
          mbar_arrive_expect_tx(&full[s], stage_bytes);
          tma_load_5d(dst, &tmK, &full[s], 0, 0, 0, hg * kDecWarps, phys);
          tma_load_5d(dst + page_bytes, &tmV, &full[s], 0, 0, 0, hg * kDecWarps, phys);
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  const int g = lane >> 2, c = lane & 3;
  const int G = p.G;
  const float sl2 = p.scale_log2;
  int it = 0;
  for (int k = blockIdx.x; k < n_items; k += gridDim.x) {
    const int b = k % p.B, qt = (k / p.B) % p.n_qt, hg = (k / (p.B * p.n_qt)) % p.n_hg;
    const int split = k / (p.B * p.n_qt * p.n_hg);
    const int h = hg * kDecWarps + warp;        // KV head of this warp
    const bool busy = warp < p.HG && h < p.Hkv;
    const int q0 = qt * 16;                     // first query head of this tile within the group
    const int rows = min(16, G - q0);           // query heads of the tile
    int L = __ldg(p.seq_lens + b);
    L = min(L, p.max_pages * 16);
    const int npages = (L + 15) >> 4;
    const int pg0 = split * PPS;
    if (pg0 >= npages) continue;
    const int pg1 = min(npages, pg0 + PPS);

    // Q fragments (A operand, rows = query heads q0 .. q0 + rows - 1 of this KV head).
    uint32_t qa[KT][4];
    {
      const __nv_bfloat16* qb = reinterpret_cast<const __nv_bfloat16*>(p.q) +
                                (static_cast<size_t>(b) * p.Hq + (busy ? h * G + q0 : 0)) * D;
#pragma unroll
      for (int kt = 0; kt < KT; ++kt) {
        const int d0 = kt * 16 + 2 * c;
        qa[kt][0] = (busy && g < rows) ? *reinterpret_cast<const uint32_t*>(qb + g * D + d0) : 0u;
        qa[kt][1] = (busy && g + 8 < rows) ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d0) : 0u;
        qa[kt][2] = (busy && g < rows) ? *reinterpret_cast<const uint32_t*>(qb + g * D + d0 + 8) : 0u;
        qa[kt][3] = (busy && g + 8 < rows) ? *reinterpret_cast<const uint32_t*>(qb + (g + 8) * D + d0 + 8) : 0u;
      }
    }
    float o[NT][4];
#pragma unroll
    for (int n = 0; n < NT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows g and g + 8

    for (int pg = pg0; pg < pg1; ++pg, ++it) {
      const int s = it % kDecStages;
      const uint32_t ph = (it / kDecStages) & 1;
      bool ok = mbar_wait(&full[s], ph, abort_flag, p.status);
      if (__any_sync(0xffffffffu, !ok)) return;
      uint8_t* kp = smem + s * stage_bytes;
      uint8_t* vp = kp + page_bytes;
      const int rem = L - pg * 16;  // valid tokens in this page (>= 1)
      if (busy) {
        if (rem < 16) {
          // tokens past the end: zero their V rows so 0 * garbage cannot poison O
          for (int idx = lane; idx < DH * 16 * 8; idx += 32) {
            const int dh = idx / 128, t = (idx / 8) % 16, ch = idx % 8;
            if (t >= rem) *reinterpret_cast<uint4*>(vp + ((warp * DH + dh) * 16 + t) * 128 + ch * 16) = make_uint4(0, 0, 0, 0);
          }
          __syncwarp();
        }
        const uint32_t kbase = smem_u32(kp) + warp * DH * 16 * 128;
        const uint32_t vbase = smem_u32(vp) + warp * DH * 16 * 128;
        // S = Q K^T over 16 tokens (two n-tiles of 8 tokens)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mi = lane >> 3, r8 = lane & 7;  // ldmatrix: matrix index and row within it
#pragma unroll
        for (int kt = 0; kt < KT; ++kt) {
          // matrices: (tokens 0-7, dims lo), (tokens 0-7, dims hi), (tokens 8-15, lo), (8-15, hi)
          const int tok = (mi >> 1) * 8 + r8;
          const int dim = kt * 16 + (mi & 1) * 8;
          const int dh = dim >> 6, ch = (dim & 63) >> 3;
          const uint32_t addr = kbase + (dh * 16 + tok) * 128 + ((ch ^ (tok & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(addr, b0, b1, b2, b3);
          mma_bf16(sc[0], qa[kt], b0, b1);
          mma_bf16(sc[1], qa[kt], b2, b3);
        }
        // mask tokens past the end, scale into the log2 domain
        float v[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int tok = nt * 8 + 2 * c + (e & 1);
            v[nt][e] = tok < rem ? sc[nt][e] * sl2 : -INFINITY;
          }
        float mx0 = fmaxf(fmaxf(v[0][0], v[0][1]), fmaxf(v[1][0], v[1][1]));
        float mx1 = fmaxf(fmaxf(v[0][2], v[0][3]), fmaxf(v[1][2], v[1][3]));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float a0 = ex2_approx(m0 - n0), a1 = ex2_approx(m1 - n1);  // exp2(-inf) = 0 on the first page
        m0 = n0;
        m1 = n1;
        float pr[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          pr[nt][0] = ex2_approx(v[nt][0] - n0);
          pr[nt][1] = ex2_approx(v[nt][1] - n0);
          pr[nt][2] = ex2_approx(v[nt][2] - n1);
          pr[nt][3] = ex2_approx(v[nt][3] - n1);
        }
        l0 = l0 * a0 + pr[0][0] + pr[0][1] + pr[1][0] + pr[1][1];
        l1 = l1 * a1 + pr[0][2] + pr[0][3] + pr[1][2] + pr[1][3];
#pragma unroll
        for (int n = 0; n < NT; ++n) {
          o[n][0] *= a0;
          o[n][1] *= a0;
          o[n][2] *= a1;
          o[n][3] *= a1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16x2(pr[0][0], pr[0][1]);
        pa[1] = pack_bf16x2(pr[0][2], pr[0][3]);
        pa[2] = pack_bf16x2(pr[1][0], pr[1][1]);
        pa[3] = pack_bf16x2(pr[1][2], pr[1][3]);
        // O += P V: V is [token][dim]; transposed ldmatrix gives the B fragments
#pragma unroll
        for (int n2 = 0; n2 < NT / 2; ++n2) {
          // matrices: (tokens 0-7, dims 16n2..+7), (8-15, same), (0-7, 16n2+8..), (8-15, 16n2+8..)
          const int tok = (mi & 1) * 8 + r8;
          const int dim = n2 * 16 + (mi >> 1) * 8;
          const int dh = dim >> 6, ch = (dim & 63) >> 3;
          const uint32_t addr = vbase + (dh * 16 + tok) * 128 + ((ch ^ (tok & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(addr, b0, b1, b2, b3);
          mma_bf16(o[2 * n2], pa, b0, b1);
          mma_bf16(o[2 * n2 + 1], pa, b2, b3);
        }
        if (rem < 16) fence_proxy_async_smem();  // generic zero-writes before the next TMA into this slot
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }

    if (busy) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
      l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
      l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
      const size_t base = (static_cast<size_t>(b) * p.n_splits + split) * p.Hq + h * G + q0;
      const float i0 = 1.f / l0, i1 = 1.f / l1;
#pragma unroll
      for (int n = 0; n < NT; ++n) {
        const int dim = n * 8 + 2 * c;
        if (g < rows)
          *reinterpret_cast<float2*>(p.part_o + (base + g) * D + dim) = make_float2(o[n][0] * i0, o[n][1] * i0);
        if (g + 8 < rows)
          *reinterpret_cast<float2*>(p.part_o + (base + g + 8) * D + dim) = make_float2(o[n][2] * i1, o[n][3] * i1);
      }
      if (c == 0) {
        if (g < rows) p.part_lse[base + g] = (m0 + log2f(l0)) * 0.69314718055994531f;
        if (g + 8 < rows) p.part_lse[base + g + 8] = (m1 + log2f(l1)) * 0.69314718055994531f;
      }
    }
  }
}

template <int D>
static cudaError_t launch_decode_t(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                                   cudaStream_t stream) {
  const int smem = 1024 + kDecStages * 2 * 16 * p.HG * D * 2 + 2 * kDecStages * 8 + 16;
  auto kern = decode_kernel<D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long items = static_cast<long long>(p.B) * p.n_splits * p.n_hg * p.n_qt;
  const int grid = items < sms ? static_cast<int>(items) : sms;
  kern<<<grid, kDecThreads, smem, stream>>>(p, tmK, tmV);
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          cudaStream_t stream) {
  if (p.D == 128) return launch_decode_t<128>(p, tmK, tmV, stream);
  if (p.D == 64) return launch_decode_t<64>(p, tmK, tmV, stream);
  return cudaErrorInvalidValue;
}

}  // namespace attn
