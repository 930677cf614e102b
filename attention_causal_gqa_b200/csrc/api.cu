// C-ABI layer: host-side validation, workspace carving, TMA tensor-map
// encoding and kernel launches. No allocation, no synchronisation on the hot calls.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "../../include/attn_b200.h"
#include "dsa.h"
#include "dsa_fp8.h"
#include "kernels.h"
#include "prologue.h"
#include "sm100.cuh"

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int ok() {
  g_last_error.clear();
  return ATTN_OK;
}

// One NVTX range per public call (named after the call), so a timeline tool shows the
// host-side span of each entry point around its kernels; free when no tool listens.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

int cuda_fail(cudaError_t e, const char* what) {
  return fail(ATTN_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr size_t kHeader = 256;  // status word lives at offset 0

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// Tiled tensor map (128-byte swizzle unless told otherwise); dims/strides innermost first, strides in bytes for dims 1..rank-1.
int make_map(CUtensorMap* m, CUtensorMapDataType dt, int rank, const void* base, const cuuint64_t* dims,
             const cuuint64_t* strides, const cuuint32_t* box, const char* what,
             CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(ATTN_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  CUresult r = fn(m, dt, static_cast<cuuint32_t>(rank), const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ATTN_ERR_CUDA, "tensor map encode failed for %s (CUresult %d)", what, (int)r);
  return ATTN_OK;
}

int clear_status(void* ws, cudaStream_t st) {
  cudaError_t e = cudaMemsetAsync(ws, 0, sizeof(int), st);
  if (e != cudaSuccess) return cuda_fail(e, "status clear");
  return ATTN_OK;
}

int decode_splits(int max_pages) {
  return (max_pages + attn::kDecodePagesPerSplit - 1) / attn::kDecodePagesPerSplit;
}

// ----------------------------------------------------------- timing hook
constexpr int kProfSlots = 4096;
struct Profiler {
  bool on = false;
  bool created = false;
  cudaEvent_t ev[2 * kProfSlots];
  int used = 0;
} g_prof;

void prof_before(cudaStream_t st) {
  if (g_prof.on && g_prof.used < kProfSlots) cudaEventRecord(g_prof.ev[2 * g_prof.used], st);
}
void prof_after(cudaStream_t st) {
  if (g_prof.on && g_prof.used < kProfSlots) {
    cudaEventRecord(g_prof.ev[2 * g_prof.used + 1], st);
    ++g_prof.used;
  }
}

}  // namespace

namespace attn {
void set_last_error(const char* msg) { g_last_error = msg; }

__global__ void selftest_wait_kernel(int* status, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // Nothing ever arrives on `bar`: the wait must give up by itself.
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&bar, 0)) {
      if (globaltimer_ns() - t0 > timeout_ns) {
        atomicOr(status, kDevErrTimeout);
        break;
      }
    }
  }
  __syncthreads();
}
// Evaluates the FMA-pipe exp2 of the softmax (exp2_fma2, sm100.cuh) on a caller buffer,
// two arguments per thread as the kernels use it.
__global__ void selftest_exp2_kernel(const float* __restrict__ z, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(z[i], i + 1 < n ? z[i + 1] : 0.f);
  const float2 r = exp2_fma2(in);
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
}
}  // namespace attn

extern "C" {

const char* attn_last_error(void) { return g_last_error.c_str(); }

// Prefill workspace: [status | cos/sin table | key operand | value operand]
//   bf16 input: key operand = rotated K in fp16 [B*Hkv, S, D]; no value operand.
//   fp32 input: key and value operands = bf16 hi parts then lo parts [2*B*Hkv, S, D] each.
size_t attn_prefill_workspace_size(int B, int Hkv, int S, int D, int dtype) {
  if (B <= 0 || Hkv <= 0 || S <= 0 || D <= 0) return kHeader;
  const size_t n = static_cast<size_t>(B) * Hkv * S * D;
  const size_t table = round_up(static_cast<size_t>(S) * (D / 2) * sizeof(float2), 256);
  if (dtype == ATTN_DTYPE_F32) return kHeader + table + 2 * round_up(2 * n * 2, 256);
  return kHeader + table + round_up(n * 2, 256);
}

int attn_prefill_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int S,
                    int D, int causal, float rope_theta, float rope_freq_scale, int rope_layout, float scale, int dtype,
                    void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("attn_prefill_ex");
  if (!q || !k || !v || !out || !lse || !workspace) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S <= 0 || D <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive (B=%d Hq=%d Hkv=%d S=%d D=%d)", B, Hq, Hkv, S, D);
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (dtype != ATTN_DTYPE_BF16 && dtype != ATTN_DTYPE_F32) return fail(ATTN_ERR_UNSUPPORTED, "dtype %d", dtype);
  const bool bf16_ops = (rope_layout & ATTN_ROPE_BF16_OPERANDS) != 0;
  rope_layout &= ~ATTN_ROPE_BF16_OPERANDS;
  if (rope_layout != ATTN_ROPE_INTERLEAVED && rope_layout != ATTN_ROPE_HALF_SPLIT)
    return fail(ATTN_ERR_INVALID_ARG, "rope_layout %d", rope_layout);
  if (!(rope_freq_scale > 0.f) || !std::isfinite(rope_freq_scale))
    return fail(ATTN_ERR_INVALID_ARG, "rope_freq_scale must be positive and finite");
  const bool half_split = rope_layout == ATTN_ROPE_HALF_SPLIT;
  const bool f32 = dtype == ATTN_DTYPE_F32;
  if (!(f32 ? D == 64 : (D == 64 || D == 128)))
    return fail(ATTN_ERR_UNSUPPORTED, "head dim %d unsupported for %s", D, f32 ? "fp32" : "bf16");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer (tensors 16 B, lse 4 B, workspace 256 B)");
  if (static_cast<long long>(B) * Hkv > (1LL << 30) || S > (1 << 24))
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  const size_t need = attn_prefill_workspace_size(B, Hkv, S, D, dtype);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale is not finite");
  if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  float2* cs = reinterpret_cast<float2*>(ws + kHeader);
  const size_t n = static_cast<size_t>(B) * Hkv * S * D;
  uint8_t* kop = ws + kHeader + round_up(static_cast<size_t>(S) * (D / 2) * sizeof(float2), 256);
  uint8_t* vop = kop + round_up(2 * n * 2, 256);  // fp32 input only
  int rc = clear_status(ws, st);
  if (rc) return rc;

  const bool rope = rope_theta > 0.f;
  if (rope && f32) {  // the fp32 operand split reads a cos/sin table
    cudaError_t e = attn::launch_rope_table(cs, S, D, static_cast<double>(rope_theta),
                                            static_cast<double>(rope_freq_scale), st);
    if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  }
  const long long rows = static_cast<long long>(B) * Hkv * S;
  const void* kbase = k;
  const void* vbase = v;
  CUtensorMapDataType kdt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t zdim = static_cast<cuuint64_t>(B) * Hkv;
  if (f32) {
    cudaError_t e =
        attn::launch_split_f32(static_cast<const float*>(k), kop, rope ? cs : nullptr, rows, S, D, half_split, st);
    if (e == cudaSuccess) e = attn::launch_split_f32(static_cast<const float*>(v), vop, nullptr, rows, S, D, false, st);
    if (e != cudaSuccess) return cuda_fail(e, "operand split launch");
    kbase = kop;
    vbase = vop;
    zdim *= 2;
  } else if (rope) {
    // one launch rotates K into the workspace and Q into `out` (see the Q operand below)
    cudaError_t e = attn::launch_rope_qk(q, out, static_cast<long long>(B) * Hq, k, kop, static_cast<long long>(B) * Hkv,
                                         S, D, static_cast<double>(rope_theta), static_cast<double>(rope_freq_scale),
                                         half_split, status, st, bf16_ops);
    if (e != cudaSuccess) return cuda_fail(e, "rope launch");
    kbase = kop;
    kdt = bf16_ops ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  }
  // Q operand. Without RoPE, bf16 Q is the operand itself. Otherwise the prologue
  // writes it into `out`, whose size is exactly that of the operand (rotated fp16 Q
  // for bf16 input; bf16 hi planes then lo planes for fp32 input). Every Q tile is
  // loaded and later overwritten by the same CTA, so the reuse is free of races.
  const long long rows_q = static_cast<long long>(B) * Hq * S;
  const void* qbase = q;
  CUtensorMapDataType qdt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  cuuint64_t zq = static_cast<cuuint64_t>(B) * Hq;
  if (f32) {
    cudaError_t e =
        attn::launch_split_f32(static_cast<const float*>(q), out, rope ? cs : nullptr, rows_q, S, D, half_split, st);
    if (e != cudaSuccess) return cuda_fail(e, "Q operand split launch");
    qbase = out;
    zq *= 2;
  } else if (rope) {  // rotated by the launch above
    qbase = out;
    qdt = bf16_ops ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  }
  const int BN = attn::prefill_block_n(D, f32);
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), zdim};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S) * D * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(BN), 1};
  const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S), zq};
  const cuuint32_t qbox[3] = {64, 128, 1};
  CUtensorMap tmQ, tmK, tmV;
  if ((rc = make_map(&tmQ, qdt, 3, qbase, qdims, strides, qbox, "Q"))) return rc;
  if ((rc = make_map(&tmK, kdt, 3, kbase, dims, strides, box, "K"))) return rc;
  if ((rc = make_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, vbase, dims, strides, box, "V"))) return rc;

  attn::PrefillParams p{};
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S;
  p.G = Hq / Hkv;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  p.n_row_blocks = (S + 127) / 128;
  p.status = status;
  const long long items = p.pair_heads ? static_cast<long long>(B) * (Hq / 2) * p.n_row_blocks
                                       : static_cast<long long>(B) * Hq * ((p.n_row_blocks + 1) / 2);
  if (items > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "too many work items");
  p.n_items = static_cast<int>(items);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = items < sms ? items : sms;  // one persistent CTA per SM
  prof_before(st);
  // rotated operands in fp16 select the f16 Q.K^T form of the kernel; bf16 ones the plain form
  cudaError_t e = attn::launch_prefill(p, tmQ, tmK, tmV, D, f32, rope && !bf16_ops, static_cast<int>(grid), st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "prefill launch");
  return ok();
}

int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int S,
                 int D, int causal, float rope_theta, float scale, int dtype, void* workspace, size_t workspace_bytes,
                 void* stream) {
  return attn_prefill_ex(q, k, v, out, lse, B, Hq, Hkv, S, D, causal, rope_theta, 1.0f, ATTN_ROPE_INTERLEAVED, scale,
                         dtype, workspace, workspace_bytes, stream);
}

// Chunked-prefill workspace: [status | cos/sin table [Sk_max, D/2] | keys fp16
// [B*Hkv, Sk_max, D] | values bf16 [B*Hkv, Sk_max, D]], Sk_max = max_cache_len + S_new.
size_t attn_prefill_chunk_workspace_size(int B, int Hkv, int S_new, int max_cache_len, int D) {
  if (B <= 0 || Hkv <= 0 || S_new <= 0 || D <= 0 || max_cache_len < 0) return kHeader;
  const size_t sk = static_cast<size_t>(max_cache_len) + S_new;
  const size_t table = round_up(sk * (D / 2) * sizeof(float2), 256);
  const size_t op = round_up(static_cast<size_t>(B) * Hkv * sk * D * 2, 256);
  return kHeader + table + 2 * op;
}

int attn_prefill_chunk_varlen(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                              const int32_t* block_table, const int32_t* cache_lens, const int32_t* new_lens, void* out,
                              float* lse, int B, int Hq, int Hkv, int S_new, int D, int page_size,
                              int max_pages_per_seq, int num_pages, int max_cache_len, float rope_theta,
                              float rope_freq_scale, int rope_layout, float scale, void* workspace,
                              size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("attn_prefill_chunk_varlen");
  if (!q || !k || !v || !k_pages || !v_pages || !block_table || !cache_lens || !out || !lse || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (new_lens && !aligned(new_lens, 4)) return fail(ATTN_ERR_INVALID_ARG, "misaligned new_lens");
  if (rope_layout != ATTN_ROPE_INTERLEAVED && rope_layout != ATTN_ROPE_HALF_SPLIT)
    return fail(ATTN_ERR_INVALID_ARG, "rope_layout %d", rope_layout);
  if (!(rope_freq_scale > 0.f) || !std::isfinite(rope_freq_scale))
    return fail(ATTN_ERR_INVALID_ARG, "rope_freq_scale must be positive and finite");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || S_new <= 0 || D <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 ||
      max_cache_len < 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive (B=%d Hq=%d Hkv=%d S_new=%d D=%d pages=%d/%d, max_cache_len=%d)",
                B, Hq, Hkv, S_new, D, max_pages_per_seq, num_pages, max_cache_len);
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d unsupported", D);
  if (page_size != 16) return fail(ATTN_ERR_UNSUPPORTED, "page size %d unsupported (16)", page_size);
  if (static_cast<long long>(max_cache_len) + S_new > static_cast<long long>(max_pages_per_seq) * page_size)
    return fail(ATTN_ERR_INVALID_ARG, "max_cache_len + S_new (%lld) exceeds the block table (%d pages)",
                static_cast<long long>(max_cache_len) + S_new, max_pages_per_seq);
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) ||
      !aligned(out, 16) || !aligned(lse, 4) || !aligned(block_table, 4) || !aligned(cache_lens, 4) ||
      !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer (tensors 16 B, lse/tables 4 B, workspace 256 B)");
  const long long rows_q = static_cast<long long>(B) * Hq * S_new;
  const long long sk = static_cast<long long>(max_cache_len) + S_new;
  if (rows_q * (D / 8) > 0x7fffffffLL || static_cast<long long>(B) * Hkv * S_new * (D / 8) > 0x7fffffffLL ||
      sk > (1 << 24))
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  const size_t need = attn_prefill_chunk_workspace_size(B, Hkv, S_new, max_cache_len, D);
  if (workspace_bytes < need) return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale is not finite");
  if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws);
  float2* cs = reinterpret_cast<float2*>(ws + kHeader);
  uint8_t* k_op = ws + kHeader + round_up(static_cast<size_t>(sk) * (D / 2) * sizeof(float2), 256);
  uint8_t* v_op = k_op + round_up(static_cast<size_t>(B) * Hkv * sk * D * 2, 256);
  int rc = clear_status(ws, st);
  if (rc) return rc;
  const bool rope = rope_theta > 0.f;
  if (rope) {
    cudaError_t e = attn::launch_rope_table(cs, static_cast<int>(sk), D, static_cast<double>(rope_theta),
                                            static_cast<double>(rope_freq_scale), st);
    if (e != cudaSuccess) return cuda_fail(e, "rope table launch");
  }
  attn::ChunkGeometry g{cache_lens, new_lens, block_table, B, Hkv, S_new, D, page_size, max_pages_per_seq,
                        num_pages, max_cache_len, rope_layout == ATTN_ROPE_HALF_SPLIT ? 1 : 0};
  const float2* rcs = rope ? cs : nullptr;
  cudaError_t e = attn::launch_kv_append(k, v, k_pages, v_pages, rcs, g, status, st);
  if (e == cudaSuccess) e = attn::launch_kv_gather(k_pages, v_pages, k_op, v_op, g, static_cast<int>(sk), status, st);
  // the prepared Q operand goes into `out` (same byte size; each tile is loaded and
  // later overwritten by the same CTA)
  if (e == cudaSuccess) e = attn::launch_rope_rows_f16(q, out, rcs, g, Hq, lse, status, st);
  if (e != cudaSuccess) return cuda_fail(e, "chunk operand launch");

  const int BN = attn::prefill_block_n(D, false);
  const cuuint64_t qdims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(S_new),
                               static_cast<cuuint64_t>(B) * Hq};
  const cuuint64_t qstr[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(S_new) * D * 2};
  const cuuint64_t kdims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(sk), static_cast<cuuint64_t>(B) * Hkv};
  const cuuint64_t kstr[2] = {static_cast<cuuint64_t>(D) * 2, static_cast<cuuint64_t>(sk) * D * 2};
  const cuuint32_t qbox[3] = {64, 128, 1};
  const cuuint32_t kbox[3] = {64, static_cast<cuuint32_t>(BN), 1};
  CUtensorMap tmQ, tmK, tmV;
  if ((rc = make_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, out, qdims, qstr, qbox, "Q"))) return rc;
  if ((rc = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, k_op, kdims, kstr, kbox, "K"))) return rc;
  if ((rc = make_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, v_op, kdims, kstr, kbox, "V"))) return rc;

  attn::PrefillParams p{};
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.S = S_new;
  p.G = Hq / Hkv;
  p.causal = 1;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.pair_heads = (p.G % 2 == 0) ? 1 : 0;
  p.n_row_blocks = (S_new + 127) / 128;
  p.status = status;
  p.q_off = cache_lens;
  p.max_off = max_cache_len;
  p.q_len = new_lens;
  const long long items = p.pair_heads ? static_cast<long long>(B) * (Hq / 2) * p.n_row_blocks
                                       : static_cast<long long>(B) * Hq * ((p.n_row_blocks + 1) / 2);
  if (items > 0x7fffffffLL) return fail(ATTN_ERR_UNSUPPORTED, "too many work items");
  p.n_items = static_cast<int>(items);
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long grid = items < sms ? items : sms;
  prof_before(st);
  e = attn::launch_prefill(p, tmQ, tmK, tmV, D, false, true, static_cast<int>(grid), st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "chunk prefill launch");
  return ok();
}

int attn_prefill_chunk_ex(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                          const int32_t* block_table, const int32_t* cache_lens, void* out, float* lse, int B, int Hq,
                          int Hkv, int S_new, int D, int page_size, int max_pages_per_seq, int num_pages,
                          int max_cache_len, float rope_theta, float rope_freq_scale, int rope_layout, float scale,
                          void* workspace, size_t workspace_bytes, void* stream) {
  return attn_prefill_chunk_varlen(q, k, v, k_pages, v_pages, block_table, cache_lens, nullptr, out, lse, B, Hq, Hkv,
                                   S_new, D, page_size, max_pages_per_seq, num_pages, max_cache_len, rope_theta,
                                   rope_freq_scale, rope_layout, scale, workspace, workspace_bytes, stream);
}

int attn_prefill_chunk(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                       const int32_t* block_table, const int32_t* cache_lens, void* out, float* lse, int B, int Hq,
                       int Hkv, int S_new, int D, int page_size, int max_pages_per_seq, int num_pages,
                       int max_cache_len, float rope_theta, float scale, void* workspace, size_t workspace_bytes,
                       void* stream) {
  return attn_prefill_chunk_ex(q, k, v, k_pages, v_pages, block_table, cache_lens, out, lse, B, Hq, Hkv, S_new, D,
                               page_size, max_pages_per_seq, num_pages, max_cache_len, rope_theta, 1.0f,
                               ATTN_ROPE_INTERLEAVED, scale, workspace, workspace_bytes, stream);
}

size_t attn_decode_paged_workspace_size(int B, int Hq, int D, int max_pages_per_seq, int page_size) {
  (void)page_size;
  if (B <= 0 || Hq <= 0 || D <= 0 || max_pages_per_seq <= 0) return kHeader;
  const size_t ns = decode_splits(max_pages_per_seq);
  return kHeader + round_up(static_cast<size_t>(B) * ns * Hq * D * sizeof(float), 256) +
         round_up(static_cast<size_t>(B) * ns * Hq * sizeof(float), 256);
}

int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int D, int page_size,
                      int max_pages_per_seq, int num_pages, float scale, int dtype, void* workspace,
                      size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("attn_decode_paged");
  if (!q || !k_pages || !v_pages || !block_table || !seq_lens || !out || !lse || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || page_size <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive");
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (dtype != ATTN_DTYPE_BF16) return fail(ATTN_ERR_UNSUPPORTED, "paged decode supports bf16 only");
  if (page_size != 16) return fail(ATTN_ERR_UNSUPPORTED, "page_size %d (only 16)", page_size);
  if (D != 64 && D != 128) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d", D);
  if (Hq > 4096 || B > (1 << 20)) return fail(ATTN_ERR_UNSUPPORTED, "problem too large (Hq %d, B %d)", Hq, B);
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
      !aligned(block_table, 4) || !aligned(seq_lens, 4) || !aligned(lse, 4) || !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  const size_t need = attn_decode_paged_workspace_size(B, Hq, D, max_pages_per_seq, page_size);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale is not finite");
  if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const int ns = decode_splits(max_pages_per_seq);
  float* part_o = reinterpret_cast<float*>(ws + kHeader);
  float* part_lse =
      reinterpret_cast<float*>(ws + kHeader + round_up(static_cast<size_t>(B) * ns * Hq * D * sizeof(float), 256));
  int rc = clear_status(ws, st);
  if (rc) return rc;

  // 5-D view of a page pool [num_pages][16][Hkv][D]: (d%64, token, d/64, head, page);
  // its shared-memory image is [head][d/64][token][64].
  const cuuint64_t row = static_cast<cuuint64_t>(Hkv) * D * 2;
  const cuuint64_t dims[5] = {64, 16, static_cast<cuuint64_t>(D / 64), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[4] = {row, 128, static_cast<cuuint64_t>(D) * 2, 16 * row};
  // one box holds up to 8 KV heads of a page (a head group); a group past Hkv reads zeros
  const int HG = Hkv < 8 ? Hkv : 8;
  const cuuint32_t box[5] = {64, 16, static_cast<cuuint32_t>(D / 64), static_cast<cuuint32_t>(HG), 1};
  CUtensorMap tmK, tmV;
  if ((rc = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, k_pages, dims, strides, box, "k_pages"))) return rc;
  if ((rc = make_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, v_pages, dims, strides, box, "v_pages"))) return rc;

  attn::DecodeParams p{};
  p.q = q;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.G = Hq / Hkv;
  p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages;
  p.n_splits = ns;
  p.HG = HG;
  p.n_hg = (Hkv + 7) / 8;
  p.n_qt = (Hq / Hkv + 15) / 16;
  if (static_cast<long long>(B) * ns * p.n_hg * p.n_qt > 0x7fffffffLL)
    return fail(ATTN_ERR_UNSUPPORTED, "too many decode work items");
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = reinterpret_cast<int*>(ws);
  prof_before(st);
  cudaError_t e = attn::launch_decode(p, tmK, tmV, st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = attn::launch_merge(part_o, part_lse, seq_lens, out, lse, B, Hq, D, ns, attn::kDecodePagesPerSplit * 16, st);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

size_t attn_decode_paged_fp8_workspace_size(int B, int Hq, int D, int max_pages_per_seq, int page_size) {
  (void)page_size;
  (void)max_pages_per_seq;
  if (B <= 0 || Hq <= 0 || D <= 0) return kHeader;
  const size_t slots = static_cast<size_t>(attn::kDecodeFp8MaxRanges) + B;  // range c, sequence b: slot c + b
  return kHeader + round_up(slots * Hq * D * sizeof(float), 256) + round_up(slots * Hq * sizeof(float), 256);
}

int attn_decode_paged_fp8(const void* q, const void* k_pages, const void* v_pages, const float* k_scale,
                          const float* v_scale, const int32_t* block_table, const int32_t* seq_lens, void* out,
                          float* lse, int B, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                          int num_pages, float scale, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("attn_decode_paged_fp8");
  if (!q || !k_pages || !v_pages || !k_scale || !v_scale || !block_table || !seq_lens || !out || !lse || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || page_size <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive");
  if (Hq % Hkv != 0) return fail(ATTN_ERR_INVALID_ARG, "Hq (%d) must be a multiple of Hkv (%d)", Hq, Hkv);
  if (page_size != 16) return fail(ATTN_ERR_UNSUPPORTED, "page_size %d (only 16)", page_size);
  if (D != 128 && D != 64) return fail(ATTN_ERR_UNSUPPORTED, "head dim %d (the FP8 cache supports 64 and 128)", D);
  if (Hkv > 8) return fail(ATTN_ERR_UNSUPPORTED, "Hkv %d > 8", Hkv);
  if (Hq / Hkv > 16) return fail(ATTN_ERR_UNSUPPORTED, "group size %d > 16", Hq / Hkv);
  if (!aligned(q, 16) || !aligned(k_pages, 16) || !aligned(v_pages, 16) || !aligned(out, 16) ||
      !aligned(k_scale, 4) || !aligned(v_scale, 4) || !aligned(block_table, 4) || !aligned(seq_lens, 4) ||
      !aligned(lse, 4) || !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  const size_t need = attn_decode_paged_fp8_workspace_size(B, Hq, D, max_pages_per_seq, page_size);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  if (!std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale is not finite");
  if (scale <= 0.f) scale = 1.0f / std::sqrt(static_cast<float>(D));

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t slots = static_cast<size_t>(attn::kDecodeFp8MaxRanges) + B;
  float* part_o = reinterpret_cast<float*>(ws + kHeader);
  float* part_lse = reinterpret_cast<float*>(ws + kHeader + round_up(slots * Hq * D * sizeof(float), 256));
  int rc = clear_status(ws, st);
  if (rc) return rc;

  // 4-D view of a page pool of codes [num_pages][16][Hkv][D]: (d, token, head, page);
  // its shared-memory image is [head][token][D bytes].
  const cuuint64_t row = static_cast<cuuint64_t>(Hkv) * D;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), 16, static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(num_pages)};
  const cuuint64_t strides[3] = {row, static_cast<cuuint64_t>(D), 16 * row};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(D), 16, static_cast<cuuint32_t>(Hkv), 1};
  CUtensorMap tmK, tmV;
  // 128-byte rows (D = 128) under the 128-byte swizzle, 64-byte rows (D = 64) under the 64-byte one
  const CUtensorMapSwizzle swz = D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  if ((rc = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, k_pages, dims, strides, box, "k_pages", swz))) return rc;
  if ((rc = make_map(&tmV, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, v_pages, dims, strides, box, "v_pages", swz))) return rc;

  attn::DecodeParams p{};
  p.q = q;
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.out = out;
  p.lse = lse;
  p.B = B;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.D = D;
  p.G = Hq / Hkv;
  p.max_pages = max_pages_per_seq;
  p.num_pages = num_pages;
  p.n_splits = 0;  // ranges, not fixed splits
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = reinterpret_cast<int*>(ws);
  p.k_scale = k_scale;
  p.v_scale = v_scale;
  prof_before(st);
  int n_ranges = 0;
  cudaError_t e = attn::launch_decode_fp8(p, tmK, tmV, &n_ranges, st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "decode launch");
  e = attn::launch_decode_range_merge(part_o, part_lse, seq_lens, out, lse, B, Hq, D, max_pages_per_seq * 16,
                                      n_ranges, st);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

// MLA workspace: [status | partial outputs (n_pairs + B) x H x Dc fp32 | partial LSE (n_pairs + B) x H]
size_t mla_decode_workspace_size(int B, int H, int Dc, int Dr, int T_max) {
  (void)Dr;
  (void)T_max;
  if (B <= 0 || H <= 0 || Dc <= 0) return kHeader;
  const size_t slots = static_cast<size_t>(attn::kMlaMaxPairs) + B;
  return kHeader + round_up(slots * H * Dc * sizeof(float), 256) + round_up(slots * H * sizeof(float), 256);
}

// The MLA decode launches after validation: partials at `parts` (the workspace past its
// header), device flags into `status`.
static int mla_run(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                   const int32_t* seq_lens, float scale, void* out, float* lse, int B, int H, int Dc, int Dr,
                   int T_max, uint8_t* parts, int* status, cudaStream_t st) {
  // the kernel's work split counts positions (tiles plus a per-sequence weight) in 32 bits
  const long long positions =
      static_cast<long long>(B) * ((T_max + attn::kMlaTile - 1) / attn::kMlaTile + attn::kMlaSegCost);
  if (positions >= (1ll << 31)) return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  const size_t slots = static_cast<size_t>(attn::kMlaMaxPairs) + B;
  float* part_o = reinterpret_cast<float*>(parts);
  float* part_lse = reinterpret_cast<float*>(parts + round_up(slots * H * Dc * sizeof(float), 256));
  int rc = ATTN_OK;

  CUtensorMap tmKV, tmPE;
  {
    const cuuint64_t d[3] = {static_cast<cuuint64_t>(Dc), static_cast<cuuint64_t>(T_max), static_cast<cuuint64_t>(B)};
    const cuuint64_t s[2] = {static_cast<cuuint64_t>(Dc) * 2, static_cast<cuuint64_t>(T_max) * Dc * 2};
    const cuuint32_t bx[3] = {64, static_cast<cuuint32_t>(attn::kMlaTile), 1};
    if ((rc = make_map(&tmKV, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, kv_cache, d, s, bx, "kv_cache"))) return rc;
  }
  {
    const cuuint64_t d[3] = {static_cast<cuuint64_t>(Dr), static_cast<cuuint64_t>(T_max), static_cast<cuuint64_t>(B)};
    const cuuint64_t s[2] = {static_cast<cuuint64_t>(Dr) * 2, static_cast<cuuint64_t>(T_max) * Dr * 2};
    // each CTA of a cluster loads its 32 of the 64 rotary columns: 64-byte rows, 64-byte swizzle
    const cuuint32_t bx[3] = {32, static_cast<cuuint32_t>(attn::kMlaTile), 1};
    if ((rc = make_map(&tmPE, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pe_cache, d, s, bx, "pe_cache",
                       CU_TENSOR_MAP_SWIZZLE_64B)))
      return rc;
  }
  attn::MlaParams p{};
  p.q_nope = q_nope;
  p.q_pe = q_pe;
  p.seq_lens = seq_lens;
  p.part_o = part_o;
  p.part_lse = part_lse;
  p.B = B;
  p.H = H;
  p.Dc = Dc;
  p.Dr = Dr;
  p.T_max = T_max;
  p.n_pairs = attn::mla_pairs_for_device();
  p.scale_log2 = scale * 1.4426950408889634f;
  p.status = status;
  prof_before(st);
  cudaError_t e = attn::launch_mla(p, tmKV, tmPE, st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "mla launch");
  e = attn::launch_mla_merge(part_o, part_lse, seq_lens, out, lse, B, H, T_max, p.n_pairs, st);
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

int mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
               const int32_t* seq_lens, float scale, void* out, float* lse, int B, int H, int Dc, int Dr, int T_max,
               void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("mla_decode");
  if (!q_nope || !q_pe || !kv_cache || !pe_cache || !seq_lens || !out || !lse || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || H <= 0 || Dc <= 0 || Dr <= 0 || T_max <= 0) return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive");
  if (H != 128 || Dc != 512 || Dr != 64)
    return fail(ATTN_ERR_UNSUPPORTED, "MLA decode supports H=128, Dc=512, Dr=64 (got %d, %d, %d)", H, Dc, Dr);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be positive");
  if (!aligned(q_nope, 16) || !aligned(q_pe, 16) || !aligned(kv_cache, 16) || !aligned(pe_cache, 16) ||
      !aligned(out, 16) || !aligned(seq_lens, 4) || !aligned(lse, 4) || !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  if (T_max > (1 << 26) || B > (1 << 20)) return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  const size_t need = mla_decode_workspace_size(B, H, Dc, Dr, T_max);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);

  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int rc = clear_status(ws, st);
  if (rc) return rc;
  return mla_run(q_nope, q_pe, kv_cache, pe_cache, seq_lens, scale, out, lse, B, H, Dc, Dr, T_max, ws + kHeader,
                 reinterpret_cast<int*>(ws), st);
}

// ------------------------------------------------ DeepSeek sparse attention
size_t dsa_index_topk_workspace_size(int B, int H_I, int d_I, int T_max, int top_k) {
  (void)B;
  (void)H_I;
  (void)d_I;
  (void)T_max;
  (void)top_k;
  return kHeader;  // the status word only
}

int dsa_index_topk(const void* q_idx, const float* w_idx, const void* k_idx, const int32_t* seq_lens, float* scores,
                   int32_t* topk_idx, int B, int H_I, int d_I, int T_max, int top_k, void* workspace,
                   size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("dsa_index_topk");
  if (!q_idx || !w_idx || !k_idx || !seq_lens || !scores || !topk_idx || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || H_I <= 0 || d_I <= 0 || T_max <= 0 || top_k <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive");
  if (d_I != attn::kDsaIndexDim) return fail(ATTN_ERR_UNSUPPORTED, "indexer width %d (supported: 128)", d_I);
  if (H_I % 16 != 0 || H_I > attn::kDsaMaxIndexHeads)
    return fail(ATTN_ERR_UNSUPPORTED, "indexer heads %d (supported: multiples of 16 up to 64)", H_I);
  if (T_max > (1 << 26) || B > 65535 || top_k > (1 << 26)) return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  if (!aligned(q_idx, 16) || !aligned(k_idx, 16) || !aligned(w_idx, 4) || !aligned(seq_lens, 4) ||
      !aligned(scores, 4) || !aligned(topk_idx, 4) || !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  const size_t need = dsa_index_topk_workspace_size(B, H_I, d_I, T_max, top_k);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = clear_status(workspace, st);
  if (rc) return rc;
  // q as (d, head, b) and k as (d, token, b), 64-column boxes with 128-byte swizzle; the Q box
  // is 64 heads high (rows past H_I read as zeros)
  CUtensorMap tmQ, tmK;
  {
    const cuuint64_t d[3] = {static_cast<cuuint64_t>(d_I), static_cast<cuuint64_t>(H_I), static_cast<cuuint64_t>(B)};
    const cuuint64_t s[2] = {static_cast<cuuint64_t>(d_I) * 2, static_cast<cuuint64_t>(H_I) * d_I * 2};
    const cuuint32_t bx[3] = {64, 64, 1};
    if ((rc = make_map(&tmQ, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, q_idx, d, s, bx, "q_idx"))) return rc;
  }
  {
    const cuuint64_t d[3] = {static_cast<cuuint64_t>(d_I), static_cast<cuuint64_t>(T_max),
                             static_cast<cuuint64_t>(B)};
    const cuuint64_t s[2] = {static_cast<cuuint64_t>(d_I) * 2, static_cast<cuuint64_t>(T_max) * d_I * 2};
    const cuuint32_t bx[3] = {64, 128, 1};
    if ((rc = make_map(&tmK, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, k_idx, d, s, bx, "k_idx"))) return rc;
  }
  attn::DsaIndexParams p{};
  p.q = q_idx;
  p.w = w_idx;
  p.k = k_idx;
  p.seq_lens = seq_lens;
  p.scores = scores;
  p.B = B;
  p.HI = H_I;
  p.T_max = T_max;
  p.status = static_cast<int*>(workspace);
  prof_before(st);
  cudaError_t e = attn::launch_dsa_index(p, tmQ, tmK, st);
  prof_after(st);
  if (e != cudaSuccess) return cuda_fail(e, "indexer launch");
  e = attn::launch_dsa_topk(scores, seq_lens, topk_idx, B, T_max, top_k, st);
  if (e != cudaSuccess) return cuda_fail(e, "top-k launch");
  return ok();
}

// workspace: [status | MLA partials | kv_sel B x top_k x Dc | pe_sel B x top_k x Dr | n_sel B]
size_t dsa_mla_decode_workspace_size(int B, int H, int Dc, int Dr, int top_k) {
  if (B <= 0 || H <= 0 || Dc <= 0 || Dr <= 0 || top_k <= 0) return kHeader;
  const size_t mla = mla_decode_workspace_size(B, H, Dc, Dr, top_k);
  const size_t rows = static_cast<size_t>(B) * top_k;
  return mla + round_up(rows * Dc * 2, 256) + round_up(rows * Dr * 2, 256) + round_up(static_cast<size_t>(B) * 4, 256);
}

// Shared by both sparse MLA entry points: the argument checks, the workspace layout
// [MLA workspace | selected latent rows bf16 | selected rotary rows bf16 | counts] and,
// after the gather `gather(kv_sel, pe_sel, n_sel, status, stream)` has filled the
// selected rows, the MLA decode over them (T_max = top_k).
extern "C++" {
template <typename Gather>
static int dsa_mla_run(const void* q_nope, const void* q_pe, const void* latent, const void* pe_cache,
                       const int32_t* seq_lens, const int32_t* topk_idx, int top_k, float scale, void* out, float* lse,
                       int B, int H, int Dc, int Dr, int T_max, void* workspace, size_t workspace_bytes, void* stream,
                       Gather&& gather) {
  if (!q_nope || !q_pe || !latent || !pe_cache || !seq_lens || !topk_idx || !out || !lse || !workspace)
    return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (B <= 0 || H <= 0 || Dc <= 0 || Dr <= 0 || T_max <= 0 || top_k <= 0)
    return fail(ATTN_ERR_INVALID_ARG, "sizes must be positive");
  if (H != 128 || Dc != 512 || Dr != 64)
    return fail(ATTN_ERR_UNSUPPORTED, "MLA decode supports H=128, Dc=512, Dr=64 (got %d, %d, %d)", H, Dc, Dr);
  if (!(scale > 0.f) || !std::isfinite(scale)) return fail(ATTN_ERR_INVALID_ARG, "scale must be positive");
  if (!aligned(q_nope, 16) || !aligned(q_pe, 16) || !aligned(latent, 16) || !aligned(pe_cache, 16) ||
      !aligned(out, 16) || !aligned(seq_lens, 4) || !aligned(topk_idx, 4) || !aligned(lse, 4) ||
      !aligned(workspace, 256))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  if (T_max > (1 << 26) || B > (1 << 20) || top_k > (1 << 26) || static_cast<long long>(B) * top_k > (1LL << 30))
    return fail(ATTN_ERR_UNSUPPORTED, "problem too large");
  const size_t need = dsa_mla_decode_workspace_size(B, H, Dc, Dr, top_k);
  if (workspace_bytes < need)
    return fail(ATTN_ERR_WORKSPACE, "workspace %zu bytes < required %zu", workspace_bytes, need);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t rows = static_cast<size_t>(B) * top_k;
  uint8_t* kv_sel = ws + mla_decode_workspace_size(B, H, Dc, Dr, top_k);
  uint8_t* pe_sel = kv_sel + round_up(rows * Dc * 2, 256);
  int32_t* n_sel = reinterpret_cast<int32_t*>(pe_sel + round_up(rows * Dr * 2, 256));
  int* status = reinterpret_cast<int*>(ws);
  int rc = clear_status(ws, st);
  if (rc) return rc;
  cudaError_t e = gather(kv_sel, pe_sel, n_sel, status, st);
  if (e != cudaSuccess) return cuda_fail(e, "gather launch");
  return mla_run(q_nope, q_pe, kv_sel, pe_sel, n_sel, scale, out, lse, B, H, Dc, Dr, top_k, ws + kHeader, status, st);
}
}  // extern "C++"

int dsa_mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                   const int32_t* seq_lens, const int32_t* topk_idx, int top_k, float scale, void* out, float* lse,
                   int B, int H, int Dc, int Dr, int T_max, void* workspace, size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("dsa_mla_decode");
  return dsa_mla_run(q_nope, q_pe, kv_cache, pe_cache, seq_lens, topk_idx, top_k, scale, out, lse, B, H, Dc, Dr, T_max,
                     workspace, workspace_bytes, stream,
                     [&](void* kv_sel, void* pe_sel, int32_t* n_sel, int* status, cudaStream_t st) {
                       return attn::launch_dsa_gather(kv_cache, pe_cache, topk_idx, seq_lens, kv_sel, pe_sel, n_sel, B,
                                                      T_max, top_k, Dc, Dr, status, st);
                     });
}

int dsa_mla_decode_fp8(const void* q_nope, const void* q_pe, const void* kv_codes, const float* kv_scale,
                       const void* pe_cache, const int32_t* seq_lens, const int32_t* topk_idx, int top_k, float scale,
                       void* out, float* lse, int B, int H, int Dc, int Dr, int T_max, void* workspace,
                       size_t workspace_bytes, void* stream) {
  NvtxRange nvtx_range("dsa_mla_decode_fp8");
  if (!kv_scale) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (!aligned(kv_scale, 4)) return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer");
  return dsa_mla_run(q_nope, q_pe, kv_codes, pe_cache, seq_lens, topk_idx, top_k, scale, out, lse, B, H, Dc, Dr, T_max,
                     workspace, workspace_bytes, stream,
                     [&](void* kv_sel, void* pe_sel, int32_t* n_sel, int* status, cudaStream_t st) {
                       return attn::launch_dsa_gather_fp8(kv_codes, kv_scale, pe_cache, topk_idx, seq_lens, kv_sel,
                                                          pe_sel, n_sel, B, T_max, top_k, Dc, Dr, status, st);
                     });
}

int attn_read_status(const void* workspace, int* flags, void* stream) {
  if (!workspace || !flags) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "stream synchronize");
  int v = 0;
  e = cudaMemcpy(&v, workspace, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status copy");
  *flags = v;
  if (v) return fail(ATTN_ERR_DEVICE, "device status flags 0x%x", v);
  return ok();
}

int attn_lse_merge(const void* o_parts, const float* lse_parts, int n_parts, long long rows, int D, void* out,
                   float* lse, void* stream) {
  NvtxRange nvtx_range("attn_lse_merge");
  if (!o_parts || !lse_parts || !out || !lse) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (n_parts < 1 || n_parts > (1 << 16) || rows < 1 || rows > (1LL << 36))
    return fail(ATTN_ERR_INVALID_ARG, "n_parts (%d) or rows (%lld) out of range", n_parts, rows);
  if (D != 64 && D != 128 && D != 256 && D != 512)
    return fail(ATTN_ERR_UNSUPPORTED, "head dim %d (64, 128, 256 or 512)", D);
  if (!aligned(o_parts, 4) || !aligned(out, 4) || !aligned(lse_parts, 4) || !aligned(lse, 4))
    return fail(ATTN_ERR_INVALID_ARG, "misaligned pointer (4 bytes)");
  cudaError_t e =
      attn::launch_parts_merge(o_parts, lse_parts, n_parts, rows, D, out, lse, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "merge launch");
  return ok();
}

double attn_rope_ntk_theta(double theta, double scale, int head_dim) {
  if (!(theta > 0.0) || !std::isfinite(theta) || !(scale >= 1.0) || !std::isfinite(scale) || head_dim < 4 ||
      head_dim % 2 != 0) {
    fail(ATTN_ERR_INVALID_ARG, "attn_rope_ntk_theta: theta > 0, scale >= 1 and an even head_dim >= 4 are required");
    return 0.0;
  }
  // the lowest rotary frequency theta^(-(D-2)/D) divided by `scale`, the highest (pair 0) unchanged
  const double r = theta * std::pow(scale, static_cast<double>(head_dim) / (head_dim - 2.0));
  if (!std::isfinite(r)) {
    fail(ATTN_ERR_INVALID_ARG, "attn_rope_ntk_theta: result overflows");
    return 0.0;
  }
  ok();
  return r;
}

double attn_rope_length_scaled_theta(double theta, int length, int base_length, double alpha) {
  if (!(theta > 0.0) || !std::isfinite(theta) || length <= 0 || base_length <= 0 || !std::isfinite(alpha)) {
    fail(ATTN_ERR_INVALID_ARG,
         "attn_rope_length_scaled_theta: theta > 0, positive lengths and a finite alpha are required");
    return 0.0;
  }
  const double r = theta * std::pow(static_cast<double>(length) / base_length, alpha);
  if (!(r > 0.0) || !std::isfinite(r)) {
    fail(ATTN_ERR_INVALID_ARG, "attn_rope_length_scaled_theta: result out of range");
    return 0.0;
  }
  ok();
  return r;
}

int attn_selftest_exp2(const float* z, float* y, int n, void* stream) {
  if (!z || !y) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (n <= 0 || n > (1 << 30)) return fail(ATTN_ERR_INVALID_ARG, "n must be within 1 .. 2^30");
  const int pairs = (n + 1) / 2;
  attn::selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(z, y, n);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

int attn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned long long timeout_ns,
                               void* stream) {
  if (!workspace) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  if (workspace_bytes < kHeader) return fail(ATTN_ERR_WORKSPACE, "workspace must hold at least 256 bytes");
  if (timeout_ns < 1000ull || timeout_ns > 10000000000ull)
    return fail(ATTN_ERR_INVALID_ARG, "timeout must be within 1e3 .. 1e10 ns");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int rc = clear_status(workspace, st);
  if (rc) return rc;
  attn::selftest_wait_kernel<<<1, 32, 0, st>>>(static_cast<int*>(workspace), timeout_ns);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, "selftest launch");
  return ok();
}

int attn_profile_enable(int on) {
  if (on && !g_prof.created) {
    for (int i = 0; i < 2 * kProfSlots; ++i) {
      cudaError_t e = cudaEventCreate(&g_prof.ev[i]);
      if (e != cudaSuccess) return cuda_fail(e, "event create");
    }
    g_prof.created = true;
  }
  g_prof.on = on != 0;
  g_prof.used = 0;
  return ok();
}

int attn_profile_collect(double* total_ms, int* count) {
  if (!total_ms || !count) return fail(ATTN_ERR_INVALID_ARG, "null pointer argument");
  double tot = 0.0;
  for (int i = 0; i < g_prof.used; ++i) {
    cudaError_t e = cudaEventSynchronize(g_prof.ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "event synchronize");
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]);
    if (e != cudaSuccess) return cuda_fail(e, "event elapsed");
    tot += ms;
  }
  *total_ms = tot;
  *count = g_prof.used;
  g_prof.used = 0;
  return ok();
}

}  // extern "C"
