// Paged decode without a caller-provided workspace.
//
// Some callers cannot allocate device memory at the point where they run
// decode: code that runs inside another framework's memory pool with
// allocation disabled, real-time paths where cudaMalloc's implicit device-wide
// synchronisation is not allowed, or embedders that only hand over buffers they
// own. For them the split partials and the status word live in one file-scope
// device array of fixed size, kept by every GPU that loads the library until the
// process exits. With CUDA's lazy module loading the array is reserved when this
// file's device code is first loaded on a device, i.e. by the first call here.
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/attn_b200.h"
#include "kernels.h"

namespace {

// ATTN_DECODE_NOALLOC_MAX_BYTES (32 MiB): enough for B * ceil(max_pages_per_seq / 32)
// * Hq * D fp32 partials plus their LSEs, e.g. 8 sequences of 32K tokens at Hq = 32, D = 128.
constexpr size_t kScratchBytes = ATTN_DECODE_NOALLOC_MAX_BYTES;
static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

namespace attn {
void set_last_error(const char* msg);  // api.cu
}

namespace {

// Device address of the array on the current device, looked up once per device with
// that device current (the array's name is only a host-side handle).
int scratch_for_current_device(void** out, const char* who) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    char buf[160];
    snprintf(buf, sizeof(buf), "%s: no usable current device", who);
    attn::set_last_error(buf);
    return ATTN_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    if (cudaGetSymbolAddress(&g_scratch_ptr[dev], g_decode_scratch) != cudaSuccess) {
      g_scratch_ptr[dev] = nullptr;
      char buf[160];
      snprintf(buf, sizeof(buf), "%s: cudaGetSymbolAddress failed", who);
      attn::set_last_error(buf);
      return ATTN_ERR_CUDA;
    }
  }
  *out = g_scratch_ptr[dev];
  return ATTN_OK;
}

}  // namespace

extern "C" {

int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                              const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int D,
                              int page_size, int max_pages_per_seq, int num_pages, float scale, int dtype,
                              void* stream) {
  const size_t need = attn_decode_paged_workspace_size(B, Hq, D, max_pages_per_seq, page_size);
  if (need > kScratchBytes) {
    char buf[256];
    snprintf(buf, sizeof(buf),
             "attn_decode_paged_noalloc: this problem needs %zu bytes of scratch, above the fixed %zu-byte "
             "array (use attn_decode_paged with a workspace)",
             need, kScratchBytes);
    attn::set_last_error(buf);
    return ATTN_ERR_WORKSPACE;
  }
  void* ptr = nullptr;
  const int rc = scratch_for_current_device(&ptr, "attn_decode_paged_noalloc");
  if (rc != ATTN_OK) return rc;
  // The existing entry point clears the status word at the start of the scratch;
  // the split partials are fully written before they are read, so nothing else
  // needs to start at zero.
  return attn_decode_paged(q, k_pages, v_pages, block_table, seq_lens, out, lse, B, Hq, Hkv, D, page_size,
                           max_pages_per_seq, num_pages, scale, dtype, ptr, kScratchBytes, stream);
}

int attn_decode_paged_noalloc_status(int* flags, void* stream) {
  if (!flags) {
    attn::set_last_error("attn_decode_paged_noalloc_status: null pointer argument");
    return ATTN_ERR_INVALID_ARG;
  }
  void* ptr = nullptr;
  const int rc = scratch_for_current_device(&ptr, "attn_decode_paged_noalloc_status");
  if (rc != ATTN_OK) return rc;
  return attn_read_status(ptr, flags, stream);
}

}  // extern "C"
