// Launch interfaces of the prologue kernels (RoPE operand preparation, KV-cache append
// and gather for chunked prefill) between the C-ABI layer and rope.cu / chunk.cu. Kept
// apart from kernels.h so the attention kernels do not depend on them.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace attn {

// RoPE prologue: cos/sin table of pos * freq_scale * theta^(-2i/D) (angles in fp64), then
// the operands. half_split: element d pairs with d + D/2 instead of 2i with 2i + 1.
cudaError_t launch_rope_table(float2* cs, int S, int D, double theta, double freq_scale, cudaStream_t stream);
// One launch rotating bf16 Q [q_heads, S, D] into q_op and K [k_heads, S, D] into k_op (fp16,
// or bf16 when bf16_out), computing each pair's cos/sin from its fp64 angle in the kernel.
cudaError_t launch_rope_qk(const void* q, void* q_op, long long q_heads, const void* k, void* k_op, long long k_heads,
                           int S, int D, double theta, double freq_scale, bool half_split, int* status,
                           cudaStream_t stream, bool bf16_out);
// fp32 X [rows, D] -> bf16 hi parts at out[0, rows) and lo parts at out[rows, 2 rows), rotating
// first when cs is non-null.
cudaError_t launch_split_f32(const float* x, void* out, const float2* cs, long long rows, int S, int D,
                             bool half_split, cudaStream_t stream);

// --------------------------------------------- chunked prefill into the paged cache
struct ChunkGeometry {
  const int32_t* cache_lens;   // [B] tokens already cached (new token i sits at cache_lens[b] + i)
  const int32_t* new_lens;     // [B] new tokens of each sequence (<= S_new), or nullptr (all S_new)
  const int32_t* block_table;  // [B, max_pages]
  int B, Hkv, S_new, D, page_size, max_pages, num_pages, max_cache_len;
  int half_split;              // RoPE pairs (i, i + D/2) instead of (2i, 2i + 1)
};
// rotate the new keys at their positions and write keys and values (bf16) into their pages
cudaError_t launch_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages, const float2* cs,
                             const ChunkGeometry& g, int* status, cudaStream_t stream);
// each sequence's cache into contiguous operands [B*Hkv, Sk_max, D]: keys fp16, values bf16, zeros past it
cudaError_t launch_kv_gather(const void* k_pages, const void* v_pages, void* k_op, void* v_op, const ChunkGeometry& g,
                             int Sk_max, int* status, cudaStream_t stream);
// new queries [B*Hq, S_new, D] rotated at their positions into fp16; rows past a sequence's
// chunk are written as zeros, and their LSE as -inf
cudaError_t launch_rope_rows_f16(const void* q, void* q_f16, const float2* cs, const ChunkGeometry& g, int Hq,
                                 float* lse, int* status, cudaStream_t stream);

}  // namespace attn
