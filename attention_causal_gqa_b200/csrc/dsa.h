// Launch interfaces of the DeepSeek sparse attention kernels (dsa.cu) for the C-ABI
// layer: lightning-indexer scores, top-k selection and the gather of the selected
// latent rows that the MLA decode kernel then attends.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace attn {

constexpr int kDevErrBadIndex = 16;  // a selected token index outside [0, seq_len) (ATTN_DEV_BAD_INDEX)
constexpr int kDsaIndexDim = 128;    // indexer query / key width
constexpr int kDsaMaxIndexHeads = 64;

struct DsaIndexParams {
  const void* q;            // [B, HI, 128] bf16 indexer queries
  const float* w;           // [B, HI] head weights
  const void* k;            // [B, T_max, 128] bf16 indexer keys
  const int32_t* seq_lens;  // [B]
  float* scores;            // [B, T_max] out: index scores, -inf past each length
  int B, HI, T_max;
  int* status;              // device status word (bounded waits)
};
// tmQ: 3-D bf16 map of q (d, head, b), box 64 x 64 x 1; tmK: 3-D bf16 map of k (d, token, b),
// box 64 x 128 x 1; both with 128-byte swizzle
cudaError_t launch_dsa_index(const DsaIndexParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK,
                             cudaStream_t stream);

// idx [B, top_k]: the min(top_k, L) best tokens in ascending order, -1 after them
cudaError_t launch_dsa_topk(const float* scores, const int32_t* seq_lens, int32_t* idx, int B, int T_max, int top_k,
                            cudaStream_t stream);

// kv_sel [B, top_k, Dc], pe_sel [B, top_k, Dr] (bf16): the rows idx[b, i] for i < n_sel[b] =
// min(seq_lens[b], top_k); an index outside [0, seq_lens[b]) is flagged and row 0 used.
cudaError_t launch_dsa_gather(const void* kv, const void* pe, const int32_t* idx, const int32_t* seq_lens,
                              void* kv_sel, void* pe_sel, int32_t* n_sel, int B, int T_max, int top_k, int Dc,
                              int Dr, int* status, cudaStream_t stream);

}  // namespace attn
