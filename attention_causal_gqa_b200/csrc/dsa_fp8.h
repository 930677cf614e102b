// Launch interface of the FP8 latent gather (dsa_fp8.cu) for the C-ABI layer.
#pragma once
#include <cstdint>
#include <cuda_runtime.h>

namespace attn {

// kv_codes [B, T_max, Dc] E4M3 with kv_scale [B, T_max, Dc / 128] (Dc = 512): the selected
// rows idx[b, i], i < n_sel[b] = min(seq_lens[b], top_k), dequantised into bf16 kv_sel
// [B, top_k, Dc]; the rotary rows copied into pe_sel [B, top_k, Dr]. An index outside
// [0, seq_lens[b]) is flagged and row 0 used.
cudaError_t launch_dsa_gather_fp8(const void* kv_codes, const float* kv_scale, const void* pe, const int32_t* idx,
                                  const int32_t* seq_lens, void* kv_sel, void* pe_sel, int32_t* n_sel, int B,
                                  int T_max, int top_k, int Dc, int Dr, int* status, cudaStream_t stream);

}  // namespace attn
