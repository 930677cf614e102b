// Launch interfaces between the C-ABI layer (api.cu) and the kernels.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <utility>

namespace attn {

// Launches kernel with programmatic dependent launch allowed: its launch overlaps the end
// of the previous kernel on the stream, so every kernel launched this way calls
// griddep_wait() before its first memory access. No kernel here triggers its dependents
// early: a dependent is scheduled only once every CTA of its predecessor has exited, so
// it can never hold resources that a not-yet-running CTA of the predecessor needs.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct PrefillParams {
  void* out;              // [B, Hq, S, D] (T)
  float* lse;             // [B, Hq, S]
  int B, Hq, Hkv, S, G;
  int causal;
  float scale_log2;       // scale * log2(e)
  int pair_heads;         // 1: the CTA's two tiles are heads h, h+1; 0: row blocks r, r+1 of one head
  int n_row_blocks;       // ceil(S / 128)
  int n_items;            // work items (pairs of query tiles); the grid walks them persistently
  const int32_t* q_off;   // [B] position of query row 0 among the keys (chunked prefill), or nullptr (0)
  int max_off;            // q_off values are clamped to [0, max_off]
  const int32_t* q_len;   // [B] valid query rows of each sequence (chunks of different lengths), or nullptr (S);
                          // rows past them are not written
  int* status;            // device status word
};

int prefill_block_n(int D, bool f32);
// tmQ: the Q operand (bf16 Q, rotated fp16 Q, or bf16 hi/lo planes of fp32 Q), 128-row boxes.
cudaError_t launch_prefill(const PrefillParams& p, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           int D, bool f32, bool rope, int grid, cudaStream_t stream);

// ----------------------------------------------------------- paged decode
constexpr int kDecodePagesPerSplit = 32;  // pages (of 16 tokens) handled by one split

struct DecodeParams {
  const void* q;            // [B, Hq, D] bf16
  const int32_t* block_table;  // [B, max_pages]
  const int32_t* seq_lens;  // [B]
  float* part_o;            // [B, n_splits, Hq, D] fp32 (normalised partial outputs)
  float* part_lse;          // [B, n_splits, Hq]
  void* out;                // [B, Hq, D] bf16
  float* lse;               // [B, Hq]
  int B, Hq, Hkv, D, G;
  int max_pages, num_pages, n_splits;
  int HG, n_hg, n_qt;       // bf16 kernel: KV heads per TMA box (min(Hkv, 8)), head groups, 16-row query tiles
  float scale_log2;
  int* status;
  const float* k_scale;     // FP8 cache only: [num_pages, Hkv] scales (nullptr: bf16 cache)
  const float* v_scale;
};
cudaError_t launch_decode(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                          cudaStream_t stream);
// FP8 (E4M3) pages: tmK / tmV are 4-D uint8 maps (d, token, head, page); D = 64 or 128.
// The persistent grid (at most kDecodeFp8MaxRanges CTAs) cuts the pages of all
// sequences into one contiguous range per CTA; range c writes the partial result of
// each sequence b it meets at slot c + b of part_o / part_lse (launch_decode_range_merge
// combines them). Returns the number of ranges through *n_ranges.
constexpr int kDecodeFp8MaxRanges = 2 * 148;  // up to two CTAs per SM (D = 64)
cudaError_t launch_decode_fp8(const DecodeParams& p, const CUtensorMap& tmK, const CUtensorMap& tmV, int* n_ranges,
                              cudaStream_t stream);
cudaError_t launch_decode_range_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out,
                                      float* lse, int B, int H, int D, int T_max, int n_ranges, cudaStream_t stream);

// ------------------------------------------------------------------ MLA
constexpr int kMlaTile = 64;        // tokens per tile
constexpr int kMlaMaxPairs = 74;    // two-CTA clusters in the persistent grid (148 SMs)
// Weight, in tiles, that the MLA work split gives each non-empty sequence on top of its
// tiles: a cluster pays a fixed cost per segment (its Q load, the drained pipeline and
// the partial-result write), so ranges are cut in units of tiles + this per sequence.
constexpr int kMlaSegCost = 8;

struct MlaParams {
  const void* q_nope;       // [B, 1, H, Dc] bf16
  const void* q_pe;         // [B, 1, H, Dr] bf16
  const int32_t* seq_lens;  // [B]
  float* part_o;            // [n_pairs + B, H, Dc] fp32 (slot = cluster + sequence)
  float* part_lse;          // [n_pairs + B, H]
  int B, H, Dc, Dr, T_max, n_pairs;
  float scale_log2;
  int* status;
};
int mla_pairs_for_device();
cudaError_t launch_mla(const MlaParams& p, const CUtensorMap& tmKV, const CUtensorMap& tmPE, cudaStream_t stream);
cudaError_t launch_mla_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out,
                             float* lse, int B, int H, int T_max, int n_pairs, cudaStream_t stream);

// ------------------------------------------------------------- LSE merge
// Combines n_valid(b) normalised partials per (b, head) into bf16 out and fp32 lse.
// n_valid(b) = ceil(len_b / tokens_per_split); len_b == 0 gives out = 0, lse = -inf.
cudaError_t launch_merge(const float* part_o, const float* part_lse, const int32_t* seq_lens, void* out, float* lse,
                         int B, int H, int D, int n_splits, int tokens_per_split, cudaStream_t stream);

// Merges n_parts bf16 partial outputs [n_parts, rows, D] with fp32 LSEs [n_parts, rows]
// over disjoint key sets into out [rows, D] bf16 and lse [rows] (D in {64, 128, 256, 512}).
cudaError_t launch_parts_merge(const void* o_parts, const float* lse_parts, int n_parts, long long rows, int D,
                               void* out, float* lse, cudaStream_t stream);

}  // namespace attn
