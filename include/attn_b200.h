/*
 * attn_b200 — exact causal GQA attention, paged GQA decode and MLA absorbed decode
 * for NVIDIA B200 (sm_100a). C ABI: plain pointers and sizes only.
 *
 * Conventions for every entry point
 *  - All tensor pointers are DEVICE pointers, contiguous, 16-byte aligned
 *    (lse arrays: 4-byte aligned). The caller owns every buffer (inputs, outputs,
 *    workspace); the library allocates nothing on these calls and keeps no pointer
 *    after it returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously; buffers must stay alive until it completes.
 *  - Return value: ATTN_OK, or an error code. Arguments are validated on the host
 *    before anything is enqueued; on error nothing is launched and
 *    attn_last_error() describes the problem (thread-local string).
 *  - Device-side problems (a bounded wait that ran out, a block-table entry outside
 *    the page pool, a length beyond the cache) are recorded as bit flags in a status
 *    word at the start of the workspace; read it with attn_read_status() after the
 *    call's work has completed. Each call clears it when it starts.
 *  - LSE is the natural logarithm of the sum of exp(scaled scores), fp32.
 *  - A sequence of length 0 yields out = 0 and lse = -inf.
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, Hq % Hkv != 0, misalignment */
  ATTN_ERR_UNSUPPORTED = 2,  /* shape or dtype outside what the kernels implement */
  ATTN_ERR_WORKSPACE = 3,    /* workspace smaller than the *_workspace_size() query */
  ATTN_ERR_CUDA = 4,         /* a CUDA runtime / driver call failed (message has details) */
  ATTN_ERR_DEVICE = 5        /* returned by attn_read_status() when the device flagged a problem */
};

enum { ATTN_DTYPE_F32 = 0, ATTN_DTYPE_BF16 = 1 };

/* RoPE pair layouts (attn_prefill_ex). */
enum { ATTN_ROPE_INTERLEAVED = 0, ATTN_ROPE_HALF_SPLIT = 1 };
/* OR-ed into attn_prefill_ex's rope_layout: rotated q and k become bf16 operands instead
 * of fp16 (for bf16 inputs whose rotated values exceed the fp16 range). */
enum { ATTN_ROPE_BF16_OPERANDS = 4 };

/* Device status flags (attn_read_status). */
enum { ATTN_DEV_TIMEOUT = 1, ATTN_DEV_BAD_PAGE = 2, ATTN_DEV_BAD_LENGTH = 4, ATTN_DEV_RANGE = 8, ATTN_DEV_BAD_INDEX = 16 };

/*
 * Causal GQA/MQA/MHA prefill with RoPE.
 * Defined by: "attention study note" (makinaruto.github.io, llm_learning/attention),
 * sections "FlashAttention的改进" / "online-softmax 分块计算原理" (tiled exact attention
 * with running max/sum) and the GQA worked table (query head h uses kv head
 * h / (Hq/Hkv)); "From 32K to 256K: DeepSeek long-context" (tqpw.cn) section 2.1
 * (RoPE on adjacent pairs, theta_i = rope_theta^(-2i/D)) and 2.5 (cos/sin cache).
 *
 *   q   [B, Hq,  S, D]   dtype (bf16, or fp32)
 *   k,v [B, Hkv, S, D]   dtype
 *   out [B, Hq,  S, D]   dtype (written). With RoPE or fp32 input it also holds the
 *                        prepared Q operand between the prologue and the main kernel
 *                        (same byte size), so it must not overlap q, k or v.
 *   lse [B, Hq,  S]      fp32  (written)
 * causal: 1 -> key j is visible to query i iff j <= i; 0 -> all keys.
 * rope_theta: > 0 applies RoPE to q and k at positions 0..S-1; <= 0 disables it.
 * scale: multiplies q.k before the softmax; <= 0 selects 1/sqrt(D).
 * Supported: dtype BF16 with D in {64, 128}; dtype F32 with D = 64.
 * Tensor-core operand precision: bf16 without RoPE multiplies the bf16 inputs as
 * they are; bf16 with RoPE rounds the rotated q and k to fp16 for Q.K^T (so
 * |rotated value| must stay <= 65504, else ATTN_DEV_RANGE is flagged); fp32 input
 * carries every operand as a bf16 hi + lo pair (three products per MMA step).
 * P.V always accumulates in fp32 from bf16 P (hi + lo for fp32 input).
 * workspace: >= attn_prefill_workspace_size(B, Hkv, S, D, dtype) bytes of device memory,
 * 256-byte aligned.
 */
size_t attn_prefill_workspace_size(int B, int Hkv, int S, int D, int dtype);
int attn_prefill(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int S,
                 int D, int causal, float rope_theta, float scale, int dtype, void* workspace,
                 size_t workspace_bytes, void* stream);

/*
 * attn_prefill with the RoPE scaling variants of "From 32K to 256K: DeepSeek
 * long-context" (tqpw.cn): section 2.2 scales the rotary frequencies by a factor and
 * section 2.4 rescales the base (theta' = theta * (L / L0)^alpha; NTK-aware scaling is
 * likewise a rescaled base), and section 2.4's embedding concatenates the two halves.
 *   rope_theta       the (possibly rescaled) base; <= 0 disables RoPE as in attn_prefill
 *   rope_freq_scale  f > 0: the angle of pair i at position p is p * f * rope_theta^(-2i/D)
 *                    (1 = plain RoPE; 1/s interpolates positions by s)
 *   rope_layout      ATTN_ROPE_INTERLEAVED: pairs (2i, 2i+1) (attn_prefill's layout);
 *                    ATTN_ROPE_HALF_SPLIT: pairs (i, i + D/2), i < D/2;
 *                    either OR ATTN_ROPE_BF16_OPERANDS (bf16 input only): the rotated q and k
 *                    are rounded to bf16 instead of fp16, so any bf16 input is served (no
 *                    ATTN_DEV_RANGE) at 8x the rounding of the fp16 operands; the fallback
 *                    for calls that reported ATTN_DEV_RANGE
 * Everything else as attn_prefill, which equals attn_prefill_ex(..., rope_freq_scale = 1,
 * ATTN_ROPE_INTERLEAVED, ...). Invalid layout or non-positive scale: ATTN_ERR_INVALID_ARG.
 */
int attn_prefill_ex(const void* q, const void* k, const void* v, void* out, float* lse, int B, int Hq, int Hkv, int S,
                    int D, int causal, float rope_theta, float rope_freq_scale, int rope_layout, float scale, int dtype,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Paged split-KV GQA decode: one query token per sequence attends to all
 * seq_lens[b] cached tokens (already rotated; no RoPE, no mask).
 * Defined by: "attention study note", section "Page Attention" (fixed-size pages
 * reached through a per-sequence table) and the online-softmax recurrence used to
 * merge per-split partial results.
 *
 *   q            [B, Hq, D]                       bf16
 *   k_pages      [num_pages, page_size, Hkv, D]   bf16
 *   v_pages      [num_pages, page_size, Hkv, D]   bf16
 *   block_table  [B, max_pages_per_seq]  int32: physical page of logical page j;
 *                entries at or past ceil(seq_lens[b]/page_size) are never read
 *   seq_lens     [B] int32, 0 <= seq_lens[b] <= max_pages_per_seq * page_size
 *   out          [B, Hq, D] bf16 (written);  lse [B, Hq] fp32 (written)
 * Supported: dtype BF16, page_size 16, D in {64, 128}, any Hkv and group size
 * G = Hq/Hkv (Hq <= 4096). KV heads are read 8 per page load; G > 16 reads each page
 * once per 16 query heads of a KV head (G <= 16 reads every cached byte once).
 * scale <= 0 selects 1/sqrt(D). Out-of-range table entries or lengths are clamped
 * (no fault) and flagged in the status word.
 */
size_t attn_decode_paged_workspace_size(int B, int Hq, int D, int max_pages_per_seq, int page_size);
int attn_decode_paged(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                      const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int D, int page_size,
                      int max_pages_per_seq, int num_pages, float scale, int dtype, void* workspace,
                      size_t workspace_bytes, void* stream);

/*
 * Paged GQA decode over an FP8 (E4M3) KV cache with one fp32 scale per (page, kv head).
 * Defined by the paged decode above, with the cached values read as
 * e4m3(code) * scale ("7 anti-patterns of DeepSeek attention optimisation" (lpnh.cn),
 * section 3.3: the FP8 E4M3 format, largest value 448, and scale factors that bring
 * tensors into its range).
 *
 *   q            [B, Hq, D] bf16
 *   k_pages      [num_pages, page_size, Hkv, D] uint8 E4M3 codes (keys already rotated)
 *   v_pages      [num_pages, page_size, Hkv, D] uint8 E4M3 codes
 *   k_scale      [num_pages, Hkv] fp32;  v_scale [num_pages, Hkv] fp32
 *   block_table, seq_lens, out, lse: as attn_decode_paged.
 * Supported: D in {64, 128}, page_size 16, Hkv <= 8, Hq/Hkv <= 16. NaN codes are out of
 * contract. Products run in fp16: codes convert exactly, q converts exactly within
 * +-65504 (else ATTN_DEV_RANGE), P carries the value scale (times 2^8) in fp16, so
 * 256 * v_scale must stay below about 6.5e4.
 * workspace: >= attn_decode_paged_fp8_workspace_size(B, Hq, D, max_pages_per_seq, page_size)
 *   (device, 256-byte aligned, caller-owned, scratch): one fp32 partial output and LSE
 *   per (page range, sequence) pair; the pages of all sequences are cut into one
 *   contiguous range per CTA of a persistent grid, so every CTA streams the same number
 *   of pages whatever the length mix.
 */
size_t attn_decode_paged_fp8_workspace_size(int B, int Hq, int D, int max_pages_per_seq, int page_size);
int attn_decode_paged_fp8(const void* q, const void* k_pages, const void* v_pages, const float* k_scale,
                          const float* v_scale, const int32_t* block_table, const int32_t* seq_lens, void* out,
                          float* lse, int B, int Hq, int Hkv, int D, int page_size, int max_pages_per_seq,
                          int num_pages, float scale, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Chunked prefill into the paged KV cache: append a chunk of S_new tokens per sequence
 * and attend the new queries over the whole cache.
 * Defined by: "From 32K to 256K: DeepSeek long-context" (tqpw.cn) chapter 1 (streaming KV
 * cache for incremental processing, long sequences cut into chunks, a PagedAttention
 * variant) and section 2.1 (RoPE); "attention study note", sections "Page Attention"
 * (block table) and the tiled online-softmax sections (the attention itself).
 *
 *   q            [B, Hq,  S_new, D]   bf16, new queries (not rotated)
 *   k, v         [B, Hkv, S_new, D]   bf16, new keys (not rotated) and values
 *   k_pages      [num_pages, page_size, Hkv, D] bf16 (keys rotated), updated in place
 *   v_pages      [num_pages, page_size, Hkv, D] bf16, updated in place
 *   block_table  [B, max_pages_per_seq] int32; must map every logical page that holds
 *                a position < cache_lens[b] + S_new
 *   cache_lens   [B] int32 (device), tokens already cached; new token i of sequence b
 *                takes position cache_lens[b] + i; 0 <= cache_lens[b] <= max_cache_len
 *   out          [B, Hq, S_new, D] bf16 (written; also holds the prepared Q operand
 *                between the prologue and the attention, so it must not overlap q/k/v)
 *   lse          [B, Hq, S_new] fp32 (written)
 * The new keys are rotated at their positions (rope_theta > 0; <= 0: no RoPE) and
 * stored with the values in bf16; query i then attends keys t <= cache_lens[b] + i (the
 * causal mask aligned to the end of the cache). scale <= 0 selects 1/sqrt(D).
 * Supported: D in {64, 128}, page_size 16. Q.K^T runs with fp16 operands (bf16 cache
 * values are exact in fp16; |values| beyond 65504 flag ATTN_DEV_RANGE); P.V in bf16.
 * Entries outside the page pool or lengths beyond max_cache_len are skipped/clamped and
 * flagged in the status word (ATTN_DEV_BAD_PAGE, ATTN_DEV_BAD_LENGTH).
 * workspace: >= attn_prefill_chunk_workspace_size(...) bytes, 256-byte aligned.
 */
size_t attn_prefill_chunk_workspace_size(int B, int Hkv, int S_new, int max_cache_len, int D);
int attn_prefill_chunk(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                       const int32_t* block_table, const int32_t* cache_lens, void* out, float* lse, int B, int Hq,
                       int Hkv, int S_new, int D, int page_size, int max_pages_per_seq, int num_pages,
                       int max_cache_len, float rope_theta, float scale, void* workspace, size_t workspace_bytes,
                       void* stream);

/*
 * attn_prefill_chunk with the RoPE variants of attn_prefill_ex (rope_freq_scale multiplies
 * every rotary frequency; rope_layout ATTN_ROPE_INTERLEAVED or ATTN_ROPE_HALF_SPLIT): the new
 * keys are stored rotated in that form, and the cached keys must have been rotated the same
 * way. attn_prefill_chunk equals this call with 1 and ATTN_ROPE_INTERLEAVED.
 */
int attn_prefill_chunk_ex(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                          const int32_t* block_table, const int32_t* cache_lens, void* out, float* lse, int B, int Hq,
                          int Hkv, int S_new, int D, int page_size, int max_pages_per_seq, int num_pages,
                          int max_cache_len, float rope_theta, float rope_freq_scale, int rope_layout, float scale,
                          void* workspace, size_t workspace_bytes, void* stream);

/*
 * attn_prefill_chunk_ex for a batch of chunks of different lengths ("From 32K to 256K:
 * DeepSeek long-context", chapter 1: long inputs are cut into chunks streamed into the
 * KV cache; sequences of a batch reach the end of their input at different points).
 *   new_lens  [B] int32 (device, read), 0 <= new_lens[b] <= S_new: sequence b appends
 *             only its first new_lens[b] tokens (rows of k, v padded to S_new) at
 *             positions cache_lens[b] .. cache_lens[b] + new_lens[b] - 1, and only those
 *             query rows attend; its rows past them are written as out = 0, lse = -inf.
 *             nullptr: every sequence takes S_new (attn_prefill_chunk_ex).
 * Lengths outside [0, S_new] are clamped and flagged (ATTN_DEV_BAD_LENGTH). Query row
 * blocks past a sequence's chunk cost no tensor-core work. Everything else as
 * attn_prefill_chunk_ex (same workspace size).
 */
int attn_prefill_chunk_varlen(const void* q, const void* k, const void* v, void* k_pages, void* v_pages,
                              const int32_t* block_table, const int32_t* cache_lens, const int32_t* new_lens, void* out,
                              float* lse, int B, int Hq, int Hkv, int S_new, int D, int page_size,
                              int max_pages_per_seq, int num_pages, int max_cache_len, float rope_theta,
                              float rope_freq_scale, int rope_layout, float scale, void* workspace,
                              size_t workspace_bytes, void* stream);

/*
 * DeepSeek MLA absorbed decode (one query token per sequence).
 * Defined by: "DeepSeek-V3 attention: einsum vs hand-optimised" (dksg.cn), absorbed
 * form: scores = (q_nope . kv_cache^T + q_pe . pe_cache^T) * scale,
 * out = softmax(scores) . kv_cache; "attention study note", MLA absorption and
 * decoupled-RoPE sections.
 *
 *   q_nope   [B, 1, H, Dc]   bf16      q_pe     [B, 1, H, Dr]  bf16
 *   kv_cache [B, T_max, Dc]  bf16      pe_cache [B, T_max, Dr] bf16
 *   seq_lens [B] int32, 0 <= seq_lens[b] <= T_max (tokens past it are never used)
 *   out      [B, 1, H, Dc]   bf16 (written);  lse [B, 1, H] fp32 (written)
 * Supported: H = 128, Dc = 512, Dr = 64. scale must be > 0.
 */
size_t mla_decode_workspace_size(int B, int H, int Dc, int Dr, int T_max);
int mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
               const int32_t* seq_lens, float scale, void* out, float* lse, int B, int H, int Dc, int Dr, int T_max,
               void* workspace, size_t workspace_bytes, void* stream);

/*
 * DeepSeek sparse attention, step 1: lightning-indexer scores and the top-k selection.
 * Defined by: "attention study note" (makinaruto), section "Lighting Indexer": indexer
 * queries q_j (one per indexer head j), one indexer key k_s per cached token, and the
 * index score sum_j w_j * ReLU(q_j . k_s); only the most relevant tokens are attended.
 *
 *   q_idx    [B, H_I, d_I] bf16   indexer queries of each sequence's decode token
 *   w_idx    [B, H_I] fp32        indexer head weights
 *   k_idx    [B, T_max, d_I] bf16 indexer keys of the cached tokens
 *   seq_lens [B] int32            cached tokens per sequence (clamped to [0, T_max])
 *   scores   [B, T_max] fp32      out: I[b, s] for s < seq_lens[b], -inf past it
 *   topk_idx [B, top_k] int32     out: the min(top_k, seq_lens[b]) tokens with the largest
 *                                 scores (ties: smaller token index first), in ascending
 *                                 token order, then -1
 * Scores are fp32 (bf16 products accumulated in fp32, then ReLU, weights and the head sum
 * in fp32); the selection is exact with respect to those scores. Supported: d_I = 128,
 * H_I a multiple of 16 up to 64. All device pointers, caller-owned; 16-byte aligned q_idx
 * and k_idx. workspace: >= dsa_index_topk_workspace_size() bytes (status word).
 */
size_t dsa_index_topk_workspace_size(int B, int H_I, int d_I, int T_max, int top_k);
int dsa_index_topk(const void* q_idx, const float* w_idx, const void* k_idx, const int32_t* seq_lens, float* scores,
                   int32_t* topk_idx, int B, int H_I, int d_I, int T_max, int top_k, void* workspace,
                   size_t workspace_bytes, void* stream);

/*
 * DeepSeek sparse attention, step 2: the MLA absorbed decode (mla_decode) over the
 * selected tokens only: scores, softmax and output use the rows kv_cache[b, t] and
 * pe_cache[b, t] for t = topk_idx[b, i], i < min(seq_lens[b], top_k) (as written by
 * dsa_index_topk; any distinct indices in [0, seq_lens[b]) are accepted, an index outside
 * it flags ATTN_DEV_BAD_INDEX and reads row 0). Same tensors, layouts and limits as
 * mla_decode. The selected rows are gathered into the workspace, then attended by the
 * MLA kernel. workspace: >= dsa_mla_decode_workspace_size(B, H, Dc, Dr, top_k) bytes,
 * 256-byte aligned, caller-owned scratch (status word first).
 */
size_t dsa_mla_decode_workspace_size(int B, int H, int Dc, int Dr, int top_k);
int dsa_mla_decode(const void* q_nope, const void* q_pe, const void* kv_cache, const void* pe_cache,
                   const int32_t* seq_lens, const int32_t* topk_idx, int top_k, float scale, void* out, float* lse,
                   int B, int H, int Dc, int Dr, int T_max, void* workspace, size_t workspace_bytes, void* stream);

/*
 * dsa_mla_decode over an FP8 (E4M3) latent cache: the latent row of token t is
 * e4m3(kv_codes[b, t, c]) * kv_scale[b, t, c / 128] ("7 anti-patterns of DeepSeek attention
 * optimisation", section 3.3: E4M3, largest value 448, with scale factors); the rotary cache
 * pe_cache stays bf16. kv_codes [B, T_max, 512] uint8, kv_scale [B, T_max, 4] fp32; the
 * other arguments, the workspace (dsa_mla_decode_workspace_size) and the limits as
 * dsa_mla_decode. The selected rows are dequantised into bf16 (the MLA kernel's operand
 * type, so each latent value is rounded to bf16) and attended by the MLA decode kernel.
 * NaN codes are out of contract.
 */
int dsa_mla_decode_fp8(const void* q_nope, const void* q_pe, const void* kv_codes, const float* kv_scale,
                       const void* pe_cache, const int32_t* seq_lens, const int32_t* topk_idx, int top_k, float scale,
                       void* out, float* lse, int B, int H, int Dc, int Dr, int T_max, void* workspace,
                       size_t workspace_bytes, void* stream);

/*
 * Paged decode for callers that cannot allocate device memory (code running
 * inside another framework's memory pool with allocation disabled, paths where
 * cudaMalloc's implicit synchronisation is not allowed, embedders that only pass
 * buffers they already own). Same arguments, layouts and results as
 * attn_decode_paged, minus the workspace: the split partials and the status
 * word live in one file-scope device array of ATTN_DECODE_NOALLOC_MAX_BYTES,
 * held by every GPU that loads the library until the process exits. The call
 * allocates nothing (the first call on a device: see below). Device-side flags
 * (bad block-table entries, lengths beyond the table, timeouts) are read with
 * attn_decode_paged_noalloc_status.
 *  - Problems whose attn_decode_paged_workspace_size() exceeds the array are
 *    rejected with ATTN_ERR_WORKSPACE and a message naming both sizes.
 *  - The first call on each device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current. With CUDA's lazy module
 *    loading (the default since CUDA 12.2) that first call may also load this
 *    library's device code and reserve the array, so make it outside any region
 *    where the caller cannot allocate, and before any stream capture.
 *  - Every call on a device shares the one array and leaves its contents behind;
 *    calls whose GPU work overlaps (different streams, or host threads) race on it
 *    and must be serialised by the caller.
 * There is no counterpart on the method's pages: it exists for these callers only.
 */
#define ATTN_DECODE_NOALLOC_MAX_BYTES (32ull << 20)
int attn_decode_paged_noalloc(const void* q, const void* k_pages, const void* v_pages, const int32_t* block_table,
                              const int32_t* seq_lens, void* out, float* lse, int B, int Hq, int Hkv, int D,
                              int page_size, int max_pages_per_seq, int num_pages, float scale, int dtype,
                              void* stream);

/*
 * Status word of the last attn_decode_paged_noalloc call on the current device (the
 * call has no workspace for attn_read_status to read): waits for `stream`, then copies
 * the word at the start of the fixed array into *flags (ATTN_DEV_BAD_PAGE,
 * ATTN_DEV_BAD_LENGTH, ATTN_DEV_TIMEOUT). Returns ATTN_OK when no flag is set,
 * ATTN_ERR_DEVICE when one is, ATTN_ERR_CUDA when the lookup or the copy fails.
 * Allocates nothing; like the entry point, it has no counterpart on the method's pages.
 */
int attn_decode_paged_noalloc_status(int* flags, void* stream);

/* Thread-local description of the last error returned on this thread ("" if none). */
const char* attn_last_error(void);

/*
 * Waits for `stream`, then copies the status word at the start of `workspace` into
 * *flags (a bitwise OR of ATTN_DEV_*). Returns ATTN_OK when no flag is set,
 * ATTN_ERR_DEVICE when one is, ATTN_ERR_CUDA when the copy fails.
 */
int attn_read_status(const void* workspace, int* flags, void* stream);

/*
 * Combines partial results of the same query rows over disjoint key sets: the slices
 * of every sequence's KV cache that the GPUs of a sequence-parallel group hold, each
 * attended with attn_decode_paged or mla_decode on its own GPU and gathered. The
 * block-level form of the online-softmax recurrence ("attention study note",
 * section "online-softmax 分块计算原理"): M = max_s lse_s, w_s = exp(lse_s - M),
 * lse = M + ln(sum_s w_s), out = sum_s w_s o_s / sum_s w_s, in part order
 * (deterministic); parts with lse = -inf (empty slices) carry no weight, and a row
 * whose parts are all empty gets out = 0, lse = -inf.
 *   o_parts   [n_parts, rows, D] bf16 (read)     lse_parts [n_parts, rows] fp32 (read)
 *   out       [rows, D] bf16 (written)            lse       [rows] fp32 (written)
 * rows = B * H of the decode (H = Hq, or the 128 MLA heads); D in {64, 128, 256, 512};
 * 1 <= n_parts <= 65536. Pointers 4-byte aligned. Asynchronous on `stream`; no workspace.
 */
int attn_lse_merge(const void* o_parts, const float* lse_parts, int n_parts, long long rows, int D, void* out,
                   float* lse, void* stream);

/*
 * RoPE base rescaling for long contexts, the values to pass as rope_theta.
 * attn_rope_ntk_theta: the NTK-aware base for a context stretched by `scale` (>= 1):
 *   theta * scale^(D / (D - 2)), which leaves the highest rotary frequency (pair 0)
 *   unchanged and divides the lowest one, theta^(-(D-2)/D), by `scale`
 *   ("From 32K to 256K: DeepSeek long-context" (tqpw.cn), section 2.2, names NTK-aware
 *   scaling; the rule is the published one).
 * attn_rope_length_scaled_theta: theta * (length / base_length)^alpha (same page,
 *   section 2.4, the length-aware base).
 * Host functions (no GPU). Invalid arguments or a non-finite result: return 0 and set
 * attn_last_error().
 */
double attn_rope_ntk_theta(double theta, double scale, int head_dim);
double attn_rope_length_scaled_theta(double theta, int length, int base_length, double alpha);

/*
 * Self-test of the exponential that part of the prefill softmax evaluates on the FMA
 * pipe instead of the MUFU (the score rate of the tensor core at head dim 128 equals
 * the MUFU rate, so 2 of every 8 exponentials of an unmasked block take this path).
 * Writes y[i] = 2^z[i] as that routine computes it: Cody-Waite reduction z = n + f with
 * n = round(z), f in [-1/2, 1/2], 2^f from a degree-3 minimax polynomial fitted for this
 * library, 2^n added to the exponent field: relative error <= 7.5e-5 for z >= -125.5
 * (normal results); just above -126 the result can be subnormal (absolute error below
 * 2^-126 * 2e-4); arguments below -126 are clamped to -126. Valid for z < 128. z, y: device arrays of n fp32 values,
 * 1 <= n <= 2^30. Asynchronous on `stream`. No counterpart on the pages: the softmax
 * they describe uses exp(); this only checks the library's own exponential.
 */
int attn_selftest_exp2(const float* z, float* y, int n, void* stream);

/*
 * Self-test of the bounded-wait mechanism every kernel uses: launches one CTA that
 * waits on an mbarrier nothing ever arrives at, with the given limit in
 * nanoseconds (1e3 .. 1e10). The wait gives up, the kernel records
 * ATTN_DEV_TIMEOUT in the workspace status word and exits normally, so the CUDA
 * context stays usable. workspace: >= 256 bytes.
 */
int attn_selftest_wait_timeout(void* workspace, size_t workspace_bytes, unsigned long long timeout_ns,
                               void* stream);

/*
 * Kernel timing hook for benchmarks. While enabled (on != 0), every call above
 * records a pair of CUDA events on its stream immediately around its main kernel
 * (prefill_kernel, decode_kernel, mla_kernel), so the time excludes the RoPE
 * prologue, the merge and host work. attn_profile_collect() waits for the recorded
 * events, returns the summed milliseconds and the number of pairs, and forgets
 * them. Enabling creates the events once (host-side resources, no device memory).
 * Not thread-safe; intended for a single benchmarking thread.
 */
int attn_profile_enable(int on);
int attn_profile_collect(double* total_ms, int* count);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
