/*
 * attn.h -- C ABI of the B200 (sm_100a) exact softmax attention library
 * (libattn_b200.so).
 *
 * What is computed ("Attention Kernel", section "问题与成本"):
 *     P = softmax(Q K^T * scale + M),   O = P V
 * with Q [B, Hq, Sq, d] and K, V [B, Hkv, Sk, d].  Several query heads share
 * one KV head (GQA); query head hq reads KV head hq / (Hq / Hkv).  The result
 * is exact: the score matrix is consumed block by block with the online
 * softmax (m, l, o) recurrence ("Attention Kernel", section "Online softmax")
 * and never written to memory; "exact" means the same mathematics within
 * floating-point rounding, not bitwise equality with another kernel.
 *
 * Conventions shared by every entry point:
 *   - Tensors are dense and contiguous (row-major in the order given).  q, k,
 *     v, o, k_cache and v_cache hold bfloat16 (attn_decode_paged_fp8's caches
 *     hold E4M3 bytes with float32 scales); the backward's d_o, dq, dk and dv
 *     hold bfloat16; lse holds float32; index arrays hold int32.
 *     Accumulation is float32.
 *   - Every pointer argument except `workspace` sizes is a DEVICE pointer on
 *     the current CUDA device.  The caller owns all memory; the library
 *     allocates nothing per call and never synchronises the stream in a
 *     launch.  Work is enqueued on `stream` and runs asynchronously.
 *   - Tensor pointers must be 16-byte aligned (a TMA requirement).
 *   - Masking: the additive mask M holds only 0 and -inf.  A key j is visible
 *     to query row i of sequence b iff j < k_len[b] and, when causal,
 *     j <= i + (k_len[b] - Sq) (causal diagonal aligned to the bottom right,
 *     so Sq = 1 sees every key and a square problem gets the usual j <= i).
 *   - A row with no visible key gets O = 0 and LSE = -inf (never NaN), as
 *     the "Online softmax" section of "Attention Kernel" requires.
 *   - LSE[b, h, i] = ln sum_j exp(scale * q_i . k_j) over the visible keys
 *     (natural log), the statistic a backward pass recomputes P from.
 *   - Return value: ATTN_OK, or an attn_status describing why nothing was
 *     launched (arguments are checked on the host before any CUDA call) or
 *     why the launch failed.  Faults found on the device (a block-table entry
 *     outside the page pool, a timed-out internal wait) set a device error
 *     word instead; read it with attn_get_device_error().
 */
#ifndef ATTN_B200_ATTN_H_
#define ATTN_B200_ATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t / CUstream; NULL is the legacy default stream. */
typedef struct CUstream_st* attn_stream_t;

typedef enum {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = 1, /* null pointer, bad extent, Hq % Hkv != 0, non-finite scale */
  ATTN_ERR_UNSUPPORTED = 2, /* head dim, page size or group size outside what is built */
  ATTN_ERR_ALIGNMENT = 3,   /* a tensor pointer is not 16-byte aligned */
  ATTN_ERR_WORKSPACE = 4,   /* decode / varlen workspace missing or too small */
  ATTN_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed (no device, launch error) */
  ATTN_ERR_DEVICE = 6       /* attn_get_device_error(): the device error word was set */
} attn_status;

/* Bits of the device error word (attn_get_device_error's flags_out). */
#define ATTN_DEVERR_WAIT_TIMEOUT 0x1u /* an internal pipeline wait exceeded its time limit */
#define ATTN_DEVERR_BAD_PAGE 0x2u     /* a block-table entry outside [0, num_pages) was skipped */
#define ATTN_DEVERR_BAD_LENGTH 0x4u   /* a k_len / seq_len / cu_seqlens entry outside its legal range */

/*
 * attn_fwd -- prefill / full-sequence attention forward.
 * Source: "Attention Kernel", sections "问题与成本" (the operation and shapes),
 * "Online softmax" (the recurrence and the zero-output contract) and
 * "FlashAttention 的稳定基础" (whole-tile causal skipping, per-element
 * predicates on boundary tiles, the saved log-sum-exp).
 *
 *   q   [B, Hq,  Sq, d] bf16      k, v [B, Hkv, Sk, d] bf16
 *   o   [B, Hq,  Sq, d] bf16 (written)
 *   lse [B, Hq,  Sq]    fp32 (written; may be NULL to skip it)
 *   B, Hq, Hkv >= 1, Hq % Hkv == 0, Sq >= 1, Sk >= 0 (Sk = 0: every row is
 *   empty), d in {64, 128}; causal in {0, 1}; scale finite (usually 1/sqrt(d)).
 * Errors: INVALID_ARG, UNSUPPORTED (d), ALIGNMENT, CUDA.  Nothing is written
 * when an error is returned before the launch.
 */
int attn_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
             int Hkv, int Sq, int Sk, int d, int causal, float scale, attn_stream_t stream);

/*
 * attn_fwd_masked -- attn_fwd with per-sequence key padding.
 * Source: as attn_fwd, plus "Attention Kernel", section "正确性契约" (padding
 * semantics and fully masked rows are part of the contract).
 *   k_lens [B] int32 device array, nullable (NULL = Sk for every sequence):
 *   sequence b sees only keys j < k_lens[b].  Values outside [0, Sk] are
 *   clamped on the device and flagged with ATTN_DEVERR_BAD_LENGTH.
 * Other arguments, layout and errors as attn_fwd.
 */
int attn_fwd_masked(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                    const int32_t* k_lens, attn_stream_t stream);

/*
 * attn_fwd_host_workspace_size -- bytes of device workspace attn_fwd_host
 * needs for these extents: two buffer sets of one chunk's Q, K, V, O and LSE
 * plus B * Hkv key lengths (a chunk is about an eighth of the B * Hkv
 * (sequence, KV head) pairs).  0 for invalid arguments.
 */
size_t attn_fwd_host_workspace_size(int B, int Hq, int Hkv, int Sq, int Sk, int d);

/*
 * attn_fwd_host -- attn_fwd_masked on tensors in HOST memory.
 * Source: as attn_fwd_masked; the result is bit-identical to it.  The batch is
 * cut into chunks of whole (sequence, KV head) pairs; each chunk's Q, K, V are
 * copied in, computed and its O, LSE copied out through two device buffer
 * sets, with the copies of one chunk overlapping the kernels of another.
 *   q, k, v, o, lse: host pointers, same shapes and layouts as attn_fwd
 *   (lse nullable).  Page-locked (pinned) memory gives the overlap; pageable
 *   memory is correct but the copies then serialise with the host.
 *   k_lens [B] int32 HOST array, nullable; values must lie in [0, Sk].
 *   workspace: device buffer of attn_fwd_host_workspace_size() bytes,
 *   16-byte aligned, caller-owned, not shared with a concurrent call.
 *   stream: the kernels run on it; the copies run on two streams the library
 *   creates once per device and keeps, ordered after the work already on
 *   `stream`.  O and LSE are complete, and q, k, v may be reused, once
 *   `stream` reaches the point where the call returned.
 *   Unlike every other entry point this one may block: when k_lens is given
 *   it synchronises `stream` once, and copies from pageable memory block.
 * Errors: as attn_fwd_masked, plus INVALID_ARG for a k_lens value outside
 * [0, Sk] and WORKSPACE for a missing or short workspace.
 */
int attn_fwd_host(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq,
                  int Hkv, int Sq, int Sk, int d, int causal, float scale, const int32_t* k_lens,
                  void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_fwd_fp8 -- attn_fwd_masked over block-scaled E4M3 Q, K and V.
 * Source: "Attention 算子加速史", section 3.3 (FP8 operands with block-level
 * scaling); the operation is attn_fwd_masked's on the dequantised values.
 *   q [B, Hq, Sq, d], k, v [B, Hkv, Sk, d]: uint8 E4M3 codes (OCP E4M3: bias
 *   7, 3 mantissa bits, no infinity; 0x7F / 0xFF are NaN and must not occur)
 *   q_scale [B, Hq, ceil(Sq/128)], k_scale, v_scale [B, Hkv, ceil(Sk/128)]
 *   fp32 device arrays: element (b, h, i, :) of a tensor is
 *   scale[b, h, i / 128] * e4m3(code).  Scales must be positive and finite.
 *   o [B, Hq, Sq, d] bf16 and lse [B, Hq, Sq] fp32 (nullable) are written as
 *   by attn_fwd_masked; causal, scale, k_lens likewise.
 *   d must be 128.  S = Q K^T runs on E4M3 tensor-core MMAs (the two block
 *   scales enter the fp32 scores); P V runs in bf16 on V widened exactly.
 * Errors: as attn_fwd_masked, plus INVALID_ARG for a NULL scale array,
 * UNSUPPORTED for d != 128, ALIGNMENT for scales not 4-byte aligned.
 */
int attn_fwd_fp8(const void* q, const void* k, const void* v, const float* q_scale,
                 const float* k_scale, const float* v_scale, void* o, float* lse, int B, int Hq,
                 int Hkv, int Sq, int Sk, int d, int causal, float scale, const int32_t* k_lens,
                 attn_stream_t stream);

/*
 * attn_fwd_paged_fp8_workspace_size -- bytes of device workspace
 * attn_fwd_paged_fp8 needs: the unit list of attn_fwd_paged, a block table
 * [B, max_pages_per_seq] and bf16 K and V pools of B * max_pages_per_seq
 * pages (the batch's pages, dequantised).  0 for invalid arguments.
 */
size_t attn_fwd_paged_fp8_workspace_size(int B, long long total_q, int max_seqlen_q,
                                         int max_pages_per_seq, int page_size, int Hkv, int d);

/*
 * attn_fwd_paged_fp8 -- attn_fwd_paged over an E4M3 paged cache.
 * Source: "Attention Kernel", sections "Paged 与 ragged KV" (the paged
 * layout) and "正确性契约" (the cache quantisation schema is part of the
 * contract): element (page, r, h, i) of the K cache is
 * k_scale[page, h] * e4m3(k_cache[page, r, h, i]) (V likewise).
 *   q [total_q, Hq, d] bf16; k_cache, v_cache [num_pages, page_size, Hkv, d]
 *   uint8 E4M3 codes (0x7F / 0xFF must not occur); k_scale, v_scale
 *   [num_pages, Hkv] fp32 device arrays; the rest as attn_fwd_paged.
 *   The call first writes the pages its sequences reach, dequantised to bf16
 *   (round to nearest of scale * value), into the workspace, then runs the
 *   bf16 paged prefill over them; no element of the cache is changed.
 *   workspace: attn_fwd_paged_fp8_workspace_size(...) bytes, 16-byte aligned,
 *   caller-owned, not shared with a concurrent call.
 * Errors: as attn_fwd_paged, plus INVALID_ARG for a NULL scale array and
 * ALIGNMENT for scales not 4-byte aligned.
 */
int attn_fwd_paged_fp8(const void* q, const void* k_cache, const void* v_cache,
                       const float* k_scale, const float* v_scale, const int32_t* block_table,
                       const int32_t* cu_seqlens_q, const int32_t* seq_lens_k, int page_size,
                       int B, int Hq, int Hkv, long long total_q, int max_seqlen_q,
                       int max_pages_per_seq, int num_pages, int d, int causal, float scale,
                       void* o, float* lse, void* workspace, size_t workspace_bytes,
                       attn_stream_t stream);

/*
 * attn_fwd_window -- causal prefill with a sliding window or a prefix-LM mask.
 * Source: "Attention Kernel", section "可编程 mask" (masks such as a sliding
 * window or a prefix-LM rule: block-level sparsity decides which tiles are
 * skipped entirely, an element-wise rule handles the tiles that remain).
 *   A query row i has key position p = i + (k_len[b] - Sq) (the causal
 *   diagonal aligned to the bottom right, as attn_fwd_masked) and sees:
 *     window > 0: keys p - window < j <= p (at most `window` keys ending at
 *                 its diagonal);
 *     prefix > 0: keys j <= p and every key j < prefix (prefix-LM);
 *     window = prefix = 0: keys j <= p (attn_fwd_masked with causal = 1);
 *   always within j < k_len[b].  window and prefix may not both be > 0.
 *   Key tiles outside a row block's visible range are skipped at both ends.
 * Other arguments, layouts and errors as attn_fwd_masked (INVALID_ARG also
 * for a negative window or prefix, or both > 0).  Document masks are ragged
 * batches (attn_fwd_varlen with one range per document); block-sparse masks
 * are attn_fwd_block_sparse.
 */
int attn_fwd_window(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                    int Hq, int Hkv, int Sq, int Sk, int d, float scale, const int32_t* k_lens,
                    int window, int prefix, attn_stream_t stream);

/*
 * attn_fwd_block_sparse -- prefill with a block-sparse mask.
 * Source: "Attention Kernel", section "可编程 mask" (block-level sparsity
 * decides which tiles are skipped entirely; the element-wise rule -- here the
 * causal / key-length one of attn_fwd_masked -- handles the tiles left).
 *   block_mask  uint8 [B, mask_heads, ceil(Sq/128), ceil(Sk/128)] device
 *               array (mask_heads 1: shared by all query heads, or Hq): entry
 *               [b][h][i/128][j/128] == 0 hides key j from query row i of
 *               head h; such 128 x 128 blocks are never loaded or computed.
 *   Rows left without a visible key get O = 0, LSE = -inf.
 * Other arguments, layouts and errors as attn_fwd_masked (INVALID_ARG also
 * for a NULL mask or mask_heads not in {1, Hq}).
 */
int attn_fwd_block_sparse(const void* q, const void* k, const void* v, void* o, float* lse, int B,
                          int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                          const int32_t* k_lens, const uint8_t* block_mask, int mask_heads,
                          attn_stream_t stream);

/*
 * attn_fwd_varlen_workspace_size -- bytes of caller-owned device workspace
 * that attn_fwd_varlen needs: the list of (sequence, 256-row query block)
 * work units the call schedules.  total_q is the number of packed query
 * tokens, B the number of sequences, max_seqlen_q an upper bound on any
 * sequence's query length.  Returns 0 for invalid arguments.
 */
size_t attn_fwd_varlen_workspace_size(int B, long long total_q, int max_seqlen_q);

/*
 * attn_fwd_varlen -- prefill attention over a ragged batch of packed
 * sequences, described by cumulative sequence lengths instead of padding.
 * Source: "Attention Kernel", section "Paged 与 ragged KV" (a ragged batch is
 * not padded into a rectangle; cumulative sequence lengths give each
 * sequence's range, and the offset type, empty sequences and accesses across
 * sequence boundaries are part of the correctness contract), with the
 * operation, masking and outputs of attn_fwd.
 *
 *   q   [total_q, Hq,  d] bf16   sequence b owns tokens [cu_q[b], cu_q[b+1])
 *   k,v [total_k, Hkv, d] bf16   sequence b owns tokens [cu_k[b], cu_k[b+1])
 *   o   [total_q, Hq,  d] bf16 (written for every token that belongs to a sequence)
 *   lse [Hq, total_q]     fp32 (written likewise; nullable)
 *   cu_seqlens_q, cu_seqlens_k  [B + 1] int32 device arrays: cu[0] = 0,
 *       non-decreasing, cu_q[B] <= total_q, cu_k[B] <= total_k.  Sequence
 *       lengths may be 0: an empty query range produces nothing, and a query
 *       range with an empty key range gets O = 0, LSE = -inf.
 *   Within sequence b the mask is attn_fwd's with Sq = len_q(b) and
 *   k_len = Sk = len_k(b) (causal diagonal aligned to the bottom right).
 *   Keys of other sequences are never visible.  A tile that straddles a
 *   boundary reads a neighbour's rows, which then get weight exactly 0, so
 *   inputs must be finite for that to leave the result untouched.
 *   max_seqlen_q >= every len_q(b), at most 2^21; B >= 1; Hq % Hkv == 0;
 *   d in {64, 128}; causal in {0, 1}; scale finite.
 *   workspace    device scratch of at least
 *                attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q)
 *                bytes, 16-byte aligned; overwritten.
 * Device-side faults: offsets that decrease, exceed the totals or give a
 * query length above max_seqlen_q make that sequence empty (nothing of it
 * is written) and flag ATTN_DEVERR_BAD_LENGTH.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA.
 */
int attn_fwd_varlen(const void* q, const void* k, const void* v, void* o, float* lse,
                    const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int B, int Hq,
                    int Hkv, long long total_q, long long total_k, int max_seqlen_q, int d,
                    int causal, float scale, void* workspace, size_t workspace_bytes,
                    attn_stream_t stream);

/*
 * attn_fwd_paged -- prefill / append over a paged KV cache: new query tokens
 * of a ragged batch attend to their sequence's keys in a page pool.
 * Source: "Attention Kernel", section "Paged 与 ragged KV" (token t of a
 * sequence lives in logical page t / page_size at offset t mod page_size; the
 * block table maps it to a physical page; the last page is partial; ragged
 * queries by cumulative lengths), with the operation and masking of attn_fwd.
 *
 *   q            [total_q, Hq, d] bf16, packed: sequence b owns query tokens
 *                [cu_q[b], cu_q[b+1])
 *   k_cache      [num_pages, page_size, Hkv, d] bf16
 *   v_cache      [num_pages, page_size, Hkv, d] bf16
 *   block_table  [B, max_pages_per_seq] int32 physical page of each logical
 *                page; entries past a sequence's last page are never read
 *   cu_seqlens_q [B + 1] int32 (as attn_fwd_varlen)
 *   seq_lens_k   [B] int32 keys of each sequence (cached + new), at most
 *                max_pages_per_seq * page_size
 *   o            [total_q, Hq, d] bf16 (written for tokens of a sequence)
 *   lse          [Hq, total_q] fp32 (nullable)
 *   Masking is attn_fwd's with Sq = len_q(b), k_len = seq_lens_k[b]: with
 *   causal = 1 the queries are the last len_q positions of the sequence
 *   (query i sees keys j <= i + seq_lens_k[b] - len_q), which is appending
 *   len_q new tokens to a cache that already holds them.
 *   page_size in {16, 32, 64, 128}; d in {64, 128}; Hq % Hkv == 0;
 *   max_seqlen_q in [1, 2^21]; workspace as attn_fwd_varlen (size from
 *   attn_fwd_varlen_workspace_size(B, total_q, max_seqlen_q)).
 *   Whole pages are read, so every slot of a referenced page must hold finite
 *   values (slots past a sequence's length get weight exactly 0).
 * Device-side faults: a page id outside [0, num_pages) is skipped and flags
 * ATTN_DEVERR_BAD_PAGE; query offsets as attn_fwd_varlen, and a seq_lens_k
 * outside [0, max_pages_per_seq * page_size], make that sequence empty and
 * flag ATTN_DEVERR_BAD_LENGTH.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA.
 */
int attn_fwd_paged(const void* q, const void* k_cache, const void* v_cache,
                   const int32_t* block_table, const int32_t* cu_seqlens_q,
                   const int32_t* seq_lens_k, int page_size, int B, int Hq, int Hkv,
                   long long total_q, int max_seqlen_q, int max_pages_per_seq, int num_pages, int d,
                   int causal, float scale, void* o, float* lse, void* workspace,
                   size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_decode_workspace_size -- bytes of caller-owned device workspace that
 * attn_decode_paged needs for the given capacity.
 * Source: "Attention 算子加速史", section 4.1-4.2 (split-K decode: each split
 * writes a partial output and its log-sum-exp; a light kernel merges them).
 * The workspace holds float32 partial outputs [B, Hq, n_split, d] and float32
 * partial log-sum-exps [B, Hq, n_split], n_split = ceil(max_pages_per_seq *
 * page_size / split_tokens) with the library's fixed split length.
 * Returns 0 for invalid arguments.
 */
size_t attn_decode_workspace_size(int B, int Hq, int max_pages_per_seq, int page_size, int d);

/*
 * attn_decode_paged -- single-query (Sq = 1) attention over a paged KV cache.
 * Source: "Attention Kernel", section "Paged 与 ragged KV" (token t of a
 * sequence lives in logical block t / page_size at offset t mod page_size;
 * the block table maps the block to a physical page; the last page is
 * partial) and "Prefill 与 decode 是两种 kernel"; "Attention 算子加速史",
 * section 4 (split-KV decode with a log-sum-exp merge).
 *
 *   q            [B, Hq, d] bf16
 *   k_cache      [num_pages, page_size, Hkv, d] bf16
 *   v_cache      [num_pages, page_size, Hkv, d] bf16
 *   block_table  [B, max_pages_per_seq] int32: physical page of each logical
 *                page; entries past the sequence's last page are never read
 *   seq_lens     [B] int32: tokens in each sequence (0 allowed: O = 0, LSE = -inf)
 *   o            [B, Hq, d] bf16 (written)
 *   lse          [B, Hq] fp32 (written; nullable)
 *   workspace    device scratch of at least attn_decode_workspace_size(...)
 *                bytes, 16-byte aligned; its contents are overwritten.
 *   page_size a positive multiple of 16 (<= 256); d in {64, 128};
 *   Hq / Hkv <= 8.
 * Device-side faults: a page id outside [0, num_pages) is skipped (its tokens
 * contribute nothing) and flags ATTN_DEVERR_BAD_PAGE; a seq_len outside
 * [0, max_pages_per_seq * page_size] is clamped and flags
 * ATTN_DEVERR_BAD_LENGTH.  The result is deterministic: the splits are merged
 * in a fixed order with no atomics.
 * Launches: two kernels on `stream`, the split kernel and the merge kernel;
 * the merge is launched with programmatic stream serialization, so that it
 * may start while the split grid drains and waits (griddepcontrol.wait) for
 * the split grid's writes before it reads them.  Both can be captured into a
 * CUDA graph.
 * Errors: INVALID_ARG, UNSUPPORTED, ALIGNMENT, WORKSPACE, CUDA.
 */
int attn_decode_paged(const void* q, const void* k_cache, const void* v_cache,
                      const int32_t* block_table, const int32_t* seq_lens, int page_size, int B,
                      int Hq, int Hkv, int d, int max_pages_per_seq, int num_pages, float scale,
                      void* o, float* lse, void* workspace, size_t workspace_bytes,
                      attn_stream_t stream);

/*
 * attn_get_device_error -- synchronise `stream`, read and clear the device
 * error word of the current device.  Returns ATTN_OK when it was zero,
 * ATTN_ERR_DEVICE when it was set (flags_out, nullable, receives the
 * ATTN_DEVERR_* bits), or ATTN_ERR_CUDA if the read itself failed.
 * The word is per device and shared by all streams and calls.
 */
int attn_get_device_error(attn_stream_t stream, unsigned int* flags_out);

/*
 * attn_decode_paged_noalloc -- attn_decode_paged without a caller-supplied
 * workspace, for callers that are not allowed to allocate device memory: code
 * that runs inside a host framework which owns every device allocation (and
 * so has no buffer of its own to lend as scratch), or a latency-critical path
 * where cudaMalloc / cudaFree, which may synchronise the device, cannot be
 * called.  The pages this library follows have no counterpart to this call;
 * it exists only for such callers.
 *
 * The split partials live in one library-owned scratch area of
 * ATTN_NOALLOC_SCRATCH_BYTES, a static device array that every GPU which
 * loads the library holds until the process exits.  Nothing is allocated by
 * this call.  Arguments, layouts and results are those of attn_decode_paged;
 * the caller still provides q, the caches, the table, the lengths and the
 * outputs.
 *   - A problem whose attn_decode_workspace_size(...) exceeds
 *     ATTN_NOALLOC_SCRATCH_BYTES is rejected with ATTN_ERR_WORKSPACE before
 *     anything is launched.
 *   - The first call on a device looks up the scratch area's device address
 *     (with that device current) and caches it; make that first call before
 *     any stream capture on that device.  The cached address belongs to the
 *     device's primary context: after cudaDeviceReset on that device it is
 *     stale, and this call must not be used again in the same process.
 *   - Every call on a device shares the same scratch area.  Calls whose
 *     kernels overlap on the GPU (different streams, or different host
 *     threads) race on it and produce garbage; serialise them.  Each call
 *     writes every scratch byte it later reads, so nothing has to be cleared
 *     between calls.
 * Errors: as attn_decode_paged, plus ATTN_ERR_CUDA if the scratch address
 * cannot be obtained.
 */
#define ATTN_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int attn_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_table, const int32_t* seq_lens, int page_size,
                              int B, int Hq, int Hkv, int d, int max_pages_per_seq, int num_pages,
                              float scale, void* o, float* lse, attn_stream_t stream);

/*
 * attn_decode_paged_fp8 -- attn_decode_paged over an FP8 (E4M3) KV cache
 * with one scale per (physical page, KV head).
 * Source: "Attention Kernel", sections "Paged 与 ragged KV" and "正确性契约"
 * (the cache quantisation schema is part of the kernel contract, with the
 * page size, block table and valid-token counts); "Attention 算子加速史",
 * section 3 (FP8 operands with scale factors) and section 4 (paged decode).
 *
 *   k_cache, v_cache  [num_pages, page_size, Hkv, d] uint8: OCP E4M3 codes
 *                     (bias 7, 3 mantissa bits, subnormals; 0x7F/0xFF are
 *                     NaN and must not occur)
 *   k_scale, v_scale  [num_pages, Hkv] fp32 device arrays: the cache element
 *                     K[page, r, h, i] is k_scale[page, h] * e4m3(code), V
 *                     likewise (finite scales; any sign)
 *   The attention computed is attn_decode_paged's over those dequantised
 *   values.  The kernel widens the codes exactly to f16 for two f16 MMAs:
 *   q K^T with q multiplied by a power of two into f16's range (exact for bf16
 *   q down to f16's subnormals), and P V with P rounded to f16; the K scale
 *   (and that power of two) multiply the fp32 scores, the V scale each page's
 *   fp32 partial output.
 * Other arguments, workspace (attn_decode_workspace_size), device-side
 * checks and errors as attn_decode_paged; INVALID_ARG also for a NULL scale
 * array, ALIGNMENT when a scale array is not 4-byte aligned (the caches need
 * 16 bytes).
 */
int attn_decode_paged_fp8(const void* q, const void* k_cache, const void* v_cache,
                          const float* k_scale, const float* v_scale, const int32_t* block_table,
                          const int32_t* seq_lens, int page_size, int B, int Hq, int Hkv, int d,
                          int max_pages_per_seq, int num_pages, float scale, void* o, float* lse,
                          void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_bwd_workspace_size -- bytes of device workspace attn_bwd needs:
 * 8 * B * Hq * ceil(Sq / 128) * 128 (two fp32 row statistics per query row,
 * padded to whole 128-row tiles).  0 for invalid arguments.
 */
size_t attn_bwd_workspace_size(int B, int Hq, int Sq);

/*
 * attn_bwd -- backward pass of attn_fwd_masked, recomputing the probabilities
 * from the saved log-sum-exp.
 * Source: "Attention Kernel", section "Backward 与重计算" (the backward
 * recomputes the local probabilities from Q, K, V, the output and the
 * log-sum-exp, with the forward's softmax scale, mask and GQA head mapping,
 * and its accumulation must be free of races); "Attention 算子加速史", FAQ Q1
 * (recompute rather than store the attention matrix).
 *   With P = softmax(scale * Q K^T + M) as in the forward and dO the gradient
 *   of O, the call writes
 *     dV = P^T dO,  dS = P * (dO V^T - rowsum(dO * O)),
 *     dQ = scale * dS K,  dK = scale * dS^T Q,
 *   dK and dV of a KV head summed over the query heads of its group.
 *   q, o, d_o, dq [B, Hq, Sq, d] bf16    k, v, dk, dv [B, Hkv, Sk, d] bf16
 *   lse [B, Hq, Sq] fp32: the forward's LSE for these q, k and mask
 *   (-inf on rows with no visible key, whose gradients are zero).
 *   o is the forward output for the same inputs; dq, dk, dv are written
 *   (every element, including keys masked by k_lens, which get zero).
 *   causal, scale, k_lens: exactly as given to attn_fwd_masked.
 *   workspace: device memory of at least attn_bwd_workspace_size(B, Hq, Sq)
 *   bytes, 16-byte aligned, owned by the caller; its contents on entry are
 *   ignored and it must not be shared with a concurrent call.
 *   Deterministic: every output element is written by one CTA in a fixed
 *   order (no atomics), so repeated calls give identical bits.
 *   Launches: three kernels on `stream` (row statistics, dK/dV, dQ); dQ is
 *   launched as a programmatic dependent of dK/dV, whose outputs it does not
 *   read, and does not complete before dK/dV has.
 * Errors: as attn_fwd_masked, plus INVALID_ARG for a NULL o, lse, d_o, dq or
 * workspace (dk, dv when Sk > 0), ALIGNMENT (o, d_o, dq, dk, dv, workspace
 * need 16 bytes, lse 4), WORKSPACE when workspace_bytes is too small.  Sk = 0
 * only zero-fills dq.
 */
int attn_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
             const void* d_o, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq, int Sk,
             int d, int causal, float scale, const int32_t* k_lens, void* workspace,
             size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_bwd_window -- backward pass of attn_fwd_window (causal, with a sliding
 * window or a prefix-LM mask).
 * Source: "Attention Kernel", section "Backward 与重计算" (the forward's mask
 * applies unchanged) and section "可编程 mask" (window and prefix rules).
 *   Arguments and layouts as attn_bwd (causal implied); window, prefix
 *   exactly as given to attn_fwd_window (>= 0, not both > 0); the workspace is
 *   attn_bwd_workspace_size(B, Hq, Sq) bytes.  Keys no visible pair reaches
 *   get zero dK, dV; rows with no visible key get zero dQ.
 * Errors: as attn_bwd, plus INVALID_ARG for a negative window or prefix, or both.
 */
int attn_bwd_window(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* d_o, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int Sq,
                    int Sk, int d, float scale, const int32_t* k_lens, int window, int prefix,
                    void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_bwd_block_sparse -- backward pass of attn_fwd_block_sparse.
 * Source: as attn_bwd_window; "可编程 mask" (block-level sparsity).
 *   block_mask, mask_heads exactly as given to attn_fwd_block_sparse: uint8
 *   [B, mask_heads, ceil(Sq/128), ceil(Sk/128)] device array, mask_heads 1 or
 *   Hq; 0 hides the 128 x 128 block, which is then neither loaded nor
 *   computed (for units of up to 4096 candidate blocks; larger ones stream
 *   it and weight it zero).  Other arguments as attn_bwd.
 * Errors: as attn_bwd, plus INVALID_ARG for a NULL block_mask or another
 * mask_heads.
 */
int attn_bwd_block_sparse(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* d_o, void* dq, void* dk, void* dv, int B,
                          int Hq, int Hkv, int Sq, int Sk, int d, int causal, float scale,
                          const int32_t* k_lens, const uint8_t* block_mask, int mask_heads,
                          void* workspace, size_t workspace_bytes, attn_stream_t stream);

/*
 * attn_bwd_varlen_workspace_size -- bytes of device workspace attn_bwd_varlen
 * needs: 8 * B * Hq * ceil(max_seqlen_q / 128) * 128 (two fp32 row statistics
 * per query row, each sequence padded to max_seqlen_q in whole 128-row tiles).
 * 0 for invalid arguments.
 */
size_t attn_bwd_varlen_workspace_size(int B, int Hq, int max_seqlen_q);

/*
 * attn_bwd_varlen -- backward pass of attn_fwd_varlen (a ragged, packed batch).
 * Source: "Attention Kernel", section "Backward 与重计算" (the backward uses
 * the forward's scale, mask and head mapping, packed-sequence boundaries must
 * agree with the forward's, and accumulation must be free of races), and
 * section "Paged 与 ragged KV" (a ragged batch is a list of sequences given by
 * cumulative lengths, each attended on its own).
 *   Sequence b owns query tokens [cu_seqlens_q[b], cu_seqlens_q[b+1]) and keys
 *   [cu_seqlens_k[b], cu_seqlens_k[b+1]); its gradients are those attn_bwd
 *   gives for that sequence alone (bottom-right causal alignment when causal).
 *   q, o, d_o, dq [total_q, Hq, d] bf16   k, v, dk, dv [total_k, Hkv, d] bf16
 *   lse [Hq, total_q] fp32 (attn_fwd_varlen's layout)
 *   cu_seqlens_q / cu_seqlens_k: device int32 [B + 1], non-decreasing from 0.
 *   max_seqlen_q / max_seqlen_k bound every sequence's query / key length.
 *   dq rows and dk, dv rows of every valid sequence are written (keys no query
 *   sees get zero); tokens outside every sequence are not touched.
 *   workspace: at least attn_bwd_varlen_workspace_size(B, Hq, max_seqlen_q)
 *   bytes, 16-byte aligned, caller-owned, not shared with a concurrent call.
 *   Deterministic (no atomics), as attn_bwd.
 * Errors: INVALID_ARG (NULL pointers, B/Hq/Hkv < 1, Hq % Hkv != 0, totals or
 * maxima out of range), UNSUPPORTED (d not 64 or 128), ALIGNMENT (tensors 16
 * bytes, lse and offsets 4), WORKSPACE.  A sequence whose offsets are not
 * valid (decreasing, outside [0, total], or longer than the maxima) is skipped
 * -- none of its rows is written -- and sets ATTN_DEVERR_BAD_LENGTH.
 * total_q = 0 does nothing; total_k = 0 only zero-fills dq.
 */
int attn_bwd_varlen(const void* q, const void* k, const void* v, const void* o, const float* lse,
                    const void* d_o, void* dq, void* dk, void* dv, const int32_t* cu_seqlens_q,
                    const int32_t* cu_seqlens_k, int B, int Hq, int Hkv, long long total_q,
                    long long total_k, int max_seqlen_q, int max_seqlen_k, int d, int causal,
                    float scale, void* workspace, size_t workspace_bytes, attn_stream_t stream);

/* attn_strerror -- static description of an attn_status value. */
const char* attn_strerror(int status);

/* attn_split_tokens -- the fixed number of tokens per decode split. */
int attn_split_tokens(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_ATTN_H_ */
