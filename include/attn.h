/*
 * attn.h - C ABI of the B200 (sm_100a) exact softmax attention library.
 *
 * Two operations, both exact scaled-dot-product attention
 *     O = softmax(Q K^T * scale + M) V
 * computed with an online softmax so that the score matrix never leaves the
 * chip ("Module 5. Modern Attention Mechanisms", section 4, the SDPA
 * definition; section 8, the FlashAttention recurrence):
 *
 *   attn_prefill       - every query row of a sequence against its own keys,
 *                        full / causal / sliding-window mask, grouped-query
 *                        heads (Hkv divides Hq; Hkv == Hq is MHA, Hkv == 1 MQA).
 *   attn_decode_paged  - one query token per sequence against a paged K/V
 *                        cache addressed through a block table
 *                        ("Module 09: Efficient Attention", "The Block Table"),
 *                        split along the sequence and merged by log-sum-exp
 *                        ("Inference attention" post, section "FlashDecoding").
 *   attn_decode_paged_window - the same decode with a sliding window, the
 *                        StreamingLLM sink positions and gpt-oss's learned
 *                        per-head sink logit ("Modern Attention Mechanisms",
 *                        sections 9, 10 and 12).
 *   attn_prefill_paged - the newest Nq positions of each sequence against its
 *                        paged context (prefix / chunked prefill).
 *   attn_prefill_backward - dQ, dK, dV of attn_prefill for an output gradient
 *                        dO, recomputing S and P tile by tile from the saved
 *                        LSE ("Inference attention" post, "FlashAttention").
 *   attn_mla_decode_paged - absorbed Multi-head Latent Attention decode over a
 *                        paged latent cache ("Modern Attention Mechanisms",
 *                        section 7; "Module 09", the MLA section).
 *
 * Conventions shared by every entry point:
 *   - Pointers named q, k, v, o, lse, k_cache, v_cache, block_table, seq_lens,
 *     out, workspace and status are DEVICE pointers owned by the caller; the
 *     library never allocates, frees or retains them.
 *   - bf16 means IEEE bfloat16 stored in 2 bytes; tensors are dense,
 *     row-major ("C order") in the layouts stated per call, and every base
 *     pointer is 16-byte aligned.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; 0 = legacy default
 *     stream). A return of ATTN_OK means the work was validated and enqueued.
 *   - Host-side argument errors return a negative status and launch nothing.
 *   - Device-side checks (block-table entries, seq_lens, bounded waits) cannot
 *     be reported by the return value; they OR a status code into *status
 *     (when status != NULL) and turn the affected output rows into NaN. The
 *     caller zeroes *status before the call and reads it after synchronising.
 *   - head dimension d must be 64 or 128 (else ATTN_ERR_UNSUPPORTED).
 *   - Query head h reads K/V head h / (Hq / Hkv): consecutive groups
 *     ("Modern Attention Mechanisms", section 6).
 */
#ifndef ATTN_B200_H
#define ATTN_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ATTN_API __attribute__((visibility("default")))
#else
#define ATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* attn_stream_t; /* the same handle as cudaStream_t */

enum attn_status {
  ATTN_OK = 0,
  ATTN_ERR_INVALID_ARG = -1,  /* bad size, null pointer, misalignment, Hq % Hkv != 0, ... */
  ATTN_ERR_UNSUPPORTED = -2,  /* valid request this build does not implement (e.g. d = 96) */
  ATTN_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed (launch, tensor map) */
  ATTN_ERR_DEVICE_CHECK = -4, /* device bit: a block-table entry or seq_len was out of range */
  ATTN_ERR_TIMEOUT = -5,      /* device bit: a bounded pipeline wait expired */
  ATTN_ERR_WORKSPACE = -6     /* workspace pointer NULL or smaller than attn_decode_workspace_bytes */
};

/* Device-side status bits OR-ed into *status. */
#define ATTN_STATUS_BIT_DEVICE_CHECK 0x1
#define ATTN_STATUS_BIT_TIMEOUT 0x2

enum attn_mask_kind {
  ATTN_MASK_FULL = 0,          /* every key visible */
  ATTN_MASK_CAUSAL = 1,        /* key j visible to query i iff j <= i */
  ATTN_MASK_SLIDING_WINDOW = 2 /* key j visible iff 0 <= i - j < window (window includes i) */
};

/*
 * attn_prefill - exact attention of N query rows against N keys per head.
 *
 * Defined by "Modern Attention Mechanisms", section 4: softmax over keys of
 * Q K^T * scale with an additive mask, causality p_k <= p_q and the window
 * 0 <= p_q - p_k < W (W positions including the current one); and section 6
 * for the GQA head map. Query and key positions are aligned (square N).
 *
 *   q     [B, Hq,  N, d] bf16      read
 *   k, v  [B, Hkv, N, d] bf16      read
 *   o     [B, Hq,  N, d] bf16      written: softmax(...) V, rounded to nearest even
 *   lse   [B, Hq,  N]    fp32      written when non-NULL: natural-log log-sum-exp
 *                                  of the scaled scores over the visible keys
 *   mask_kind  ATTN_MASK_*; window is read only for ATTN_MASK_SLIDING_WINDOW and
 *              must then be >= 1 (window >= N behaves exactly as CAUSAL).
 *   scale      the score scale, typically 1/sqrt(d); must be finite and > 0.
 *   status     device int32 or NULL (bounded-wait timeout bit).
 *
 * Every row of every mask kind sees at least its own key, so no row is fully
 * masked. Errors: ATTN_ERR_INVALID_ARG for non-positive sizes, Hq % Hkv != 0,
 * NULL q/k/v/o, misaligned pointers, window < 1 with SLIDING_WINDOW, bad scale;
 * ATTN_ERR_UNSUPPORTED for d not in {64, 128}; ATTN_ERR_CUDA on launch failure.
 */
ATTN_API int attn_prefill(const void* q, const void* k, const void* v, void* o, float* lse, int B, int Hq, int Hkv,
                 int N, int d, int mask_kind, int window, float scale, int32_t* status, attn_stream_t stream);

/*
 * attn_prefill_paged - prefix (chunked) prefill: the newest Nq positions of
 * each sequence attend to its whole cached context, read through a block
 * table.
 *
 * Positions are bottom-right aligned ("Modern Attention Mechanisms", section 4:
 * after a prefix of length P, query row i has position P + i): sequence b has
 * seq_lens[b] cached tokens (its Nq new tokens already appended, as in
 * "Module 09: Efficient Attention", "Chunked Prefill"), so query row i sits at
 * position seq_lens[b] - Nq + i. Key j is visible to it under CAUSAL iff
 * j <= seq_lens[b] - Nq + i, under SLIDING_WINDOW iff additionally
 * seq_lens[b] - Nq + i - j < window, under FULL iff j < seq_lens[b]. The cache
 * layout and addressing are those of attn_decode_paged.
 *
 *   q            [B, Hq, Nq, d] bf16                        read
 *   k_cache,
 *   v_cache      [num_blocks, block_size, Hkv, d] bf16      read (only referenced slots)
 *   block_table  [B, max_blocks_per_seq] int32              read: the entries covering
 *                the keys each query row sees must lie in [0, num_blocks)
 *   seq_lens     [B] int32, each in [Nq, max_seq_len]       read
 *   o            [B, Hq, Nq, d] bf16                        written
 *   lse          [B, Hq, Nq] fp32, natural log              written when non-NULL
 *   block_size   16, 32, 64 or 128 (else ATTN_ERR_UNSUPPORTED)
 *   max_seq_len  >= Nq and <= max_blocks_per_seq * block_size
 *   status       device int32 or NULL.
 *
 * A seq_len outside [Nq, max_seq_len] or a needed block-table entry outside
 * the pool is never dereferenced: that sequence's rows of o and lse are NaN
 * and ATTN_STATUS_BIT_DEVICE_CHECK is OR-ed into *status. With seq_lens[b] ==
 * Nq for every b and a contiguous block table this equals attn_prefill.
 *
 * Errors (nothing is launched): ATTN_ERR_INVALID_ARG for NULL or misaligned
 * pointers, non-positive sizes, max_seq_len < Nq, Hq % Hkv != 0,
 * max_blocks_per_seq * block_size < max_seq_len, a bad mask, window or scale;
 * ATTN_ERR_UNSUPPORTED for d other than 64 or 128, another block_size, or
 * B * Hq * Nq of 2^31 or more; ATTN_ERR_CUDA when a launch fails.
 */
ATTN_API int attn_prefill_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                                const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int Nq, int d,
                                int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len,
                                int mask_kind, int window, float scale, int32_t* status, attn_stream_t stream);

/*
 * attn_decode_plan - the split-KV plan attn_decode_paged uses (host only, no
 * GPU needed). Long sequences are cut into chunks of *chunk_tokens tokens
 * (a multiple of 16); each (sequence, K/V head, chunk) is one unit of work
 * ("Inference attention" post, "FlashDecoding": split keys along the
 * sequence so that small batches fill the GPU). A unit covers 16 query
 * heads of a K/V head, or 32 when Hq / Hkv is above 16 (one such CTA takes
 * the place of two). With at least two units per SM the chunks are 2048
 * tokens; with fewer (a single long sequence, a small batch) the chunk count
 * fills whole waves of resident CTAs, each chunk at most 4096 tokens. num_sms
 * is the device's SM count. Returns ATTN_OK or ATTN_ERR_INVALID_ARG.
 */
ATTN_API int attn_decode_plan(int B, int Hq, int Hkv, int max_seq_len, int num_sms, int* chunk_tokens, int* num_splits);

/*
 * attn_decode_workspace_bytes - bytes of device workspace attn_decode_paged
 * needs for these sizes on the current device (partial outputs fp32
 * [B, Hq, splits, d], partial log-sum-exp fp32 [B, Hq, splits], then the
 * split merge's ticket counters and a work counter, a few uint64 per
 * (sequence, K/V head)).
 * Returns 0 for invalid sizes.
 */
ATTN_API size_t attn_decode_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seq_len, int block_size);

/*
 * attn_decode_paged - one new query token per sequence against its whole
 * cached context, read through a block table.
 *
 * Defined by "Module 09: Efficient Attention", "Code: A Paged KV Cache from
 * Scratch": the pool has shape (num_blocks, block_size, num_kv_heads,
 * head_dim) and token t of sequence b sits in slot t % block_size of physical
 * block block_table[b][t / block_size]. The query attends to all seq_lens[b]
 * cached tokens, its own K/V already appended ("USAAIO Lesson 90", part 2), so
 * no mask applies. Split partials are merged with the online softmax's
 * rescaling ("Inference attention" post, "FlashDecoding"), inside the same
 * single launch: the last CTA to finish a sequence's splits merges them (a
 * second, dependent launch merges when a sequence has more partials than one
 * CTA stages at once).
 *
 * Reproducibility: a plan with fixed chunks gives bit-identical results on
 * every call. A plan whose CTAs all fit on the GPU at once (few sequences,
 * no window, at most 16 query heads per K/V head) hands the chunks' 32-token
 * grains to whichever CTA is free at run time, so repeated calls agree to the
 * rounding of a different summation order.
 *
 *   q            [B, Hq, d] bf16                            read
 *   k_cache,
 *   v_cache      [num_blocks, block_size, Hkv, d] bf16      read (only referenced slots)
 *   block_table  [B, max_blocks_per_seq] int32              read: entries
 *                0 .. ceil(seq_lens[b] / block_size) - 1 must lie in [0, num_blocks);
 *                later entries are never read (may hold -1)
 *   seq_lens     [B] int32, each in [1, max_seq_len]        read
 *   o            [B, Hq, d] bf16                            written
 *   lse          [B, Hq] fp32, natural log                  written when non-NULL
 *   block_size   a multiple of 16 (the pages' default is 16)
 *   max_seq_len  <= max_blocks_per_seq * block_size
 *   workspace    device scratch of at least attn_decode_workspace_bytes(...)
 *                bytes, 16-byte aligned; contents on entry are irrelevant
 *                (the counters carry a 32-bit tag that changes with every
 *                call; a counter without this call's tag is taken as zero).
 *                Calls whose kernels overlap on the GPU must not share a
 *                workspace.
 *   status       device int32 or NULL.
 *
 * A referenced block-table entry outside [0, num_blocks) or a seq_len outside
 * [1, max_seq_len] is never dereferenced: the affected rows of o and lse are
 * NaN and ATTN_STATUS_BIT_DEVICE_CHECK is OR-ed into *status.
 *
 * Errors (nothing is launched): ATTN_ERR_INVALID_ARG for NULL or misaligned
 * pointers, non-positive sizes, Hq % Hkv != 0, max_blocks_per_seq *
 * block_size < max_seq_len or a non-positive or non-finite scale;
 * ATTN_ERR_UNSUPPORTED for d other than 64 or 128, block_size not a multiple
 * of 16, B above 65535 or Hkv * ceil(Hq / Hkv / 16) above 65535;
 * ATTN_ERR_WORKSPACE for a missing, misaligned or short workspace;
 * ATTN_ERR_CUDA when the device query or the launch fails.
 */
ATTN_API int attn_decode_paged(const void* q, const void* k_cache, const void* v_cache, const int32_t* block_table,
                      const int32_t* seq_lens, void* o, float* lse, int B, int Hq, int Hkv, int d,
                      int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len, float scale,
                      void* workspace, size_t workspace_bytes, int32_t* status, attn_stream_t stream);

/*
 * attn_decode_window_workspace_bytes - bytes of device workspace
 * attn_decode_paged_window needs for these sizes, window and n_sink (the split
 * plan covers only the sub-blocks a windowed query can see). Equal to
 * attn_decode_workspace_bytes when window == 0 or window >= max_seq_len.
 * Returns 0 for invalid sizes.
 */
ATTN_API size_t attn_decode_window_workspace_bytes(int B, int Hq, int Hkv, int d, int max_seq_len, int block_size,
                                                   int window, int n_sink);

/*
 * attn_decode_paged_window - attn_decode_paged with a sliding window, sink
 * positions and learned sink logits.
 *
 * Defined by "Module 5. Modern Attention Mechanisms": section 4/9 (a window
 * of W positions includes the current one: the query at position
 * n - 1 = seq_lens[b] - 1 sees positions p with 0 <= n - 1 - p < W), section
 * 10 and the mask builder of section 12 (StreamingLLM: the first n_sink
 * positions stay visible beside a finite window), and section 10's gpt-oss
 * sink: each query head h owns a logit sinks[h] that is appended to the row's
 * scaled scores, normalised with them and dropped before the product with V
 * (it takes probability mass and contributes no value).
 *
 * Arguments as for attn_decode_paged, plus
 *   sinks        [Hq] fp32 device array of sink logits (natural-log units, the
 *                same units as scale * q.k), or NULL for none. A non-finite
 *                logit turns that head's rows into NaN and sets
 *                ATTN_STATUS_BIT_DEVICE_CHECK.
 *   window       W >= 1, or 0 for no window (every cached token visible).
 *                W >= max_seq_len behaves as 0.
 *   n_sink       0 <= n_sink <= max_seq_len; n_sink > 0 needs window > 0
 *                (else ATTN_ERR_INVALID_ARG).
 *   workspace    at least attn_decode_window_workspace_bytes(...) bytes.
 *
 *   o            softmax over the visible tokens and the sink column, times V.
 *   lse          log(sum over visible tokens of exp(scale * q.k) + exp(sinks[h])):
 *                the log of the full softmax denominator (without sinks, the
 *                log-sum-exp over the visible tokens).
 *
 * Only table entries of blocks that hold a visible token are read: a rolling
 * cache may leave the entries of evicted middle blocks as -1. Out-of-range
 * entries that are read, and seq_lens outside [1, max_seq_len], are handled
 * as in attn_decode_paged.
 *
 * Errors: those of attn_decode_paged, plus ATTN_ERR_INVALID_ARG for window < 0,
 * n_sink < 0, n_sink > max_seq_len, n_sink > 0 with window == 0, or a
 * misaligned sinks pointer.
 */
ATTN_API int attn_decode_paged_window(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_table, const int32_t* seq_lens, const float* sinks, void* o,
                                      float* lse, int B, int Hq, int Hkv, int d, int num_blocks, int block_size,
                                      int max_blocks_per_seq, int max_seq_len, int window, int n_sink, float scale,
                                      void* workspace, size_t workspace_bytes, int32_t* status,
                                      attn_stream_t stream);

/*
 * attn_prefill_backward_workspace_bytes - bytes of device workspace
 * attn_prefill_backward needs: D = rowsum(dO * O) and LSE * log2(e), each fp32
 * [B, Hq, Npad] with Npad = N rounded up to a multiple of 128. Returns 0 for
 * invalid sizes.
 */
ATTN_API size_t attn_prefill_backward_workspace_bytes(int B, int Hq, int N);

/*
 * attn_prefill_backward - gradients of attn_prefill.
 *
 * The pages say the backward pass recomputes S and P tile by tile instead of
 * storing them ("Inference attention" post, section "FlashAttention"); the
 * gradients are the chain rule of the forward definition ("Module 5. Modern
 * Attention Mechanisms", section 4; head map of section 6):
 *   P = exp(scale Q K^T - LSE) on visible pairs (0 elsewhere),
 *   dV = P^T dO, dP = dO V^T, dS = P * (dP - D), D = rowsum(dO * O),
 *   dQ = scale dS K, dK = scale dS^T Q,
 * with dK and dV of a K/V head summed over the Hq / Hkv query heads that read it.
 *
 *   q, o, d_o    [B, Hq, N, d] bf16                          read (o, lse: attn_prefill's outputs)
 *   k, v         [B, Hkv, N, d] bf16                         read
 *   lse          [B, Hq, N] fp32, natural log                read
 *   dq           [B, Hq, N, d] bf16                          written
 *   dk, dv       [B, Hkv, N, d] bf16                         written
 *   mask_kind, window, scale   as passed to attn_prefill
 *   workspace    at least attn_prefill_backward_workspace_bytes(B, Hq, N)
 *                bytes, 16-byte aligned
 *   status       device int32 or NULL (bounded-wait expiry: NaN outputs and
 *                ATTN_STATUS_BIT_TIMEOUT)
 *
 * Errors: ATTN_ERR_INVALID_ARG for NULL or misaligned tensors, non-positive
 * sizes, Hq % Hkv != 0, a bad mask or scale; ATTN_ERR_UNSUPPORTED for d other
 * than 64 or 128, B or Hq above 65535, or B * Hq * N of 2^31 or more;
 * ATTN_ERR_WORKSPACE for a missing or short workspace.
 */
ATTN_API int attn_prefill_backward(const void* q, const void* k, const void* v, const void* o, const void* d_o,
                                   const float* lse, void* dq, void* dk, void* dv, int B, int Hq, int Hkv, int N,
                                   int d, int mask_kind, int window, float scale, void* workspace,
                                   size_t workspace_bytes, int32_t* status, attn_stream_t stream);

/*
 * attn_mla_decode_workspace_bytes - bytes of device workspace
 * attn_mla_decode_paged needs (fp32 partial latent outputs [B, H, splits, 512]
 * and partial log-sum-exps [B, H, splits]). Returns 0 for invalid or
 * unsupported sizes.
 */
ATTN_API size_t attn_mla_decode_workspace_bytes(int B, int H, int d_latent, int d_rope, int max_seq_len);

/*
 * attn_mla_decode_paged - one new query token per sequence, H heads, against a
 * paged cache of Multi-head Latent Attention rows, in the absorbed form.
 *
 * Defined by "Module 5. Modern Attention Mechanisms", section 7 (with
 * k_t = A c_t and v_t = B c_t: q.k_t = (A^T q).c_t and
 * sum_t p_t v_t = B (sum_t p_t c_t); a separate positional key whose term is
 * added to the logit) and "Module 09: Efficient Attention", the MLA section
 * (key and query are the concatenations [content ; rope], the logit is their
 * dot product over sqrt(d_head + d_h^R), the cache holds d_c + d_h^R numbers
 * per token). Token t of sequence b is row [c_t ; k^R_t] in slot
 * t % block_size of block block_table[b][t / block_size]; head h's query is
 * [A_h^T q^C_h ; q^R_h]; every cached token is visible. The output is the
 * latent sum_t p_t c_t: the caller applies the value up-projection B_h.
 *
 *   q            [B, H, d_latent + d_rope] bf16                         read
 *   cache        [num_blocks, block_size, d_latent + d_rope] bf16       read (only referenced rows)
 *   block_table  [B, max_blocks_per_seq] int32, as for attn_decode_paged read
 *   seq_lens     [B] int32, each in [1, max_seq_len]                     read
 *   o            [B, H, d_latent] bf16                                   written
 *   lse          [B, H] fp32, natural log, or NULL                      written
 *   d_latent, d_rope   must be 512 and 64 (DeepSeek-V2's widths), else
 *                ATTN_ERR_UNSUPPORTED
 *   block_size   16, 32, 64 or 128
 *   scale        the logit scale, 1 / sqrt(d_head + d_rope) per the pages
 *   workspace    at least attn_mla_decode_workspace_bytes(...) bytes, 16-byte aligned
 *
 * Bad referenced table entries and seq_lens are handled as in
 * attn_decode_paged (NaN rows, ATTN_STATUS_BIT_DEVICE_CHECK).
 *
 * Errors (nothing is launched): ATTN_ERR_INVALID_ARG for NULL or misaligned
 * pointers, non-positive sizes, max_blocks_per_seq * block_size < max_seq_len
 * or a non-positive or non-finite scale; ATTN_ERR_UNSUPPORTED for other
 * widths or block sizes, or B above 65535; ATTN_ERR_WORKSPACE for a missing,
 * misaligned or short workspace; ATTN_ERR_CUDA when the device query or a
 * launch fails.
 */
ATTN_API int attn_mla_decode_paged(const void* q, const void* cache, const int32_t* block_table,
                                   const int32_t* seq_lens, void* o, float* lse, int B, int H, int d_latent,
                                   int d_rope, int num_blocks, int block_size, int max_blocks_per_seq,
                                   int max_seq_len, float scale, void* workspace, size_t workspace_bytes,
                                   int32_t* status, attn_stream_t stream);

/*
 * attn_paged_gather - walk every sequence's block table into a contiguous
 * cache (the "gather" of "Module 09: Efficient Attention", "Code: A Paged KV
 * Cache from Scratch"). Bit-exact copy; used to check block-table indexing.
 *
 *   cache        [num_blocks, block_size, Hkv, d] bf16       read
 *   out          [B, Hkv, max_seq_len, d] bf16               written: token t of
 *                sequence b for t < seq_lens[b], zero for the rest
 *   block_table, seq_lens as for attn_decode_paged (seq_lens[b] may be 0 here).
 * Invalid referenced entries: that token's row is NaN and the device-check
 * bit is set.
 *
 * Errors (nothing is launched): ATTN_ERR_INVALID_ARG for NULL or misaligned
 * pointers, non-positive sizes or max_blocks_per_seq * block_size <
 * max_seq_len; ATTN_ERR_UNSUPPORTED for d not a multiple of 8; ATTN_ERR_CUDA
 * when the launch fails.
 */
ATTN_API int attn_paged_gather(const void* cache, const int32_t* block_table, const int32_t* seq_lens, void* out, int B,
                      int Hkv, int d, int num_blocks, int block_size, int max_blocks_per_seq, int max_seq_len,
                      int32_t* status, attn_stream_t stream);

/*
 * attn_decode_paged_noalloc - attn_decode_paged for callers that cannot
 * allocate device memory. No passage of the pages corresponds to it; it
 * exists for the library's users.
 *
 * Some callers cannot call cudaMalloc or hand the library a workspace: code
 * living inside a host framework that owns every device byte through its own
 * allocator, or a latency-critical loop that must not pay for an allocation
 * (which may synchronise the device) on the decode path. This variant takes
 * the same arguments as attn_decode_paged minus workspace/workspace_bytes and
 * keeps the split partials in a static device array of
 * ATTN_DECODE_NOALLOC_SCRATCH_BYTES bytes that the library holds on every GPU
 * it is loaded on until the process exits. It calls no allocating routine.
 *
 *   - Requests whose split workspace (attn_decode_workspace_bytes) exceeds
 *     ATTN_DECODE_NOALLOC_SCRATCH_BYTES are rejected with ATTN_ERR_WORKSPACE
 *     before anything is launched.
 *   - The first call on each device looks up that device's address of the
 *     array (a set-up step, done once per device with the device current);
 *     make that first call before any stream capture. The address is kept
 *     for the life of the process: after cudaDeviceReset (or any teardown of
 *     the device's primary context) it is stale, so do not call this entry
 *     point on that device again in the same process.
 *   - Every call on a device shares the one array and leaves its contents
 *     behind. Nothing in it has to start at zero: each call writes every
 *     partial it later reads, and the merge's ticket counters carry a tag
 *     that changes with every call (the array is zero when the library
 *     loads). Calls whose kernels overlap on the GPU (two streams, or two
 *     host threads) race on the array: serialise them.
 * Outputs, errors and device checks are exactly those of attn_decode_paged.
 */
#define ATTN_DECODE_NOALLOC_SCRATCH_BYTES (32u << 20) /* 32 MiB */
ATTN_API int attn_decode_paged_noalloc(const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_table, const int32_t* seq_lens, void* o, float* lse,
                                       int B, int Hq, int Hkv, int d, int num_blocks, int block_size,
                                       int max_blocks_per_seq, int max_seq_len, float scale, int32_t* status,
                                       attn_stream_t stream);

/* attn_status_string - static English description of a status code. */
ATTN_API const char* attn_status_string(int status);

/* attn_version - library version, major * 10000 + minor * 100 + patch. */
ATTN_API int attn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_B200_H */
