/*
 * gqa_decode.h -- C ABI of the B200 (sm_100a) paged GQA/MQA decode-attention library.
 *
 * The library computes, for one new query token per sequence,
 *
 *     out[b, h, :] = sum_t softmax_t( scale * <q[b, h, :], K_b[t, kvh(h), :]> ) * V_b[t, kvh(h), :]
 *
 * over the sequence's cached keys/values K_b, V_b, t in [0, seq_lens[b]), where
 * the cache is paged and addressed through a per-sequence block table.  It also
 * provides the scatter that writes each step's new K/V row into its page.
 *
 * Sources (web pages the method is described on):
 *   - "TensorRT对Multi-Query Attention的专项优化支持": each decoded token re-reads all
 *     cached K/V of its sequence (the bandwidth-bound step); MHA keeps K_i, V_i per
 *     head, MQA shares one K, V among all query heads (cache h*d_k*s -> d_k*s);
 *     multi-head Q against shared K/V is computed without copying or broadcasting
 *     K/V; QK^T and AV with tiled shared-memory K/V prefetch; fixed-length pages
 *     ("Page-Based管理机制").  Its plugin entry launch_mqa_kernel(q, k, v, out,
 *     batch, heads, seq_q, seq_kv, head_dim, stream) is the model for the call shape.
 *   - tiny-llm "优化" page: GQA (num_kv_heads may differ from num_heads, section 3);
 *     preallocated KV cache and its size formula (section 2); paged KV "strategy 1"
 *     = block table + scatter/gather; FlashDecoding for long-context decode
 *     (planned-optimisation table).
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *   All tensor arguments are DEVICE pointers to row-major, contiguous memory on the
 *   current CUDA device, owned by the caller; the library never frees or retains them
 *   beyond the call.  bf16 means IEEE bfloat16 stored as 16-bit words.
 *
 *     q, out             [num_seqs, num_heads, head_dim]                 bf16
 *     k_pages, v_pages   [num_pages, num_kv_heads, page_size, head_dim]   bf16
 *     block_table        [num_seqs, max_blocks_per_seq]                   int32
 *     seq_lens           [num_seqs]                                       int32
 *     positions          [num_seqs]                                       int32
 *     k_new, v_new       [num_seqs, num_kv_heads, head_dim]               bf16
 *
 *   Token t of sequence b is slot (t % page_size) of page block_table[b][t / page_size];
 *   query head h reads kv head h / (num_heads / num_kv_heads).  Block-table entries
 *   past ceil(seq_lens[b] / page_size) are never used and may hold any value (the
 *   decode kernels load rows of the table 32 entries at a time, so such entries inside
 *   the [num_seqs, max_blocks_per_seq] array may be loaded, never dereferenced).
 *
 *   `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Calls
 *   only enqueue work: they never synchronise the stream and never read device data
 *   on the host.
 *
 *   Errors: a negative gqa_status.  Argument errors are detected on the host before
 *   anything is launched, and gqa_last_error_string() explains them.  Errors that
 *   depend on device data (a page id outside [0, num_pages), a position or seq_len
 *   beyond max_blocks_per_seq * page_size, a negative length, a bounded wait that
 *   ran out) cannot be seen at launch time: the kernels skip the offending work,
 *   never fault or trap, and set a per-device error word that
 *   gqa_check_device_error() reports.
 *
 *   Scratch memory: gqa_paged_decode_attn needs a per-device workspace (split
 *   partial results and per-segment arrival counters).  The library allocates it with
 *   cudaMalloc on the first call per device and grows it when a call needs more;
 *   it is freed at process exit.  Calls on different streams of the same device that
 *   overlap in time share that workspace and must not run concurrently.
 */
#ifndef GQA_DECODE_H_
#define GQA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  GQA_OK = 0,
  GQA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, misaligned pointer        */
  GQA_ERR_UNSUPPORTED = -2,   /* valid but not built: head_dim, page_size, limits  */
  GQA_ERR_CUDA = -3,          /* a CUDA runtime/driver call failed                 */
  GQA_ERR_DEVICE_BOUNDS = -4, /* device-side index out of range (work skipped)     */
  GQA_ERR_TIMEOUT = -5,       /* a kernel's bounded wait ran out (work skipped)    */
  GQA_ERR_OUT_OF_PAGES = -6   /* gqa_pager.h: the free list is too short           */
} gqa_status;

/*
 * gqa_kv_append -- scatter one new K and V row per (sequence, kv head) into the
 * paged cache (the "scatter" half of the block-table scheme on the tiny-llm
 * "优化" page; the decode step's "append pos").
 *
 *   k_pages[block_table[b][p / page_size], kvh, p % page_size, :] = k_new[b, kvh, :]
 *   v_pages[...same slot...]                                      = v_new[b, kvh, :]
 *   with p = positions[b], for every b < num_seqs and kvh < num_kv_heads.
 *
 * Bits are copied unchanged (bit-exact); no other byte of the pools is written.
 * Requirements: head_dim % 8 == 0, page_size >= 1, all bf16 pointers 16-byte
 * aligned, num_seqs >= 0 (0 launches nothing).  A position outside
 * [0, max_blocks_per_seq * page_size) or a page id outside [0, num_pages) skips that
 * sequence's row and sets GQA_ERR_DEVICE_BOUNDS in the device error word.
 */
gqa_status gqa_kv_append(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                         const int32_t* block_table, const int32_t* positions, int num_seqs,
                         int num_kv_heads, int head_dim, int page_size, int max_blocks_per_seq,
                         int num_pages, void* stream);

/*
 * gqa_paged_decode_attn -- decode attention of one query token per sequence over the
 * paged cache, with num_heads query heads sharing num_kv_heads K/V heads (MQA when
 * num_kv_heads == 1, MHA when equal, GQA between): the definition at the top of this
 * file, written to out as bf16 (round to nearest even) from fp32 accumulation.
 *
 * Each kv head's K/V are read from HBM once for all of its query heads.  Long
 * contexts are split across the GPU (FlashDecoding, named on the tiny-llm page);
 * partial results are merged with their log-sum-exp: inside the same launch for
 * groups of up to 16 query heads per kv head, by a second kernel on the same stream
 * (launched to overlap the first one's end) for larger groups.
 *
 *   scale           multiplier of q.k (usually 1/sqrt(head_dim)), finite.
 *   seq_lens[b]     context length of sequence b including any token appended this
 *                   step; 0 gives an all-zero output row.
 * Requirements: head_dim in {64, 128}; page_size a multiple of 16 in [16, 256];
 * num_heads % num_kv_heads == 0; q 16-byte and out 8-byte aligned; k_pages, v_pages 16-byte
 * aligned; num_seqs <= 65536.  Slots at or beyond seq_lens[b] and unused pages may
 * hold any bits (NaN included) without affecting out.
 */
gqa_status gqa_paged_decode_attn(const void* q, const void* k_pages, const void* v_pages,
                                 const int32_t* block_table, const int32_t* seq_lens, void* out,
                                 int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                 int page_size, float scale, int max_blocks_per_seq,
                                 int num_pages, void* stream);

/*
 * gqa_decode_step -- one decode step: gqa_kv_append of this step's K/V rows (at
 * positions[b]), then gqa_paged_decode_attn over seq_lens[b] tokens, on `stream`.
 * Same arguments, layouts, requirements and errors as the two calls.  The decode launch
 * overlaps the append (programmatic dependent launch): its prologue and block-table
 * reads run while the append finishes, and its first K/V copy waits for it.  This is
 * the step tiny-llm's "优化" page describes (append position, then attention over the
 * block table) as one call.  Calls never synchronise or read device data on the host, so
 * after a first call on the device (which sets up the workspace) the step can be captured
 * in a CUDA graph and replayed with new contents of the same buffers.
 */
gqa_status gqa_decode_step(const void* q, const void* k_new, const void* v_new, void* k_pages,
                           void* v_pages, const int32_t* block_table, const int32_t* positions,
                           const int32_t* seq_lens, void* out, int num_seqs, int num_heads,
                           int num_kv_heads, int head_dim, int page_size, float scale,
                           int max_blocks_per_seq, int num_pages, void* stream);

/*
 * Several query tokens per sequence (speculative verification, chunked prefill over the
 * cache).  The MQA plugin's entry point on the TensorRT MQA page carries a query length
 * (seq_q) beside the KV length; here the q_len query tokens of sequence b are its q_len
 * newest tokens, at positions seq_lens[b] - q_len .. seq_lens[b] - 1, and query token i
 * attends to positions 0 .. seq_lens[b] - q_len + i: itself and everything before it,
 * as one decode step per token would.  A token whose window is empty (seq_lens[b] <
 * q_len - i) gets zeros.  q_len = 1 is gqa_paged_decode_attn.
 *
 * gqa_kv_append_multi -- q_len new rows per sequence: k_new, v_new [num_seqs, q_len,
 *   num_kv_heads, head_dim]; row i of sequence b goes to position positions[b] + i (all
 *   of them inside max_blocks_per_seq * page_size, else that sequence's rows are skipped
 *   and reported as GQA_ERR_DEVICE_BOUNDS).  Otherwise as gqa_kv_append.
 * gqa_paged_multi_query_attn -- q, out [num_seqs, q_len, num_heads, head_dim] bf16; the
 *   other arguments, layouts, requirements and errors as gqa_paged_decode_attn.  Each kv
 *   head's K/V are read once for all q_len x (num_heads / num_kv_heads) query rows; that
 *   product must be <= 128 when q_len > 1 (GQA_ERR_UNSUPPORTED otherwise).
 * gqa_multi_query_step -- gqa_kv_append_multi, then gqa_paged_multi_query_attn, as
 *   gqa_decode_step does for one token (the attention launch overlaps the append).
 */
gqa_status gqa_kv_append_multi(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                               const int32_t* block_table, const int32_t* positions, int num_seqs,
                               int q_len, int num_kv_heads, int head_dim, int page_size,
                               int max_blocks_per_seq, int num_pages, void* stream);
gqa_status gqa_paged_multi_query_attn(const void* q, const void* k_pages, const void* v_pages,
                                      const int32_t* block_table, const int32_t* seq_lens, void* out,
                                      int num_seqs, int q_len, int num_heads, int num_kv_heads,
                                      int head_dim, int page_size, float scale, int max_blocks_per_seq,
                                      int num_pages, void* stream);
gqa_status gqa_multi_query_step(const void* q, const void* k_new, const void* v_new, void* k_pages,
                                void* v_pages, const int32_t* block_table, const int32_t* positions,
                                const int32_t* seq_lens, void* out, int num_seqs, int q_len,
                                int num_heads, int num_kv_heads, int head_dim, int page_size,
                                float scale, int max_blocks_per_seq, int num_pages, void* stream);

/*
 * 8-bit (e4m3) K/V cache.  The TensorRT MQA page calibrates Q, K and V separately with
 * their own per-tensor scales in 8-bit mode (one shared scale loses precision to their
 * different ranges); the TensorRT-LLM guide names FP8 for throughput.  Here the pools
 * hold e4m3 codes (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; no infinities;
 * S.1111.111 is NaN; largest value 448) and K and V each carry one fp32 scale per kv
 * head (k_scales, v_scales: [num_kv_heads] device arrays; a per-tensor scale is the case
 * of equal entries).  A cached value is code * scale of its kv head.  The pools take
 * half the bytes of bf16 ones, the quantity decode attention is bound by.
 *
 *     k_pages, v_pages   [num_pages, num_kv_heads, page_size, head_dim]   e4m3 codes (uint8)
 *
 * Writing a bf16 value x stores the code nearest to the fp32 quotient x / scale (IEEE
 * division, round to nearest even), saturating to +-448; NaN stays NaN.  q, out,
 * k_new, v_new stay bf16.
 *
 * gqa_kv_quantize_fp8 -- codes of a whole bf16 pool: dst[p, kvh, t, :] = code of
 *   src[p, kvh, t, :] / scales[kvh] (src [num_pages, num_kv_heads, page_size, head_dim]
 *   bf16, dst the same shape in e4m3; both 16-byte aligned; head_dim % 16 == 0).
 * gqa_kv_append_fp8 -- gqa_kv_append into coded pools, K rows with k_scales and V rows
 *   with v_scales; same arguments otherwise (head_dim % 16 == 0, pools 16-byte aligned).
 * gqa_paged_decode_attn_fp8 -- gqa_paged_decode_attn over coded pools: the definition at
 *   the top of this file with K_b, V_b the cached values code * scale.  The kernel widens
 *   codes to fp16 (exactly), converts q to fp16 (round to nearest: exact for 2^-17 <=
 *   |q| <= 65504, saturating above) and accumulates in fp32.  Requirements as
 *   gqa_paged_decode_attn, and num_heads / num_kv_heads <= 16 (GQA_ERR_UNSUPPORTED
 *   otherwise).
 * gqa_decode_step_fp8 -- gqa_kv_append_fp8, then gqa_paged_decode_attn_fp8, as
 *   gqa_decode_step does for a bf16 cache.
 */
gqa_status gqa_kv_quantize_fp8(const void* src, void* dst, const float* scales, int num_pages,
                               int num_kv_heads, int page_size, int head_dim, void* stream);
gqa_status gqa_kv_append_fp8(const void* k_new, const void* v_new, void* k_pages, void* v_pages,
                             const float* k_scales, const float* v_scales, const int32_t* block_table,
                             const int32_t* positions, int num_seqs, int num_kv_heads, int head_dim,
                             int page_size, int max_blocks_per_seq, int num_pages, void* stream);
gqa_status gqa_paged_decode_attn_fp8(const void* q, const void* k_pages, const void* v_pages,
                                     const float* k_scales, const float* v_scales,
                                     const int32_t* block_table, const int32_t* seq_lens, void* out,
                                     int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                     int page_size, float scale, int max_blocks_per_seq, int num_pages,
                                     void* stream);
gqa_status gqa_decode_step_fp8(const void* q, const void* k_new, const void* v_new, void* k_pages,
                               void* v_pages, const float* k_scales, const float* v_scales,
                               const int32_t* block_table, const int32_t* positions,
                               const int32_t* seq_lens, void* out, int num_seqs, int num_heads,
                               int num_kv_heads, int head_dim, int page_size, float scale,
                               int max_blocks_per_seq, int num_pages, void* stream);

/*
 * gqa_paged_decode_attn_noalloc -- the same decode attention as gqa_paged_decode_attn
 * (same arguments, layouts and result), for callers that cannot allocate device memory:
 * an engine that has already reserved nearly all of the GPU for its own caching
 * allocator or KV pool (an extra cudaMalloc would fail or fragment it), a step loop that
 * cannot afford the device-wide synchronisation cudaMalloc/cudaFree imply, or a plugin
 * whose host framework hands it no workspace.  The pages describe no such variant; it
 * exists only for these callers.
 *
 * Scratch: instead of the per-device workspace, the call uses a fixed 16 MiB array
 * compiled into the library's device image.  Every GPU that loads the library holds
 * that array until the process exits.  This call never allocates: no cudaMalloc, no
 * cudaFree, no allocating library routine.
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call before any
 *     stream capture.
 *   - Sharing: all calls use the same array and it keeps the last call's contents; each
 *     call clears the part that must start at zero (error word, split counters) on
 *     `stream`.  Calls whose execution overlaps on the GPU (other streams, other host
 *     threads) race on the array and must be ordered by the caller.
 *   - Limits: at most 16384 segments (num_seqs * num_kv_heads * head tiles; a head tile
 *     holds 8 or 16 query heads for groups up to 16, up to 128 otherwise); when the
 *     split partials of the default number of workers do not fit, fewer workers are
 *     used.  A call beyond the limits returns GQA_ERR_UNSUPPORTED and launches nothing.
 *   - Device-side errors (bad page ids or lengths, a bounded wait that ran out) skip
 *     the offending work as in gqa_paged_decode_attn and set an error word kept in the
 *     array itself.  The word accumulates across calls until gqa_check_device_error,
 *     which reads and clears it together with the regular one (with cudaMemcpy and
 *     cudaMemset on the array: that call allocates nothing either).
 */
gqa_status gqa_paged_decode_attn_noalloc(const void* q, const void* k_pages, const void* v_pages,
                                         const int32_t* block_table, const int32_t* seq_lens,
                                         void* out, int num_seqs, int num_heads, int num_kv_heads,
                                         int head_dim, int page_size, float scale,
                                         int max_blocks_per_seq, int num_pages, void* stream);

/*
 * gqa_check_device_error -- synchronise `stream`, then read and clear the current
 * device's error words: the workspace's (every call but the allocation-free decode) and
 * the allocation-free decode's own, each only if a call has set it up on this device
 * (this call creates and allocates nothing).  Returns GQA_OK, GQA_ERR_DEVICE_BOUNDS,
 * GQA_ERR_TIMEOUT (takes precedence when both are set; it also resets the decode
 * workspace counters a timed-out launch may have left behind) or GQA_ERR_CUDA.
 */
gqa_status gqa_check_device_error(void* stream);

/* Human-readable message of the last error returned on this host thread. */
const char* gqa_last_error_string(void);

/*
 * gqa_kv_cache_bytes -- bytes of a bf16 K+V cache for one sequence:
 * 2 x num_layers x num_kv_heads x head_dim x seq_len x 2 bytes (tiny-llm "优化" page,
 * section 2).  Returns 0 for negative arguments.
 */
size_t gqa_kv_cache_bytes(int num_layers, int num_kv_heads, int head_dim, int64_t seq_len);

/*
 * gqa_set_num_workers -- number of split workers (CTAs) used by the next
 * gqa_paged_decode_attn calls on this process; 0 (default) picks it from the SM count.
 * A fixed count changes how the context is split, never the result beyond fp32
 * rounding order; tests use it to force many or few splits.  Returns
 * GQA_ERR_INVALID_ARG for n < 0.
 */
gqa_status gqa_set_num_workers(int n);

/*
 * gqa_set_wait_limit_ns -- upper bound on any single wait inside the kernels
 * (default 1e9 ns).  When `arm_without_copy` is non-zero the next decode launches arm
 * their copy barriers without issuing the copies, so every wait runs out: this
 * exercises the GQA_ERR_TIMEOUT path without faulting anything.  Tests only.
 */
gqa_status gqa_set_wait_limit_ns(int64_t limit_ns, int arm_without_copy);

/* Kernels launched by this library since the process started (all devices). */
uint64_t gqa_launch_count(void);

/* ABI version of this header: 1. */
int gqa_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* GQA_DECODE_H_ */
