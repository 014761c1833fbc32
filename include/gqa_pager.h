/*
 * gqa_pager.h -- host-side page bookkeeping for the paged K/V cache of gqa_decode.h.
 *
 * The tiny-llm "优化" page preallocates the whole K/V cache once (section "已实现的优化",
 * item 2: KVCacheManager, no allocation during decode), keeps it paged (table "计划中的
 * 优化", row "分页 KV（策略 1）": block table + scatter/gather) and lists continuous
 * batching as the scheduler-side next step (row "连续批处理"); the TensorRT page on
 * in-flight batching names the same serving pattern.  This is that bookkeeping, kept
 * outside the kernels: which pool pages each sequence slot owns, in token order, so that
 * a step's block table, positions and lengths can be handed to gqa_kv_append /
 * gqa_paged_decode_attn / gqa_decode_step.
 *
 * Model.  A pager owns the ids 0 .. num_pages-1 of one preallocated pool (the pool's
 * memory stays with the caller) and max_seqs sequence slots.  Slot s holds a length
 * L_s >= 0 and the pages of its first ceil(L_s / page_size) blocks: token t of slot s is
 * row t % page_size of page block_table[s][t / page_size].  A page belongs to at most one
 * slot; pages of no slot are on a free list (last freed, first reused).  Table entries
 * past a slot's pages are -1.
 *
 * Every mutating call is all-or-nothing: on an error nothing changes.  Errors:
 * GQA_ERR_INVALID_ARG (bad slot, negative count, duplicate slot in a step, a length
 * beyond max_blocks_per_seq * page_size), GQA_ERR_OUT_OF_PAGES (the free list is too
 * short), with gqa_last_error_string() explaining.  Calls are host-only, never touch a
 * GPU, and are not thread-safe: one pager is used by one thread at a time.
 */
#ifndef GQA_PAGER_H_
#define GQA_PAGER_H_

#include <stdint.h>

#include "gqa_decode.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct gqa_pager gqa_pager; /* opaque */

/* A pager over num_pages pages of page_size tokens for max_seqs slots of at most
 * max_blocks_per_seq pages each; every slot starts empty, every page free.  *out is
 * set on success (release it with gqa_pager_destroy). */
gqa_status gqa_pager_create(int num_pages, int page_size, int max_seqs, int max_blocks_per_seq,
                            gqa_pager** out);
void gqa_pager_destroy(gqa_pager* pager);

/* Slot seq grows by n_tokens (>= 0) tokens, taking the pages its new blocks need from the
 * free list (a prompt's tokens, or a draft of several tokens). */
gqa_status gqa_pager_extend(gqa_pager* pager, int seq, int n_tokens);

/* One decode step: every slot seqs[0..n) grows by one token.  positions[i] receives the
 * new token's index (the slot's length before the step) and seq_lens[i] its length after,
 * the layouts gqa_kv_append and gqa_paged_decode_attn take for a batch in that order.
 * Either output may be NULL.  A slot may appear once. */
gqa_status gqa_pager_step(gqa_pager* pager, const int32_t* seqs, int n, int32_t* positions,
                          int32_t* seq_lens);

/* Slot seq shrinks to new_len tokens (0 <= new_len <= its length), returning the pages
 * of blocks past the new end to the free list (rejected draft tokens, a finished
 * sequence with new_len 0). */
gqa_status gqa_pager_truncate(gqa_pager* pager, int seq, int new_len);

/* Block-table rows and lengths of slots seqs[0..n), in that order, into host buffers
 * block_table[n][max_blocks_per_seq] (entries past a slot's pages -1) and seq_lens[n]
 * (either may be NULL): the batch a decode call reads. */
gqa_status gqa_pager_gather(const gqa_pager* pager, const int32_t* seqs, int n, int32_t* block_table,
                            int32_t* seq_lens);

/* Pages on the free list; length of a slot (-1 for a bad slot). */
int gqa_pager_free_pages(const gqa_pager* pager);
int gqa_pager_seq_len(const gqa_pager* pager, int seq);

#ifdef __cplusplus
}
#endif

#endif /* GQA_PAGER_H_ */
