/*
 * pkv_pages.h -- host-side page allocator for the paged KV pools of libpkv:
 * the bookkeeping a continuous-batching loop runs between decode steps.
 *
 * What it does, after the pages: the cache is cut into fixed-size pages,
 * allocated on demand as tokens are generated, named per request by a
 * block table that maps logical positions to physical pages
 * ("TensorRT-LLM Guide: High-Throughput GPU Inference Engine", section
 * "2. Paged KV Cache & Memory Virtualization"); when a sequence finishes its
 * pages return to the pool at once and a waiting request takes the freed
 * batch slot in the next iteration (same page, section "1. In-Flight
 * Batching: Continuous Iteration Scheduling"; "Scaling TensorRT-LLM: Kernel
 * Fusion and Inflight Batching in Production", section "What the Scheduler
 * Actually Does"); pages can be shared by requests with a common prefix,
 * such as a common system prompt ("TensorRT-LLM: NVIDIA's Optimized
 * Inference Engine", section "The paged KV cache, in-flight batching and
 * CUDA graphs").
 *
 * Model: max_batch slots, each free or holding one request with L tokens in
 * the cache (seq_lens[slot] = L) and ceil(L / P) pages or more in its row of
 * the block table (int32 [max_batch][max_blocks_per_seq], -1 past its
 * pages).  Every physical page is free or referenced by one or more slots;
 * a page's reference count is the number of slots whose table names it, and
 * a page returns to the free list when that count drops to zero.  Only full
 * pages are shared (a shared prefix of S tokens shares floor(S / P) pages),
 * so appends, which write position L of the appending slot, never touch a
 * shared page.  The free list is a stack (the most recently freed page is
 * handed out first).  Host memory only; not thread-safe (one scheduler
 * thread); no CUDA call.
 *
 * Errors: every call returns a pkv_status; a failed call changes nothing.
 */
#ifndef PKV_PAGES_H
#define PKV_PAGES_H

#include <stdint.h>

#include "pkv.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pkv_pages pkv_pages;

/* num_pages physical pages of page_size tokens; all pages free, all slots
 * free, the block table all -1, seq_lens all 0. */
pkv_status pkv_pages_create(int num_pages, int page_size, int max_batch, int max_blocks_per_seq,
                            pkv_pages** out);

/* NULL is accepted. */
pkv_status pkv_pages_destroy(pkv_pages* pp);

/* Puts a request with `len` tokens already in the cache (its prefill done)
 * into free slot `slot`, with pages for positions 0 .. len - 1.  If
 * share_slot >= 0, the first floor(share_tokens / P) pages are the ones of
 * that (active) slot's table, shared (reference count + 1); share_tokens
 * must not exceed len nor the sharing slot's length.  The other pages come
 * off the free list.  PKV_ERR_OOM if the free list is too short,
 * PKV_ERR_INVALID_ARG for a busy or bad slot, a bad length or share. */
pkv_status pkv_pages_admit(pkv_pages* pp, int slot, int len, int share_slot, int share_tokens);

/* Before a step that appends q_len tokens to every active slot: makes sure
 * each active slot has pages for positions L .. L + q_len - 1, allocating on
 * a page crossing.  All or nothing: PKV_ERR_OOM (nothing allocated) if the
 * free list cannot cover every slot. */
pkv_status pkv_pages_reserve(pkv_pages* pp, int q_len);

/* After the step: L += q_len for every active slot. */
pkv_status pkv_pages_advance(pkv_pages* pp, int q_len);

/* The request in `slot` is done: every page of its row loses one reference,
 * pages left with none go back on the free list, the slot is free again. */
pkv_status pkv_pages_release(pkv_pages* pp, int slot);

/* Views of the bookkeeping (owned by pp, valid until the next call):
 * block table int32 [max_batch][max_blocks_per_seq], seq_lens int32
 * [max_batch] (0 for free slots), active flag int32 [max_batch], reference
 * count int32 [num_pages]. */
const int32_t* pkv_pages_block_table(const pkv_pages* pp);
const int32_t* pkv_pages_seq_lens(const pkv_pages* pp);
const int32_t* pkv_pages_active(const pkv_pages* pp);
const int32_t* pkv_pages_refcount(const pkv_pages* pp);

/* Pages on the free list; -1 for NULL. */
int pkv_pages_free_count(const pkv_pages* pp);

/* The block-table writes since the previous call (admissions, pages added by
 * pkv_pages_reserve, rows cleared by pkv_pages_release) as (slot, index,
 * value) int32 triples written to out: an entry written more than once
 * appears once, with its last value (so the triples can be applied in any
 * order, in parallel), in the order of those last writes.  A caller that
 * keeps a copy of the table (on the device, say: pkv_table_sync) applies
 * them instead of copying the whole table each step.  Returns the number of
 * triples, or -1 when there were more than max_changes (or more writes than
 * the log holds, about num_pages), in which case the contents of out are
 * unspecified and the caller should copy the whole table.  Either way the
 * log starts empty again. */
int pkv_pages_take_changes(pkv_pages* pp, int32_t* out, int max_changes);

#ifdef __cplusplus
}
#endif
#endif
