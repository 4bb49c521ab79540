/*
 * pa_block_manager.h -- C ABI of the host-side page pool that drives the
 * paged KV cache kernels of pa_b200.h.
 *
 * What it implements, from the pages on vLLM / PagedAttention:
 *  - "4. vLLM核心机制：PagedAttention、Continuous Batching、动态批处理",
 *    section 4.2: the cache is a pool of fixed-size physical pages; a
 *    sequence's page table maps its logical page i to any physical page;
 *    a sequence gets pages as it grows and the pool takes them back when it
 *    ends; pages holding a common prefix (parallel sampling, shared system
 *    prompts) are named by several tables at once.
 *    Section 4.4: under memory pressure a running sequence is preempted and
 *    its pages are moved to a CPU-side pool, to be brought back later.
 *  - pinggu.org forum post, section "PagedAttention：让显存像虚拟内存一样灵活":
 *    pages are handed out on demand and returned when a request finishes.
 *
 * Readings where the pages give no mechanism:
 *  - Sharing is reference counted per physical page.  A sequence that is
 *    about to write into a page it shares with others, and that page is only
 *    partly filled, first gets a private copy of it (copy-on-write): the
 *    manager allocates a fresh page, drops one reference to the shared one
 *    and reports the (shared, fresh) pair, which the caller copies with
 *    pa_copy_blocks before the step's pa_write_kv.  A full shared page is
 *    never written again, so appending past it just allocates a new page.
 *  - Swapping moves whole sequences.  A device page named by several of the
 *    sequences being swapped is copied once and stays shared on the other
 *    side; a page still named by a sequence that stays keeps its device copy.
 *  - Free pages are reused last-freed-first; a fresh pool hands out ids in
 *    ascending order.  Everything is deterministic.
 *
 * Conventions
 *  - The manager is host-only: no call touches a GPU or launches anything.
 *    It owns only its own bookkeeping; all arrays passed in are the
 *    caller's (host memory) and are not retained.
 *  - Sequence ids are caller-chosen int64 values.  Device page ids are in
 *    [0, num_device_blocks), host page ids in [0, num_host_blocks): two
 *    separate pools with the same page geometry.
 *  - Every call returns PA_BM_OK (0) or a negative PA_BM_ERR_* code and
 *    changes nothing when it fails (all-or-nothing).  Calls on one manager are
 *    serialised by an internal lock.
 */
#ifndef PA_BLOCK_MANAGER_H
#define PA_BLOCK_MANAGER_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define PA_BM_OK 0
#define PA_BM_ERR_ARG (-20)        /* a size or pointer argument is invalid */
#define PA_BM_ERR_NO_SPACE (-21)   /* not enough free pages in the pool the call needs */
#define PA_BM_ERR_UNKNOWN (-22)    /* no sequence with this id */
#define PA_BM_ERR_EXISTS (-23)     /* a sequence with this id already exists */
#define PA_BM_ERR_STATE (-24)      /* the sequence is in the other pool (swapped out / in) */
#define PA_BM_ERR_CAPACITY (-25)   /* an output array or the table stride is too small */
#define PA_BM_ERR_HOST_MEMORY (-26) /* the manager's own bookkeeping could not get host memory */

typedef struct pa_block_manager pa_block_manager;

/* A manager over num_device_blocks device pages and num_host_blocks host
 * pages of block_size tokens each.  Returns NULL on a bad argument or when
 * memory for the bookkeeping cannot be had.  block_size > 0; pools >= 0. */
pa_block_manager *pa_bm_create(int32_t block_size, int64_t num_device_blocks, int64_t num_host_blocks);
void pa_bm_destroy(pa_block_manager *bm);

/* Pool state. */
int64_t pa_bm_num_free_device_blocks(const pa_block_manager *bm);
int64_t pa_bm_num_free_host_blocks(const pa_block_manager *bm);
/* References held on page `block` of the device pool (host_pool = 0) or of
 * the host pool (host_pool != 0); -1 if the id is outside the pool. */
int32_t pa_bm_ref_count(const pa_block_manager *bm, int32_t host_pool, int64_t block);

/* A new sequence holding num_tokens tokens (its prompt), all in fresh device
 * pages: ceil(num_tokens / block_size) of them.  The slots its prompt's KV
 * goes to follow from pa_bm_slots. */
int pa_bm_add_sequence(pa_block_manager *bm, int64_t seq_id, int64_t num_tokens);

/* child starts as a copy of parent that shares all of its pages (each page
 * gains one reference).  parent must be on the device pool. */
int pa_bm_fork(pa_block_manager *bm, int64_t parent_id, int64_t child_id);

/* Ends a sequence: one reference dropped from each of its pages; pages with
 * none left go back to their pool's free list. */
int pa_bm_free_sequence(pa_block_manager *bm, int64_t seq_id);

/* Number of tokens of the sequence (>= 0), or a negative error code. */
int64_t pa_bm_num_tokens(const pa_block_manager *bm, int64_t seq_id);

/* 1 if the sequence is in the host pool (swapped out), 0 if on the device, or
 * a negative error code. */
int pa_bm_is_swapped(const pa_block_manager *bm, int64_t seq_id);

/* Copies the sequence's page table (ids in its current pool) into
 * table[0..capacity); *num_blocks gets its length (also when the capacity is
 * too small, which returns PA_BM_ERR_CAPACITY). */
int pa_bm_block_table(const pa_block_manager *bm, int64_t seq_id, int32_t *table, int64_t capacity,
                      int64_t *num_blocks);

/* Device slots (page * block_size + row) of tokens [first, first + count) of
 * a sequence on the device pool: slots[i] for token first + i.  All of them
 * must already have pages. */
int pa_bm_slots(const pa_block_manager *bm, int64_t seq_id, int64_t first, int64_t count, int64_t *slots);

/* Reserves the slot of one new token at the end of a device-pool sequence:
 * a fresh page when the last one is full (or there is none), a private copy
 * of the last page when it is partly full and shared.  *slot gets the slot;
 * *copy_src / *copy_dst get the copy-on-write pair or -1 / -1. */
int pa_bm_append_slot(pa_block_manager *bm, int64_t seq_id, int64_t *slot, int64_t *copy_src,
                      int64_t *copy_dst);

/* One decode step of a continuous batch: for each of the num_seqs sequences
 * (all on the device pool, distinct ids) reserve the slot of its new token
 * as pa_bm_append_slot does, then fill
 *   block_tables   int32 [num_seqs][table_stride], rows padded with -1;
 *   context_lens   int32 [num_seqs], tokens including the new one;
 *   slot_mapping   int64 [num_seqs], the new token's slot;
 *   copy_pairs     int64 [copy_capacity][2], the copy-on-write pairs, in
 *                  order; *num_copies gets their number.
 * The pairs never overlap (each destination is a fresh page), so one
 * pa_copy_blocks call applies them.  The whole step fails without change if
 * the pool runs out, a table is longer than table_stride, or the copy array
 * is too small (num_seqs pairs always suffice).  The one exception:
 * *num_copies is written as soon as the step is planned, so on
 * PA_BM_ERR_NO_SPACE, or PA_BM_ERR_CAPACITY from a too-small copy array, it
 * holds the number of pairs the step needs (to size copy_pairs with); on
 * earlier failures it is left as it was. */
int pa_bm_build_decode_step(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t table_stride,
                            int32_t *block_tables, int32_t *context_lens, int64_t *slot_mapping,
                            int64_t *copy_pairs, int64_t copy_capacity, int64_t *num_copies);

/* One prefill (or chunked-prefill) step of a continuous batch: sequence i
 * (device pool, distinct ids) brings new_tokens[i] >= 0 tokens.  Their slots
 * are reserved as num_new successive pa_bm_append_slot calls would (a private
 * copy of a shared, partly full last page before the first of them, a fresh
 * page at every page boundary), then the step's arrays for pa_write_kv and
 * pa_prefill are filled:
 *   block_tables   int32 [num_seqs][table_stride], rows padded with -1;
 *   query_start    int32 [num_seqs + 1], query_start[0] = 0, the new tokens'
 *                  prefix sum (sequence i's rows of q are query_start[i] ..);
 *   context_lens   int32 [num_seqs], tokens including the new ones;
 *   slot_mapping   int64 [slot_capacity], the new tokens' slots in row order
 *                  (sequence by sequence); the total must fit;
 *   copy_pairs     int64 [copy_capacity][2], the copy-on-write pairs, in
 *                  order; *num_copies gets their number (num_seqs pairs
 *                  always suffice).
 * A sequence with no new tokens gets its table and length only.  The whole
 * step fails without change if the pool runs out, a table is longer than
 * table_stride, a length or the token total passes int32, or an output array
 * is too small; as for pa_bm_build_decode_step, *num_copies alone is written
 * once the step is planned (on PA_BM_ERR_NO_SPACE or a too-small slot or copy
 * array it holds the pairs the step needs). */
int pa_bm_build_prefill_step(pa_block_manager *bm, const int64_t *seq_ids, const int64_t *new_tokens,
                             int64_t num_seqs, int64_t table_stride, int32_t *block_tables, int32_t *query_start,
                             int32_t *context_lens, int64_t *slot_mapping, int64_t slot_capacity,
                             int64_t *copy_pairs, int64_t copy_capacity, int64_t *num_copies);

/* What a step would take, without taking it: sequence i (device pool,
 * distinct ids) brings new_tokens[i] >= 0 tokens (1 each for a decode step).
 * *pages gets the fresh device pages the step needs (copy-on-write copies
 * included), *copies the copy-on-write pairs it would produce.  Compare with
 * pa_bm_num_free_device_blocks to decide admission or preemption before
 * building the step. */
int pa_bm_step_needs(const pa_block_manager *bm, const int64_t *seq_ids, const int64_t *new_tokens, int64_t num_seqs,
                     int64_t *pages, int64_t *copies);

/* Moves num_seqs device-pool sequences to the host pool (preemption).
 * mapping int64 [capacity][2] gets the (device page, host page) pairs to
 * copy with pa_swap_blocks (device pools as source, host pools as
 * destination), *num_pairs their number (at most the total pages of the
 * sequences; set also when the call fails with PA_BM_ERR_NO_SPACE or
 * PA_BM_ERR_CAPACITY, to the number the call would need).  Device pages
 * that no other sequence names return to the free list: copy them out
 * before the pages are handed out again. */
int pa_bm_swap_out(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t *mapping,
                   int64_t capacity, int64_t *num_pairs);

/* The reverse: host-pool sequences back to fresh device pages; mapping gets
 * (host page, device page) pairs for pa_swap_blocks with the host pools as
 * source. */
int pa_bm_swap_in(pa_block_manager *bm, const int64_t *seq_ids, int64_t num_seqs, int64_t *mapping,
                  int64_t capacity, int64_t *num_pairs);

#ifdef __cplusplus
}
#endif

#endif /* PA_BLOCK_MANAGER_H */
