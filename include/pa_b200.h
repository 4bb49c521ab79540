/*
 * pa_b200.h -- C ABI of the B200 (sm_100a) paged decode attention library.
 *
 * The operations come from web pages describing vLLM / PagedAttention:
 *  - "4. vLLM核心机制：PagedAttention、Continuous Batching、动态批处理",
 *    section 4.2: the KV cache is cut into fixed-size pages (16 or 32 tokens);
 *    a per-sequence page table maps logical page i to any physical page of
 *    the pool; attention walks the pages through the table; prefix pages may
 *    be named by several tables.  Section 4.3: each decode iteration produces
 *    the new token and the updated KV cache.
 *  - "vLLM：大型语言模型推理优化的革命性突破", section 2.1: the attention kernel
 *    indexes the scattered blocks through the table, with no data movement
 *    and no zero padding.
 * Grouped-query heads (several query heads reading one KV head) are part of
 * the problem statement this library serves, not of the pages.
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees or retains them.  The library allocates no device memory on
 *    any call; its device state is statically allocated __device__ data: one
 *    status word per device, and the fixed scratch array behind
 *    pa_decode_static_workspace.
 *  - Storage elements are 2-byte floats: PA_FLOAT16 (IEEE binary16) or
 *    PA_BFLOAT16.  Strides are in ELEMENTS.
 *  - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream) and returns a PA_* status.  A negative status means the
 *    arguments were rejected on the host and nothing was launched (or the
 *    launch itself failed: PA_ERR_CUDA, text in pa_last_cuda_error()).
 *  - Problems that only the device can see (a block id outside the pool, a
 *    context length outside the table, a slot outside the pool, a bounded
 *    wait that ran out) set bits in the device status word and never trap;
 *    read them with pa_get_device_status().
 *  - Cache layout: k_cache and v_cache are [num_blocks][num_kv_heads]
 *    [block_size][head_dim], contiguous, so one (block, kv head) slab of
 *    block_size * head_dim elements is contiguous in memory.
 *  - Supported shapes: head_dim in {64, 128}; block_size in {16, 32};
 *    num_q_heads a multiple of num_kv_heads (query head hq reads kv head
 *    hq / (num_q_heads / num_kv_heads)).  All tensor base pointers must be
 *    16-byte aligned and every token/sequence stride a multiple of 8 elements.
 */
#ifndef PA_B200_H
#define PA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- host status codes ---- */
#define PA_OK 0
#define PA_ERR_NULL (-1)        /* a required pointer is NULL */
#define PA_ERR_DTYPE (-2)       /* dtype is not PA_FLOAT16 / PA_BFLOAT16 */
#define PA_ERR_SHAPE (-3)       /* a size is negative or inconsistent */
#define PA_ERR_ALIGN (-4)       /* a pointer or stride breaks the 16-byte rule */
#define PA_ERR_UNSUPPORTED (-5) /* head_dim or block_size outside the supported set */
#define PA_ERR_HEADS (-6)       /* num_q_heads is not a multiple of num_kv_heads */
#define PA_ERR_WORKSPACE (-7)   /* workspace missing, too small or misaligned */
#define PA_ERR_PARTITION (-8)   /* partition_tokens negative or not a multiple of 16 */
#define PA_ERR_CUDA (-9)        /* a CUDA runtime call failed; see pa_last_cuda_error() */
#define PA_ERR_STATIC_WORKSPACE (-10) /* the problem needs more scratch than PA_STATIC_WORKSPACE_BYTES */
#define PA_ERR_ADDRESS (-11)    /* a pointer is neither this device's memory nor pinned host memory mapped for it */

/* Size of the fixed scratch array behind pa_decode_static_workspace (32 MiB). */
#define PA_STATIC_WORKSPACE_BYTES (32u * 1024u * 1024u)

/* ---- device status bits (pa_get_device_status) ---- */
#define PA_DEV_ERR_BLOCK_ID 0x1u    /* a table entry a sequence needs is outside [0, num_blocks) */
#define PA_DEV_ERR_CONTEXT 0x2u     /* context_len < 0 or > block_table_stride * block_size */
#define PA_DEV_ERR_CONTEXT_HINT 0x4u /* context_len > the max_context_len the call was given */
#define PA_DEV_ERR_SLOT 0x8u        /* a slot_mapping entry >= num_blocks * block_size */
#define PA_DEV_ERR_TIMEOUT 0x10u    /* a bounded wait on a bulk copy ran out */
#define PA_DEV_ERR_INTERNAL 0x20u   /* debug builds only: an internal index check failed; that access was skipped */
#define PA_DEV_ERR_PLAN 0x40u       /* a cascade plan disagrees with the call: a group member's table differs on the
                                       shared prefix or its context ends inside it, or a plan index is out of range */

/* ---- build flags (pa_build_flags) ---- */
#define PA_BUILD_DEBUG 0x1u /* built with PA_DEBUG: every derived index is checked on the device before use */

typedef enum { PA_FLOAT16 = 1, PA_BFLOAT16 = 2 } pa_dtype;

/*
 * pa_write_kv -- store this step's new K and V rows into their cache slots
 * ("4. vLLM核心机制" section 4.3, with the page layout of section 4.2).
 *
 * For every token t < num_tokens and kv head h:
 *   slot = slot_mapping[t];  if slot < 0 the token is skipped (padding);
 *   k_cache[slot / block_size][h][slot % block_size][:] = k[t][h][:]
 *   v_cache[...same...]                                  = v[t][h][:]
 * The copy is bit for bit.
 *
 *   k, v           [num_tokens][num_kv_heads][head_dim]; token stride
 *                  k_token_stride / v_token_stride, heads contiguous.
 *   k_cache,v_cache [num_blocks][num_kv_heads][block_size][head_dim].
 *   slot_mapping   int64 [num_tokens].
 * Slots must be distinct (two tokens writing one slot race).  A slot
 * >= num_blocks * block_size is skipped and sets PA_DEV_ERR_SLOT.
 * num_tokens == 0 launches nothing and returns PA_OK.
 */
int pa_write_kv(const void *k, const void *v, void *k_cache, void *v_cache, const int64_t *slot_mapping,
                int64_t num_tokens, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                int64_t num_blocks, int64_t k_token_stride, int64_t v_token_stride, int32_t dtype,
                void *stream);

/*
 * pa_decode_workspace_size -- bytes of device workspace pa_decode needs for
 * these sizes and this partition_tokens (see pa_decode) on the current
 * device.  It does not depend on the storage type.  Returns 0 on bad input.
 */
size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int32_t max_context_len, int32_t partition_tokens);

/*
 * pa_decode -- single-token decode attention over the block-paged KV cache
 * ("4. vLLM核心机制" section 4.2; "vLLM：大型语言模型推理优化的革命性突破" 2.1).
 *
 * For every sequence s and query head hq, with h = hq / (num_q_heads /
 * num_kv_heads) and L = context_lens[s]:
 *   token j < L lives in physical block block_tables[s][j / block_size],
 *   row j % block_size;
 *   z_j = scale * <q[s][hq][:], K_j>;  w = softmax(z);  out[s][hq][:] = sum_j w_j V_j.
 * Arithmetic is fp32 (storage values widened exactly); the result is rounded
 * to nearest-even into out's storage type (= dtype).  L == 0 gives zeros.
 *
 *   q               [num_seqs][num_q_heads][head_dim], sequence stride q_seq_stride.
 *   k_cache,v_cache as for pa_write_kv.
 *   block_tables    int32 [num_seqs][block_table_stride]; only entries
 *                   j < ceil(L / block_size) of row s are read.
 *   context_lens    int32 [num_seqs].
 *   out             [num_seqs][num_q_heads][head_dim], sequence stride out_seq_stride.
 *   max_context_len host-side upper bound of every context_len; it sizes the
 *                   split over the token axis.  A sequence above it (or above
 *                   the table's capacity) gets a zero output row and sets
 *                   PA_DEV_ERR_CONTEXT_HINT (or PA_DEV_ERR_CONTEXT).
 *   partition_tokens how the work is cut.  The tiles of 16 tokens of every
 *                   (sequence, kv head, group of up to 8 query heads) are laid
 *                   in one stream, ordered by sequence, then head group, then
 *                   position, and the stream is cut into chunks of
 *                   consecutive tiles that the GPU's warps take in turn.
 *                   0 = balanced: one chunk per resident warp, so every warp
 *                   gets the same number of tiles whatever the length mix;
 *                   otherwise a positive multiple of 16: chunks of
 *                   partition_tokens / 16 tiles.  A sequence cut across chunks
 *                   is finished by a second kernel that merges the partial
 *                   softmax states in a fixed order: results are deterministic
 *                   run to run for the same arguments and device.
 *   workspace       device scratch of at least pa_decode_workspace_size()
 *                   bytes, 16-byte aligned.  Contents need no initialisation
 *                   and are overwritten.  Calls that run concurrently must not
 *                   share one workspace.
 * num_seqs is at most 32768.
 * A table entry outside [0, num_blocks) is never dereferenced: the affected
 * (sequence, head) rows are zeroed and PA_DEV_ERR_BLOCK_ID is set.
 * num_seqs == 0 launches nothing and returns PA_OK.
 */
int pa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
              const int32_t *context_lens, float scale, void *out, int32_t num_seqs, int32_t num_q_heads,
              int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks,
              int32_t block_table_stride, int32_t max_context_len, int64_t q_seq_stride, int64_t out_seq_stride,
              int32_t partition_tokens, int32_t dtype, void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_prefill -- causal attention of each sequence's NEW tokens (a prompt, or
 * the next chunk of one) over its paged context ("4. vLLM核心机制" section
 * 4.3: the prompt's tokens enter the cache before decoding starts, possibly
 * a piece per iteration).  Sequence s brings
 * n_s = query_start[s+1] - query_start[s] new tokens whose K/V rows are
 * ALREADY in the cache (write them with pa_write_kv first); its context
 * holds L_s = context_lens[s] >= n_s tokens, the new ones last.  New token t
 * (0 <= t < n_s) is at logical position p = L_s - n_s + t and attends to the
 * tokens 0..p only:
 *   out[query_start[s] + t][hq][:] = softmax_j(scale * q . K[j]) V[j],  j = 0..p,
 * K/V rows gathered through block_tables as in pa_decode (kv head
 * hq / (num_q_heads / num_kv_heads)).  n_s = 1 is a decode step.
 *   q            [num_query_tokens][num_q_heads][head_dim], token stride
 *                q_token_stride (elements, multiple of 8);
 *   query_start  int32 [num_seqs + 1], query_start[0] = 0, non-decreasing,
 *                query_start[num_seqs] <= num_query_tokens;
 *   context_lens int32 [num_seqs];
 *   out          like q, token stride out_token_stride;
 *   max_query_len >= every n_s (sizes the grid); a sequence with more new
 *                tokens sets PA_DEV_ERR_CONTEXT_HINT and its rows past
 *                max_query_len (rounded up to 256) are not written.
 * Runs on the tensor cores (tcgen05, tensor memory accumulators): work items
 * of 256 new tokens of one query head, taken from a per-call queue by
 * persistent CTAs; computes in fp32 with P rounded to the storage type.
 * The queue is one of 64 work counters in the library's device memory,
 * handed to successive calls in turn and cleared on the call's stream before
 * its launch: at most 64 calls may execute at the same time on one device
 * (calls on one stream never overlap), and a call captured in a CUDA graph
 * keeps the counter it was captured with.
 * Sequences with one new token cost a whole 128-row tile each here: batch
 * them through pa_decode; sequences with none cost a few microseconds per
 * thousand (query tile, head) slots of max_query_len.  Device-side errors: L_s < n_s or L_s > block_table_stride *
 * block_size -> PA_DEV_ERR_CONTEXT and zero rows; query_start entries that
 * leave [0, num_query_tokens] -> PA_DEV_ERR_CONTEXT and that sequence is not
 * written; a needed table entry outside the pool -> PA_DEV_ERR_BLOCK_ID and
 * zero rows.
 */
int pa_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
               const int32_t *query_start, const int32_t *context_lens, float scale, void *out, int32_t num_seqs,
               int64_t num_query_tokens, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
               int32_t block_size, int64_t num_blocks, int32_t block_table_stride, int32_t max_query_len,
               int64_t q_token_stride, int64_t out_token_stride, int32_t dtype, void *stream);

/*
 * pa_copy_blocks -- copy whole blocks inside one pair of caches: for every
 * pair i, block block_mapping[i][0] is copied (all kv heads, rows and dims, K
 * and V) to block block_mapping[i][1].  This is the copy a sequence needs
 * before it appends to a block it shares with others (a prefix page named
 * by several tables, "4. vLLM核心机制" section 4.2): it gets a private copy
 * first (copy-on-write).
 *   block_mapping  int64 [num_pairs][2], 8-byte aligned, in device memory
 *                  or pinned host memory (checked as for pa_swap_blocks).
 * A pair with a negative entry is skipped; an entry >= num_blocks is skipped
 * and sets PA_DEV_ERR_BLOCK_ID.  Destinations must be distinct and must not
 * be the source of another pair (pairs run concurrently).  Bit-exact copy.
 */
int pa_copy_blocks(void *k_cache, void *v_cache, const int64_t *block_mapping, int64_t num_pairs,
                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int64_t num_blocks, void *stream);

/*
 * pa_swap_blocks -- copy whole blocks from one pool (src_k, src_v with
 * src_num_blocks blocks) to another (dst_k, dst_v with dst_num_blocks), with
 * the same layout.  Either pool may be pinned host memory (reached through
 * unified addressing): this moves a preempted sequence's pages to a
 * CPU-side pool and back ("4. vLLM核心机制" section 4.4).  block_mapping
 * pairs are (source block, destination block), device-accessible; rules as
 * for pa_copy_blocks (entries checked against their own pool's size).
 * Every pointer (pools and mapping) is checked with the runtime before the
 * launch: device memory of the current device and pinned host memory are
 * accepted (host pointers are translated to their device addresses);
 * anything else (pageable host memory, another device's memory) returns
 * PA_ERR_ADDRESS with nothing launched.  Host-side pools move over the host
 * link, so a swap runs at that link's bandwidth.
 */
int pa_swap_blocks(const void *src_k, const void *src_v, void *dst_k, void *dst_v, const int64_t *block_mapping,
                   int64_t num_pairs, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                   int64_t src_num_blocks, int64_t dst_num_blocks, void *stream);

/*
 * pa_get_device_status -- wait for `stream`, then copy the current device's
 * status word (PA_DEV_ERR_* bits accumulated by earlier calls) to
 * *status_out; clear it when `clear` is non-zero.  Synchronises `stream`.
 */
int pa_get_device_status(uint32_t *status_out, int32_t clear, void *stream);

/* pa_status_string -- static text for a PA_* status code. */
const char *pa_status_string(int32_t status);

/* pa_last_cuda_error -- text of the last CUDA failure seen by this thread ("" if none). */
const char *pa_last_cuda_error(void);

/* pa_launch_count -- kernels this library has launched in this process (all devices). */
uint64_t pa_launch_count(void);

/*
 * pa_debug_wait_timeout -- self-test of the bounded wait used by the decode
 * kernel: launches one warp that waits on a shared-memory barrier that
 * nothing will ever complete, giving up after limit_ns nanoseconds (clamped
 * to [1e3, 1e9]); the kernel then sets PA_DEV_ERR_TIMEOUT and returns.
 * Touches no caller memory.
 */
int pa_debug_wait_timeout(int64_t limit_ns, void *stream);

/*
 * pa_decode_static_workspace -- pa_decode for callers that cannot allocate
 * device memory.  The pages have no counterpart to this entry point; it
 * exists for the library's users.
 *
 * Some callers may not call cudaMalloc (or any allocator) at run time: a
 * plugin inside a host framework that owns every device allocation, or a
 * server that fixes its memory budget at start-up and must not allocate,
 * fragment memory or pay an allocator's implicit device synchronisation in
 * the middle of a step.  Such callers cannot provide pa_decode's workspace.
 * This variant takes the same arguments as pa_decode minus the workspace
 * and uses instead a scratch array of PA_STATIC_WORKSPACE_BYTES (32 MiB)
 * compiled into the library as a static __device__ variable.  Every GPU on
 * which the library is loaded holds that array until the process exits.
 *
 * - It allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 * - A problem whose split-context scratch (pa_decode_workspace_size for the
 *   same sizes and partition_tokens) exceeds PA_STATIC_WORKSPACE_BYTES is
 *   rejected with PA_ERR_STATIC_WORKSPACE before anything is launched; use
 *   pa_decode with a caller workspace, or a larger partition_tokens.
 * - The first call on each device looks up the array's device address with
 *   cudaGetSymbolAddress while that device is current and caches it; make
 *   that first call before any stream capture begins.
 * - All calls on a device share the one array, and it keeps whatever the
 *   last call left there.  The decode kernels write every scratch entry
 *   before reading it, so nothing needs clearing between calls; but two
 *   calls that can run at the same time on the GPU (different streams with
 *   no ordering between them) race on the array and may corrupt each
 *   other's results.  Order them on one stream, or use pa_decode.
 * Results equal pa_decode's for the same arguments.
 */
int pa_decode_static_workspace(const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *block_tables, const int32_t *context_lens, float scale, void *out,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int64_t num_blocks, int32_t block_table_stride,
                               int32_t max_context_len, int64_t q_seq_stride, int64_t out_seq_stride,
                               int32_t partition_tokens, int32_t dtype, void *stream);

/*
 * pa_read_bandwidth_probe -- reads `bytes` bytes at `src` (device memory,
 * 16-byte aligned, bytes a multiple of 16) once, with every SM streaming
 * 16-byte loads that bypass L1, and folds them into *sink (one device word,
 * XOR-accumulated; its value means nothing).  A measurement aid with no
 * counterpart on the pages: timed with events around it over a buffer much
 * larger than L2, it gives the read-only HBM rate against which the decode
 * kernels (which read K/V and write almost nothing) are best compared.
 * bytes == 0 launches nothing.
 */
int pa_read_bandwidth_probe(const void *src, int64_t bytes, uint32_t *sink, void *stream);

/*
 * pa_build_flags -- PA_BUILD_* bits of this build.  A PA_DEBUG build
 * (libpa_b200_debug.so) checks, before each access, every index the kernels
 * derive rather than read (the tile a stream position maps to, table-window
 * entries, cache rows, chunk and piece rows of the workspace, output rows,
 * prefill items); a failed check skips the access and sets
 * PA_DEV_ERR_INTERNAL.  Results are otherwise the same as the release
 * build's.  It stands in for a memory checker on small cases.
 */
uint32_t pa_build_flags(void);

/* ---- cascade decode: shared-prefix groups read once ("4. vLLM核心机制" section 4.2) ----
 *
 * When several sequences' tables name the same leading blocks (one prompt
 * sampled several times, a shared system prompt: the pages' copy-free prefix
 * sharing), pa_decode reads those blocks once per sequence.  The cascade
 * calls compute the same attention with every shared tile fetched once per
 * group: the host finds the groups (pa_find_prefix_groups) and builds a plan
 * (pa_cascade_plan), the caller copies the plan to the device with the
 * step's other inputs, and pa_decode_cascade runs it.  The plan depends on
 * the groups, the head counts, block_size and max_context_len only, not on
 * the exact lengths, so a plan serves every step until a group changes.
 */
typedef struct pa_cascade_info {
  int32_t num_seqs, num_q_heads, num_kv_heads, block_size, max_context_len;
  int32_t num_jobs;      /* jobs: num_prefix_jobs prefix jobs first, then the suffix jobs */
  int32_t num_prefix_jobs;
  int32_t num_members;   /* entries of the plan's member list */
  int32_t num_pieces;    /* partial states merged per (sequence, head) in total over the sequences */
  int32_t rows_per_head; /* partial rows of the workspace per kv head */
  int64_t plan_ints;     /* int32 entries of the plan */
} pa_cascade_info;

/*
 * pa_find_prefix_groups -- host-side grouping of a batch by shared leading
 * blocks.  All pointers are HOST memory.  block_tables int32
 * [num_seqs][block_table_stride], context_lens int32 [num_seqs].  Sequences
 * whose first table entries agree form a candidate group (only full blocks,
 * j < context_len / block_size, count); its prefix is the longest run of
 * leading entries every member shares.  A group is reported when it has at
 * least two members and prefix >= max(1, min_prefix_blocks).  Output (caller
 * arrays of num_seqs + 1, num_seqs, num_seqs int32): group g's members are
 * group_members[group_offsets[g] .. group_offsets[g+1]) in increasing order,
 * sharing group_prefix_blocks[g] blocks; groups are ordered by first member;
 * *num_groups is their count.  Sequences in no group are not listed.
 * Contexts outside [0, block_table_stride * block_size] -> PA_ERR_SHAPE.
 */
int pa_find_prefix_groups(const int32_t *block_tables, const int32_t *context_lens, int32_t num_seqs,
                          int32_t block_table_stride, int32_t block_size, int32_t min_prefix_blocks,
                          int32_t *group_offsets, int32_t *group_members, int32_t *group_prefix_blocks,
                          int32_t *num_groups);

/*
 * pa_cascade_plan -- host-side work plan of pa_decode_cascade.  All pointers
 * are HOST memory.  Groups as pa_find_prefix_groups reports them (any
 * sequence at most once; sequences in no group, and groups with a zero
 * prefix, attend through their own tables only); every member of group g
 * must hold at least group_prefix_blocks[g] * block_size tokens, and
 * group_prefix_blocks[g] * block_size <= max_context_len.  num_q_heads /
 * num_kv_heads must be at most 8 (PA_ERR_UNSUPPORTED otherwise).
 * chunk_tokens: tokens per job along the context, 0 = 320, else a positive
 * multiple of 16 (PA_ERR_PARTITION).  Fills *info; writes the plan
 * (info->plan_ints int32) to `plan` unless it is NULL (a size query).
 * plan_capacity (entries) smaller than needed -> PA_ERR_WORKSPACE, with
 * *info filled.
 * Jobs: per group, per column set of up to 4 * (8 / G) members, per chunk
 * of the shared tiles; per sequence, per chunk of the tiles from its
 * prefix to ceil(max_context_len / 16).
 */
int pa_cascade_plan(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t block_size,
                    int32_t max_context_len, int32_t chunk_tokens, int32_t num_groups, const int32_t *group_offsets,
                    const int32_t *group_members, const int32_t *group_prefix_blocks, int32_t *plan,
                    int64_t plan_capacity, pa_cascade_info *info);

/* pa_cascade_workspace_size -- device workspace bytes pa_decode_cascade needs for this plan (0 on bad input). */
size_t pa_cascade_workspace_size(const pa_cascade_info *info, int32_t head_dim);

/*
 * pa_decode_cascade -- the attention of pa_decode (same definition, same
 * fp32 arithmetic, rounded to nearest even), computed by the plan's jobs:
 * each job streams 16-token tiles of one table row once and applies them to
 * all of its members' query heads, leaving partial softmax states in the
 * workspace; a second kernel merges every (sequence, head)'s pieces in plan
 * order (deterministic).  Sizes (num_seqs, heads, block_size,
 * max_context_len) come from *info (host); `plan` is the plan in DEVICE
 * memory, unchanged until the call has run.  Other arguments as pa_decode.
 * Device-side errors: a context outside [0, min(block_table_stride *
 * block_size, max_context_len)] -> zero row and PA_DEV_ERR_CONTEXT(_HINT);
 * a member whose table differs from its group's first member on the shared
 * blocks, or whose context ends inside them, or a plan index out of range
 * -> PA_DEV_ERR_PLAN and zero rows for the sequences concerned; table
 * entries outside the pool -> PA_DEV_ERR_BLOCK_ID and zero rows.
 * info->num_seqs == 0 launches nothing.
 */
int pa_decode_cascade(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                      const int32_t *context_lens, float scale, void *out, int32_t head_dim, int64_t num_blocks,
                      int32_t block_table_stride, int64_t q_seq_stride, int64_t out_seq_stride, int32_t dtype,
                      const int32_t *plan, const pa_cascade_info *info, void *workspace, size_t workspace_bytes,
                      void *stream);

/* pa_version -- library ABI version (major * 10000 + minor * 100 + patch). */
int32_t pa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* PA_B200_H */
