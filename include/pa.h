/*
 * pa.h — C ABI of libpagedattn: paged KV-cache decode attention for B200 (sm_100a).
 *
 * The operations (sources: web pages on PagedAttention):
 *
 *   pa_decode            Batched single-token decode attention that reads each
 *                        sequence's keys and values from a pool of fixed-size
 *                        blocks through a per-sequence block table ("PagedAttention"
 *                        concept card, 实现要点: the kernel takes the block table and
 *                        reads K/V scatter-gather; 核心思想: logical block index to
 *                        physical block).  The attention math is unchanged
 *                        ("什么是分页注意力", 边界与常见误解): for query head h of
 *                        sequence b, o = softmax(scale * q.K^T) V over the sequence's
 *                        tokens.
 *   pa_decode_append     pa_reshape_and_cache of the step's tokens and pa_decode in one
 *                        call; the balanced decode kernel writes the tokens itself.
 *   pa_reshape_and_cache Scatter the step's new K/V rows into their slots (each step
 *                        computes one key and value per token and caches them:
 *                        "什么是 LLM 中的分页注意力", 快速回顾:KV 缓存; slot addressing
 *                        as in its section 块表).
 *   pa_copy_blocks       Copy-on-write copy of whole blocks before a forked sequence
 *                        writes into a block it shares (concept card, 实现要点;
 *                        "深入解析 PagedAttention", 多序列共享).
 *   pa_alloc_*           Host-side block allocator with reference counts: on-demand
 *                        blocks, fork = share + refcount, free at refcount 0, copy on
 *                        write ("深入解析 PagedAttention", 核心创新 and 多序列共享;
 *                        concept card, 带来的能力 and 实现要点).
 *
 * Conventions shared by every entry point
 *   - Device pointers are caller-owned.  No entry point allocates or frees device
 *     memory, and none synchronises: kernels are queued on `stream` and the call
 *     returns.  The split-context workspace is caller-provided
 *     (pa_decode_workspace_size).
 *   - Every function returns a pa_status; no exception or abort crosses the ABI.
 *     Argument errors are detected on the host before anything is queued, and a
 *     failing call changes no state.
 *   - Data corruption that only the device can see (a block id outside
 *     [0, num_blocks), a sequence length outside [0, max_blocks*block_size], a slot
 *     outside the pool) never faults: the kernel ORs a PA_DEVERR_* bit into
 *     *dev_err_flag (if non-NULL), skips or clamps the access, and the affected
 *     output is unspecified.  Read the flag after synchronising and map it with
 *     pa_status_from_device_flag.
 *   - Layouts (row-major, innermost last):
 *       q, out          [B][Hq][D]
 *       k_pool, v_pool  [num_blocks][block_size][Hkv][D]
 *       block_tables    [B][max_blocks] int32; entries at logical index
 *                       >= ceil(seq_lens[b] / block_size) are never read (may be -1)
 *       seq_lens        [B] int32, tokens of sequence b including this step's token
 *       key, value      [T][Hkv][D]
 *       slot_mapping    [T] int64; slot s = physical block (s / block_size), offset
 *                       (s % block_size); s < 0 skips the token
 *       pairs           [n][2] int32 (src, dst) physical block ids
 *   - Query head h reads KV head h / (Hq / Hkv) (grouped-query attention).
 *   - Element types: PA_BF16 (bfloat16 storage, fp32 arithmetic, one final rounding
 *     to bfloat16) or PA_F32 (fp32 throughout, no TF32).  All of q, pools and out
 *     share the dtype.  Supported: D in {64, 128}; block_size in {4, 8, 16, 32};
 *     Hq % Hkv == 0; q/out/pool/key/value pointers 16-byte aligned.
 */
#ifndef PAGED_KV_CACHE_350_B200_PA_H
#define PAGED_KV_CACHE_350_B200_PA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same underlying type as cudaStream_t; NULL means the legacy default stream. */
typedef struct CUstream_st* pa_stream_t;

typedef enum pa_status {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,    /* bad size, pointer, alignment or combination */
  PA_ERR_UNSUPPORTED = 2,    /* valid but not implemented (e.g. D not in {64,128}) */
  PA_ERR_OUT_OF_BLOCKS = 3,  /* allocator has no free block; state unchanged */
  PA_ERR_BAD_BLOCK_ID = 4,   /* device flag: a block id outside [0, num_blocks) */
  PA_ERR_CUDA = 5,           /* a CUDA runtime call failed (launch, driver entry point) */
  PA_ERR_NOT_FOUND = 6,      /* allocator: unknown sequence id */
  PA_ERR_EXISTS = 7,         /* allocator: sequence id already in use */
  PA_ERR_BAD_SEQ_LEN = 8,    /* device flag: seq_lens[b] outside [0, max_blocks*block_size] */
  PA_ERR_BAD_SLOT = 9,       /* device flag: slot >= num_blocks*block_size */
  PA_ERR_TIMEOUT = 10,       /* device flag: a bounded pipeline wait gave up */
  PA_ERR_SCRATCH_LIMIT = 11, /* pa_decode_no_alloc: the shape needs more than its static scratch */
  PA_ERR_HOST_MEMORY = 12    /* allocator: a host allocation failed; state unchanged */
} pa_status;

typedef enum pa_dtype { PA_F32 = 0, PA_BF16 = 1 } pa_dtype;

/* Bits a kernel ORs into *dev_err_flag. */
#define PA_DEVERR_BAD_BLOCK_ID 0x1
#define PA_DEVERR_BAD_SEQ_LEN 0x2
#define PA_DEVERR_BAD_SLOT 0x4
#define PA_DEVERR_TIMEOUT 0x8

/* Static, NUL-terminated description of a status. */
const char* pa_status_string(pa_status status);

/* Map a device error flag word to the status of its lowest set bit (PA_OK if 0). */
pa_status pa_status_from_device_flag(int32_t flag);

/* Library version string, e.g. "0.1.0". */
const char* pa_version(void);

/* ---------------------------------------------------------------------------
 * Decode attention
 * ------------------------------------------------------------------------- */

typedef enum pa_decode_path {
  PA_PATH_AUTO = 0,     /* tensor-core path when eligible, else the CUDA-core path */
  PA_PATH_GENERIC = 1,  /* CUDA-core path (any supported shape and dtype) */
  PA_PATH_TENSOR = 2    /* bf16 tensor-core path: Hq/Hkv <= 16, block_size in {8,16,32};
                           PA_ERR_UNSUPPORTED if not eligible */
} pa_decode_path;

/* Kernels a decode call can run (reported by pa_decode_plan). */
typedef enum pa_decode_kernel {
  PA_KERNEL_NONE = 0,          /* empty batch */
  PA_KERNEL_GENERIC = 1,       /* CUDA cores, one CTA per (sequence, KV head, heads, partition) */
  PA_KERNEL_TC_PARTITION = 2,  /* tensor cores, one CTA per (sequence, KV head, partition) */
  PA_KERNEL_TC_STREAM = 3      /* tensor cores, one persistent wave; every consumer warp owns
                                  an equal range of the batch's 16-token tiles */
} pa_decode_kernel;

typedef struct pa_decode_opts {
  /* Tokens per context partition.  0 = automatic.  Otherwise a positive multiple of
   * block_size (and of 16 on the tensor-core path), and the partition kernels are used:
   * a sequence longer than one partition is split; each partition writes a partial
   * (max, sum, unnormalised output) to the workspace and a reduce kernel merges them by
   * log-sum-exp. */
  int partition_tokens;
  int path;             /* pa_decode_path */
  /* Upper bound on the CTAs of the balanced tensor-core kernel (0 = one full wave).
   * Changes only the schedule, not the result's definition. */
  int max_ctas;
} pa_decode_opts;

/* Bytes of workspace pa_decode needs on the current device for B sequences of at most
 * max_seq_len tokens, for every kernel the call could choose (partition_tokens as in
 * pa_decode_opts; 0 = automatic).  Returns (size_t)-1 for invalid arguments. */
size_t pa_decode_workspace_size(int B, int Hq, int Hkv, int D, int max_seq_len,
                                int block_size, int partition_tokens);

/* out[b][h][:] = sum_t softmax_t(scale * q[b][h].k_t) v_t over t < seq_lens[b], with
 * k_t = k_pool[block_tables[b][t / block_size]][t % block_size][h / (Hq/Hkv)][:]
 * (v_t likewise).  seq_lens[b] == 0 gives a zero row.  `workspace` may be NULL when
 * workspace_bytes is 0; with the automatic partitioning an insufficient workspace
 * makes every sequence a single partition.  dev_err_flag may be NULL. */
pa_status pa_decode(void* out, const void* q, const void* k_pool, const void* v_pool,
                    const int32_t* block_tables, const int32_t* seq_lens, int B, int Hq,
                    int Hkv, int D, int block_size, int max_blocks, int num_blocks,
                    float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                    int32_t* dev_err_flag, pa_stream_t stream);

/* What pa_decode_ex would launch for these arguments on the current device (host
 * only, queues nothing). */
typedef struct pa_decode_plan_info {
  int kernel;            /* pa_decode_kernel */
  int partition_tokens;  /* partition kernels: tokens per partition */
  int max_parts;         /* partition kernels: partitions of the longest possible sequence */
  int grid;              /* CTAs of the main kernel (stream kernel: one wave) */
  int launches;          /* kernel launches: 0, 1, or 2 with a reduce */
} pa_decode_plan_info;

pa_status pa_decode_plan(int B, int Hq, int Hkv, int D, int block_size, int max_blocks,
                         pa_dtype dtype, size_t workspace_bytes, const pa_decode_opts* opts,
                         pa_decode_plan_info* info);

/* pa_decode with explicit options (opts may be NULL = defaults). */
pa_status pa_decode_ex(void* out, const void* q, const void* k_pool, const void* v_pool,
                       const int32_t* block_tables, const int32_t* seq_lens, int B, int Hq,
                       int Hkv, int D, int block_size, int max_blocks, int num_blocks,
                       float scale, pa_dtype dtype, void* workspace, size_t workspace_bytes,
                       int32_t* dev_err_flag, pa_stream_t stream, const pa_decode_opts* opts);

/* One decode step with the cache write fused in.  For every row b with L = seq_lens[b]
 * >= 1, position L-1 is the step's token: its key and value (k_new[b], v_new[b], each
 * [B][Hkv][D] in the pools' dtype, 16-byte aligned) are written to slot
 * block_tables[b][(L-1) / block_size] * block_size + (L-1) % block_size of the pools
 * (a new token fills the next free slot of the sequence's current block: "什么是 LLM
 * 中的分页注意力", 使用分页注意力), and out is pa_decode over positions 0 .. L-1 with
 * that token included.  The result, out and pools, is the same as pa_reshape_and_cache
 * with those slots followed by pa_decode_ex.  Rows with L = 0 write nothing (zero
 * output row); a row whose length is out of range or whose table entry is outside
 * [0, num_blocks) writes nothing and raises its PA_DEVERR_* bit.
 *   - The block receiving row b's token must not be read by another row of the call
 *     (the allocator's copy-on-write guarantees this); such a row could see the old or
 *     the new values.
 *   - The balanced tensor-core kernel writes the token itself (the step is that
 *     kernel and its reduce); the other kernels run after a one-launch append kernel,
 *     so pa_decode_plan's `launches` is one more for them.
 * Arguments, workspace and options otherwise as pa_decode_ex. */
pa_status pa_decode_append(void* out, const void* q, const void* k_new, const void* v_new,
                           void* k_pool, void* v_pool, const int32_t* block_tables,
                           const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                           int block_size, int max_blocks, int num_blocks, float scale,
                           pa_dtype dtype, void* workspace, size_t workspace_bytes,
                           int32_t* dev_err_flag, pa_stream_t stream,
                           const pa_decode_opts* opts);

/* Decode for a batch in which groups of sequences share their leading blocks: samples
 * forked from one prompt, or requests with a common system prompt ("深入解析 PagedAttention",
 * 多序列共享; "什么是 LLM 中的分页注意力", 跨请求的内存共享).  Same result as pa_decode, but each
 * group's shared tokens are read from HBM once for the whole group: the members' query heads
 * are stacked as the rows of one tensor-core tile (members x Hq/Hkv <= 64 rows) that streams
 * the shared tokens and then each member's own tokens with the other members' rows masked
 * out of the softmax.
 *   group_of      [B] device int32: group of batch row b, or -1
 *   group_prefix  [ngroups] device int32: shared tokens of the group, a multiple of
 *                 PA_SHARED_PREFIX_ALIGN and <= every member's length; members' tables must
 *                 hold the same block ids for those tokens.  0 is allowed (the group then
 *                 shares no tokens; its members' own tokens are still read as one unit)
 *   group_members [ngroups][max_members] device int32: the group's batch rows, -1 padded
 * pa_alloc_prefix_groups builds these from the allocator.  bf16 tensor-core shapes only
 * (PA_ERR_UNSUPPORTED otherwise); max_members <= 32, max_members * (Hq/Hkv) <= 64;
 * B + ngroups <= 8192.
 * One launch: a persistent kernel with one CTA per SM, the tile math on the 5th-generation
 * tensor cores.  A unit split between CTAs is merged by the CTA holding its first chunk
 * (its owner): each later CTA publishes its piece's partial (per-row max, sum and
 * unnormalised output) in the workspace with a flag tagged for this call, and the owner
 * waits for those flags (bounded: every CTA of the grid is resident), merges, writes the
 * rows and clears the flags it consumed, so that a replay of a captured launch waits for
 * fresh partials.
 * Workspace: pa_decode_shared_prefix_workspace_size (on the current device); its contents
 * need no initialisation, and calls whose kernels may overlap on the GPU must not share
 * one. */
#define PA_SHARED_PREFIX_ALIGN 32
size_t pa_decode_shared_prefix_workspace_size(int B, int Hq, int Hkv, int D, int block_size,
                                              int ngroups);
pa_status pa_decode_shared_prefix(void* out, const void* q, const void* k_pool,
                                  const void* v_pool, const int32_t* block_tables,
                                  const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                                  int block_size, int max_blocks, int num_blocks, float scale,
                                  pa_dtype dtype, const int32_t* group_of,
                                  const int32_t* group_prefix, const int32_t* group_members,
                                  int ngroups, int max_members, void* workspace,
                                  size_t workspace_bytes, int32_t* dev_err_flag,
                                  pa_stream_t stream);

/* Decode without any device allocation.  The source pages have no counterpart: this
 * entry point exists for callers that cannot allocate device memory, so cannot provide
 * pa_decode's workspace: e.g. a serving runtime that owns every device buffer through
 * its own pool and forbids further allocations, or a latency-critical caller that
 * cannot afford cudaMalloc (which may synchronise the device).
 *
 * Same arguments and result as pa_decode, minus the workspace.  Runs the balanced
 * tensor-core kernel with its scratch in a static device array of the library
 * (PA_NO_ALLOC_SCRATCH_BYTES per device that loads the library, held until exit); it
 * calls no cudaMalloc, cudaFree or allocating library routine.
 *   - The array is device memory reserved when the library's module loads on a device:
 *     at context creation under CUDA_MODULE_LOADING=EAGER (then even by processes that
 *     never call this function), or inside the first call under lazy loading (the
 *     default).
 *   - The first call on each device looks up the array's address (cudaGetSymbolAddress
 *     with that device current) and caches it for the current context; a new context on
 *     the device (e.g. after cudaDeviceReset) is detected and the address looked up
 *     again.  Make that first call before any stream capture, so that neither the module
 *     load nor the lookup happens inside one.
 *   - All calls on a device share the array, which keeps the last call's contents;
 *     nothing in it has to start at zero.  Calls whose kernels overlap on the GPU race
 *     on the array: order them (e.g. one stream).
 *   - PA_ERR_UNSUPPORTED for shapes the tensor-core path does not take (fp32, block
 *     size 4, Hq/Hkv > 16, B > 8192); PA_ERR_SCRATCH_LIMIT, before anything is queued,
 *     if the shape's one-wave schedule on this device needs more than
 *     PA_NO_ALLOC_SCRATCH_BYTES (2 partial slots x G rows x (D+2) floats per consumer
 *     warp of the wave). */
#define PA_NO_ALLOC_SCRATCH_BYTES (32u << 20)
pa_status pa_decode_no_alloc(void* out, const void* q, const void* k_pool, const void* v_pool,
                             const int32_t* block_tables, const int32_t* seq_lens, int B, int Hq,
                             int Hkv, int D, int block_size, int max_blocks, int num_blocks,
                             float scale, pa_dtype dtype, int32_t* dev_err_flag,
                             pa_stream_t stream);

/* Self-test of the kernels' bounded waits (the pages have no counterpart; it exists for
 * the failure-detection test).  One warp waits, through the same bounded wait the decode
 * kernels use, on a barrier phase that nothing completes, limited to limit_us
 * (1 .. 1000000) microseconds.  The wait runs out, ORs PA_DEVERR_TIMEOUT into
 * *dev_err_flag (device memory, required) and the kernel returns: the context stays
 * usable.  PA_ERR_INVALID_ARG for a NULL flag or a limit out of range. */
pa_status pa_selftest_bounded_wait(int32_t* dev_err_flag, unsigned limit_us,
                                   pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Cache maintenance
 *
 * Both kernels are queued as programmatic dependents of the kernel before them on the
 * stream: their blocks may be scheduled while that kernel drains, and wait for its
 * completion before any memory access.  Stream order is unchanged; a step of copy,
 * cache write and decode just pays no launch gap between its kernels.
 * ------------------------------------------------------------------------- */

/* For t < T with s = slot_mapping[t] >= 0: k_pool[s / block_size][s % block_size][:][:]
 * = key[t][:][:], same for value.  Non-negative slots must be distinct within a call. */
pa_status pa_reshape_and_cache(const void* key, const void* value, void* k_pool, void* v_pool,
                               const int64_t* slot_mapping, int T, int Hkv, int D,
                               int block_size, int num_blocks, pa_dtype dtype,
                               int32_t* dev_err_flag, pa_stream_t stream);

/* For i < n: block pairs[i][1] of both pools = block pairs[i][0] (all block_size slots,
 * every head).  `pairs` is a DEVICE array.  Destinations must be distinct and no
 * destination may also be a source in the same call. */
pa_status pa_copy_blocks(void* k_pool, void* v_pool, const int32_t* pairs, int n,
                         int block_size, int Hkv, int D, int num_blocks, pa_dtype dtype,
                         int32_t* dev_err_flag, pa_stream_t stream);

/* ---------------------------------------------------------------------------
 * Host block allocator (opaque, library-owned; destroy with pa_alloc_destroy)
 *
 * Policy: the free list is a LIFO stack whose initial pops return 0, 1, 2, ... or,
 * with shuffle_seed != 0, a Fisher-Yates permutation drawn from splitmix64(seed)
 * (index next() % (i+1) for i = n-1 .. 1).  A sequence of n tokens holds
 * ceil(n / block_size) blocks.  Appending takes a fresh block when the last block is
 * full (or absent); when the last block is partial and shared (refcount > 1) the
 * append copies on write: it takes a fresh block dst, reports (src, dst), decrements
 * refcount(src) and points the table at dst.  Freed blocks are pushed in table order
 * when their refcount reaches 0.  A failing call changes no state, including one that
 * runs out of host memory (PA_ERR_HOST_MEMORY: every allocation a call needs is made
 * before it changes anything).  Not thread-safe.
 * ------------------------------------------------------------------------- */

typedef struct pa_allocator pa_allocator;

pa_status pa_alloc_create(int num_blocks, int block_size, uint64_t shuffle_seed,
                          pa_allocator** out);
/* Like pa_alloc_create with an explicit initial pop order (a permutation of
 * [0, num_blocks), host array, copied). */
pa_status pa_alloc_create_ordered(int num_blocks, int block_size, const int32_t* pop_order,
                                  pa_allocator** out);
void pa_alloc_destroy(pa_allocator* a);

/* Register a sequence already holding num_tokens tokens: ceil(num_tokens/bs) fresh blocks. */
pa_status pa_alloc_add_seq(pa_allocator* a, int64_t seq_id, int num_tokens);
/* child shares every block of parent (refcount +1 each) and its token count. */
pa_status pa_alloc_fork(pa_allocator* a, int64_t parent_id, int64_t child_id);
/* Reserve the slot of the sequence's next token; *cow_src = *cow_dst = -1 if no copy. */
pa_status pa_alloc_append_slot(pa_allocator* a, int64_t seq_id, int64_t* slot,
                               int32_t* cow_src, int32_t* cow_dst);
/* append_slot for n distinct sequences, in order, all or nothing: on any error no
 * sequence is changed.  Writes slot_mapping[n]; copy pairs to cow_pairs[2*k..] (room
 * for n pairs) and their count to *n_pairs. */
pa_status pa_alloc_append_slots(pa_allocator* a, const int64_t* seq_ids, int n,
                                int64_t* slot_mapping, int32_t* cow_pairs, int* n_pairs);
/* Drop a sequence; blocks whose refcount reaches 0 return to the free list. */
pa_status pa_alloc_free_seq(pa_allocator* a, int64_t seq_id);
/* Keep only the first num_tokens tokens (0 <= num_tokens <= current count), e.g. to roll
 * back rejected speculative tokens.  Blocks past ceil(num_tokens / block_size) are
 * released in table order (refcount - 1; free at 0).  A now-partial shared last block is
 * copied on write at the next append, as usual. */
pa_status pa_alloc_truncate(pa_allocator* a, int64_t seq_id, int num_tokens);
/* Beam-search step: beam i (seq_ids[i], n distinct live sequences) continues from beam
 * parent_idx[i] (0 <= parent_idx[i] < n).  Every new beam first takes a shared reference
 * to its parent's blocks and token count; then the beams' old tables are released, beam
 * 0 first, each in table order (refcount - 1; free at 0).  Allocates nothing. */
pa_status pa_alloc_beam_select(pa_allocator* a, const int64_t* seq_ids, const int32_t* parent_idx,
                               int n);

/* Copy the sequence's table (up to cap entries) to out; *n = its length, *num_tokens. */
pa_status pa_alloc_block_table(const pa_allocator* a, int64_t seq_id, int32_t* out, int cap,
                               int* n, int* num_tokens);
/* Fill block_tables[n][max_blocks] (padded with -1) and seq_lens[n] for n sequences. */
pa_status pa_alloc_block_tables(const pa_allocator* a, const int64_t* seq_ids, int n,
                                int32_t* block_tables, int max_blocks, int32_t* seq_lens);
/* PA_OK if every listed sequence exists (else PA_ERR_NOT_FOUND) and its table would still
 * fit max_blocks entries after one more token (else PA_ERR_INVALID_ARG).  Changes nothing. */
pa_status pa_alloc_check_append_fits(const pa_allocator* a, const int64_t* seq_ids, int n,
                                     int max_blocks);
/* Slots of all tokens of a sequence, token t at
 * table[t / block_size] * block_size + t % block_size (up to cap); *n = its token count.
 * Used to write a prompt's K/V (prefill) with pa_reshape_and_cache. */
pa_status pa_alloc_seq_slots(const pa_allocator* a, int64_t seq_id, int64_t* slots, int cap,
                             int* n);
/* Group a batch for pa_decode_shared_prefix (host arrays).  Batch rows whose tables start
 * with the same block are taken in batch order, in chunks of max_members; a chunk of >= 2
 * rows becomes a group whose shared prefix is the leading table entries all its members
 * hold, capped at the shortest member's length and rounded down to align_tokens; a chunk
 * whose prefix rounds to 0 is not grouped.  Writes group_of[n], group_prefix[ngroups],
 * group_members[ngroups][max_members] (-1 padded; room for n groups) and *ngroups. */
pa_status pa_alloc_prefix_groups(const pa_allocator* a, const int64_t* seq_ids, int n,
                                 int max_members, int align_tokens, int32_t* group_of,
                                 int32_t* group_prefix, int32_t* group_members, int* ngroups);
int pa_alloc_refcount(const pa_allocator* a, int32_t block);   /* -1 if out of range */
int pa_alloc_num_free(const pa_allocator* a);
/* Sum over live sequences of (blocks * block_size - tokens). */
int64_t pa_alloc_internal_waste_slots(const pa_allocator* a);
/* Free stack bottom-to-top into out (up to cap); returns its length. */
int pa_alloc_free_list(const pa_allocator* a, int32_t* out, int cap);

/* ---------------------------------------------------------------------------
 * Decode-step pipeline: one call per step of a serving loop
 *
 * Each step: the allocator reserves every sequence's next slot (pa_alloc_append_slots;
 * copy-on-write pairs for partial blocks still shared) and writes the padded tables and
 * lengths (pa_alloc_block_tables) into a pinned host input slot behind the step's q / new
 * K / new V, which the caller wrote there; one host->device copy moves the slot; then
 * pa_copy_blocks (if the step has pairs) and pa_decode_append run, and the output is
 * copied back to a pinned host output slot.  Copies run on their own streams and steps
 * are queued back to back over `depth` slots, so the host prepares step t+1 and the copy
 * engines move neighbouring steps' data while the GPU decodes step t ("深入解析
 * PagedAttention", 核心创新: blocks are allocated on demand as each sequence grows;
 * "什么是 LLM 中的分页注意力", 使用分页注意力: each new token fills the next slot of the
 * sequence's current block).
 *
 * With shared_prefix_members > 0 a step is the parallel-sampling one ("深入解析
 * PagedAttention", 多序列共享): after the appends the allocator also groups the rows whose
 * tables share leading blocks (pa_alloc_prefix_groups, up to shared_prefix_members rows a
 * group, PA_SHARED_PREFIX_ALIGN) and writes the slot mapping, and the kernels are
 * pa_copy_blocks, pa_reshape_and_cache and pa_decode_shared_prefix, which reads each
 * group's shared blocks once.
 *
 * Ownership: every buffer and stream is the caller's; the pipeline creates only CUDA
 * events (no device memory).  The allocator is borrowed: it must outlive the pipeline and
 * not be used by another thread during a call.  Not thread-safe.
 * ------------------------------------------------------------------------- */

typedef struct pa_pipeline pa_pipeline;

typedef struct pa_pipeline_desc {
  int B, Hq, Hkv, D, block_size, max_blocks, num_blocks;  /* the batch shape, fixed */
  pa_dtype dtype;
  int depth;                  /* staging slots, 1 .. 64 */
  void* k_pool;               /* device pools [num_blocks][block_size][Hkv][D] */
  void* v_pool;
  void* workspace;            /* device, pa_decode_workspace_size bytes (may be NULL) */
  size_t workspace_bytes;
  int32_t* dev_err_flag;      /* device, nullable */
  void* const* host_in;       /* [depth] pinned host, pa_pipeline_input_bytes each */
  void* const* dev_in;        /* [depth] device, pa_pipeline_input_bytes each, 256-B aligned */
  void* const* host_out;      /* [depth] pinned host [B][Hq][D] */
  void* const* dev_out;       /* [depth] device [B][Hq][D], 16-B aligned */
  pa_stream_t compute;        /* kernels */
  pa_stream_t copy_in;        /* host->device copies */
  pa_stream_t copy_out;       /* device->host copies */
  int shared_prefix_members;  /* 0: pa_decode_append; 1 .. 32: the shared-prefix step, for
                                 shapes pa_decode_shared_prefix takes (bf16, members *
                                 Hq/Hkv <= 64, ...) and a workspace of at least
                                 pa_decode_shared_prefix_workspace_size(B, .., B / 2) bytes
                                 (checked by pa_pipeline_create: PA_ERR_INVALID_ARG) */
} pa_pipeline_desc;

/* Bytes of one input slot; offsets[6] (nullable) receives the byte offsets of its
 * sections: q [B][Hq][D], k_new [B][Hkv][D], v_new [B][Hkv][D] (written by the caller),
 * block_tables [B][max_blocks] int32, seq_lens [B] int32 and copy pairs [B][2] int32
 * (written by the pipeline).  0 for invalid arguments. */
size_t pa_pipeline_input_bytes(int B, int Hq, int Hkv, int D, int max_blocks, pa_dtype dtype,
                               size_t* offsets);
/* The same for a pipeline with shared_prefix_members = m: offsets[10] (nullable) adds,
 * after those six, slot_mapping [B] int64, group_of [B], group_prefix [B] and
 * group_members [B][m] int32 (all written by the pipeline).  With m = 0 it equals
 * pa_pipeline_input_bytes.  0 for invalid arguments (m outside 0 .. 32). */
size_t pa_pipeline_input_bytes_prefix(int B, int Hq, int Hkv, int D, int max_blocks,
                                      pa_dtype dtype, int shared_prefix_members,
                                      size_t* offsets);
/* The descriptor's arrays are copied.  PA_ERR_INVALID_ARG for a bad descriptor. */
pa_status pa_pipeline_create(pa_allocator* alloc, const pa_pipeline_desc* desc,
                             pa_pipeline** out);
/* Waits for every queued step, then frees the pipeline (not the caller's buffers). */
void pa_pipeline_destroy(pa_pipeline* p);
/* *slot = the input slot of the next step, once its previous host->device copy has
 * finished: the caller then writes q, k_new and v_new there and calls submit. */
pa_status pa_pipeline_next_slot(pa_pipeline* p, int* slot);
/* Queue one step for seq_ids[B] (distinct live sequences; the batch order of q/k/v).
 * *step (nullable) = its index (0, 1, ...), *h2d_bytes (nullable) = bytes copied in.
 * Returns once the step is queued.  An allocator error (e.g. PA_ERR_OUT_OF_BLOCKS) leaves
 * everything unchanged, except that a failure of the shared-prefix grouping (host memory
 * only) leaves the step's appends made; after PA_ERR_CUDA the pipeline should be
 * destroyed. */
pa_status pa_pipeline_submit(pa_pipeline* p, const int64_t* seq_ids, float scale,
                             int64_t* step, size_t* h2d_bytes);
/* Waits for step's output copy; *slot = the host_out slot holding it, valid until step +
 * depth is submitted.  PA_ERR_INVALID_ARG for a step not yet queued or no longer held. */
pa_status pa_pipeline_result(pa_pipeline* p, int64_t step, int* slot);
/* Waits for every queued step. */
pa_status pa_pipeline_sync(pa_pipeline* p);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_CACHE_350_B200_PA_H */
