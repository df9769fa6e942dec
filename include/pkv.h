/*
 * pkv.h -- C ABI of the B200 paged KV-cache library (sm_100a).
 *
 * The library implements the data-parallel hot path of PagedAttention:
 *   - pkv_kv_cache_write          scatter each new token's K/V into its slot;
 *   - pkv_paged_attention_decode  single-query decode attention over a cache
 *                                 held in fixed-size physical blocks reached
 *                                 through a per-request block table;
 *   - pkv_paged_attention_decode_append  the append of each request's new
 *                                 token and the decode, in one launch where
 *                                 the decode's layout allows;
 *   - pkv_copy_blocks             copy-on-write copy of shared blocks;
 *   - pkv_paged_attention_decode_prefix  the same decode with the blocks a
 *                                 group of requests shares read once per group.
 *
 * Sources (web pages on the subject; cited by title and section):
 *   [KVOPT]  "KV Cache Optimization and PagedAttention" (intro prose).
 *   [PAMEM]  "PagedAttention: Optimizing KV Cache Utilization in Large Language
 *            Models": "The Mechanics of PagedAttention", "The Math: Block
 *            Attention Calculation", "Serving Advantages", "Conclusion".
 *   [KVMGMT] "KV Cache Management": "The Solution: PagedAttention (vLLM)",
 *            "The Bonus: Zero-Copy Sharing", "Watch Out For".
 *
 * Conventions shared by every call
 *   - Pointers are DEVICE pointers of the current CUDA device unless a comment
 *     says "host".  The caller owns and allocates all memory; the library
 *     allocates nothing (decode scratch is a caller-provided workspace).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  The returned status reports host-side validation and
 *     launch errors only.
 *   - Cache layout: k_cache / v_cache are [num_blocks, num_kv_heads,
 *     block_size, head_dim], row-major, so each (block, kv head) is one
 *     contiguous block_size*head_dim run.  The token at logical position t of a
 *     request lives in physical block block_tables[b][t / block_size] at offset
 *     t % block_size; a slot id is physical_block * block_size + offset.
 *   - Query head h reads kv head h / (num_q_heads / num_kv_heads).
 *   - Indices the device finds out of range (a slot, a block id, a sequence
 *     longer than its block table) are skipped and raise a bit in a per-device
 *     error word; pkv_get_device_error reads and clears it.  Kernels never trap.
 *   - Supported: head_dim 64 or 128; block_size a power of two in [1, 256];
 *     element types PKV_F32 and PKV_BF16 (decode, write, copy) and
 *     PKV_FP8_E4M3 caches (see the fp8 calls).
 */
#ifndef PKV_H_
#define PKV_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t, spelled without the CUDA headers. */
typedef struct CUstream_st* pkv_stream_t;

typedef enum pkv_status {
    PKV_OK = 0,
    PKV_ERR_INVALID_ARG = 1,   /* null pointer, bad size, inconsistent dims      */
    PKV_ERR_UNSUPPORTED = 2,   /* valid but not implemented (dtype, head_dim...) */
    PKV_ERR_WORKSPACE = 3,     /* workspace null or smaller than required        */
    PKV_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed           */
    PKV_ERR_DEVICE_INDEX = 5,  /* pkv_get_device_error found a device-side flag  */
    PKV_ERR_OUT_OF_BLOCKS = 6  /* block allocator: not enough free blocks        */
} pkv_status;

typedef enum pkv_dtype {
    PKV_F32 = 0,
    PKV_BF16 = 1,
    PKV_FP8_E4M3 = 2
} pkv_dtype;

/* Bits of the device error word (pkv_get_device_error). */
#define PKV_DEVERR_BAD_SLOT 0x1u       /* write: slot >= num_blocks*block_size      */
#define PKV_DEVERR_BAD_BLOCK 0x2u      /* decode: table entry outside [0,num_blocks) */
#define PKV_DEVERR_BAD_SEQ_LEN 0x4u    /* decode: seq_len < 0 or > max_blocks*bs    */
#define PKV_DEVERR_BAD_PAIR 0x8u       /* copy/swap: block id out of range; copy:
                                          a dst repeated or also a src            */
#define PKV_DEVERR_TIMEOUT 0x10u       /* a bounded in-kernel wait gave up          */
#define PKV_DEVERR_PREFIX 0x20u        /* prefix decode: bad group id, length or size */

/* Human-readable name of a status code (static string). */
const char* pkv_status_string(pkv_status status);

/* Library version, major*10000 + minor*100 + patch. */
int pkv_version(void);

/*
 * pkv_kv_cache_write -- append new tokens' K and V to the paged cache.
 *
 * [PAMEM] "The Mechanics of PagedAttention": as tokens are generated, their K
 * and V vectors are written into the request's allocated physical blocks,
 * wherever those blocks sit in memory.
 *
 *   k, v          [num_tokens, num_kv_heads, head_dim], element type dtype.
 *   slot_mapping  [num_tokens] int64; token t goes to block slot/block_size at
 *                 offset slot%block_size.  slot < 0 marks padding: skipped.
 *                 slot >= num_blocks*block_size: skipped, PKV_DEVERR_BAD_SLOT.
 *                 Slots must be distinct within one call (else the result of
 *                 the colliding tokens is unspecified).
 *   k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim].
 * The copy is bit-exact.  num_tokens == 0 launches nothing and returns PKV_OK.
 */
pkv_status pkv_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                              void* k_cache, void* v_cache, int32_t num_tokens,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int32_t num_blocks, pkv_dtype dtype, pkv_stream_t stream);

/*
 * pkv_kv_cache_write_fp8 -- append new tokens to an fp8 (e4m3) cache.
 *
 * "KV Cache Management", "Watch Out For" and "What to Read Next": long
 * contexts call for quantising the KV cache to 8 bits.  Each value is stored
 * as the e4m3 code of x / scale[h] (one fp32 scale per kv head, the quotient
 * rounded as an IEEE fp32 division, then rounded to nearest even and saturated
 * at +-448), and read back as code * scale[h].
 *   k, v          [num_tokens, num_kv_heads, head_dim] bf16.
 *   k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim] uint8 codes.
 *   k_scale, v_scale  [num_kv_heads] fp32 (device).
 * Slots as in pkv_kv_cache_write.
 */
pkv_status pkv_kv_cache_write_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                                  void* k_cache, void* v_cache, const float* k_scale,
                                  const float* v_scale, int32_t num_tokens, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  pkv_stream_t stream);

/*
 * pkv_decode_workspace_bytes -- bytes of device scratch that
 * pkv_paged_attention_decode needs for these sizes on the CURRENT device.
 * max_seq_len bounds every seq_lens entry of the calls that will use it;
 * partition_size as in the decode call (0 = automatic).  Returns 0 for
 * invalid sizes.
 */
size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                  int32_t num_kv_heads, int32_t head_dim,
                                  int32_t block_size, int32_t max_seq_len,
                                  int32_t partition_size);

/*
 * pkv_decode_workspace_init -- zero a decode workspace (asynchronous on
 * `stream`).  Call once after allocating a workspace, before its first decode.
 * Decode calls leave the workspace ready for the next call (the ready flags
 * of the partial results they use return to zero), so re-initialising is
 * needed only if a call reported PKV_DEVERR_TIMEOUT.
 */
pkv_status pkv_decode_workspace_init(void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream);

/*
 * pkv_paged_attention_decode -- one decode step of attention for a batch.
 *
 * [PAMEM] "The Math: Block Attention Calculation": for query q_i the page
 * table gives the physical location of every key K_j and the scores are
 * Softmax(q_i K^T / sqrt(d_k)).  The printed per-block softmax is read as the
 * block's slice of ONE softmax over all of the request's tokens; the output
 * is that softmax applied to the V rows:
 *     out[b,h,:] = sum_t softmax_t(scale * q[b,h,:] . K_t) V_t
 * over the seq_lens[b] tokens of request b (seq_lens counts the token
 * appended this step).  seq_lens[b] == 0 gives an all-zero row.
 *
 *   q             [num_seqs, num_q_heads, head_dim], element type q_dtype
 *                 (PKV_F32 with an fp32 cache, PKV_BF16 with bf16/fp8 caches).
 *   k_cache, v_cache  cache layout above, element type kv_dtype.
 *   block_tables  [num_seqs, max_blocks_per_seq] int32; entries past
 *                 ceil(seq_len/block_size) are never read.
 *   seq_lens      [num_seqs] int32.
 *   out           [num_seqs, num_q_heads, head_dim], element type out_dtype
 *                 (PKV_F32 or PKV_BF16; round to nearest even).
 *   k_scale, v_scale  [num_kv_heads] fp32 dequantisation scales for an fp8
 *                 cache (value = code * scale); NULL otherwise.
 *   scale         softmax scale (1/sqrt(head_dim) for standard attention).
 *   max_seq_len   an upper bound of seq_lens (sizes the workspace check).
 *   partition_size  0 = automatic split of the whole batch's KV into equal
 *                 shares, one per resident CTA; else tokens per split unit
 *                 (a multiple of 32).
 *   Ordering: the kernel is launched as a programmatic dependent of the
 *                 previous kernel in the stream and reads seq_lens and
 *                 block_tables while that kernel drains; it waits for it before
 *                 touching q, the caches, out or the workspace.  So seq_lens and
 *                 block_tables must not be written by the kernel immediately
 *                 before this call if that kernel releases its dependents early
 *                 (griddepcontrol.launch_dependents); host copies and ordinary
 *                 kernels are fine, and so is pkv_kv_cache_write.  With
 *                 partition_size > 0 on the bf16/fp8 path a merge kernel
 *                 follows on the same stream.
 *   workspace     device scratch of at least pkv_decode_workspace_bytes(...)
 *                 bytes, 256-byte aligned, zeroed once by
 *                 pkv_decode_workspace_init.  Calls that overlap in time need
 *                 distinct workspaces.
 * Accumulation is fp32.  Out-of-range table entries are skipped (their tokens
 * do not take part) and flag PKV_DEVERR_BAD_BLOCK; seq_lens outside
 * [0, max_blocks_per_seq*block_size] are clamped and flag
 * PKV_DEVERR_BAD_SEQ_LEN.
 */
pkv_status pkv_paged_attention_decode(const void* q, const void* k_cache,
                                      const void* v_cache, const int32_t* block_tables,
                                      const int32_t* seq_lens, int32_t block_size,
                                      float scale, void* out, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t max_blocks_per_seq,
                                      int32_t num_blocks, int32_t max_seq_len,
                                      pkv_dtype q_dtype, pkv_dtype kv_dtype,
                                      pkv_dtype out_dtype, const float* k_scale,
                                      const float* v_scale, int32_t partition_size,
                                      void* workspace, size_t workspace_bytes,
                                      pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_append -- each request's new token appended to
 * the cache, then pkv_paged_attention_decode.
 *
 * [PAMEM] "The Mechanics of PagedAttention": the new token's K and V go to the
 * slot its block table names; "The Math: Block Attention Calculation": the
 * decode.  Request b's new token is the last of its seq_lens[b] tokens: K row
 * k_new[b] and V row v_new[b] are written at position L-1 (L = seq_lens[b]) as
 * the table names it -- physical block block_tables[b][(L-1)/block_size], row
 * (L-1) % block_size -- the same bytes pkv_kv_cache_write writes for that
 * slot; the decode then runs exactly as pkv_paged_attention_decode (same
 * arguments, same result).  When the decode runs one CTA per SM (groups of at
 * most 8 query heads per kv head and fewer than 4 (request, kv head) pairs per
 * SM), the row is written inside the decode launch, by the CTA that fetches
 * its block, just before fetching it: one launch.  Otherwise (many short
 * groups, where that CTA's single producer would be held up) a small append
 * kernel runs first and the decode overlaps its start: two launches.
 *   k_new, v_new  [num_seqs, num_kv_heads, head_dim] bf16, 16-byte aligned.
 *   Other arguments as pkv_paged_attention_decode.  bf16 q and caches on the
 *   tensor-core path (block_size >= 2, not 1) only: other configurations
 *   return PKV_ERR_UNSUPPORTED (use pkv_kv_cache_write + the decode).  A
 *   request with seq_lens[b] == 0 appends nothing; an out-of-range table entry
 *   skips the copy and flags PKV_DEVERR_BAD_BLOCK, as the decode does.
 */
pkv_status pkv_paged_attention_decode_append(
    const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
    const int32_t* block_tables, const int32_t* seq_lens, int32_t block_size, float scale,
    void* out, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_seq_len, pkv_dtype out_dtype,
    int32_t partition_size, void* workspace, size_t workspace_bytes, pkv_stream_t stream);

/*
 * pkv_decode_prefix_workspace_bytes -- workspace bytes of
 * pkv_paged_attention_decode_prefix for these sizes on the CURRENT device:
 * the decode's own scratch plus one partial result per (split of the shared
 * pass, request, query head).  max_prefix_members bounds the requests of any
 * one group; max_prefix_len bounds every prefix_lens entry.  0 if invalid.
 */
size_t pkv_decode_prefix_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int32_t max_seq_len,
                                         int32_t num_prefixes, int32_t max_prefix_members,
                                         int32_t max_prefix_len);

/*
 * pkv_paged_attention_decode_prefix -- pkv_paged_attention_decode for a batch
 * in which groups of requests share the physical blocks of a common prefix.
 *
 * [KVMGMT] "The Bonus: Zero-Copy Sharing" and [KVOPT]: requests forked from
 * one prompt point their block tables at the same physical blocks, stored
 * once.  This call also READS them once per group: a shared pass streams the
 * group's prefix blocks a single time for all of the group's query heads (a
 * dense contraction over the group's q rows), leaving one partial softmax
 * state per (request, query head); each request's own pass then covers only
 * the tokens after the prefix and merges the two states.  The result is the
 * same attention as pkv_paged_attention_decode over the full tables (up to
 * fp32 rounding order); nothing about the output depends on the grouping.
 *
 *   prefix_of     [num_seqs] int32: the group of request b, or -1 for none.
 *   prefix_lens   [num_prefixes] int32: tokens of group g's prefix, a multiple
 *                 of block_size, <= max_prefix_len.  Contract: for every
 *                 member b, block_tables[b][j] is the same physical block for
 *                 all j < prefix_lens[g] / block_size (the shared blocks of a
 *                 fork; the partly filled block a fork copies is not part of
 *                 it).  A member shorter than the prefix attends to its own
 *                 seq_lens[b] tokens only.  The shared pass reads the table of
 *                 the group's longest member.
 *   num_prefixes, max_prefix_members, max_prefix_len  as for
 *                 pkv_decode_prefix_workspace_bytes; the workspace must be at
 *                 least that size.
 *   Other arguments as pkv_paged_attention_decode (partition_size automatic).
 *   Supported: q and caches PKV_BF16, head_dim 64 or 128, block_size >= 8;
 *   other configurations return PKV_ERR_UNSUPPORTED.
 *   Ordering: three kernels on `stream`: the shared pass, each request's own
 *   pass, and the merge of the two; the first two read seq_lens,
 *   block_tables, prefix_of and prefix_lens before waiting for the previous
 *   kernel, with the same rule as pkv_paged_attention_decode.
 *   Device checks: a group id >= num_prefixes, a prefix length that is not a
 *   multiple of block_size or exceeds max_prefix_len (it is clamped and
 *   rounded down), and a group with more than max_prefix_members requests
 *   raise PKV_DEVERR_PREFIX; the outputs of members past that bound are
 *   undefined.
 */
pkv_status pkv_paged_attention_decode_prefix(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* seq_lens, int32_t block_size, float scale, void* out, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq,
    int32_t num_blocks, int32_t max_seq_len, pkv_dtype q_dtype, pkv_dtype kv_dtype,
    pkv_dtype out_dtype, const int32_t* prefix_of, const int32_t* prefix_lens,
    int32_t num_prefixes, int32_t max_prefix_members, int32_t max_prefix_len, void* workspace,
    size_t workspace_bytes, pkv_stream_t stream);

/*
 * pkv_paged_attention_decode_noalloc -- pkv_paged_attention_decode for callers
 * that cannot allocate device memory.
 *
 * The pages have no counterpart of this call; it exists for integration.  A
 * serving engine that reserves nearly all device memory for its KV pool up
 * front may not let an extension allocate, and on a latency-critical path the
 * device-wide synchronisation of cudaMalloc may not be acceptable.  This
 * variant takes the same arguments minus the workspace and runs the same
 * decode with its scratch in a fixed array inside the library's device image
 * (pkv_decode_noalloc_scratch_bytes() bytes, held by every device that loads
 * the library until the process exits).  It allocates nothing.
 *   - Sizes whose scratch (pkv_decode_workspace_bytes) exceeds that maximum are
 *     refused with PKV_ERR_WORKSPACE; nothing is launched.
 *   - The first call on a device finds the array's device address (with that
 *     device current) and zeroes it on `stream`; make that first call before
 *     any stream capture.
 *   - Each call clears, on `stream`, the part of the array that must start at
 *     zero; the rest keeps the previous call's contents.
 *   - All calls on a device share the array: calls that overlap on the GPU
 *     (other streams, other host threads) race.  Order them.
 */
pkv_status pkv_paged_attention_decode_noalloc(const void* q, const void* k_cache,
                                              const void* v_cache,
                                              const int32_t* block_tables,
                                              const int32_t* seq_lens, int32_t block_size,
                                              float scale, void* out, int32_t num_seqs,
                                              int32_t num_q_heads, int32_t num_kv_heads,
                                              int32_t head_dim, int32_t max_blocks_per_seq,
                                              int32_t num_blocks, int32_t max_seq_len,
                                              pkv_dtype q_dtype, pkv_dtype kv_dtype,
                                              pkv_dtype out_dtype, const float* k_scale,
                                              const float* v_scale, int32_t partition_size,
                                              pkv_stream_t stream);

/* Size in bytes of the fixed scratch array pkv_paged_attention_decode_noalloc uses. */
size_t pkv_decode_noalloc_scratch_bytes(void);

/*
 * pkv_copy_blocks -- copy whole physical blocks (copy-on-write fork).
 *
 * [KVOPT] intro and [KVMGMT] "The Bonus: Zero-Copy Sharing": requests with a
 * common prefix point their block tables at the same physical blocks; before
 * a request appends into a shared, partially filled block it takes a private
 * copy of it.  For every pair: k_cache[dst] = k_cache[src] and
 * v_cache[dst] = v_cache[src] (all kv heads, all slots), bit-exact.
 *
 *   block_mapping [num_pairs, 2] int64 (src, dst).  dst ids must be distinct
 *                 and no dst may also be a src in the same call (then the
 *                 copies touch disjoint blocks and their order is immaterial);
 *                 the device checks this and raises PKV_DEVERR_BAD_PAIR for a
 *                 call that breaks it, whose result is then unspecified.
 *                 Out-of-range ids: pair skipped, PKV_DEVERR_BAD_PAIR.
 *   elem_bytes of dtype: 4 (F32), 2 (BF16), 1 (FP8_E4M3).
 */
pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                           int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, pkv_dtype dtype,
                           pkv_stream_t stream);

/*
 * pkv_swap_blocks -- copy whole blocks between two pools, e.g. the device cache
 * and a host pool, for preemption.
 *
 * "PagedAttention: Optimizing KV Cache Utilization in Large Language Models",
 * "Conclusion": when generation runs out of physical blocks, requests are
 * preempted and their KV cache recomputed or swapped out, then swapped back in.
 * For every pair: dst_k_cache[dst] = src_k_cache[src] (same for V), all kv
 * heads and slots, bit-exact.  Pools have the cache layout above with
 * src_num_blocks / dst_num_blocks blocks.
 *
 *   All five pointers must be reachable from the current device: device
 *   memory, or pinned host memory mapped into its address space (cudaHostAlloc /
 *   torch pin_memory).  Anything else (pageable host memory, another device's
 *   memory) is refused with PKV_ERR_INVALID_ARG before any launch.
 *   block_mapping [num_pairs, 2] int64 (src, dst); out-of-range ids: pair
 *   skipped, PKV_DEVERR_BAD_PAIR.  dst ids distinct.
 */
pkv_status pkv_swap_blocks(const void* src_k_cache, const void* src_v_cache, void* dst_k_cache,
                           void* dst_v_cache, const int64_t* block_mapping, int32_t num_pairs,
                           int32_t src_num_blocks, int32_t dst_num_blocks, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, pkv_dtype dtype,
                           pkv_stream_t stream);

/*
 * pkv_get_device_error -- synchronise `stream`, then read and clear the error
 * word of the current device into *flags (PKV_DEVERR_* bits; 0 = clean).
 * Returns PKV_ERR_DEVICE_INDEX if any bit was set, PKV_OK if none.  The word
 * is shared by every stream of the device.
 */
pkv_status pkv_get_device_error(pkv_stream_t stream, uint32_t* flags /* host */);

/* ==========================================================================
 * Host-side block manager (no GPU work; all pointers below are HOST pointers)
 *
 * "KV Cache Optimization and PagedAttention" (intro), "PagedAttention:
 * Optimizing KV Cache Utilization in Large Language Models" ("The Mechanics of
 * PagedAttention") and "KV Cache Management" ("The Solution: PagedAttention
 * (vLLM)", "The Bonus: Zero-Copy Sharing"): physical blocks are handed out on
 * demand as a request's tokens arrive; a per-request block table maps logical
 * to physical blocks; requests with a common prefix share physical blocks, each
 * carrying a reference count, and a request that must write into a shared,
 * partially filled block first gets a private copy (copy-on-write).
 * Not thread-safe: one allocator per host thread, or external locking.
 * ========================================================================== */

typedef struct pkv_allocator pkv_allocator;

typedef struct pkv_allocator_stats {
    int32_t num_blocks;      /* pool size                                   */
    int32_t free_blocks;     /* on the free list                            */
    int32_t used_blocks;     /* referenced by at least one sequence         */
    int32_t shared_blocks;   /* referenced by more than one sequence        */
    int32_t num_seqs;
    int64_t stored_tokens;   /* valid slots in used blocks (shared counted once) */
    int64_t logical_tokens;  /* sum of the sequences' lengths               */
    int64_t unused_slots;    /* empty slots in used blocks (internal waste)  */
} pkv_allocator_stats;

/* Pool of num_blocks blocks of block_size slots (power of two <= 256). */
pkv_status pkv_allocator_create(int32_t num_blocks, int32_t block_size, pkv_allocator** out);
void pkv_allocator_destroy(pkv_allocator* allocator);

/* Register an empty sequence (seq_id must be new). */
pkv_status pkv_allocator_add_seq(pkv_allocator* allocator, int64_t seq_id);

/* New sequence `child` sharing every block of `parent` (reference counts + 1). */
pkv_status pkv_allocator_fork(pkv_allocator* allocator, int64_t parent, int64_t child);

/*
 * Append num_tokens tokens to seq_id.  Writes their slot ids to slots[0..n)
 * (for pkv_kv_cache_write).  If the sequence's last block is shared and only
 * partially filled, it is first replaced by a private copy: *num_cow = 1 and
 * cow_pair = {src, dst} (run pkv_copy_blocks on it before writing); else
 * *num_cow = 0.  PKV_ERR_OUT_OF_BLOCKS (nothing changed) if the pool cannot
 * supply the blocks needed.
 */
pkv_status pkv_allocator_append(pkv_allocator* allocator, int64_t seq_id, int32_t num_tokens,
                                int64_t* slots, int64_t* cow_pair, int32_t* num_cow);

/* Drop a sequence; blocks whose reference count reaches 0 return to the pool. */
pkv_status pkv_allocator_free_seq(pkv_allocator* allocator, int64_t seq_id);

/* Copy the sequence's block table into table[0..capacity); report its size. */
pkv_status pkv_allocator_block_table(const pkv_allocator* allocator, int64_t seq_id,
                                     int32_t* table, int32_t capacity, int32_t* num_blocks,
                                     int64_t* num_tokens);

pkv_status pkv_allocator_get_stats(const pkv_allocator* allocator, pkv_allocator_stats* out);

/* Reference count of a physical block (-1 for an invalid id). */
int32_t pkv_allocator_refcount(const pkv_allocator* allocator, int32_t block);

/*
 * Waste of the two reservation schemes the pages contrast ("KV Cache
 * Optimization and PagedAttention", intro and its waste example): a
 * contiguous region of reserve_len slots per request versus whole blocks of
 * block_size slots.  Also how many of the requests, taken in order, fit at
 * once in a pool of pool_slots slots under each scheme.
 */
typedef struct pkv_waste_report {
    int64_t used_slots;           /* sum of the lengths                       */
    int64_t contiguous_reserved;  /* n * reserve_len                          */
    int64_t paged_reserved;       /* sum of ceil(L / block_size) * block_size */
    int32_t contiguous_admitted;
    int32_t paged_admitted;
} pkv_waste_report;

pkv_status pkv_waste_compare(const int32_t* lengths, int32_t n, int32_t reserve_len,
                             int32_t block_size, int64_t pool_slots, pkv_waste_report* out);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H_ */
