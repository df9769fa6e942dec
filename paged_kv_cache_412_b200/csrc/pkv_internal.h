// pkv_internal.h -- host-side declarations shared by the library's translation
// units (launchers, per-device state).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

// Per-device facts the launchers need, queried once per device.
struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int max_smem_optin = 0;
    unsigned* error_word = nullptr;  // device address of the error word
};

// Info for the current device (thread-safe, cached).  nullptr on failure.
const DeviceInfo* current_device_info();

// Workspace bound of one decode call.  It covers both decode kernels (the
// tensor-core one groups up to 16 query heads per kv-head pass, the CUDA-core
// one up to 8), so one size fits whichever path the call takes.
//
// Layout of a workspace of B bytes: the records' ready flags first, in a
// region whose size depends only on B (sync_region_bytes(B)), then the partial
// records.  A given buffer therefore always keeps its flags in the same words,
// which every call returns to zero; records are always written before they are
// read in the same call and need no clearing, whatever the sizes of the next
// call.
struct DecodePlan {
    int rec_gp;        // floats per record row = largest query-head group of either path
    size_t n_bg_max;   // (request, head group) pairs, largest over the paths
    size_t units_max;  // upper bound of split units
    size_t records;    // partial-result records
    size_t rec_bytes;  // records + their (max, sum) pairs + per-group meta
    size_t off_ml, off_meta;  // offsets inside the record region
    size_t off_extra;         // caller-specific scratch after the records
    size_t bytes;      // smallest workspace that fits
};

// Bytes at the start of a B-byte workspace reserved for the merge's
// synchronisation words, all of which return to zero at the end of every call:
// one ready flag per partial record in its first half, per-group arrival
// counters in its second half.
inline size_t sync_region_bytes(size_t workspace_bytes) {
    return (workspace_bytes / 128 + 255) / 256 * 256;
}
inline size_t sync_counters_offset(size_t workspace_bytes) {
    return sync_region_bytes(workspace_bytes) / 2;
}

// Fill a plan for these sizes on the current device (false if invalid).
// extra_bytes: scratch placed after the records (no clearing needed).
bool make_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int max_seq_len, int partition_size, DecodePlan* plan,
                      size_t extra_bytes = 0);

// Kernel arguments of the decode path (plain values, passed by value).
struct DecodeParams {
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    void* out;
    const float* k_scale;
    const float* v_scale;
    float* rec_acc;   // [records][group_pad][head_dim]
    float* rec_ml;    // [records][group_pad][2]  (running max in log2 units, sum)
    int32_t* meta;    // [num_seqs * num_hg][2]   (first unit, number of units)
    unsigned* ready;  // [records] 1 once a partial record is written (zero between calls)
    unsigned* err;
    int num_seqs, num_q_heads, num_kv_heads, group, num_sub, num_hg;
    int block_size, log2_bs, max_blocks, num_blocks;
    int fixed_units;  // 0 = automatic
    int max_len_hint;  // the caller's bound of seq_lens (a guess of the first table window)
    int defer_merge;  // 1: parts of a split group only publish records (+ meta);
                      // a separate merge kernel combines them
    int row_copy;     // 1: blocks of 2 or 4 rows -- one bulk copy per (block, K or V)
                      // into a skewed stage layout instead of TMA boxes
    unsigned* counters;  // [num_seqs * num_hg] arrivals per split group (zero between calls)
    long long rec_cap;  // records the workspace holds
    int out_dtype;
    float scale_log2;  // softmax scale * log2(e)
    // Shared prefixes (prefix_of == nullptr: none).  Request b's own pass
    // starts at the end of its group's prefix and its output folds in the
    // shared pass's partial results (pfx_*), one per split of that pass.
    const int32_t* prefix_of;    // [num_seqs] group or -1
    const int32_t* prefix_lens;  // [num_prefixes] tokens
    const float* pfx_acc;        // [pfx_splits][num_seqs][num_q_heads][head_dim]
    const float* pfx_ml;         // [pfx_splits][num_seqs][num_q_heads][2]
    int num_prefixes, max_prefix_len, pfx_splits;
    // Bound of every in-kernel wait (ns of global time), and a test-only fault
    // (DecodeFault) that makes one wait run out; 0 = none.
    unsigned long long wait_ns;
    int fault_mode, fault_arg;
    // Fused append (pkv_paged_attention_decode_append): request b's new K/V rows
    // [num_seqs][num_kv_heads][head_dim] bf16, written at position seq_lens[b]-1
    // before the decode reads that block; nullptr: no append.
    const void* k_new;
    const void* v_new;
};

// Test-only faults of the tensor-core decode, set for the next decode call of
// the calling host thread by pkv_internal_decode_fault (exported, not part of
// the public header).  Each one makes a bounded wait run out so the give-up
// path (PKV_DEVERR_TIMEOUT, workspace re-initialisation) can be exercised
// without faulting the GPU:
//   kFaultMergeFlag: the merger of a split group also waits for its own
//     ready flag, which nothing sets;
//   kFaultSkipStage: CTA 0's producer never arrives on the full barrier of its
//     chunk fault_arg (no copy is issued for it), so that stage never fills.
enum DecodeFault { kFaultNone = 0, kFaultMergeFlag = 1, kFaultSkipStage = 2 };

// Host argument checks of a decode call (everything but the workspace):
// null pointers, sizes, dtypes, head_dim, alignment.  PKV_OK if the call may
// proceed.
pkv_status check_decode_args(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* seq_lens,
                             int32_t block_size, float scale, const void* out, int32_t num_seqs,
                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                             int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_seq_len,
                             pkv_dtype q_dtype, pkv_dtype kv_dtype, pkv_dtype out_dtype,
                             const float* k_scale, const float* v_scale, int32_t partition_size);

// Kernel arguments of the shared pass of pkv_paged_attention_decode_prefix.
// CTA x handles split (x % splits) of row tile ((x / splits) % row_tiles) of
// kv head ((x / splits / row_tiles) % num_kv_heads) of group
// (x / splits / row_tiles / num_kv_heads); a row tile is 64 (member, query
// head) rows of the group, members in request order.
struct PrefixParams {
    const void* q;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    const int32_t* prefix_of;
    const int32_t* prefix_lens;
    float* pfx_acc;  // as DecodeParams
    float* pfx_ml;
    unsigned* err;
    int num_seqs, num_q_heads, num_kv_heads, group;
    int block_size, log2_bs, max_blocks, num_blocks;
    int num_prefixes, max_members, max_prefix_len, splits, row_tiles;
    float scale_log2;
};

// Rows of (member, query head) pairs one CTA of the shared pass covers.
constexpr int kPrefixRows = 128;
// CTAs of the shared pass resident per SM; the launch sizes its splits for one
// wave of that many.  (Two fit -- 256 tensor-memory columns and under half the
// shared memory each -- but doubled the partial records to merge and shared one
// SM's issue slots between two softmax chains: slower.)
constexpr int kPrefixCtasPerSm = 1;

pkv_status launch_decode_prefix(const PrefixParams& p, const void* k_cache, const void* v_cache,
                                int head_dim, cudaStream_t stream);

pkv_status launch_decode_simt(const DecodeParams& p, int head_dim, pkv_dtype kv_dtype,
                              int group_pad, cudaStream_t stream, int* grid_out);

bool decode_mma_supported(int head_dim, int block_size, pkv_dtype q_dtype, pkv_dtype kv_dtype);

pkv_status launch_decode_mma(const DecodeParams& p, int head_dim, int group_pad, bool fp8,
                             cudaStream_t stream, int* grid_out);

// TMA view of a cache [num_blocks, Hkv, block_size, head_dim] as rows x
// head_dim: bf16 boxes of 64 columns x box_rows rows with the 128-byte
// swizzle (both_halves at head_dim 128: 3-D boxes holding both 64-column
// halves); fp8 boxes of whole rows with the swizzle of their width.  False if
// the driver entry point is missing or the encoder rejects the view.
bool encode_cache_map(CUtensorMap* map, const void* base, long long rows, int head_dim,
                      int box_rows, bool fp8, bool both_halves = false);

// Launch config with programmatic dependent launch: the kernel may start while
// the previous kernel in the stream drains; it waits (griddepcontrol.wait)
// before touching memory.
struct PdlLaunch {
    cudaLaunchConfig_t cfg{};
    cudaLaunchAttribute attr[1];
    PdlLaunch(dim3 grid, dim3 block, size_t smem, cudaStream_t s) {
        cfg.gridDim = grid;
        cfg.blockDim = block;
        cfg.dynamicSmemBytes = smem;
        cfg.stream = s;
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
    }
};

pkv_status launch_kv_cache_write(const void* k, const void* v, const int64_t* slots,
                                 void* k_cache, void* v_cache, int num_tokens, int num_kv_heads,
                                 int head_dim, int block_size, int num_blocks, int elem_bytes,
                                 unsigned* err, cudaStream_t stream);

// Each request's new token (position seq_lens[b] - 1) appended through its
// block table: bf16 rows k[b], v[b] of [num_seqs, num_kv_heads, head_dim].
pkv_status launch_append_by_table(const void* k, const void* v, const int32_t* block_tables,
                                  const int32_t* seq_lens, void* k_cache, void* v_cache,
                                  int num_seqs, int num_kv_heads, int head_dim, int block_size,
                                  int log2_bs, int max_blocks, int num_blocks,
                                  cudaStream_t stream);

// Whether the tensor-core decode of this call appends inside its own launch
// (the one-CTA-per-SM layout); otherwise the append runs as its own kernel.
bool decode_mma_fuses_append(const DecodeParams& p, int group_pad);

pkv_status launch_kv_cache_write_fp8(const void* k, const void* v, const int64_t* slots,
                                     void* k_cache, void* v_cache, const float* k_scale,
                                     const float* v_scale, int num_tokens, int num_kv_heads,
                                     int head_dim, int block_size, int num_blocks, unsigned* err,
                                     cudaStream_t stream);

pkv_status launch_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                              const int64_t* pairs, int num_pairs, size_t block_bytes,
                              int src_blocks, int dst_blocks, unsigned* err,
                              cudaStream_t stream);

pkv_status launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int num_pairs,
                              size_t block_bytes, int num_blocks, unsigned* err,
                              cudaStream_t stream);

}  // namespace pkv
