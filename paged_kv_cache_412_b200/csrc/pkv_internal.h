// pkv_internal.h -- host-side declarations shared by the library's translation
// units (launchers, per-device state).  Not part of the public ABI.
#pragma once

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

// Decomposition of one decode call, shared by the workspace sizing and the
// launch so both agree.
struct DecodePlan {
    int group_pad;     // query heads per head group, padded to 1/2/4/8
    int num_sub;       // head groups per kv head (ceil(G / 8) when G > 8)
    int num_hg;        // head groups per request = num_kv_heads * num_sub
    int chunk_tokens;  // tokens per pipeline stage
    int fixed_units;   // chunks per split unit when partition_size > 0, else 0
    int grid;          // persistent CTAs
    size_t units_max;  // upper bound of split units
    size_t records;    // partial-result records
    size_t bytes;      // workspace bytes
};

// Fill a plan for these sizes on the current device (false if invalid).
bool make_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int max_seq_len, int partition_size, int ctas_per_sm,
                      DecodePlan* plan);

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
    unsigned* err;
    int num_seqs, num_q_heads, num_kv_heads, group, num_sub, num_hg;
    int block_size, log2_bs, max_blocks, num_blocks;
    int fixed_units;  // 0 = automatic
    long long rec_cap;  // records the workspace holds
    int out_dtype;
    float scale_log2;  // softmax scale * log2(e)
};

pkv_status launch_decode_simt(const DecodeParams& p, int head_dim, pkv_dtype kv_dtype,
                              int group_pad, cudaStream_t stream, int* grid_out);

pkv_status launch_kv_cache_write(const void* k, const void* v, const int64_t* slots,
                                 void* k_cache, void* v_cache, int num_tokens, int num_kv_heads,
                                 int head_dim, int block_size, int num_blocks, int elem_bytes,
                                 unsigned* err, cudaStream_t stream);

pkv_status launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int num_pairs,
                              size_t block_bytes, int num_blocks, unsigned* err,
                              cudaStream_t stream);

}  // namespace pkv
