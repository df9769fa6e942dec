// api.cu -- the extern "C" entry points declared in include/pkv.h: host-side
// validation, workspace planning, per-device state and the error word.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {

// The per-device error word (PKV_DEVERR_* bits).  Kernels receive its address
// as an argument; pkv_get_device_error reads and clears it.
__device__ unsigned g_error_word = 0;

namespace {

constexpr int kMaxDevices = 64;
constexpr int kChunkTokens = 32;  // tokens per decode pipeline stage
constexpr int kMaxCtasPerSm = 4;  // cap of resident decode CTAs per SM

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int log2_int(int x) {
    int r = 0;
    while ((1 << r) < x) ++r;
    return r;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int elem_size(pkv_dtype t) {
    switch (t) {
        case PKV_F32: return 4;
        case PKV_BF16: return 2;
        case PKV_FP8_E4M3: return 1;
        default: return 0;
    }
}

// Splits of the shared prefix pass: as many (group, kv head, row tile, split)
// CTAs as fit one wave (the pass holds one CTA per SM; a partial second wave
// would double the pass), at most one per 64-token chunk of the longest prefix.
int prefix_splits_for(int num_sms, int num_prefixes, int num_kv_heads, int row_tiles,
                      int max_prefix_len) {
    const long long base = (long long)num_prefixes * num_kv_heads * row_tiles;
    const long long nch = (max_prefix_len + 63) / 64;
    if (base <= 0 || nch <= 0) return 1;
    long long s = (long long)num_sms * kPrefixCtasPerSm / base;
    s = std::min(s, nch);
    s = std::min(s, 64LL);
    return (int)std::max(s, 1LL);
}

int prefix_row_tiles(int max_members, int group) {
    return (int)(((long long)max_members * group + kPrefixRows - 1) / kPrefixRows);
}

size_t prefix_record_bytes(int splits, int num_seqs, int num_q_heads, int head_dim) {
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t rows = (size_t)splits * num_seqs * num_q_heads;
    return up(rows * head_dim * sizeof(float)) + up(rows * 2 * sizeof(float));
}

int group_pad_of(int group) {
    if (group >= 8) return 8;
    int g = 1;
    while (g < group) g <<= 1;
    return g;
}

}  // namespace

const DeviceInfo* current_device_info() {
    static std::mutex mu;
    static DeviceInfo infos[kMaxDevices];
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    DeviceInfo& di = infos[dev];
    if (di.device == dev) return &di;
    DeviceInfo tmp;
    tmp.device = dev;
    if (cudaDeviceGetAttribute(&tmp.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return nullptr;
    if (cudaDeviceGetAttribute(&tmp.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
        return nullptr;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return nullptr;
    tmp.error_word = static_cast<unsigned*>(addr);
    di = tmp;
    return &di;
}

bool make_decode_plan(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int max_seq_len, int partition_size, DecodePlan* plan,
                      size_t extra_bytes) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_seq_len < 0 || partition_size < 0)
        return false;
    if (num_q_heads % num_kv_heads) return false;
    if (partition_size % kChunkTokens) return false;
    const DeviceInfo* di = current_device_info();
    if (!di) return false;
    const int group = num_q_heads / num_kv_heads;
    DecodePlan pl{};
    // CUDA-core path: groups of <= 8 query heads; tensor-core path: <= 16.
    pl.rec_gp = group > 8 ? 16 : 8;
    pl.n_bg_max = (size_t)num_seqs * num_kv_heads * ((group + 7) / 8);
    size_t units = (size_t)di->num_sms * kMaxCtasPerSm;
    if (partition_size > 0) {
        // fixed split units: W = partition / stage tokens (32 or 64), at least 1
        for (int ch : {32, 64}) {
            const size_t w = std::max(1, partition_size / ch);
            const size_t chunks = (size_t)((max_seq_len + ch - 1) / ch);
            units = std::max(units, pl.n_bg_max * chunks / w + 1);
        }
    }
    pl.units_max = units;
    pl.records = pl.n_bg_max + units;
    auto up = [](size_t x) { return (x + 255) / 256 * 256; };
    const size_t acc_bytes = pl.records * pl.rec_gp * head_dim * sizeof(float);
    const size_t ml_bytes = pl.records * pl.rec_gp * 2 * sizeof(float);
    const size_t meta_bytes = pl.n_bg_max * 2 * sizeof(int32_t);
    pl.off_ml = up(acc_bytes);
    pl.off_meta = pl.off_ml + up(ml_bytes);
    pl.off_extra = pl.off_meta + up(meta_bytes);
    pl.rec_bytes = pl.off_extra + up(extra_bytes);
    // smallest B with sync region(B) + records <= B, a flag for every record
    // and a counter for every group
    size_t b = up(pl.rec_bytes + 2 * pl.records * sizeof(uint32_t));
    while (sync_region_bytes(b) + pl.rec_bytes > b ||
           sync_counters_offset(b) < pl.records * sizeof(uint32_t) ||
           sync_region_bytes(b) - sync_counters_offset(b) < pl.n_bg_max * sizeof(uint32_t))
        b += 256;
    pl.bytes = b;
    *plan = pl;
    return true;
}

}  // namespace pkv

using namespace pkv;

extern "C" {

const char* pkv_status_string(pkv_status status) {
    switch (status) {
        case PKV_OK: return "PKV_OK";
        case PKV_ERR_INVALID_ARG: return "PKV_ERR_INVALID_ARG: invalid argument";
        case PKV_ERR_UNSUPPORTED: return "PKV_ERR_UNSUPPORTED: unsupported configuration";
        case PKV_ERR_WORKSPACE: return "PKV_ERR_WORKSPACE: workspace missing or too small";
        case PKV_ERR_CUDA: return "PKV_ERR_CUDA: CUDA runtime or launch failure";
        case PKV_ERR_DEVICE_INDEX: return "PKV_ERR_DEVICE_INDEX: device reported a bad index";
        case PKV_ERR_OUT_OF_BLOCKS: return "PKV_ERR_OUT_OF_BLOCKS: not enough free blocks";
        default: return "PKV_ERR_UNKNOWN";
    }
}

int pkv_version(void) { return 100; }

pkv_status pkv_kv_cache_write(const void* k, const void* v, const int64_t* slot_mapping,
                              void* k_cache, void* v_cache, int32_t num_tokens,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int32_t num_blocks, pkv_dtype dtype, pkv_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        !is_pow2(block_size) || block_size > 256)
        return PKV_ERR_INVALID_ARG;
    const int es = elem_size(dtype);
    if (es == 0) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PKV_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8))
        return PKV_ERR_INVALID_ARG;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    return launch_kv_cache_write(k, v, slot_mapping, k_cache, v_cache, num_tokens, num_kv_heads,
                                 head_dim, block_size, num_blocks, es, di->error_word,
                                 reinterpret_cast<cudaStream_t>(stream));
}

pkv_status pkv_kv_cache_write_fp8(const void* k, const void* v, const int64_t* slot_mapping,
                                  void* k_cache, void* v_cache, const float* k_scale,
                                  const float* v_scale, int32_t num_tokens, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks,
                                  pkv_stream_t stream) {
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        !is_pow2(block_size) || block_size > 256)
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k || !v || !slot_mapping || !k_cache || !v_cache || !k_scale || !v_scale)
        return PKV_ERR_INVALID_ARG;
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(slot_mapping, 8) || !aligned(k_scale, 4) || !aligned(v_scale, 4))
        return PKV_ERR_INVALID_ARG;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    return launch_kv_cache_write_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale,
                                     num_tokens, num_kv_heads, head_dim, block_size, num_blocks,
                                     di->error_word, reinterpret_cast<cudaStream_t>(stream));
}

size_t pkv_decode_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t max_seq_len,
                                  int32_t partition_size) {
    if (!is_pow2(block_size) || block_size > 256) return 0;
    DecodePlan pl;
    if (!make_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                          partition_size, &pl))
        return 0;
    return pl.bytes;
}

pkv_status pkv_decode_workspace_init(void* workspace, size_t workspace_bytes,
                                     pkv_stream_t stream) {
    if (!workspace || workspace_bytes == 0) return PKV_ERR_INVALID_ARG;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? PKV_OK
               : PKV_ERR_CUDA;
}

}  // extern "C"

namespace pkv {

pkv_status check_decode_args(const void* q, const void* k_cache, const void* v_cache,
                             const int32_t* block_tables, const int32_t* seq_lens,
                             int32_t block_size, float scale, const void* out, int32_t num_seqs,
                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                             int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_seq_len,
                             pkv_dtype q_dtype, pkv_dtype kv_dtype, pkv_dtype out_dtype,
                             const float* k_scale, const float* v_scale, int32_t partition_size) {
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        max_blocks_per_seq <= 0 || num_blocks <= 0 || max_seq_len < 0 || partition_size < 0)
        return PKV_ERR_INVALID_ARG;
    if (num_q_heads % num_kv_heads) return PKV_ERR_INVALID_ARG;
    if (!is_pow2(block_size) || block_size > 256) return PKV_ERR_INVALID_ARG;
    if (partition_size % kChunkTokens) return PKV_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return PKV_ERR_INVALID_ARG;
    if (elem_size(q_dtype) == 0 || elem_size(kv_dtype) == 0 || elem_size(out_dtype) == 0)
        return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (out_dtype == PKV_FP8_E4M3) return PKV_ERR_UNSUPPORTED;
    const bool f32_pair = q_dtype == PKV_F32 && kv_dtype == PKV_F32;
    const bool bf16_pair = q_dtype == PKV_BF16 && kv_dtype == PKV_BF16;
    const bool fp8_cache = q_dtype == PKV_BF16 && kv_dtype == PKV_FP8_E4M3;
    if (!f32_pair && !bf16_pair && !fp8_cache) return PKV_ERR_INVALID_ARG;
    if (fp8_cache && block_size < 8) return PKV_ERR_UNSUPPORTED;  // tensor-core path only
    if (fp8_cache && (!k_scale || !v_scale)) return PKV_ERR_INVALID_ARG;
    if ((long long)max_blocks_per_seq * block_size > 0x7fffffffLL) return PKV_ERR_INVALID_ARG;
    if (num_seqs == 0) return PKV_OK;
    if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !out)
        return PKV_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
        !aligned(block_tables, 4) || !aligned(seq_lens, 4) || !aligned(out, elem_size(out_dtype)))
        return PKV_ERR_INVALID_ARG;
    return PKV_OK;
}

namespace {

// Test-only fault of the next decode call on this host thread (DecodeFault).
struct PendingFault {
    int mode = kFaultNone;
    int arg = 0;
    unsigned long long wait_ns = 0;
};
thread_local PendingFault t_fault;

// Shared-prefix arguments of pkv_paged_attention_decode_prefix.
struct PrefixArgs {
    const int32_t* prefix_of;
    const int32_t* prefix_lens;
    int num_prefixes, max_members, max_prefix_len;
};

pkv_status decode_entry(const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, const int32_t* seq_lens, int32_t block_size,
                        float scale, void* out, int32_t num_seqs, int32_t num_q_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq,
                        int32_t num_blocks, int32_t max_seq_len, pkv_dtype q_dtype,
                        pkv_dtype kv_dtype, pkv_dtype out_dtype, const float* k_scale,
                        const float* v_scale, int32_t partition_size, void* workspace,
                        size_t workspace_bytes, pkv_stream_t stream, const PrefixArgs* pa,
                        const void* k_new = nullptr, const void* v_new = nullptr) {
    {
        const pkv_status cs = check_decode_args(
            q, k_cache, v_cache, block_tables, seq_lens, block_size, scale, out, num_seqs,
            num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len,
            q_dtype, kv_dtype, out_dtype, k_scale, v_scale, partition_size);
        if (cs != PKV_OK || num_seqs == 0) return cs;
    }
    if (k_new || v_new) {  // fused append: bf16 caches on the tensor-core path
        if (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16))
            return PKV_ERR_INVALID_ARG;
        if (!decode_mma_supported(head_dim, block_size, q_dtype, kv_dtype) ||
            kv_dtype != PKV_BF16 || (pa && pa->num_prefixes > 0))
            return PKV_ERR_UNSUPPORTED;
    }
    const DeviceInfo* di0 = current_device_info();
    if (!di0) return PKV_ERR_CUDA;
    const bool use_prefix = pa && pa->num_prefixes > 0;
    int pfx_splits = 0, pfx_tiles = 0;
    size_t pfx_bytes = 0;
    if (pa) {
        if (pa->num_prefixes < 0 || pa->max_members < 1 || pa->max_prefix_len < 0)
            return PKV_ERR_INVALID_ARG;
        if (partition_size != 0) return PKV_ERR_INVALID_ARG;
        if (use_prefix) {
            if (!pa->prefix_of || !pa->prefix_lens || !aligned(pa->prefix_of, 4) ||
                !aligned(pa->prefix_lens, 4))
                return PKV_ERR_INVALID_ARG;
            if (!(q_dtype == PKV_BF16 && kv_dtype == PKV_BF16) || block_size < 8 ||
                !decode_mma_supported(head_dim, block_size, q_dtype, kv_dtype))
                return PKV_ERR_UNSUPPORTED;
            pfx_tiles = prefix_row_tiles(pa->max_members, num_q_heads / num_kv_heads);
            pfx_splits = prefix_splits_for(di0->num_sms, pa->num_prefixes, num_kv_heads,
                                           pfx_tiles, pa->max_prefix_len);
            pfx_bytes = prefix_record_bytes(pfx_splits, num_seqs, num_q_heads, head_dim);
        }
    }
    DecodePlan pl;
    if (!make_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                          partition_size, &pl, pfx_bytes))
        return PKV_ERR_INVALID_ARG;  // the device was queried above: the sizes are at fault
    if (!workspace || workspace_bytes < pl.bytes || !aligned(workspace, 256))
        return PKV_ERR_WORKSPACE;
    if ((long long)num_blocks * num_kv_heads * block_size > 0x7fffffffLL)
        return PKV_ERR_UNSUPPORTED;  // cache rows must fit the 32-bit TMA row coordinate
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;

    const int group = num_q_heads / num_kv_heads;
    const bool mma = decode_mma_supported(head_dim, block_size, q_dtype, kv_dtype);
    // heads per kv-head pass: 8 or 16 on the tensor-core path, 1/2/4/8 otherwise
    const int group_pad = mma ? (group > 8 ? 16 : 8) : group_pad_of(group);
    const int per_pass = mma ? (group > 8 ? 16 : 8) : 8;
    const int num_sub = (group + per_pass - 1) / per_pass;

    unsigned char* ws = static_cast<unsigned char*>(workspace);
    DecodeParams p{};
    p.q = q;
    p.k_cache = k_cache;
    p.v_cache = v_cache;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.out = out;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    const size_t cnt_region = sync_region_bytes(workspace_bytes);
    if (cnt_region + pl.rec_bytes > workspace_bytes ||
        sync_counters_offset(workspace_bytes) < pl.records * sizeof(uint32_t) ||
        cnt_region - sync_counters_offset(workspace_bytes) < pl.n_bg_max * sizeof(uint32_t))
        return PKV_ERR_WORKSPACE;
    p.ready = reinterpret_cast<unsigned*>(ws);
    p.counters = reinterpret_cast<unsigned*>(ws + sync_counters_offset(workspace_bytes));
    p.rec_acc = reinterpret_cast<float*>(ws + cnt_region);
    p.rec_ml = reinterpret_cast<float*>(ws + cnt_region + pl.off_ml);
    p.meta = reinterpret_cast<int32_t*>(ws + cnt_region + pl.off_meta);
    p.err = di->error_word;
    p.num_seqs = num_seqs;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = group;
    p.num_sub = num_sub;
    p.num_hg = num_kv_heads * num_sub;
    p.block_size = block_size;
    p.log2_bs = log2_int(block_size);
    p.max_blocks = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.max_len_hint = max_seq_len;
    p.fixed_units = partition_size > 0 ? std::max(1, partition_size / (mma ? 64 : 32)) : 0;
    // Fixed partitions and prefix groups on the tensor-core path: merge in a
    // separate kernel, so a group split into many parts (or folded with many
    // splits of a shared prefix) is combined in parallel instead of by one
    // warp of the decode kernel (which would stall that warp's CTA).
    p.defer_merge = (mma && (partition_size > 0 || use_prefix)) ? 1 : 0;
    p.row_copy = (mma && block_size < 8) ? 1 : 0;
    p.rec_cap = (long long)pl.records;
    p.out_dtype = out_dtype;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.wait_ns = kWaitLimitNs;
    p.k_new = k_new;
    p.v_new = v_new;
    if (t_fault.mode != kFaultNone) {  // consumed by this call
        p.fault_mode = t_fault.mode;
        p.fault_arg = t_fault.arg;
        p.wait_ns = t_fault.wait_ns;
        t_fault = PendingFault{};
    }
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (use_prefix) {
        const size_t rows = (size_t)pfx_splits * num_seqs * num_q_heads;
        unsigned char* pfx = ws + cnt_region + pl.off_extra;
        float* pfx_acc = reinterpret_cast<float*>(pfx);
        float* pfx_ml = reinterpret_cast<float*>(pfx + (rows * head_dim * sizeof(float) + 255) /
                                                           256 * 256);
        p.prefix_of = pa->prefix_of;
        p.prefix_lens = pa->prefix_lens;
        p.num_prefixes = pa->num_prefixes;
        p.max_prefix_len = pa->max_prefix_len;
        p.pfx_acc = pfx_acc;
        p.pfx_ml = pfx_ml;
        p.pfx_splits = pfx_splits;
        PrefixParams pp{};
        pp.q = q;
        pp.block_tables = block_tables;
        pp.seq_lens = seq_lens;
        pp.prefix_of = pa->prefix_of;
        pp.prefix_lens = pa->prefix_lens;
        pp.pfx_acc = pfx_acc;
        pp.pfx_ml = pfx_ml;
        pp.err = di->error_word;
        pp.num_seqs = num_seqs;
        pp.num_q_heads = num_q_heads;
        pp.num_kv_heads = num_kv_heads;
        pp.group = group;
        pp.block_size = block_size;
        pp.log2_bs = p.log2_bs;
        pp.max_blocks = max_blocks_per_seq;
        pp.num_blocks = num_blocks;
        pp.num_prefixes = pa->num_prefixes;
        pp.max_members = pa->max_members;
        pp.max_prefix_len = pa->max_prefix_len;
        pp.splits = pfx_splits;
        pp.row_tiles = pfx_tiles;
        pp.scale_log2 = p.scale_log2;
        const pkv_status ps = launch_decode_prefix(pp, k_cache, v_cache, head_dim, st);
        if (ps != PKV_OK) return ps;
    }
    if (k_new && !decode_mma_fuses_append(p, group_pad)) {
        // Many (request, head group) pairs or 16-head groups: one producer per
        // CTA, which the append would hold up; the append runs first as its
        // own kernel (the decode overlaps its start through programmatic
        // dependent launch).
        p.k_new = p.v_new = nullptr;
        const pkv_status as = launch_append_by_table(
            k_new, v_new, block_tables, seq_lens, const_cast<void*>(k_cache),
            const_cast<void*>(v_cache), num_seqs, num_kv_heads, head_dim, block_size, p.log2_bs,
            max_blocks_per_seq, num_blocks, st);
        if (as != PKV_OK) return as;
    }
    if (mma)
        return launch_decode_mma(p, head_dim, group_pad, kv_dtype == PKV_FP8_E4M3, st, nullptr);
    return launch_decode_simt(p, head_dim, kv_dtype, group_pad, st, nullptr);
}

}  // namespace
}  // namespace pkv

extern "C" {

pkv_status pkv_paged_attention_decode(const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, const int32_t* seq_lens,
                                      int32_t block_size, float scale, void* out,
                                      int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t max_blocks_per_seq,
                                      int32_t num_blocks, int32_t max_seq_len, pkv_dtype q_dtype,
                                      pkv_dtype kv_dtype, pkv_dtype out_dtype,
                                      const float* k_scale, const float* v_scale,
                                      int32_t partition_size, void* workspace,
                                      size_t workspace_bytes, pkv_stream_t stream) {
    return decode_entry(q, k_cache, v_cache, block_tables, seq_lens, block_size, scale, out,
                        num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                        num_blocks, max_seq_len, q_dtype, kv_dtype, out_dtype, k_scale, v_scale,
                        partition_size, workspace, workspace_bytes, stream, nullptr);
}

pkv_status pkv_paged_attention_decode_append(
    const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
    const int32_t* block_tables, const int32_t* seq_lens, int32_t block_size, float scale,
    void* out, int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    int32_t max_blocks_per_seq, int32_t num_blocks, int32_t max_seq_len, pkv_dtype out_dtype,
    int32_t partition_size, void* workspace, size_t workspace_bytes, pkv_stream_t stream) {
    if (num_seqs > 0 && (!k_new || !v_new)) return PKV_ERR_INVALID_ARG;
    return decode_entry(q, k_cache, v_cache, block_tables, seq_lens, block_size, scale, out,
                        num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                        num_blocks, max_seq_len, PKV_BF16, PKV_BF16, out_dtype, nullptr, nullptr,
                        partition_size, workspace, workspace_bytes, stream, nullptr, k_new, v_new);
}

size_t pkv_decode_prefix_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                         int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int32_t max_seq_len,
                                         int32_t num_prefixes, int32_t max_prefix_members,
                                         int32_t max_prefix_len) {
    if (!is_pow2(block_size) || block_size > 256) return 0;
    if (num_prefixes < 0 || max_prefix_members < 1 || max_prefix_len < 0) return 0;
    if (num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads) return 0;
    const DeviceInfo* di = current_device_info();
    if (!di) return 0;
    size_t extra = 0;
    if (num_prefixes > 0) {
        const int tiles = prefix_row_tiles(max_prefix_members, num_q_heads / num_kv_heads);
        const int splits = prefix_splits_for(di->num_sms, num_prefixes, num_kv_heads, tiles,
                                             max_prefix_len);
        extra = prefix_record_bytes(splits, num_seqs, num_q_heads, head_dim);
    }
    DecodePlan pl;
    if (!make_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                          0, &pl, extra))
        return 0;
    return pl.bytes;
}

pkv_status pkv_paged_attention_decode_prefix(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* seq_lens, int32_t block_size, float scale, void* out, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq,
    int32_t num_blocks, int32_t max_seq_len, pkv_dtype q_dtype, pkv_dtype kv_dtype,
    pkv_dtype out_dtype, const int32_t* prefix_of, const int32_t* prefix_lens,
    int32_t num_prefixes, int32_t max_prefix_members, int32_t max_prefix_len, void* workspace,
    size_t workspace_bytes, pkv_stream_t stream) {
    const PrefixArgs pa{prefix_of, prefix_lens, num_prefixes, max_prefix_members, max_prefix_len};
    return decode_entry(q, k_cache, v_cache, block_tables, seq_lens, block_size, scale, out,
                        num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                        num_blocks, max_seq_len, q_dtype, kv_dtype, out_dtype, nullptr, nullptr, 0,
                        workspace, workspace_bytes, stream, &pa);
}

pkv_status pkv_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping,
                           int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, pkv_dtype dtype,
                           pkv_stream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        !is_pow2(block_size) || block_size > 256)
        return PKV_ERR_INVALID_ARG;
    const int es = elem_size(dtype);
    if (es == 0) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !block_mapping) return PKV_ERR_INVALID_ARG;
    if (!aligned(k_cache, 16) || !aligned(v_cache, 16) || !aligned(block_mapping, 8))
        return PKV_ERR_INVALID_ARG;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * es;
    return launch_copy_blocks(k_cache, v_cache, block_mapping, num_pairs, block_bytes, num_blocks,
                              di->error_word, reinterpret_cast<cudaStream_t>(stream));
}

namespace {

// Device address of p if the current device can dereference it (device or
// managed memory, or pinned host memory mapped into the device's address
// space); nullptr otherwise (pageable host memory, another device's memory).
void* device_view(const void* p) {
    cudaPointerAttributes a{};
    if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
        cudaGetLastError();  // clear the sticky-free error of an unknown pointer
        return nullptr;
    }
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return nullptr;
    if (a.type == cudaMemoryTypeDevice) return a.device == dev ? a.devicePointer : nullptr;
    if (a.type == cudaMemoryTypeManaged || a.type == cudaMemoryTypeHost) return a.devicePointer;
    return nullptr;
}

}  // namespace

pkv_status pkv_swap_blocks(const void* src_k_cache, const void* src_v_cache, void* dst_k_cache,
                           void* dst_v_cache, const int64_t* block_mapping, int32_t num_pairs,
                           int32_t src_num_blocks, int32_t dst_num_blocks, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, pkv_dtype dtype,
                           pkv_stream_t stream) {
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || src_num_blocks <= 0 ||
        dst_num_blocks <= 0 || !is_pow2(block_size) || block_size > 256)
        return PKV_ERR_INVALID_ARG;
    const int es = elem_size(dtype);
    if (es == 0) return PKV_ERR_INVALID_ARG;
    if (head_dim != 64 && head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!src_k_cache || !src_v_cache || !dst_k_cache || !dst_v_cache || !block_mapping)
        return PKV_ERR_INVALID_ARG;
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    // every pointer must be reachable from the device: refuse rather than fault
    void* sk = device_view(src_k_cache);
    void* sv = device_view(src_v_cache);
    void* dk = device_view(dst_k_cache);
    void* dv = device_view(dst_v_cache);
    void* bm = device_view(block_mapping);
    if (!sk || !sv || !dk || !dv || !bm) return PKV_ERR_INVALID_ARG;
    if (!aligned(sk, 16) || !aligned(sv, 16) || !aligned(dk, 16) || !aligned(dv, 16) ||
        !aligned(bm, 8))
        return PKV_ERR_INVALID_ARG;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * es;
    return launch_swap_blocks(sk, sv, dk, dv, static_cast<const int64_t*>(bm), num_pairs,
                              block_bytes, src_num_blocks, dst_num_blocks, di->error_word,
                              reinterpret_cast<cudaStream_t>(stream));
}

pkv_status pkv_get_device_error(pkv_stream_t stream, uint32_t* flags) {
    if (!flags) return PKV_ERR_INVALID_ARG;
    *flags = 0;
    if (cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return PKV_ERR_CUDA;
    unsigned v = 0;
    if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof v) != cudaSuccess) return PKV_ERR_CUDA;
    if (v) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof zero) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    *flags = v;
    return v ? PKV_ERR_DEVICE_INDEX : PKV_OK;
}

}  // extern "C"

// Not declared in the public header: arms a test-only fault (pkv::DecodeFault)
// for the next decode call made by the calling host thread, with every
// in-kernel wait of that call bounded by wait_ns instead of the default 2 s.
// Used by the failure-detection tests to make a bounded wait run out.
extern "C" pkv_status pkv_internal_decode_fault(int32_t mode, int32_t arg,
                                                unsigned long long wait_ns) {
    if (mode < pkv::kFaultNone || mode > pkv::kFaultSkipStage || arg < 0 || wait_ns == 0 ||
        wait_ns > pkv::kWaitLimitNs)
        return PKV_ERR_INVALID_ARG;
    pkv::t_fault.mode = mode;
    pkv::t_fault.arg = arg;
    pkv::t_fault.wait_ns = wait_ns;
    return PKV_OK;
}
