// noalloc.cu -- a decode entry point that allocates nothing.
//
// Some callers cannot hand this library a scratch buffer: a serving engine
// that reserves almost all device memory for its KV pool up front and does not
// let extensions call cudaMalloc, or code on a latency-critical path where the
// device-wide synchronisation of an allocation is not acceptable.  For them,
// pkv_paged_attention_decode_noalloc runs the same decode with its scratch in a
// fixed-size array that lives in the library's own device image (a file-scope
// __device__ array), so the call itself allocates nothing.
//
// Costs and limits of that choice:
//   * every GPU that loads the library holds kScratchBytes for the life of the
//     process, whether or not this entry point is used;
//   * all calls on a device share the one array, so calls that overlap on the
//     GPU (different streams, or different threads) race; callers must order
//     them (one stream, or events);
//   * problems whose scratch would exceed kScratchBytes are refused with
//     PKV_ERR_WORKSPACE.
#include <mutex>

#include "pkv_internal.h"

namespace pkv {
namespace {

// 16 MiB: enough for, e.g., 400 requests x 8 kv heads at head_dim 128 with the
// automatic split; see pkv_decode_workspace_bytes for any other shape.
constexpr size_t kScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device.  The first call
// on a device looks the address up (with that device current) and zeroes the
// array on `stream`.
pkv_status scratch_address(cudaStream_t stream, void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PKV_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || !ptr)
            return PKV_ERR_CUDA;
        if (cudaMemsetAsync(ptr, 0, kScratchBytes, stream) != cudaSuccess) return PKV_ERR_CUDA;
        g_scratch_ptr[dev] = ptr;
    }
    *out = g_scratch_ptr[dev];
    return PKV_OK;
}

}  // namespace
}  // namespace pkv

extern "C" size_t pkv_decode_noalloc_scratch_bytes(void) { return pkv::kScratchBytes; }

extern "C" pkv_status pkv_paged_attention_decode_noalloc(
    const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
    const int32_t* seq_lens, int32_t block_size, float scale, void* out, int32_t num_seqs,
    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t max_blocks_per_seq,
    int32_t num_blocks, int32_t max_seq_len, pkv_dtype q_dtype, pkv_dtype kv_dtype,
    pkv_dtype out_dtype, const float* k_scale, const float* v_scale, int32_t partition_size,
    pkv_stream_t stream) {
    using namespace pkv;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // Every argument check comes before the scratch array is touched, so a
    // rejected call puts no work on the stream (nor on a graph being captured).
    const pkv_status cs = check_decode_args(
        q, k_cache, v_cache, block_tables, seq_lens, block_size, scale, out, num_seqs,
        num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, num_blocks, max_seq_len, q_dtype,
        kv_dtype, out_dtype, k_scale, v_scale, partition_size);
    if (cs != PKV_OK || num_seqs == 0) return cs;
    DecodePlan pl;
    if (!make_decode_plan(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size, max_seq_len,
                          partition_size, &pl))
        return current_device_info() ? PKV_ERR_INVALID_ARG : PKV_ERR_CUDA;
    if (pl.bytes > kScratchBytes) return PKV_ERR_WORKSPACE;  // beyond the fixed maximum
    void* ws = nullptr;
    {
        const pkv_status s = scratch_address(st, &ws);
        if (s != PKV_OK) return s;
        // The array keeps the previous call's contents; the record-ready
        // flags and arrival counters this call can use must start at zero, so
        // clear them (no allocation: memset nodes).
        unsigned char* base = static_cast<unsigned char*>(ws);
        if (cudaMemsetAsync(base, 0, pl.records * sizeof(uint32_t), st) != cudaSuccess ||
            cudaMemsetAsync(base + sync_counters_offset(kScratchBytes), 0,
                            pl.n_bg_max * sizeof(uint32_t), st) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    return pkv_paged_attention_decode(q, k_cache, v_cache, block_tables, seq_lens, block_size,
                                      scale, out, num_seqs, num_q_heads, num_kv_heads, head_dim,
                                      max_blocks_per_seq, num_blocks, max_seq_len, q_dtype,
                                      kv_dtype, out_dtype, k_scale, v_scale, partition_size, ws,
                                      kScratchBytes, stream);
}
