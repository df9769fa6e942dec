// cache_ops.cu -- the cache-mutating kernels: KV append (scatter into slots)
// and copy-on-write block copy.  Both are pure byte movement, done in 16-byte
// vectors with coalesced loads and stores; both are bit-exact.
//
// kv_cache_write: "PagedAttention: Optimizing KV Cache Utilization in Large
// Language Models", "The Mechanics of PagedAttention" -- new tokens' K and V
// vectors are written into their allocated blocks, wherever those sit.
// copy_blocks: "KV Cache Optimization and PagedAttention" (intro) and "KV Cache
// Management", "The Bonus: Zero-Copy Sharing" -- shared prefix blocks are
// stored once; a request privately copies a shared block before appending.
#include <cuda_fp8.h>

#include <algorithm>

#include "pkv_device.cuh"
#include "pkv_internal.h"

namespace pkv {
namespace {

constexpr int kWriteVecs = 2;  // 16-byte vectors (of K and of V) per thread
constexpr int kCopyVecs = 4;   // 16-byte vectors per thread of a block copy

// Each thread moves kWriteVecs 16-byte vectors of K and of V (vector i of the
// rows t * Hkv + h, i = base + j * blockDim.x, so a warp's accesses stay
// contiguous), every load issued before any store.  Row r = t * Hkv + h of k/v
// goes to cache row ((blk * Hkv + h) * bs + off).
__global__ void kv_cache_write_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                      const int64_t* __restrict__ slots, uint4* __restrict__ kc,
                                      uint4* __restrict__ vc, long long total_vecs,
                                      int vecs_per_row, int num_kv_heads, int block_size,
                                      int num_blocks, unsigned* err) {
    // The previous kernel (a decode reading this cache) must be done first.
    griddep_wait();
    griddep_launch_dependents();
    const long long base = (long long)blockIdx.x * blockDim.x * kWriteVecs + threadIdx.x;
    uint4 kv[kWriteVecs], vv[kWriteVecs];
    size_t dst[kWriteVecs];
    bool ok[kWriteVecs];
#pragma unroll
    for (int j = 0; j < kWriteVecs; ++j) {
        const long long i = base + (long long)j * blockDim.x;
        ok[j] = false;
        if (i >= total_vecs) continue;
        const long long row = i / vecs_per_row;
        const int vec = (int)(i - row * vecs_per_row);
        const long long t = row / num_kv_heads;
        const int h = (int)(row - t * num_kv_heads);
        const int64_t slot = __ldg(slots + t);
        if (slot < 0) continue;  // padding token
        if (slot >= (int64_t)num_blocks * block_size) {
            if (h == 0 && vec == 0) raise_error(err, PKV_DEVERR_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int off = (int)(slot - blk * block_size);
        dst[j] = (((size_t)blk * num_kv_heads + h) * block_size + off) * vecs_per_row + vec;
        kv[j] = __ldg(k + i);
        vv[j] = __ldg(v + i);
        ok[j] = true;
    }
#pragma unroll
    for (int j = 0; j < kWriteVecs; ++j) {
        if (!ok[j]) continue;
        kc[dst[j]] = kv[j];
        vc[dst[j]] = vv[j];
    }
}

// Append of each request's new token through its block table (the decode
// step: request b's token is its last, position L - 1, L = seq_lens[b]
// clamped to the table's capacity as the decode clamps it): one thread per
// 16-byte vector of a (request, kv head) row, K and V together.  A request of
// length 0 appends nothing; an entry outside the pool is skipped (the decode
// that reads the block flags it).
__global__ void append_by_table_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                       const int32_t* __restrict__ block_tables,
                                       const int32_t* __restrict__ seq_lens,
                                       uint4* __restrict__ kc, uint4* __restrict__ vc,
                                       long long total_vecs, int vecs_per_row, int num_kv_heads,
                                       int block_size, int log2_bs, int max_blocks,
                                       int num_blocks) {
    griddep_wait();  // the previous kernel may read this cache or write the new rows
    griddep_launch_dependents();
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= total_vecs) return;
    const long long row = i / vecs_per_row;  // b * Hkv + h
    const int vec = (int)(i - row * vecs_per_row);
    const int b = (int)(row / num_kv_heads);
    const int h = (int)(row - (long long)b * num_kv_heads);
    const int L = min(__ldg(seq_lens + b), max_blocks * block_size);
    if (L <= 0) return;
    const int t = L - 1;
    const int phys = __ldg(block_tables + (size_t)b * max_blocks + (t >> log2_bs));
    if (phys < 0 || phys >= num_blocks) return;
    const size_t dst =
        (((size_t)phys * num_kv_heads + h) * block_size + (t & (block_size - 1))) * vecs_per_row + vec;
    const uint4 kv = __ldg(k + i), vv = __ldg(v + i);
    kc[dst] = kv;
    vc[dst] = vv;
}

// fp8 append: one thread per 16 output bytes (16 elements) of one (token, kv
// head) row, K and V together.  code = e4m3(x / scale[h]): the quotient is the
// correctly rounded fp32 division, the conversion rounds to nearest even and
// saturates at +-448 ("KV Cache Management", "Watch Out For": compress the KV
// cache to 8-bit floats to fit long contexts).
__global__ void kv_cache_write_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                          const int64_t* __restrict__ slots,
                                          uint4* __restrict__ kc, uint4* __restrict__ vc,
                                          const float* __restrict__ k_scale,
                                          const float* __restrict__ v_scale, long long total_vecs,
                                          int vecs_per_row, int num_kv_heads, int block_size,
                                          int num_blocks, unsigned* err) {
    griddep_wait();
    griddep_launch_dependents();
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total_vecs; i += stride) {
        const long long row = i / vecs_per_row;
        const int vec = (int)(i - row * vecs_per_row);
        const long long t = row / num_kv_heads;
        const int h = (int)(row - t * num_kv_heads);
        const int64_t slot = __ldg(slots + t);
        if (slot < 0) continue;
        if (slot >= (int64_t)num_blocks * block_size) {
            if (h == 0 && vec == 0) raise_error(err, PKV_DEVERR_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int off = (int)(slot - blk * block_size);
        const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * vecs_per_row + vec;
        const float ks = __ldg(k_scale + h), vs = __ldg(v_scale + h);
#pragma unroll
        for (int which = 0; which < 2; ++which) {
            const uint4* src = (which == 0 ? k : v) + 2 * i;  // 16 bf16 = 32 bytes
            const float sc = which == 0 ? ks : vs;
            const uint4 a = __ldg(src), b = __ldg(src + 1);
            float f[16];
            bf16x8_to_f32(a, f);
            bf16x8_to_f32(b, f + 8);
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f[4 * q], sc), __fdiv_rn(f[4 * q + 1], sc)),
                    __NV_SATFINITE, __NV_E4M3);
                const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(
                    make_float2(__fdiv_rn(f[4 * q + 2], sc), __fdiv_rn(f[4 * q + 3], sc)),
                    __NV_SATFINITE, __NV_E4M3);
                w[q] = (uint32_t)lo | ((uint32_t)hi << 16);
            }
            (which == 0 ? kc : vc)[dst] = make_uint4(w[0], w[1], w[2], w[3]);
        }
    }
}

// Copy-on-write contract of one call, checked for pair i by one CTA: its
// destination is no other pair's destination and no pair's source (its own
// included).  Under it the pairs' copies touch disjoint blocks, so their order
// does not matter; a call that breaks it has an unspecified result and raises
// PKV_DEVERR_BAD_PAIR.  Block-uniform; every thread must call it.
__device__ __forceinline__ void check_cow_contract(const int64_t* __restrict__ pairs,
                                                   int num_pairs, int i, int64_t dst,
                                                   unsigned* err) {
    bool clash = false;
    for (int j = threadIdx.x; j < num_pairs; j += blockDim.x) {
        const int64_t sj = __ldg(pairs + 2 * j), dj = __ldg(pairs + 2 * j + 1);
        clash |= (j != i && dj == dst) || sj == dst;
    }
    if (__syncthreads_or(clash) && threadIdx.x == 0) raise_error(err, PKV_DEVERR_BAD_PAIR);
}

// grid.x = pair, grid.y = 0 (K) / 1 (V), grid.z = slice of the block.
__global__ void copy_blocks_kernel(uint4* __restrict__ kc, uint4* __restrict__ vc,
                                   const int64_t* __restrict__ pairs, int num_pairs,
                                   long long vecs_per_block, int slice_vecs, int num_blocks,
                                   unsigned* err) {
    const int64_t src = __ldg(pairs + 2 * blockIdx.x);
    const int64_t dst = __ldg(pairs + 2 * blockIdx.x + 1);
    if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            raise_error(err, PKV_DEVERR_BAD_PAIR);
        return;
    }
    if (blockIdx.y == 0 && blockIdx.z == 0)
        check_cow_contract(pairs, num_pairs, blockIdx.x, dst, err);
    uint4* base = blockIdx.y == 0 ? kc : vc;
    const uint4* s = base + src * vecs_per_block;
    uint4* d = base + dst * vecs_per_block;
    const long long lo = (long long)blockIdx.z * slice_vecs;
    const long long hi = min(lo + slice_vecs, vecs_per_block);
    // slice_vecs = kCopyVecs * blockDim.x: all of a thread's loads, then its stores
    uint4 x[kCopyVecs];
#pragma unroll
    for (int j = 0; j < kCopyVecs; ++j) {
        const long long i = lo + threadIdx.x + (long long)j * blockDim.x;
        if (i < hi) x[j] = s[i];
    }
#pragma unroll
    for (int j = 0; j < kCopyVecs; ++j) {
        const long long i = lo + threadIdx.x + (long long)j * blockDim.x;
        if (i < hi) d[i] = x[j];
    }
}

// Block copy between two pools (either may be pinned host memory reached over
// the bus): grid.x = pair, grid.y = 0 (K) / 1 (V), grid.z = slice of the block.
__global__ void swap_blocks_kernel(const uint4* __restrict__ sk, const uint4* __restrict__ sv,
                                   uint4* __restrict__ dk, uint4* __restrict__ dv,
                                   const int64_t* __restrict__ pairs, long long vecs_per_block,
                                   int slice_vecs, int src_blocks, int dst_blocks, unsigned* err) {
    const int64_t src = pairs[2 * blockIdx.x];
    const int64_t dst = pairs[2 * blockIdx.x + 1];
    if (src < 0 || dst < 0 || src >= src_blocks || dst >= dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
            raise_error(err, PKV_DEVERR_BAD_PAIR);
        return;
    }
    const uint4* s = (blockIdx.y == 0 ? sk : sv) + src * vecs_per_block;
    uint4* d = (blockIdx.y == 0 ? dk : dv) + dst * vecs_per_block;
    const long long lo = (long long)blockIdx.z * slice_vecs;
    const long long hi = min(lo + slice_vecs, vecs_per_block);
    uint4 x[kCopyVecs];
#pragma unroll
    for (int j = 0; j < kCopyVecs; ++j) {
        const long long i = lo + threadIdx.x + (long long)j * blockDim.x;
        if (i < hi) x[j] = s[i];
    }
#pragma unroll
    for (int j = 0; j < kCopyVecs; ++j) {
        const long long i = lo + threadIdx.x + (long long)j * blockDim.x;
        if (i < hi) d[i] = x[j];
    }
}

}  // namespace

pkv_status launch_swap_blocks(const void* src_k, const void* src_v, void* dst_k, void* dst_v,
                              const int64_t* pairs, int num_pairs, size_t block_bytes,
                              int src_blocks, int dst_blocks, unsigned* err,
                              cudaStream_t stream) {
    if (num_pairs == 0) return PKV_OK;
    const long long vecs = (long long)(block_bytes / 16);
    const int threads = 256;
    const int slice = threads * kCopyVecs;
    const long long slices = (vecs + slice - 1) / slice;
    if (slices > 65535) return PKV_ERR_UNSUPPORTED;
    dim3 grid(num_pairs, 2, (unsigned)slices);
    swap_blocks_kernel<<<grid, threads, 0, stream>>>(
        static_cast<const uint4*>(src_k), static_cast<const uint4*>(src_v),
        static_cast<uint4*>(dst_k), static_cast<uint4*>(dst_v), pairs, vecs, slice, src_blocks,
        dst_blocks, err);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status launch_kv_cache_write(const void* k, const void* v, const int64_t* slots,
                                 void* k_cache, void* v_cache, int num_tokens, int num_kv_heads,
                                 int head_dim, int block_size, int num_blocks, int elem_bytes,
                                 unsigned* err, cudaStream_t stream) {
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    const int vecs_per_row = head_dim * elem_bytes / 16;
    const long long total = (long long)num_tokens * num_kv_heads * vecs_per_row;
    if (total == 0) return PKV_OK;
    const int threads = 256;
    const long long grid = (total + (long long)threads * kWriteVecs - 1) / ((long long)threads * kWriteVecs);
    if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
    PdlLaunch L(dim3((unsigned)grid), dim3(threads), 0, stream);
    const cudaError_t e = cudaLaunchKernelEx(
        &L.cfg, kv_cache_write_kernel, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        slots, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), total, vecs_per_row,
        num_kv_heads, block_size, num_blocks, err);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status launch_append_by_table(const void* k, const void* v, const int32_t* block_tables,
                                  const int32_t* seq_lens, void* k_cache, void* v_cache,
                                  int num_seqs, int num_kv_heads, int head_dim, int block_size,
                                  int log2_bs, int max_blocks, int num_blocks,
                                  cudaStream_t stream) {
    const int vecs_per_row = head_dim * 2 / 16;  // bf16 rows
    const long long total = (long long)num_seqs * num_kv_heads * vecs_per_row;
    if (total == 0) return PKV_OK;
    const int threads = 256;
    const long long grid = (total + threads - 1) / threads;
    if (grid > 0x7fffffffLL) return PKV_ERR_UNSUPPORTED;
    PdlLaunch L(dim3((unsigned)grid), dim3(threads), 0, stream);
    const cudaError_t e = cudaLaunchKernelEx(
        &L.cfg, append_by_table_kernel, static_cast<const uint4*>(k), static_cast<const uint4*>(v),
        block_tables, seq_lens, static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), total,
        vecs_per_row, num_kv_heads, block_size, log2_bs, max_blocks, num_blocks);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status launch_kv_cache_write_fp8(const void* k, const void* v, const int64_t* slots,
                                     void* k_cache, void* v_cache, const float* k_scale,
                                     const float* v_scale, int num_tokens, int num_kv_heads,
                                     int head_dim, int block_size, int num_blocks, unsigned* err,
                                     cudaStream_t stream) {
    const DeviceInfo* di = current_device_info();
    if (!di) return PKV_ERR_CUDA;
    const int vecs_per_row = head_dim / 16;  // 16-byte vectors of fp8 codes
    const long long total = (long long)num_tokens * num_kv_heads * vecs_per_row;
    if (total == 0) return PKV_OK;
    const int threads = 256;
    const long long want = (total + threads - 1) / threads;
    const int grid = (int)std::min<long long>(want, (long long)di->num_sms * 8);
    PdlLaunch L(dim3(grid), dim3(threads), 0, stream);
    const cudaError_t e = cudaLaunchKernelEx(
        &L.cfg, kv_cache_write_fp8_kernel, static_cast<const uint4*>(k),
        static_cast<const uint4*>(v), slots, static_cast<uint4*>(k_cache),
        static_cast<uint4*>(v_cache), k_scale, v_scale, total, vecs_per_row, num_kv_heads,
        block_size, num_blocks, err);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status launch_copy_blocks(void* k_cache, void* v_cache, const int64_t* pairs, int num_pairs,
                              size_t block_bytes, int num_blocks, unsigned* err,
                              cudaStream_t stream) {
    if (num_pairs == 0) return PKV_OK;
    const long long vecs = (long long)(block_bytes / 16);
    const int threads = 256;
    const int slice = threads * kCopyVecs;  // 16 KB per CTA
    const long long slices = (vecs + slice - 1) / slice;
    if (slices > 65535 || num_pairs > 2147483647) return PKV_ERR_UNSUPPORTED;
    dim3 grid(num_pairs, 2, (unsigned)slices);
    copy_blocks_kernel<<<grid, threads, 0, stream>>>(static_cast<uint4*>(k_cache),
                                                      static_cast<uint4*>(v_cache), pairs,
                                                      num_pairs, vecs, slice, num_blocks, err);
    return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace pkv
