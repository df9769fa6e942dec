// pkv_device.cuh -- device-side building blocks shared by the library's kernels:
// inline-PTX wrappers for mbarriers and bulk (TMA) copies, bounded waits,
// element conversions and the error word.  sm_100a only.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pkv.h"

namespace pkv {

constexpr unsigned FULL_MASK = 0xffffffffu;

// Upper bound of any in-kernel wait: after this the kernel raises
// PKV_DEVERR_TIMEOUT and stops instead of spinning for ever.
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s

__device__ __forceinline__ void raise_error(unsigned* err, unsigned bits) {
    if (err) atomicOr(err, bits);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---- mbarrier -------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

// Make mbarrier initialisation visible to the async (TMA) proxy.
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return done != 0;
}

// Wait for the phase with the given parity to complete; false on timeout
// (after limit_ns of global time, or 2^30 polls, whichever comes first).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          uint64_t limit_ns = kWaitLimitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0 && global_timer_ns() - t0 > limit_ns) return false;
    }
    return false;
}

// ---- flags between CTAs ------------------------------------------------------

// Acquire load of a flag at GPU scope: what its releasing writer wrote before
// the release is visible to this thread (and, after a warp barrier, to the
// rest of the warp) once the value is seen.
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Release store of a flag at GPU scope: the writes this thread, and the
// threads synchronised with it by a barrier before, made are visible to an
// acquirer that reads the value.
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ---- bulk copies (TMA, non-tensor, no multicast) ---------------------------

// L2 policy for data read exactly once (streamed K/V tiles).
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// L2 policy for data several CTAs read in turn (a shared prefix's tiles).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// Global -> shared copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned) completing on `bar` as transaction bytes.
__device__ __forceinline__ void bulk_load(void* dst_smem, const void* src_gmem, uint32_t bytes,
                                          uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst_smem)),
        "l"(src_gmem), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// ---- programmatic dependent launch ------------------------------------------

// Wait until the previous kernel in the stream has completed and its writes are
// visible (no-op when the kernel was not launched as a dependent).
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Let the next kernel in the stream begin launching.
__device__ __forceinline__ void griddep_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---- named barriers ---------------------------------------------------------

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---- element conversions -----------------------------------------------------

// 16 bytes of bf16 (8 values) -> 8 floats (exact).
__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ void f32x4_from_u4(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
}

// Element traits: storage type -> elements per 16-byte vector and unpacking.
template <typename T>
struct Elem;

template <>
struct Elem<float> {
    static constexpr int kBytes = 4;
    static constexpr int kPerVec = 4;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) { f32x4_from_u4(u, f); }
    __device__ __forceinline__ static void store(float* dst, float v) { *dst = v; }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kBytes = 2;
    static constexpr int kPerVec = 8;
    __device__ __forceinline__ static void unpack(const uint4& u, float* f) { bf16x8_to_f32(u, f); }
    __device__ __forceinline__ static void store(__nv_bfloat16* dst, float v) {
        *dst = __float2bfloat16_rn(v);
    }
};

__device__ __forceinline__ void store_out(void* out, size_t idx, float v, int out_dtype) {
    if (out_dtype == PKV_F32)
        static_cast<float*>(out)[idx] = v;
    else
        static_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

// 2^x for softmax weights (scores are kept in the log2 domain): the hardware
// exponential alone (ex2.approx.ftz: about 2 ulp; results below 2^-126 flush
// to 0, weights that small vanish beside the row maximum's 1; 2^-inf = 0).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

}  // namespace pkv
