// common.cuh -- internal helpers shared by the libw4 translation units.
//
// Host side: status plumbing, the cached sm_100 device check, the per-device
// error word that kernels raise when a bounded wait runs out.
// Device side: bounded mbarrier waits and thin inline-PTX wrappers for the
// sm_100a instructions the kernels use (mbarrier, TMA bulk copies, tcgen05).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "w4.h"

namespace w4 {

// ---------------------------------------------------------------------------
// host helpers (defined in abi.cu)
// ---------------------------------------------------------------------------

// W4_OK if the current device is compute capability 10.0; cached per device.
int check_device();
// Device address of the error word of the current device (lazily resolved).
int* device_error_word();
// Record a CUDA error for w4_last_cuda_error() and return W4_ERR_CUDA.
int cuda_fail(cudaError_t e);
// Check cudaGetLastError() after a launch.
int launch_status();
// SM count of the current device (cached).
int sm_count();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Device-side index checks of the debug build (compiled with -DW4_DEBUG:
// libw4_debug.so).  W4_CHECK(cond, err) is true when cond holds; when it does
// not, the kernel records W4_ERR_BOUNDS in the device error word (the first
// error sticks) and the caller skips the guarded access.  No trap, no fault:
// a failed check leaves the context usable.  Release builds compile every
// check to `true`.
#ifdef W4_DEBUG
__device__ __forceinline__ bool debug_check(bool ok, int* err) {
    if (!ok && err) atomicCAS(err, 0, (int)W4_ERR_BOUNDS);
    return ok;
}
#define W4_CHECK(cond, err) (::w4::debug_check((cond), (err)))
#else
#define W4_CHECK(cond, err) (true)
#endif

// Upper bound of any single wait inside a kernel.  Far above any legitimate
// wait (kernels here run for micro- to milliseconds).
constexpr unsigned long long kWaitLimitNs = 4000000000ull;

// ---------------------------------------------------------------------------
// device helpers
// ---------------------------------------------------------------------------

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait with a suspend-time hint: the thread sleeps in hardware until the
// phase completes or `hint_ns` passes, instead of re-polling the barrier word
// (hundreds of threads polling shared-memory barriers congested the
// shared-memory pipeline of the other warps).
constexpr uint32_t kSuspendHintNs = 1000000u;

__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    return ok != 0;
}

// Wait until the phase with the given parity of `bar` has completed, asleep
// in try_wait between checks.  Gives up when `abort_flag` (shared; may be
// null for drain waits that must not be cut short) is raised by another
// thread, or after the limit (kWaitLimitNs for mbar_wait), in which case it
// raises the flag and the device error word.  Returns false if it gave up.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag, int* err_word,
                                              unsigned long long limit_ns) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try_wait(a, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(a, parity)) return true;
        if (abort_flag && *abort_flag) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            if (abort_flag) *abort_flag = 1;
            if (err_word) atomicExch(err_word, (int)W4_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag, int* err_word) {
    return mbar_wait_for(bar, parity, abort_flag, err_word, kWaitLimitNs);
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Generic-proxy shared-memory writes -> visible to the async proxy (TMA,
// tensor cores).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 2-D tiled TMA load, global -> shared, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const void* tmap, uint64_t* bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load_1d(void* smem_dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(smem_dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

__device__ __forceinline__ uint32_t lane_id() {
    uint32_t l;
    asm volatile("mov.u32 %0, %%laneid;" : "=r"(l));
    return l;
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "elect.sync _|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(pred));
    return pred != 0;
}

// The int8 code of one activation, x -> clamp(rint(fl(x / dx)), -127, 127),
// given the block's dx != 0 and rcp = RN(1 / dx).  q = RN(x * rcp) differs
// from the exact quotient x / dx by at most 2^-16 when |x / dx| <= 127 (rcp
// and the product are each within half an ulp, 2^-24 relative), and the IEEE
// quotient fl(x / dx) by at most half an ulp more; so when q lies farther than
// 2^-14 from a half-integer, q, x / dx and fl(x / dx) all round to the same
// integer.  Closer to a half-integer (rare), the IEEE division itself decides.
// A subnormal dx (block amax below 127 * 2^-126) can make 1 / dx overflow;
// every element of such a block takes the IEEE division (the test is uniform
// across the block).  Shared by the quantiser and the GEMV that quantises its
// activations in place, so both give the same codes.
//
// Rounding without conversions: for |v| < 2^22, v + 1.5 * 2^23 rounds v to an
// integer (ties to even, the fp32 addition's own rounding) whose value sits in
// the mantissa bits, so the code is the float's bits minus those of 1.5 * 2^23
// (one add and one integer subtract instead of the quarter-rate conversion).
// With a normal dx, |x| <= amax gives |x / dx| <= 127 (1 + 2^-23), so the code
// never leaves [-127, 127]; a subnormal dx (rounded on the coarse subnormal
// grid) can make |x / dx| reach 128, and that path clamps.
constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23
constexpr int kRoundMagicBits = 0x4B400000;

__device__ __forceinline__ int q8_code_subnormal(float x, float dx) {
    const float qf = rintf(__fdiv_rn(x, dx));
    return (int)fminf(fmaxf(qf, -127.0f), 127.0f);
}

// The rare fallback kept out of line, so that the per-element fast path stays
// compact (measured 3 % faster on a 259 MB activation stream than inlined).
static __device__ __noinline__ float q8_div_magic(float x, float dx) { return __fdiv_rn(x, dx) + kRoundMagic; }

__device__ __forceinline__ int q8_code_normal(float x, float dx, float rcp) {
    const float q = x * rcp;
    float t = q + kRoundMagic;  // rint(q), in the mantissa
    // |q - rint(q)| <= 1/2 (exact: Sterbenz), so "within 2^-14 of a
    // half-integer" is one compare
    if (fabsf(q - (t - kRoundMagic)) > 0.5f - 0x1p-14f) t = q8_div_magic(x, dx);
    return __float_as_int(t) - kRoundMagicBits;
}

__device__ __forceinline__ int q8_code(float x, float dx, float rcp) {
    return dx < 0x1p-126f ? q8_code_subnormal(x, dx) : q8_code_normal(x, dx, rcp);
}

}  // namespace w4
