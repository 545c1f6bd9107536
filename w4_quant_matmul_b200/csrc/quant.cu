// quant.cu -- activation quantiser to int8 blocks of 32 (the Q8_1-style MMQ
// layout the hipfire prefill path pre-quantises activations to: "What
// changed" list of the hipfire HFQ4-G256 MMQ article).
//
// Per (token t, block b of 32 consecutive k):
//   amax = max |x|;  dx = amax / 127 (IEEE fp32 division);
//   amax == 0 -> dx = 0, qa = 0, S = 0;
//   else qa = clamp(rint(x / dx), -127, 127) (ties to even);  S = sum(qa).
//
// HBM-bound: 2 bytes read and 1.25 bytes written per element.  Each thread
// owns 8 consecutive elements (one 16-byte load) per chunk and four chunks a
// grid stride apart, loaded before any is converted; four adjacent lanes form
// a block and reduce amax and S with two xor-shuffles.  K % 32 == 0 means a
// block never straddles a row, so the flattened [M][K] array is processed as
// one stream.
//
// Division.  A full IEEE division per element made the kernel issue-bound.
// All 32 elements of a block share the divisor dx, so each element's quotient
// is formed by Markstein's correction of a reciprocal product (P. Markstein,
// IBM J. Res. Dev. 34(1), 1990; also Cornea, Harrison and Tang, "Scientific
// Computing on Itanium-based Systems", 2002): r = RN(1/dx) once per block,
// q0 = x r, e = x - q0 dx (one FMA, exact), q = q0 + e r.  q is within an
// ulp of the IEEE quotient fl(x / dx) (|q| <= ~127 here, ulp <= 2^-16), so
// rint(q) = rint(fl(x / dx)) whenever q is farther than 2^-14 from a
// half-integer; elements that land closer (rare) take the IEEE division
// itself.  The codes therefore equal clamp(rint(fl(x / dx))) exactly.
#include "common.cuh"

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// One 8-element chunk (a quarter of a block) held by this lane: amax and the
// code sum are reduced over the block's four lanes (xor 1, 2).
__device__ __forceinline__ void quantize_quarter(uint4 v, bool live, int64_t i, int64_t n8,
                                                 int8_t* __restrict__ qa, float* __restrict__ dx,
                                                 int32_t* __restrict__ bsum, int* err) {
    float f[8] = {bf16_lo(v.x), bf16_hi(v.x), bf16_lo(v.y), bf16_hi(v.y),
                  bf16_lo(v.z), bf16_hi(v.z), bf16_lo(v.w), bf16_hi(v.w)};
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const float scale = __fdiv_rn(amax, 127.0f);
    int sum = 0;
    uint32_t packed[2] = {0u, 0u};
    if (amax != 0.0f) {
        const float rcp = __frcp_rn(scale);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const int qi = w4::q8_code(f[j], scale, rcp);
            sum += qi;
            packed[j >> 2] |= ((uint32_t)qi & 0xFFu) << (8 * (j & 3));
        }
    }
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    if (live && W4_CHECK(i >= 0 && i < n8, err)) {
        reinterpret_cast<uint2*>(qa)[i] = make_uint2(packed[0], packed[1]);
        if ((i & 3) == 0) {
            dx[i >> 2] = (amax == 0.0f) ? 0.0f : scale;
            bsum[i >> 2] = sum;
        }
    }
}

// Each thread takes kUnroll chunks, a grid stride apart, and issues all their
// 16-byte loads before converting any, so that kUnroll loads per thread are
// in flight (one per thread left HBM under-occupied).
constexpr int kUnroll = 4;

__global__ void __launch_bounds__(256) q8_quantize_kernel(const uint16_t* __restrict__ x,
                                                          int64_t n8, int8_t* __restrict__ qa,
                                                          float* __restrict__ dx,
                                                          int32_t* __restrict__ bsum,
                                                          int* err) {
    // a dependent kernel (the W4A8 product) may launch and run its prologue
    // now; it waits for this grid's completion before reading its outputs
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    // n8 (number of 8-element chunks) is a multiple of 4, so every warp-wide
    // iteration is either all live or all dead within each group of 4 lanes;
    // the loop bound keeps whole warps together for the shuffles.
    const int64_t n8_warp = (n8 + 31) & ~int64_t(31);
    for (int64_t i0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i0 < n8_warp;
         i0 += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            v[u] = i < n8 ? __ldg(reinterpret_cast<const uint4*>(x) + i) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            if (i - threadIdx.x % 32 >= n8_warp) break;  // uniform across the warp
            quantize_quarter(v[u], i < n8, i, n8, qa, dx, bsum, err);
        }
    }
}

}  // namespace

extern "C" int q8_quantize_act(const uint16_t* x_bf16, int64_t M, int64_t K, int8_t* qa,
                               float* dx, int32_t* bsum, void* stream) {
    if (M < 0 || K < 0 || K % 32 != 0) return W4_ERR_SHAPE;
    if (M == 0 || K == 0) return W4_OK;
    if (!x_bf16 || !qa || !dx || !bsum) return W4_ERR_NULL;
    if (!w4::aligned16(x_bf16) || !w4::aligned16(qa) || !w4::aligned16(dx) ||
        !w4::aligned16(bsum))
        return W4_ERR_ALIGN;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    const int64_t n8 = M * K / 8;
    // enough threads for kUnroll chunks each, at most 8 resident CTAs per SM
    int64_t blocks = (n8 + 256 * kUnroll - 1) / (256 * kUnroll);
    const int64_t cap = (int64_t)w4::sm_count() * 8;
    if (blocks > cap) blocks = cap;
    q8_quantize_kernel<<<(int)blocks, 256, 0, (cudaStream_t)stream>>>(x_bf16, n8, qa, dx, bsum,
                                                                       w4::device_error_word());
    return w4::launch_status();
}
