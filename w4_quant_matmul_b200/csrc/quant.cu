// quant.cu -- activation quantiser to int8 blocks of 32 (the Q8_1-style MMQ
// layout the hipfire prefill path pre-quantises activations to: "What
// changed" list of the hipfire HFQ4-G256 MMQ article).
//
// Per (token t, block b of 32 consecutive k):
//   amax = max |x|;  dx = amax / 127 (IEEE fp32 division);
//   amax == 0 -> dx = 0, qa = 0, S = 0;
//   else qa = clamp(rint(x / dx), -127, 127) (ties to even);  S = sum(qa).
//
// HBM-bound: 2 bytes read and 1.25 bytes written per element.  One thread
// owns one block (four 16-byte loads) per grid-stride step; the kernel is
// register-capped at four CTAs of 256 threads per SM (64 registers), so that
// 32 warps keep their loads in flight (measured on a 259 MB stream: 4211 GB/s
// against 3720 GB/s for two blocks per thread at three CTAs per SM).  No
// shuffles: amax comes from the largest 15-bit magnitude field of the bf16
// words (for non-negative floats the integer order of the bit patterns is the
// numeric order), two halves at a time with a 16-bit SIMD max.  K % 32 == 0
// means a block never straddles a row, so the flattened [M][K] array is one
// stream of blocks.
//
// Division.  A full IEEE division per element made the kernel issue-bound.
// All 32 elements of a block share the divisor dx, so each element's quotient
// is the product with r = RN(1/dx), formed once per block; the product rounds
// to the same integer as the IEEE quotient unless it lies within 2^-14 of a
// half-integer, where the element takes the IEEE division itself (see
// q8_code).  The codes therefore equal clamp(rint(fl(x / dx))) exactly.
#include "common.cuh"

namespace {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Largest magnitude of 32 bf16 values (16 words), as fp32.
__device__ __forceinline__ float block_amax(const uint32_t (&w)[16]) {
    uint32_t m = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = __vmaxu2(m, w[i] & 0x7FFF7FFFu);
    const uint32_t hi = m >> 16, lo = m & 0xFFFFu;
    return __uint_as_float((hi > lo ? hi : lo) << 16);
}

// Quantise one block of 32 (its 16 words) and store its codes, dx and S.
__device__ __forceinline__ void quantize_block(const uint32_t (&w)[16], int64_t blk,
                                               int8_t* __restrict__ qa, float* __restrict__ dx,
                                               int32_t* __restrict__ bsum, int64_t nblocks,
                                               int* err) {
    const float amax = block_amax(w);
    uint32_t packed[8];
    int sum = 0;
    float scale = 0.0f;
    if (amax != 0.0f) {
        scale = __fdiv_rn(amax, 127.0f);
        int q[32];
        if (scale < 0x1p-126f) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                q[2 * i] = w4::q8_code_subnormal(bf16_lo(w[i]), scale);
                q[2 * i + 1] = w4::q8_code_subnormal(bf16_hi(w[i]), scale);
            }
        } else {
            const float rcp = __frcp_rn(scale);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                q[2 * i] = w4::q8_code_normal(bf16_lo(w[i]), scale, rcp);
                q[2 * i + 1] = w4::q8_code_normal(bf16_hi(w[i]), scale, rcp);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) sum += q[i];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            packed[i] = __byte_perm(__byte_perm((uint32_t)q[4 * i], (uint32_t)q[4 * i + 1], 0x0040),
                                    __byte_perm((uint32_t)q[4 * i + 2], (uint32_t)q[4 * i + 3], 0x0040),
                                    0x5410);
    } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) packed[i] = 0u;
    }
    if (W4_CHECK(blk >= 0 && blk < nblocks, err)) {
        uint4* dst = reinterpret_cast<uint4*>(qa + blk * 32);
        dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
        dx[blk] = scale;
        bsum[blk] = sum;
    }
}

// Grid-stride loop, one block per thread and step.
__global__ void __launch_bounds__(256, 4) q8_quantize_kernel(const uint16_t* __restrict__ x,
                                                          int64_t nblocks, int8_t* __restrict__ qa,
                                                          float* __restrict__ dx,
                                                          int32_t* __restrict__ bsum,
                                                          int* err) {
    // a dependent kernel (the W4A8 product) may launch and run its prologue
    // now; it waits for this grid's completion before reading its outputs
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t b0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b0 < nblocks; b0 += stride) {
        uint32_t w0[16];
        const uint4* s0 = reinterpret_cast<const uint4*>(x) + b0 * 4;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 v = __ldg(s0 + i);
            w0[4 * i] = v.x; w0[4 * i + 1] = v.y; w0[4 * i + 2] = v.z; w0[4 * i + 3] = v.w;
        }
        quantize_block(w0, b0, qa, dx, bsum, nblocks, err);
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
    const int64_t nblocks = M * K / 32;
    // two blocks per thread; at most 8 resident CTAs of 256 threads per SM
    int64_t ctas = (nblocks + 256 - 1) / 256;
    const int64_t cap = (int64_t)w4::sm_count() * 8;
    if (ctas > cap) ctas = cap;
    q8_quantize_kernel<<<(int)ctas, 256, 0, (cudaStream_t)stream>>>(x_bf16, nblocks, qa, dx, bsum,
                                                                     w4::device_error_word());
    return w4::launch_status();
}
