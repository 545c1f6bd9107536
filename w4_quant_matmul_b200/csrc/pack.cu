// pack.cu -- W4-G256 weight quantiser/packer and the nibble pack/unpack pair.
//
// Format: groups of 256 consecutive k per row, 4-bit codes plus one fp16
// scale d and one fp16 min m per group, w = d*q + m ("HFQ4-G256", hipfire
// MMQ prefill article).  Byte j of a code row holds k = 2j in bits 0-3 and
// k = 2j+1 in bits 4-7.  The same quantiser also packs groups of 32 (the
// asymmetric int4 group-32 W4A16 scheme of the ROCM_OCTAVE page,
// "Validation"), with d and m planes of K/32 columns.  These kernels are off
// the timed path (weights are packed once); they are written for exactness
// first, bandwidth second.
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int kGroup = 256;
constexpr int kGroup32 = 32;

// One pass of a warp covers 32 / (GROUP / 8) consecutive (row, group) units:
// GROUP / 8 lanes per group, each owning 8 consecutive weights (one warp per
// group at 256, eight groups per warp at 32).
//   mn, mx -> d16 = fp16_rn((mx - mn) / 15), m16 = fp16_rn(mn)
//   q = d16 == 0 ? 0 : clamp(rint((w - m16) / d16), 0, 15)
// All fp32 operations are the IEEE round-to-nearest intrinsics so that the
// result does not depend on contraction or fast-math settings.
template <int GROUP>
__global__ void __launch_bounds__(256) w4_pack_kernel(const float* __restrict__ w, int64_t N,
                                                      int64_t K, uint8_t* __restrict__ codes,
                                                      __half* __restrict__ d,
                                                      __half* __restrict__ m, int* err) {
    constexpr int kLanes = GROUP / 8;       // lanes per group
    constexpr int kPerPass = 32 / kLanes;   // groups per warp pass
    static_assert(kLanes >= 1 && kLanes <= 32 && 32 % kLanes == 0, "group of 8..256");
    const int64_t G = K / GROUP;
    const int64_t groups = N * G;
    const int lane = threadIdx.x & 31;
    const int sub = lane / kLanes, part = lane % kLanes;
    const int64_t warps_total = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t base = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kPerPass;
         base < groups; base += warps_total * kPerPass) {
        const int64_t gi = base + sub;
        const bool live = gi < groups;  // the same for all lanes of a group
        const int64_t n = live ? gi / G : 0, g = live ? gi % G : 0;
        float v[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
        if (live && W4_CHECK(n < N && g < G && part < kLanes, err)) {
            const float4* src = reinterpret_cast<const float4*>(w + n * K + g * GROUP + part * 8);
            const float4 a = __ldg(src), b = __ldg(src + 1);
            v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
            v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
        }
        float mn = v[0], mx = v[0];
#pragma unroll
        for (int i = 1; i < 8; ++i) {
            mn = fminf(mn, v[i]);
            mx = fmaxf(mx, v[i]);
        }
        // xor offsets below kLanes stay inside the group's lanes
#pragma unroll
        for (int off = kLanes / 2; off > 0; off >>= 1) {
            mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        }
        // a zero minimum or maximum is taken as +0, so that d and m do not
        // depend on where a -0 sits in the group (fminf/fmaxf may return
        // either zero)
        if (mn == 0.0f) mn = 0.0f;
        if (mx == 0.0f) mx = 0.0f;
        const __half d16 = __float2half_rn(__fdiv_rn(__fsub_rn(mx, mn), 15.0f));
        const __half m16 = __float2half_rn(mn);
        const float df = __half2float(d16), mf = __half2float(m16);
        uint32_t packed = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            float qf = 0.0f;
            if (df != 0.0f) {
                qf = rintf(__fdiv_rn(__fsub_rn(v[i], mf), df));
                qf = fminf(fmaxf(qf, 0.0f), 15.0f);
            }
            packed |= (uint32_t)qf << (4 * i);
        }
        if (live && W4_CHECK(n < N && g < G, err)) {
            reinterpret_cast<uint32_t*>(codes + n * (K / 2) + g * (GROUP / 2))[part] = packed;
            if (part == 0) {
                d[n * G + g] = d16;
                m[n * G + g] = m16;
            }
        }
    }
}

// q (one code per byte) -> packed codes.  Thread handles 16 output bytes.
__global__ void pack_codes_kernel(const uint8_t* __restrict__ q, int64_t pairs,
                                  uint8_t* __restrict__ codes) {
    const int64_t vec = pairs / 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < vec; i += stride) {
        const uint4* s = reinterpret_cast<const uint4*>(q) + 2 * i;
        uint4 a = s[0], b = s[1];
        uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t out[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            // 8 input bytes (two words) -> 4 output bytes
            uint32_t lo = in[2 * j] & 0x0F0F0F0Fu, hi = in[2 * j + 1] & 0x0F0F0F0Fu;
            uint32_t r = 0;
#pragma unroll
            for (int b2 = 0; b2 < 2; ++b2) {
                r |= (((lo >> (16 * b2)) & 0xFu) | (((lo >> (16 * b2 + 8)) & 0xFu) << 4)) << (8 * b2);
                r |= (((hi >> (16 * b2)) & 0xFu) | (((hi >> (16 * b2 + 8)) & 0xFu) << 4))
                     << (8 * (b2 + 2));
            }
            out[j] = r;
        }
        reinterpret_cast<uint4*>(codes)[i] = make_uint4(out[0], out[1], out[2], out[3]);
    }
    // scalar tail
    for (int64_t p = vec * 16 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < pairs;
         p += stride) {
        codes[p] = (uint8_t)((q[2 * p] & 0xFu) | ((q[2 * p + 1] & 0xFu) << 4));
    }
}

// packed codes -> q (one code per byte).  Thread handles 16 input bytes.
__global__ void unpack_kernel(const uint8_t* __restrict__ codes, int64_t pairs,
                              uint8_t* __restrict__ q) {
    const int64_t vec = pairs / 16;
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < vec; i += stride) {
        uint4 c = reinterpret_cast<const uint4*>(codes)[i];
        uint32_t in[4] = {c.x, c.y, c.z, c.w};
        uint32_t out[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t lo = in[j] & 0x0F0F0F0Fu;         // k = 0, 2, 4, 6
            const uint32_t hi = (in[j] >> 4) & 0x0F0F0F0Fu;  // k = 1, 3, 5, 7
            out[2 * j] = __byte_perm(lo, hi, 0x5140);
            out[2 * j + 1] = __byte_perm(lo, hi, 0x7362);
        }
        uint4* d = reinterpret_cast<uint4*>(q) + 2 * i;
        d[0] = make_uint4(out[0], out[1], out[2], out[3]);
        d[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    for (int64_t p = vec * 16 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < pairs;
         p += stride) {
        const uint8_t b = codes[p];
        q[2 * p] = b & 0xFu;
        q[2 * p + 1] = b >> 4;
    }
}

int grid_for(int64_t work, int threads) {
    int64_t blocks = (work + threads - 1) / threads;
    const int64_t cap = (int64_t)w4::sm_count() * 32;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    return (int)blocks;
}

template <int GROUP>
int pack_grouped(const float* w, int64_t N, int64_t K, uint8_t* codes, uint16_t* d_f16,
                 uint16_t* m_f16, void* stream) {
    if (N < 0 || K < 0 || K % GROUP != 0) return W4_ERR_SHAPE;
    if (N == 0 || K == 0) return W4_OK;
    if (!w || !codes || !d_f16 || !m_f16) return W4_ERR_NULL;
    if (!w4::aligned16(w) || !w4::aligned16(codes) || !w4::aligned16(d_f16) ||
        !w4::aligned16(m_f16))
        return W4_ERR_ALIGN;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    // one thread per 8 weights: N * K / 8 threads in warp passes
    const int64_t threads = N * (K / 8);
    w4_pack_kernel<GROUP><<<grid_for(threads, 256), 256, 0, (cudaStream_t)stream>>>(
        w, N, K, codes, reinterpret_cast<__half*>(d_f16), reinterpret_cast<__half*>(m_f16),
        w4::device_error_word());
    return w4::launch_status();
}

}  // namespace

extern "C" {

int w4_pack(const float* w, int64_t N, int64_t K, uint8_t* codes, uint16_t* d_f16,
            uint16_t* m_f16, void* stream) {
    return pack_grouped<kGroup>(w, N, K, codes, d_f16, m_f16, stream);
}

int w4_pack_g32(const float* w, int64_t N, int64_t K, uint8_t* codes, uint16_t* d_f16,
                uint16_t* m_f16, void* stream) {
    return pack_grouped<kGroup32>(w, N, K, codes, d_f16, m_f16, stream);
}

int w4_pack_codes(const uint8_t* q, int64_t N, int64_t K, uint8_t* codes, void* stream) {
    if (N < 0 || K < 0 || K % 2 != 0) return W4_ERR_SHAPE;
    if (N == 0 || K == 0) return W4_OK;
    if (!q || !codes) return W4_ERR_NULL;
    if (!w4::aligned16(q) || !w4::aligned16(codes)) return W4_ERR_ALIGN;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    const int64_t pairs = N * K / 2;
    pack_codes_kernel<<<grid_for(pairs / 16 + 1, 256), 256, 0, (cudaStream_t)stream>>>(q, pairs,
                                                                                       codes);
    return w4::launch_status();
}

int w4_unpack(const uint8_t* codes, int64_t N, int64_t K, uint8_t* q, void* stream) {
    if (N < 0 || K < 0 || K % 2 != 0) return W4_ERR_SHAPE;
    if (N == 0 || K == 0) return W4_OK;
    if (!q || !codes) return W4_ERR_NULL;
    if (!w4::aligned16(q) || !w4::aligned16(codes)) return W4_ERR_ALIGN;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    const int64_t pairs = N * K / 2;
    unpack_kernel<<<grid_for(pairs / 16 + 1, 256), 256, 0, (cudaStream_t)stream>>>(codes, pairs,
                                                                                   q);
    return w4::launch_status();
}

}  // extern "C"
