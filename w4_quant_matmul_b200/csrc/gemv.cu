// gemv.cu -- decode GEMV over W4-G256 weights, dequantisation fused into the
// weight stream (the batch-1..8 "quant-GEMM bandwidth ladder" of the
// GFX1100-TG150 spec and GFX1100-TG200 campaign pages).
//
//   y[t][n] = sum_g ( d[n][g] * sum_{k in g} q[n][k] x[t][k]
//                     + m[n][g] * sum_{k in g} x[t][k] )
//
// Design (HBM-bound: 0.515625 bytes of weight per multiply-add at M = 1):
//  * A half-warp (16 lanes) owns RH whole rows; lane j streams 16-byte code
//    chunks (32 codes) c = j, j+16, ... of each row with non-allocating
//    128-bit loads, U chunks ahead, so every lane keeps U*RH loads in flight.
//    No cross-warp reduction: a 4-step xor-shuffle inside the half-warp
//    finishes each row.
//  * The activations are staged once per CTA into shared memory as fp32 in
//    a chunk-minor layout (sub-block i of chunk c at [i][c]) so that the 16
//    lanes, which read 16 different chunks, hit 16 different banks; the
//    per-chunk sums Sx[t][c] are staged beside them.  When M*K*4 bytes do not
//    fit, x stays bf16 in shared memory and is widened on use.
//  * Dequantisation never materialises w: a code q becomes the float
//    1 + q/16 by placing its nibble in the top mantissa bits of 1.0f (one
//    shift and one logic op), so per chunk
//      A = sum x * (1 + q/16)   and   sum q*x = 16 * (A - Sx),
//    and the group's contribution is 16 d (A - Sx) + m Sx, applied once per
//    chunk.  Accumulation is fp32 in a fixed order (bitwise deterministic).
//  * Persistent grid: CTAs loop over blocks of 16*RH rows, so the activation
//    staging is paid once per CTA.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kHalfWarps = kThreads / 16;
constexpr int kSmemBudget = 200 * 1024;

__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ld_f16_as_f32(const __half* p) { return __half2float(__ldg(p)); }

// 1 + q/16 for the nibble at bit position 4*i of w.
template <int I>
__device__ __forceinline__ float nib_f(uint32_t w) {
    constexpr int s = 19 - 4 * I;
    const uint32_t v = (s >= 0) ? (w << (s >= 0 ? s : 0)) : (w >> (s < 0 ? -s : 0));
    return __uint_as_float((v & 0x00780000u) | 0x3F800000u);
}

template <int M, bool XF32>
struct XStage {
    // fp32: float4 xs[M][8][C] ; bf16: uint4 xs[M][4][C]
    static constexpr int kVecPerChunk = XF32 ? 8 : 4;
};

template <int M, int RH, int U, bool XF32>
__global__ void __launch_bounds__(kThreads) w4_gemv_kernel(
    const uint8_t* __restrict__ codes, const __half* __restrict__ d, const __half* __restrict__ m,
    int N, int K, const uint16_t* __restrict__ x, void* __restrict__ y, int out_f32) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = K >> 5;  // 32-code chunks per row
    const int G = K >> 8;  // groups per row
    constexpr int VPC = XStage<M, XF32>::kVecPerChunk;
    uint4* xs = reinterpret_cast<uint4*>(smem);                       // [M][VPC][C]
    float* sx = reinterpret_cast<float*>(smem + (size_t)M * VPC * C * 16);  // [M][C]

    // ---- stage x (and the per-chunk sums) once per CTA ----
    const int nvec = M * C * 4;  // uint4 (8 bf16) units of x
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
        const int t = v / (C * 4);
        const int r = v - t * C * 4;
        const int c = r >> 2, q4 = r & 3;  // chunk, quarter (8 values)
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x) + v);
        if (XF32) {
            float4 a, b;
            a.x = __uint_as_float(raw.x << 16); a.y = __uint_as_float(raw.x & 0xFFFF0000u);
            a.z = __uint_as_float(raw.y << 16); a.w = __uint_as_float(raw.y & 0xFFFF0000u);
            b.x = __uint_as_float(raw.z << 16); b.y = __uint_as_float(raw.z & 0xFFFF0000u);
            b.z = __uint_as_float(raw.w << 16); b.w = __uint_as_float(raw.w & 0xFFFF0000u);
            float4* xf = reinterpret_cast<float4*>(xs);
            xf[((size_t)t * 8 + 2 * q4) * C + c] = a;
            xf[((size_t)t * 8 + 2 * q4 + 1) * C + c] = b;
        } else {
            xs[((size_t)t * 4 + q4) * C + c] = raw;
        }
    }
    __syncthreads();
    for (int v = threadIdx.x; v < M * C; v += kThreads) {
        const int t = v / C, c = v - t * C;
        float s = 0.0f;
        if (XF32) {
            const float4* xf = reinterpret_cast<const float4*>(xs);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 a = xf[((size_t)t * 8 + i) * C + c];
                s += a.x; s += a.y; s += a.z; s += a.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 a = xs[((size_t)t * 4 + i) * C + c];
                s += __uint_as_float(a.x << 16); s += __uint_as_float(a.x & 0xFFFF0000u);
                s += __uint_as_float(a.y << 16); s += __uint_as_float(a.y & 0xFFFF0000u);
                s += __uint_as_float(a.z << 16); s += __uint_as_float(a.z & 0xFFFF0000u);
                s += __uint_as_float(a.w << 16); s += __uint_as_float(a.w & 0xFFFF0000u);
            }
        }
        sx[v] = s;
    }
    __syncthreads();

    const int hw = threadIdx.x >> 4;   // half-warp in CTA
    const int j = threadIdx.x & 15;    // lane in half-warp
    const int rows_per_cta = kHalfWarps * RH;
    const int nblocks = (N + rows_per_cta - 1) / rows_per_cta;
    const size_t row_bytes = (size_t)(K >> 1);

    for (int blk = blockIdx.x; blk < nblocks; blk += gridDim.x) {
        int rows[RH];
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            const int n = blk * rows_per_cta + hw * RH + i;
            rows[i] = n < N ? n : N - 1;  // tail rows re-read row N-1; results dropped
        }
        float yacc[M][RH];
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) yacc[t][i] = 0.0f;

        for (int c0 = j; c0 < C; c0 += 16 * U) {
            uint4 wq[U][RH];
            float dv[U][RH], mv[U][RH];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 16 * u;
                const bool live = c < C;
                const int g = (live ? c : 0) >> 3;
#pragma unroll
                for (int i = 0; i < RH; ++i) {
                    wq[u][i] = live ? ld_nc_v4(codes + rows[i] * row_bytes + (size_t)c * 16)
                                    : make_uint4(0, 0, 0, 0);
                    dv[u][i] = live ? ld_f16_as_f32(d + (size_t)rows[i] * G + g) : 0.0f;
                    mv[u][i] = live ? ld_f16_as_f32(m + (size_t)rows[i] * G + g) : 0.0f;
                }
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int c = c0 + 16 * u;
                if (c >= C) break;
                float a[M][RH];
#pragma unroll
                for (int t = 0; t < M; ++t)
#pragma unroll
                    for (int i = 0; i < RH; ++i) a[t][i] = 0.0f;
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    float xv[M][8];
#pragma unroll
                    for (int t = 0; t < M; ++t) {
                        if (XF32) {
                            const float4* xf = reinterpret_cast<const float4*>(xs);
                            const float4 p = xf[((size_t)t * 8 + 2 * wi) * C + c];
                            const float4 q = xf[((size_t)t * 8 + 2 * wi + 1) * C + c];
                            xv[t][0] = p.x; xv[t][1] = p.y; xv[t][2] = p.z; xv[t][3] = p.w;
                            xv[t][4] = q.x; xv[t][5] = q.y; xv[t][6] = q.z; xv[t][7] = q.w;
                        } else {
                            const uint4 p = xs[((size_t)t * 4 + wi) * C + c];
                            xv[t][0] = __uint_as_float(p.x << 16);
                            xv[t][1] = __uint_as_float(p.x & 0xFFFF0000u);
                            xv[t][2] = __uint_as_float(p.y << 16);
                            xv[t][3] = __uint_as_float(p.y & 0xFFFF0000u);
                            xv[t][4] = __uint_as_float(p.z << 16);
                            xv[t][5] = __uint_as_float(p.z & 0xFFFF0000u);
                            xv[t][6] = __uint_as_float(p.w << 16);
                            xv[t][7] = __uint_as_float(p.w & 0xFFFF0000u);
                        }
                    }
#pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const uint32_t w = wi == 0 ? wq[u][i].x
                                         : wi == 1 ? wq[u][i].y
                                         : wi == 2 ? wq[u][i].z
                                                   : wq[u][i].w;
                        float f[8];
                        f[0] = nib_f<0>(w); f[1] = nib_f<1>(w); f[2] = nib_f<2>(w);
                        f[3] = nib_f<3>(w); f[4] = nib_f<4>(w); f[5] = nib_f<5>(w);
                        f[6] = nib_f<6>(w); f[7] = nib_f<7>(w);
#pragma unroll
                        for (int t = 0; t < M; ++t)
#pragma unroll
                            for (int e = 0; e < 8; ++e) a[t][i] = fmaf(xv[t][e], f[e], a[t][i]);
                    }
                }
#pragma unroll
                for (int t = 0; t < M; ++t) {
                    const float s = sx[t * C + c];
#pragma unroll
                    for (int i = 0; i < RH; ++i) {
                        const float dd = dv[u][i] * 16.0f;
                        yacc[t][i] = fmaf(dd, a[t][i] - s, fmaf(mv[u][i], s, yacc[t][i]));
                    }
                }
            }
        }
        // reduce the 16 lanes of the half-warp (xor < 16 stays inside it)
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                float v = yacc[t][i];
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                yacc[t][i] = v;
            }
        // lane (t*RH + i) of the half-warp stores element (t, i)
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                if (j == ((t * RH + i) & 15)) {
                    const int n = blk * rows_per_cta + hw * RH + i;
                    if (n < N) {
                        if (out_f32)
                            reinterpret_cast<float*>(y)[(size_t)t * N + n] = yacc[t][i];
                        else
                            reinterpret_cast<__nv_bfloat16*>(y)[(size_t)t * N + n] =
                                __float2bfloat16_rn(yacc[t][i]);
                    }
                }
            }
    }
}

template <int M, int RH, int U, bool XF32>
int launch(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
           const uint16_t* x, void* y, int out_f32, cudaStream_t st) {
    auto kern = w4_gemv_kernel<M, RH, U, XF32>;
    const int C = K / 32;
    const size_t smem = (size_t)M * (XF32 ? 8 : 4) * C * 16 + (size_t)M * C * 4;
    // Per-instantiation cache: one device, a few shared-memory sizes.
    struct Entry { int dev; size_t smem; int per_sm; };
    static thread_local Entry cache[8];
    static thread_local int ncache = 0;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBudget + 16 * 1024);
        if (e != cudaSuccess) return w4::cuda_fail(e);
        attr_dev = dev;
        ncache = 0;
    }
    int per_sm = 0;
    for (int i = 0; i < ncache; ++i)
        if (cache[i].dev == dev && cache[i].smem == smem) per_sm = cache[i].per_sm;
    if (per_sm == 0) {
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem);
        if (e != cudaSuccess) return w4::cuda_fail(e);
        if (per_sm < 1) per_sm = 1;
        cache[ncache & 7] = Entry{dev, smem, per_sm};
        if (ncache < 8) ++ncache;
    }
    const int rows_per_cta = kHalfWarps * RH;
    const int nblocks = (N + rows_per_cta - 1) / rows_per_cta;
    int grid = per_sm * w4::sm_count();
    if (grid > nblocks) grid = nblocks;
    kern<<<grid, kThreads, smem, st>>>(codes, reinterpret_cast<const __half*>(d),
                                      reinterpret_cast<const __half*>(m), N, K, x, y, out_f32);
    return w4::launch_status();
}

template <int M>
int dispatch_m(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
               const uint16_t* x, void* y, int out_f32, cudaStream_t st) {
    const int C = K / 32;
    const bool f32 = (size_t)M * 8 * C * 16 + (size_t)M * C * 4 <= (size_t)kSmemBudget;
    // rows per half-warp: enough row-blocks to cover the SMs, else fewer rows
    // per half-warp (more independent streams).
    const int sms = w4::sm_count();
    const bool big = N >= 16 * 4 * sms * 2;
    if (M <= 2) {
        if (big) return f32 ? launch<M, 4, 2, true>(codes, d, m, N, K, x, y, out_f32, st)
                            : launch<M, 4, 2, false>(codes, d, m, N, K, x, y, out_f32, st);
        return f32 ? launch<M, 1, 8, true>(codes, d, m, N, K, x, y, out_f32, st)
                   : launch<M, 1, 8, false>(codes, d, m, N, K, x, y, out_f32, st);
    }
    if (big) return f32 ? launch<M, 2, 2, true>(codes, d, m, N, K, x, y, out_f32, st)
                        : launch<M, 2, 2, false>(codes, d, m, N, K, x, y, out_f32, st);
    return f32 ? launch<M, 1, 4, true>(codes, d, m, N, K, x, y, out_f32, st)
               : launch<M, 1, 4, false>(codes, d, m, N, K, x, y, out_f32, st);
}

}  // namespace

extern "C" int w4_gemv(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                       int64_t N, int64_t K, const uint16_t* x_bf16, int M, void* y,
                       int out_dtype, void* stream) {
    if (M < 1 || M > 8 || N < 1 || K < 256 || K % 256 != 0) return W4_ERR_SHAPE;
    if (N > (int64_t)1 << 30 || K > (int64_t)1 << 20) return W4_ERR_SHAPE;
    if (N * (K / 2) > ((int64_t)1 << 40)) return W4_ERR_SHAPE;
    if (out_dtype != W4_OUT_BF16 && out_dtype != W4_OUT_F32) return W4_ERR_SHAPE;
    if (!codes || !d_f16 || !m_f16 || !x_bf16 || !y) return W4_ERR_NULL;
    if (!w4::aligned16(codes) || !w4::aligned16(d_f16) || !w4::aligned16(m_f16) ||
        !w4::aligned16(x_bf16) || !w4::aligned16(y))
        return W4_ERR_ALIGN;
    // x must fit shared memory at least as bf16 (M * K * 2 bytes + sums)
    if ((int64_t)M * K * 2 + (int64_t)M * (K / 32) * 4 > kSmemBudget) return W4_ERR_SHAPE;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    const int out_f32 = out_dtype == W4_OUT_F32;
    cudaStream_t st = (cudaStream_t)stream;
    const int n = (int)N, k = (int)K;
    switch (M) {
        case 1: return dispatch_m<1>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 2: return dispatch_m<2>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 3: return dispatch_m<3>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 4: return dispatch_m<4>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 5: return dispatch_m<5>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 6: return dispatch_m<6>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        case 7: return dispatch_m<7>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
        default: return dispatch_m<8>(codes, d_f16, m_f16, n, k, x_bf16, y, out_f32, st);
    }
}
