// gemv.cu -- decode GEMV over W4-G256 weights, dequantisation fused into the
// weight stream (the batch-1..8 "quant-GEMM bandwidth ladder" of the
// GFX1100-TG150 spec and GFX1100-TG200 campaign pages).
//
//   y[t][n] = sum_g ( d[n][g] * sum_{k in g} q[n][k] x[t][k]
//                     + m[n][g] * sum_{k in g} x[t][k] )
//
// HBM-bound at M = 1 (0.515625 weight bytes per multiply-add), so the design
// goal is a weight stream that keeps enough bytes in flight and an inner loop
// cheap enough not to become the limit:
//
//  * Work split.  A half-warp (16 lanes) owns RH rows and one of KS K-slices;
//    lane j streams the 16-byte code chunks (32 codes) c = j, j+16, ... of its
//    slice with non-allocating 128-bit loads, U chunks ahead per row.  With
//    KS > 1 the slices of a row are summed in fixed order through shared
//    memory (small-N shapes need the extra streams); with KS = 1 a 4-step
//    xor-shuffle finishes the row.  CTAs loop over row blocks.
//  * Dequantisation.  Two codes at a time become a bf16x2 pair (128 + q) by
//    OR-ing their nibbles, shifted to bits 0-3 of each half, into the bf16
//    exponent of 128: one logic op for k and k+4 of a word, a shift and a logic
//    op for the other three pairs.  The mixed-precision fma.rn.f32.bf16 then
//    accumulates x * (128 + q) in fp32 at full FMA rate, exactly (8-bit x 8-bit
//    products), so per 32-code chunk
//        A = sum x (128 + q)   and   sum q x = A - 128 * Sx,
//    and the chunk adds d (A - 128 Sx) + m Sx (Sx = sum of its 32 x).
//  * Activations.  x is staged once per CTA into shared memory as bf16 pairs
//    permuted to match the code pairs, chunk-minor (sub-word w of chunk c at
//    [w][c]) so the 16 lanes of a half-warp hit 16 different banks; the chunk
//    sums Sx are staged beside them (fp32, fixed order).
//  * Programmatic dependent launch.  Before griddepcontrol.wait the CTA only
//    asks L2 to prefetch its first batch of weights (bulk L2 prefetch; L2 is
//    the point of coherence, so a prefetch can never observe stale data even
//    if the preceding kernel writes the weights).  In a chain of launches the
//    first HBM round trip of this GEMV overlaps the tail of the previous
//    kernel; every load that feeds arithmetic happens after the wait.
// Accumulation is fp32 in a fixed order: results are bitwise deterministic.
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

__device__ __forceinline__ uint16_t ld_nc_u16(const void* p) {
    uint16_t r;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(r) : "l"(p));
    return r;
}

// acc += lo(xp) * lo(fp) + hi(xp) * hi(fp), each product exact, fp32 accumulate.
__device__ __forceinline__ float fma_bf16x2(uint32_t xp, uint32_t fp, float acc) {
    asm("{\n\t.reg .b16 xl, xh, fl, fh;\n\t"
        "mov.b32 {xl, xh}, %1;\n\t"
        "mov.b32 {fl, fh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, xl, fl, %0;\n\t"
        "fma.rn.f32.bf16 %0, xh, fh, %0;\n\t}\n"
        : "+f"(acc)
        : "r"(xp), "r"(fp));
    return acc;
}

// bf16x2 (128 + q_lo, 128 + q_hi) from the nibbles at bits [s, s+4) and
// [s+16, s+20) of a code word.
template <int S>
__device__ __forceinline__ uint32_t code_pair(uint32_t w) {
    return ((w >> S) & 0x000F000Fu) | 0x43004300u;
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Bulk prefetch of [p, p + bytes) into L2 (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void l2_prefetch(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <int RH, int U>
struct Batch {
    uint4 wq[U][RH];
    uint16_t dv[U][RH], mv[U][RH];
};

template <int RH, int U>
__device__ __forceinline__ void load_batch(Batch<RH, U>& b, const uint8_t* __restrict__ codes,
                                           const __half* __restrict__ d,
                                           const __half* __restrict__ m, const int (&rows)[RH],
                                           size_t row_bytes, int G, int c0, int c_end) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c = c0 + 16 * u;
        const bool live = c < c_end;
        const int g = (live ? c : 0) >> 3;
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            if (live) {
                b.wq[u][i] = ld_nc_v4(codes + rows[i] * row_bytes + (size_t)c * 16);
                b.dv[u][i] = ld_nc_u16(d + (size_t)rows[i] * G + g);
                b.mv[u][i] = ld_nc_u16(m + (size_t)rows[i] * G + g);
            } else {
                b.wq[u][i] = make_uint4(0, 0, 0, 0);
                b.dv[u][i] = 0;
                b.mv[u][i] = 0;
            }
        }
    }
}

template <int M, int RH, int U>
__device__ __forceinline__ void consume_batch(const Batch<RH, U>& b, const uint4* __restrict__ xs,
                                              const float* __restrict__ sx, int C, int c0,
                                              int c_end, float (&yacc)[M][RH]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c = c0 + 16 * u;
        if (c >= c_end) break;
        float a[M][RH];
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) a[t][i] = 0.0f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            uint4 xv[M];
#pragma unroll
            for (int t = 0; t < M; ++t) xv[t] = xs[((size_t)t * 4 + wi) * C + c];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                const uint32_t w = wi == 0 ? b.wq[u][i].x
                                 : wi == 1 ? b.wq[u][i].y
                                 : wi == 2 ? b.wq[u][i].z
                                           : b.wq[u][i].w;
                const uint32_t f0 = code_pair<0>(w), f1 = code_pair<4>(w);
                const uint32_t f2 = code_pair<8>(w), f3 = code_pair<12>(w);
#pragma unroll
                for (int t = 0; t < M; ++t) {
                    a[t][i] = fma_bf16x2(xv[t].x, f0, a[t][i]);
                    a[t][i] = fma_bf16x2(xv[t].y, f1, a[t][i]);
                    a[t][i] = fma_bf16x2(xv[t].z, f2, a[t][i]);
                    a[t][i] = fma_bf16x2(xv[t].w, f3, a[t][i]);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < M; ++t) {
            const float s = sx[t * C + c];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                const float dd = __half2float(__ushort_as_half(b.dv[u][i]));
                const float mm = __half2float(__ushort_as_half(b.mv[u][i]));
                yacc[t][i] = fmaf(dd, fmaf(-128.0f, s, a[t][i]), fmaf(mm, s, yacc[t][i]));
            }
        }
    }
}

template <int M, int RH, int U>
__global__ void __launch_bounds__(kThreads) w4_gemv_kernel(
    const uint8_t* __restrict__ codes, const __half* __restrict__ d, const __half* __restrict__ m,
    int N, int K, int KS, const uint16_t* __restrict__ x, void* __restrict__ y, int out_f32) {
    extern __shared__ __align__(16) unsigned char smem[];
    const int C = K >> 5;  // 32-code chunks per row
    const int G = K >> 8;  // groups per row
    uint4* xs = reinterpret_cast<uint4*>(smem);                                // [M][4][C]
    float* sx = reinterpret_cast<float*>(smem + (size_t)M * 4 * C * 16);         // [M][C]
    float* red = sx + (size_t)M * C;  // [KS][rows_per_cta][M] partial sums (KS > 1)

    const int hw = threadIdx.x >> 4;  // half-warp in CTA
    const int j = threadIdx.x & 15;   // lane in half-warp
    const int groups = kHalfWarps / KS;  // row groups per CTA
    const int rg = hw / KS, s = hw - (hw / KS) * KS;
    const bool active = rg < groups;
    const int rows_per_cta = groups * RH;
    const int nblocks = (N + rows_per_cta - 1) / rows_per_cta;
    const size_t row_bytes = (size_t)(K >> 1);
    const int cs = (int)(((long long)C * s) / KS), ce = (int)(((long long)C * (s + 1)) / KS);

    // ---- first batch of this CTA's weights: independent of earlier kernels ----
    int blk = blockIdx.x;
    int rows[RH];
#pragma unroll
    for (int i = 0; i < RH; ++i) {
        const int n = blk * rows_per_cta + (active ? rg : 0) * RH + i;
        rows[i] = n < N ? n : N - 1;  // tail rows re-read row N-1; results dropped
    }
    if (blk < nblocks && active && j == 0) {
        const int c_last = min(cs + 16 * U, ce);
        if (c_last > cs) {
#pragma unroll
            for (int i = 0; i < RH; ++i)
                l2_prefetch(codes + rows[i] * row_bytes + (size_t)cs * 16,
                            (uint32_t)(c_last - cs) * 16u);
        }
    }

    // ---- everything below may depend on the previous kernel in the stream ----
    pdl_wait();
    Batch<RH, U> bt;
    if (blk < nblocks && active) load_batch(bt, codes, d, m, rows, row_bytes, G, cs + j, ce);

    // ---- x and its chunk sums, once per CTA ----
    const int nvec = M * C * 4;  // uint4 (8 bf16) units of x
    for (int v = threadIdx.x; v < nvec; v += kThreads) {
        const int t = v / (C * 4);
        const int r = v - t * C * 4;
        const int c = r >> 2, wi = r & 3;
        const uint4 raw = __ldg(reinterpret_cast<const uint4*>(x) + v);
        uint4 o;  // pairs (x0,x4) (x1,x5) (x2,x6) (x3,x7) of these 8 values
        o.x = __byte_perm(raw.x, raw.z, 0x5410);
        o.y = __byte_perm(raw.x, raw.z, 0x7632);
        o.z = __byte_perm(raw.y, raw.w, 0x5410);
        o.w = __byte_perm(raw.y, raw.w, 0x7632);
        xs[((size_t)t * 4 + wi) * C + c] = o;
    }
    __syncthreads();
    for (int v = threadIdx.x; v < M * C; v += kThreads) {
        const int t = v / C, c = v - t * C;
        float acc = 0.0f;
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            const uint4 p = xs[((size_t)t * 4 + wi) * C + c];
            acc += bf16_lo(p.x); acc += bf16_lo(p.y); acc += bf16_lo(p.z); acc += bf16_lo(p.w);
            acc += bf16_hi(p.x); acc += bf16_hi(p.y); acc += bf16_hi(p.z); acc += bf16_hi(p.w);
        }
        sx[v] = acc;
    }
    __syncthreads();
    pdl_launch_dependents();

    for (; blk < nblocks; blk += gridDim.x) {
        float yacc[M][RH];
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) yacc[t][i] = 0.0f;
        if (active) {
            for (int c0 = cs + j; c0 < ce; c0 += 16 * U) {
                if (c0 != cs + j) load_batch(bt, codes, d, m, rows, row_bytes, G, c0, ce);
                consume_batch<M, RH, U>(bt, xs, sx, C, c0, ce, yacc);
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
        // next row block's first batch goes out before the store/reduction
        const int nblk = blk + gridDim.x;
        int nrows[RH];
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            const int n = nblk * rows_per_cta + (active ? rg : 0) * RH + i;
            nrows[i] = n < N ? n : N - 1;
        }
        if (nblk < nblocks && active)
            load_batch(bt, codes, d, m, nrows, row_bytes, G, cs + j, ce);

        if (KS == 1) {
#pragma unroll
            for (int t = 0; t < M; ++t)
#pragma unroll
                for (int i = 0; i < RH; ++i) {
                    if (active && j == ((t * RH + i) & 15)) {
                        const int n = blk * rows_per_cta + rg * RH + i;
                        if (n < N) {
                            if (out_f32)
                                reinterpret_cast<float*>(y)[(size_t)t * N + n] = yacc[t][i];
                            else
                                reinterpret_cast<__nv_bfloat16*>(y)[(size_t)t * N + n] =
                                    __float2bfloat16_rn(yacc[t][i]);
                        }
                    }
                }
        } else {
            if (active && j == 0) {
#pragma unroll
                for (int i = 0; i < RH; ++i)
#pragma unroll
                    for (int t = 0; t < M; ++t)
                        red[((size_t)s * rows_per_cta + rg * RH + i) * M + t] = yacc[t][i];
            }
            __syncthreads();
            for (int e = threadIdx.x; e < rows_per_cta * M; e += kThreads) {
                const int r = e / M, t = e - r * M;
                float v = 0.0f;
                for (int q = 0; q < KS; ++q) v += red[((size_t)q * rows_per_cta + r) * M + t];
                const int n = blk * rows_per_cta + r;
                if (n < N) {
                    if (out_f32)
                        reinterpret_cast<float*>(y)[(size_t)t * N + n] = v;
                    else
                        reinterpret_cast<__nv_bfloat16*>(y)[(size_t)t * N + n] =
                            __float2bfloat16_rn(v);
                }
            }
            __syncthreads();
        }
#pragma unroll
        for (int i = 0; i < RH; ++i) rows[i] = nrows[i];
    }
}

size_t smem_bytes(int M, int C, int KS, int RH) {
    const int rows_per_cta = (kHalfWarps / KS) * RH;
    return (size_t)M * 4 * C * 16 + (size_t)M * C * 4 +
           (KS > 1 ? (size_t)KS * rows_per_cta * M * 4 : 0);
}

template <int M, int RH>
int launch(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K, int KS,
           const uint16_t* x, void* y, int out_f32, cudaStream_t st) {
    constexpr int U = 8 / RH;
    auto kern = w4_gemv_kernel<M, RH, U>;
    const int C = K / 32;
    const size_t smem = smem_bytes(M, C, KS, RH);
    // Per-instantiation cache: one device, a few shared-memory sizes.
    struct Entry {
        int dev;
        size_t smem;
        int per_sm;
    };
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
    const int rows_per_cta = (kHalfWarps / KS) * RH;
    const int nblocks = (N + rows_per_cta - 1) / rows_per_cta;
    int grid = per_sm * w4::sm_count();
    if (grid > nblocks) grid = nblocks;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, codes, reinterpret_cast<const __half*>(d),
                           reinterpret_cast<const __half*>(m), N, K, KS, x, y, out_f32);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    return w4::launch_status();
}

// Rows per half-warp and K-split: enough independent half-warp streams to
// cover the SMs (~64 per SM), each K-slice at least one chunk per lane.
void pick_split(int N, int C, int sms, int* rh, int* ks) {
    const long long target = (long long)sms * 64;
    if ((long long)N / 4 >= target) { *rh = 4; *ks = 1; return; }
    if ((long long)N / 2 >= target) { *rh = 2; *ks = 1; return; }
    *rh = 1;
    int k = 1;
    while (k < 16 && (long long)N * k < target && C / (2 * k) >= 16) k *= 2;
    *ks = k;
}

template <int M>
int dispatch_m(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
               const uint16_t* x, void* y, int out_f32, cudaStream_t st) {
    int rh, ks;
    pick_split(N, K / 32, w4::sm_count(), &rh, &ks);
    if (M >= 4 && rh > 2) rh = 2;  // register budget: M * RH accumulators twice
    if (smem_bytes(M, K / 32, ks, rh) > (size_t)kSmemBudget) ks = 1;
    if constexpr (M < 4) {
        if (rh == 4) return launch<M, 4>(codes, d, m, N, K, ks, x, y, out_f32, st);
    }
    if (rh >= 2) return launch<M, 2>(codes, d, m, N, K, ks, x, y, out_f32, st);
    return launch<M, 1>(codes, d, m, N, K, ks, x, y, out_f32, st);
}

}  // namespace

extern "C" int w4_gemv(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                       int64_t N, int64_t K, const uint16_t* x_bf16, int M, void* y,
                       int out_dtype, void* stream) {
    if (M < 1 || M > 8 || N < 1 || K < 256 || K % 256 != 0) return W4_ERR_SHAPE;
    if (N > (int64_t)1 << 30 || K > (int64_t)1 << 20) return W4_ERR_SHAPE;
    if (out_dtype != W4_OUT_BF16 && out_dtype != W4_OUT_F32) return W4_ERR_SHAPE;
    if (!codes || !d_f16 || !m_f16 || !x_bf16 || !y) return W4_ERR_NULL;
    if (!w4::aligned16(codes) || !w4::aligned16(d_f16) || !w4::aligned16(m_f16) ||
        !w4::aligned16(x_bf16) || !w4::aligned16(y))
        return W4_ERR_ALIGN;
    // x (M*K bf16) and its chunk sums must fit the shared-memory stage
    if (smem_bytes(M, (int)(K / 32), 1, 1) > (size_t)kSmemBudget) return W4_ERR_SHAPE;
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
