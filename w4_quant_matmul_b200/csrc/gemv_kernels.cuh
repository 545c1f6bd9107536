// gemv_kernels.cuh -- decode GEMV over W4-G256 weights, dequantisation fused into the
// weight stream (the batch-1..8 "quant-GEMM bandwidth ladder" of the
// GFX1100-TG150 spec and GFX1100-TG200 campaign pages).
//
//   y[t][n] = sum_g ( d[n][g] * sum_{k in g} q[n][k] x[t][k]
//                     + m[n][g] * sum_{k in g} x[t][k] )
//
// HBM-bound at M = 1 (0.515625 weight bytes per multiply-add); on B200 the
// CUDA-core instruction issue rate, not the FMA rate, is what a dequant-fused
// GEMV runs into first, so the inner loop is built on integer dot products:
//
//  * Activations, per 32-element chunk (once per CTA, in shared memory): the
//    chunk's largest exponent E fixes sigma = 2^(14 - E), and every element
//    becomes the 16-bit integer X = rint(x * sigma), split X = 256 Xh + Xl
//    (Xh signed, Xl unsigned bytes).  Every element within a factor 2^7 of
//    the chunk's largest magnitude is represented exactly (bf16 carries 8
//    significant bits); smaller ones are rounded with an absolute error of at
//    most 2^-15 of the chunk's largest magnitude.  The chunk sum Sx of the
//    original values (fp32, fixed order) is kept for the min term.
//  * Weights: a code word (8 nibbles) splits into the bytes of its low and
//    high nibbles with three logic ops; dp4a multiplies four codes by four
//    activation bytes and accumulates in int32, so 8 codes cost 3 logic ops +
//    4 dp4a per token, and sum_k q X is exact: 256 * sum(q Xh) + sum(q Xl)
//    (|.| <= 32 * 15 * 32640 < 2^24, exact in fp32 too).  Per chunk
//        sum q x ~= (sum q X) / sigma,    y += d * that + m * Sx.
//
// Two ways of feeding that inner loop, chosen by the size of the weight stream:
//
//  * Row kernel (large streams, e.g. the lm_head).  A half-warp (16 lanes)
//    owns RH rows and one of KS K-slices; lane j streams the 16-byte code
//    chunks c = j, j+16, ... of its slice with non-allocating 128-bit loads, U
//    chunks ahead per row, and each activation word it reads serves RH rows.
//    With KS > 1 the slices of a row are summed in fixed order through shared
//    memory; with KS = 1 a 4-step xor-shuffle finishes the row.  CTAs loop
//    over row blocks.
//  * Ring kernel (streams below 16 MB, where a few latency-bound rounds of the
//    row kernel and their imbalance dominate).  Every CTA gets one contiguous
//    range of rows of equal length; a producer lane streams it with bulk TMA
//    copies (cp.async.bulk, 16 rows x a 1280-byte K-chunk per stage) through a
//    4-stage shared-memory ring completed on mbarriers, so the whole range is
//    in flight without registers; 16 consumer half-warps run the same inner
//    loop, one row each, from shared memory.
//  * Programmatic dependent launch.  The ring kernel's producer lane reads
//    only the weight planes and never waits for the preceding kernel, so in a
//    chain of launches this GEMV's ring fills while the previous kernel is
//    still running; its consumers also request their first d and m, and the
//    row kernel its first batch of codes, d and m, before they wait
//    (griddepcontrol.wait) and read the activations.  The weight planes must
//    therefore not be written by the kernel launched immediately before on
//    the same stream.  The row kernel is launched this way for streams below
//    64 MB and in plain stream order above (the lm_head: its many early CTAs
//    cost more than the overlap gained).
//  * Activation forms.  The same kernels also take the activations as int8
//    blocks of 32 (qa, dx, S from q8_quantize_act: the 32-code chunk is one
//    block, two dp4a per code word give its exact dot product P, then
//    y += d * (dx * P) + m * (dx * S)), or as bf16 quantised to those blocks in
//    shared memory with the quantiser's own code function.
//  * Group size.  Both kernels apply d and m per 32-code chunk, taking those
//    of group c >> GSH: GSH = 3 for W4-G256, 0 for group-32 weights (the
//    asymmetric int4 group-32 scheme of the ROCM_OCTAVE page, "Validation").
// Integer sums are exact and the float reductions run in a fixed order:
// results are bitwise deterministic (for a given shape, which fixes the kernel).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "common.cuh"

namespace {

constexpr int kThreads = 256;
constexpr int kHalfWarps = kThreads / 16;
constexpr int kSmemBudget = 200 * 1024;

// Activations: bf16 x [M][K] as 16-bit fixed-point words (kActBf16); int8
// blocks of 32 with their scales and sums (kActInt8: qa [M][K], dx and S
// [M][K/32]); or bf16 x [M][K] quantised to those int8 blocks in shared
// memory, with the quantiser's arithmetic (kActBf16ToInt8).
constexpr int kActBf16 = 0;
constexpr int kActInt8 = 1;
constexpr int kActBf16ToInt8 = 2;

// Staged activation word of one 8-code slice of a 32-element chunk: the bf16
// form holds {Xh even k, Xh odd k, Xl even k, Xl odd k} (16 bytes), the int8
// forms {qa even k, qa odd k} (8 bytes).
template <int AM>
struct XWord {
    using T = uint4;
};
template <>
struct XWord<kActInt8> {
    using T = uint2;
};
template <>
struct XWord<kActBf16ToInt8> {
    using T = uint2;
};
__host__ __device__ constexpr int xword_bytes(int AM) { return AM == kActBf16 ? 16 : 8; }

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

// Group size as a shift of the 32-code chunk index: a chunk c takes the d, m
// of group c >> GSH (kG256 = 3: groups of 256; kG32 = 0: groups of 32).
constexpr int kG256 = 3;
constexpr int kG32 = 0;

template <int RH, int U>
struct Batch {
    uint4 wq[U][RH];
    uint32_t dm[U][RH];
};

template <int RH, int U, int GSH>
__device__ __forceinline__ void load_batch(Batch<RH, U>& b, const uint8_t* __restrict__ codes,
                                           const __half* __restrict__ d,
                                           const __half* __restrict__ m, const int (&rows)[RH],
                                           size_t row_bytes, int G, int c0, int c_end, int N,
                                           int* err) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c = c0 + 16 * u;
        const bool live = c < c_end;
        const int g = (live ? c : 0) >> GSH;
#pragma unroll
        for (int i = 0; i < RH; ++i) {
            if (live && W4_CHECK(rows[i] >= 0 && rows[i] < N && (size_t)c * 16 < row_bytes &&
                                     (c >> GSH) < G, err)) {
                b.wq[u][i] = ld_nc_v4(codes + rows[i] * row_bytes + (size_t)c * 16);
                b.dm[u][i] = (uint32_t)ld_nc_u16(d + (size_t)rows[i] * G + g) |
                             ((uint32_t)ld_nc_u16(m + (size_t)rows[i] * G + g) << 16);
            } else {
                b.wq[u][i] = make_uint4(0, 0, 0, 0);
                b.dm[u][i] = 0;
            }
        }
    }
}

// kDump (test instantiation, int8 forms): also store every chunk's exact
// block product to dump[t][row][chunk].
template <int M, int RH, int U, int AM, bool kDump>
__device__ __forceinline__ void consume_batch(const Batch<RH, U>& b,
                                              const typename XWord<AM>::T* __restrict__ xq,
                                              const float* __restrict__ sx,
                                              const float* __restrict__ inv, int C, int c0,
                                              int c_end, float (&yacc)[M][RH],
                                              int32_t* __restrict__ dump, int N,
                                              const int (&rows)[RH], int* err) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
        const int c = c0 + 16 * u;
        if (c >= c_end) break;
        if (!W4_CHECK(c < C, err)) break;  // activation words [M][4][C]
        int ah[M][RH], al[M][RH];
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                ah[t][i] = 0;
                al[t][i] = 0;
            }
#pragma unroll
        for (int wi = 0; wi < 4; ++wi) {
            typename XWord<AM>::T xv[M];  // this slice's activation word per token
#pragma unroll
            for (int t = 0; t < M; ++t) xv[t] = xq[((size_t)t * 4 + wi) * C + c];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                const uint32_t w = wi == 0 ? b.wq[u][i].x
                                 : wi == 1 ? b.wq[u][i].y
                                 : wi == 2 ? b.wq[u][i].z
                                           : b.wq[u][i].w;
                const uint32_t lo = w & 0x0F0F0F0Fu;         // codes of k = 0, 2, 4, 6
                const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // codes of k = 1, 3, 5, 7
#pragma unroll
                for (int t = 0; t < M; ++t) {
                    ah[t][i] = __dp4a((int)lo, (int)xv[t].x, ah[t][i]);
                    ah[t][i] = __dp4a((int)hi, (int)xv[t].y, ah[t][i]);
                    if constexpr (AM == kActBf16) {
                        al[t][i] = (int)__dp4a(lo, xv[t].z, (unsigned)al[t][i]);
                        al[t][i] = (int)__dp4a(hi, xv[t].w, (unsigned)al[t][i]);
                    }
                }
            }
        }
        if constexpr (kDump) {
            // rows past N were clamped to N - 1: they store row N - 1's value again
#pragma unroll
            for (int t = 0; t < M; ++t)
#pragma unroll
                for (int i = 0; i < RH; ++i)
                    dump[((size_t)t * N + rows[i]) * C + c] = ah[t][i];
        }
#pragma unroll
        for (int t = 0; t < M; ++t) {
            const float s = sx[t * C + c], iv = inv[t * C + c];
#pragma unroll
            for (int i = 0; i < RH; ++i) {
                const float dd = __half2float(__ushort_as_half((unsigned short)(b.dm[u][i] & 0xFFFFu)));
                const float mm = __half2float(__ushort_as_half((unsigned short)(b.dm[u][i] >> 16)));
                // int8 blocks: the exact block dot P times dx; else (sum q X) / sigma
                const float qx = (AM != kActBf16 ? (float)ah[t][i] : (float)(ah[t][i] * 256 + al[t][i])) * iv;
                yacc[t][i] = fmaf(dd, qx, fmaf(mm, s, yacc[t][i]));
            }
        }
    }
}

// One quarter (8 values) of a 32-element activation chunk -> its activation
// word; lanes 4q..4q+3 of a warp hold the four quarters of one chunk.  Writes
// the word and (lane quarter 0) the chunk sum and 1/sigma.  Every lane of the
// warp must call it (the chunk reductions are xor-shuffles); `live` = false
// lanes contribute nothing and store nothing.
__device__ __forceinline__ void stage_quarter(uint4 raw, bool live, uint4* __restrict__ word_dst,
                                              float* __restrict__ sum_dst,
                                              float* __restrict__ inv_dst, int quarter) {
    float f[8] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y),
                  bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w)};
    float s = 0.0f;
    uint32_t emax = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        s += f[e];
        emax = max(emax, (__float_as_uint(f[e]) >> 23) & 0xFFu);
    }
    // fixed-order chunk sum: (q0 + q1) + (q2 + q3)
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, 1));
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, 2));
    // sigma = 2^(14 - E) with E = emax - 127, as an exponent field in [1, 253]
    int se = 268 - (int)emax;
    se = se < 1 ? 1 : (se > 253 ? 253 : se);
    const float sigma = __uint_as_float((uint32_t)se << 23);
    int X[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        // rint(f * sigma) exactly: f * sigma is exact and |.| < 2^15, so adding
        // 1.5 * 2^23 rounds to the nearest integer, which sits in the mantissa
        const float t = fmaf(f[e], sigma, 12582912.0f);
        X[e] = emax == 0 ? 0 : (int)(__float_as_uint(t) - 0x4B400000u);
    }
    // bytes: even k -> (X0, X2, X4, X6), odd k -> (X1, X3, X5, X7)
    const uint32_t e01 = __byte_perm((uint32_t)X[0], (uint32_t)X[2], 0x0040);
    const uint32_t e23 = __byte_perm((uint32_t)X[4], (uint32_t)X[6], 0x0040);
    const uint32_t o01 = __byte_perm((uint32_t)X[1], (uint32_t)X[3], 0x0040);
    const uint32_t o23 = __byte_perm((uint32_t)X[5], (uint32_t)X[7], 0x0040);
    const uint32_t eh01 = __byte_perm((uint32_t)X[0], (uint32_t)X[2], 0x0051);
    const uint32_t eh23 = __byte_perm((uint32_t)X[4], (uint32_t)X[6], 0x0051);
    const uint32_t oh01 = __byte_perm((uint32_t)X[1], (uint32_t)X[3], 0x0051);
    const uint32_t oh23 = __byte_perm((uint32_t)X[5], (uint32_t)X[7], 0x0051);
    if (live) {
        *word_dst = make_uint4(__byte_perm(eh01, eh23, 0x5410), __byte_perm(oh01, oh23, 0x5410),
                               __byte_perm(e01, e23, 0x5410), __byte_perm(o01, o23, 0x5410));
        if (quarter == 0) {
            *sum_dst = s;
            *inv_dst = emax == 0 ? 0.0f : __uint_as_float((uint32_t)(254 - se) << 23);
        }
    }
}

// Activation forms (the Act pointers below).
struct Act {
    const void* x;
    const float* dx;
    const int32_t* S;
    int32_t* dump;  // test instantiation only: exact block products [M][N][K/32]
};

// One int8 activation block (32 values of token t, chunk c) -> the words the
// dp4a loop reads: word wi holds the bytes of k = 8 wi + {0, 2, 4, 6} (.x) and
// k = 8 wi + {1, 3, 5, 7} (.y), matching the low / high nibbles of a code word;
// the chunk's "sum" slot holds dx * S and its "inverse scale" slot dx.
__device__ __forceinline__ void stage_block_a8(const Act& a, int C, int t, int c,
                                               uint2* __restrict__ xq, float* __restrict__ sx,
                                               float* __restrict__ inv) {
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const int8_t*>(a.x) + ((size_t)t * C + c) * 32);
    const uint4 q0 = __ldg(src), q1 = __ldg(src + 1);
    const uint32_t w[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi)
        xq[((size_t)t * 4 + wi) * C + c] =
            make_uint2(__byte_perm(w[2 * wi], w[2 * wi + 1], 0x6420),
                       __byte_perm(w[2 * wi], w[2 * wi + 1], 0x7531));
    const float dxv = __ldg(a.dx + (size_t)t * C + c);
    sx[t * C + c] = dxv * (float)__ldg(a.S + (size_t)t * C + c);
    inv[t * C + c] = dxv;
}

// One bf16 activation block (32 values of token t, chunk c) quantised to int8
// exactly as q8_quantize_act does (dx = fl(amax / 127), codes by q8_code,
// S = sum of codes), then staged like stage_block_a8.
__device__ __forceinline__ void stage_block_q8x(const Act& a, int C, int t, int c,
                                                uint2* __restrict__ xq, float* __restrict__ sx,
                                                float* __restrict__ inv) {
    const uint4* src = reinterpret_cast<const uint4*>(
        reinterpret_cast<const uint16_t*>(a.x) + ((size_t)t * C + c) * 32);
    uint32_t raw[16];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 v = __ldg(src + i);
        raw[4 * i] = v.x;
        raw[4 * i + 1] = v.y;
        raw[4 * i + 2] = v.z;
        raw[4 * i + 3] = v.w;
    }
    // amax: the largest 15-bit magnitude field of the bf16 words (for finite,
    // non-negative floats the integer order of the bit patterns is the
    // numeric order), two halves at a time
    uint32_t mx = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) mx = __vmaxu2(mx, raw[i] & 0x7FFF7FFFu);
    const float amax = __uint_as_float(max(mx >> 16, mx & 0xFFFFu) << 16);
    const float dxv = __fdiv_rn(amax, 127.0f);
    uint32_t w[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};  // the 32 codes, 4 per word
    int S = 0;
    if (amax != 0.0f) {
        // the subnormal-dx test once per block (q8_code takes it per element)
        int q[32];
        if (dxv < 0x1p-126f) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                q[2 * i] = w4::q8_code_subnormal(bf16_lo(raw[i]), dxv);
                q[2 * i + 1] = w4::q8_code_subnormal(bf16_hi(raw[i]), dxv);
            }
        } else {
            const float rcp = __frcp_rn(dxv);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                q[2 * i] = w4::q8_code_normal(bf16_lo(raw[i]), dxv, rcp);
                q[2 * i + 1] = w4::q8_code_normal(bf16_hi(raw[i]), dxv, rcp);
            }
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) S += q[i];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = __byte_perm(__byte_perm((uint32_t)q[4 * i], (uint32_t)q[4 * i + 1], 0x0040),
                               __byte_perm((uint32_t)q[4 * i + 2], (uint32_t)q[4 * i + 3], 0x0040),
                               0x5410);
    }
#pragma unroll
    for (int wi = 0; wi < 4; ++wi)
        xq[((size_t)t * 4 + wi) * C + c] =
            make_uint2(__byte_perm(w[2 * wi], w[2 * wi + 1], 0x6420),
                       __byte_perm(w[2 * wi], w[2 * wi + 1], 0x7531));
    const float dxs = amax == 0.0f ? 0.0f : dxv;
    sx[t * C + c] = dxs * (float)S;
    inv[t * C + c] = dxs;
}

// Resident CTAs per SM the register allocation is sized for: small M needs
// many warps in flight to cover HBM latency.  At M = 5..8 two CTAs (128
// registers, a few spilled) beat one CTA with 248 registers: measured at
// M = 8 on the lm_head, 188 against 199 us (bf16 x), 123 against 133 us
// (int8 x), 218 against 268 us (group-32 weights).
template <int M>
struct MinCtas {
    static constexpr int value = M == 1 ? 3 : 2;
};

template <int M, int RH, int U, int AM, int GSH = kG256, bool kDump = false>
__global__ void __launch_bounds__(kThreads, MinCtas<M>::value) w4_gemv_rows_kernel(
    const uint8_t* __restrict__ codes, const __half* __restrict__ d, const __half* __restrict__ m,
    int N, int K, int KS, const Act act, void* __restrict__ y, int out_f32, int* err) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int C = K >> 5;  // 32-code chunks per row
    const int G = K >> (5 + GSH);  // groups per row
    using XW = typename XWord<AM>::T;
    XW* xq = reinterpret_cast<XW*>(smem);                                        // [M][4][C]
    float* sx = reinterpret_cast<float*>(smem + (size_t)M * 4 * C * sizeof(XW)); // [M][C]
    float* inv = sx + (size_t)M * C;                                             // [M][C]
    float* red = inv + (size_t)M * C;  // [KS][rows_per_cta][M] partial sums (KS > 1)

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

    // the first batch of codes, d and m: weights, requested before the wait
    // for the preceding kernel so that their latency overlaps the activation
    // staging (not with in-place quantisation, whose registers would then spill)
    constexpr bool kEarlyBatch = AM != kActBf16ToInt8;
    Batch<RH, U> bt;
    if (kEarlyBatch && blk < nblocks && active)
        load_batch<RH, U, GSH>(bt, codes, d, m, rows, row_bytes, G, cs + j, ce, N, err);

    // ---- everything below may depend on the previous kernel in the stream ----
    pdl_wait();

    // ---- activation words, chunk sums and scales, once per CTA ----
    if constexpr (AM == kActInt8) {
        for (int v = threadIdx.x; v < M * C; v += kThreads)
            stage_block_a8(act, C, v / C, v - (v / C) * C, xq, sx, inv);
    } else if constexpr (AM == kActBf16ToInt8) {
        for (int v = threadIdx.x; v < M * C; v += kThreads)
            stage_block_q8x(act, C, v / C, v - (v / C) * C, xq, sx, inv);
    } else {
        const int nq = M * C * 4;  // quarters (8 values) of chunks; a multiple of 4
        for (int base = 0; base < nq; base += kThreads) {
            const int v = base + threadIdx.x;
            const bool live = v < nq;
            const int vv = live ? v : 0;
            const int t = vv / (C * 4);
            const int r = vv - t * C * 4;
            const int c = r >> 2, q4 = r & 3;
            const uint4 raw = live ? __ldg(reinterpret_cast<const uint4*>(act.x) + vv)
                                   : make_uint4(0, 0, 0, 0);
            if constexpr (AM == kActBf16)
                stage_quarter(raw, live, &xq[((size_t)t * 4 + q4) * C + c], &sx[t * C + c],
                              &inv[t * C + c], q4);
        }
    }
    __syncthreads();
    pdl_launch_dependents();
    if (!kEarlyBatch && blk < nblocks && active)
        load_batch<RH, U, GSH>(bt, codes, d, m, rows, row_bytes, G, cs + j, ce, N, err);

    for (; blk < nblocks; blk += gridDim.x) {
        float yacc[M][RH];
#pragma unroll
        for (int t = 0; t < M; ++t)
#pragma unroll
            for (int i = 0; i < RH; ++i) yacc[t][i] = 0.0f;
        if (active) {
            for (int c0 = cs + j; c0 < ce; c0 += 16 * U) {
                if (c0 != cs + j)
                    load_batch<RH, U, GSH>(bt, codes, d, m, rows, row_bytes, G, c0, ce, N, err);
                consume_batch<M, RH, U, AM, kDump>(bt, xq, sx, inv, C, c0, ce, yacc, act.dump,
                                                   N, rows, err);
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
            load_batch<RH, U, GSH>(bt, codes, d, m, nrows, row_bytes, G, cs + j, ce, N, err);

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

size_t smem_bytes(int M, int C, int KS, int RH, int AM) {
    const int rows_per_cta = (kHalfWarps / KS) * RH;
    return (size_t)M * 4 * C * xword_bytes(AM) + (size_t)M * C * 8 +
           (KS > 1 ? (size_t)KS * rows_per_cta * M * 4 : 0);
}

template <int M, int RH, int AM, int GSH = kG256, bool kDump = false>
int launch_rows(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K, int KS,
           const Act& x, void* y, int out_f32, cudaStream_t st) {
    // code chunks in flight per lane: 8 over the RH rows; 4 from M = 6 on, where
    // the loop is issue-bound and a larger batch only spills (lm_head at
    // M = 8: 164 against 192 us with bf16 x, 186 against 218 us with group-32
    // weights, 118 against 123 us with int8 x)
    constexpr int U = (M >= 6 ? 4 : 8) / RH > 0 ? (M >= 6 ? 4 : 8) / RH : 1;
    auto kern = w4_gemv_rows_kernel<M, RH, U, AM, GSH, kDump>;
    const int C = K / 32;
    const size_t smem = smem_bytes(M, C, KS, RH, AM);
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

    // Programmatic dependent launch for streams below 64 MB (the layer shapes):
    // the CTAs launched early issue their first batch of weights before the
    // dependency wait (per-token chain 1023 -> 1062 tok/s).  The lm_head stays
    // in plain stream order: launched early behind a ring-kernel GEMV, its
    // many resident-but-waiting CTAs cost more than the overlap gains
    // (measured ~10 us per five-GEMV decode step).
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    const bool pdl = (size_t)N * (size_t)K / 2 < ((size_t)64 << 20);
    cfg.attrs = pdl ? attr : nullptr;
    cfg.numAttrs = pdl ? 1 : 0;
    e = cudaLaunchKernelEx(&cfg, kern, codes, reinterpret_cast<const __half*>(d),
                           reinterpret_cast<const __half*>(m), N, K, KS, x, y, out_f32,
                           w4::device_error_word());
    if (e != cudaSuccess) return w4::cuda_fail(e);
    return w4::launch_status();
}

// Rows per half-warp and K-split: enough independent half-warp streams to
// cover the SMs (~64 per SM), each K-slice at least one chunk per lane.
// slots = resident CTAs of the row kernel (0: no wave rule).  Two rows per
// half-warp are then taken only when their row blocks fill the last wave of
// CTAs about as well as one row per half-warp does: with a stream of a few
// waves, the last, partly filled wave is the kernel's tail (measured on
// 19456 x 2560 at M = 1: 608 blocks of 32 rows over 444 CTAs, the median CTA
// done 3 us before the last; one row per half-warp took the per-token chain
// from 954 to 976 tok/s).
void pick_split(int N, int C, int sms, int slots, int* rh, int* ks) {
    const long long target = (long long)sms * 64;
    if ((long long)N / 4 >= target) { *rh = 4; *ks = 1; return; }
    if ((long long)N / 2 >= target && slots == 0) { *rh = 2; *ks = 1; return; }
    if ((long long)N / 2 >= target) {
        // fill of the last wave, in parts of a wave, for blocks of 32 / 16 rows
        const long long b2 = (N + 2 * kHalfWarps - 1) / (2 * kHalfWarps);
        const long long b1 = (N + kHalfWarps - 1) / kHalfWarps;
        const double f2 = (double)b2 / (double)(((b2 + slots - 1) / slots) * slots);
        const double f1 = (double)b1 / (double)(((b1 + slots - 1) / slots) * slots);
        *rh = f2 + 0.1 >= f1 ? 2 : 1;
        *ks = 1;
        return;
    }
    *rh = 1;
    int k = 1;
    while (k < 16 && (long long)N * k < target && C / (2 * k) >= 16) k *= 2;
    *ks = k;
}

template <int M, int AM, int GSH = kG256, bool kDump = false>
int dispatch_m(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
               const Act& x, void* y, int out_f32, cudaStream_t st) {
    int rh, ks;
    pick_split(N, K / 32, w4::sm_count(), M == 1 ? MinCtas<M>::value * w4::sm_count() : 0, &rh,
               &ks);
    if (M >= 4 && rh > 2) rh = 2;  // register budget: M * RH accumulators twice
    if (smem_bytes(M, K / 32, ks, rh, AM) > (size_t)kSmemBudget) ks = 1;
    if constexpr (M < 4) {
        if (rh == 4)
            return launch_rows<M, 4, AM, GSH, kDump>(codes, d, m, N, K, ks, x, y, out_f32, st);
    }
    if (rh >= 2)
        return launch_rows<M, 2, AM, GSH, kDump>(codes, d, m, N, K, ks, x, y, out_f32, st);
    return launch_rows<M, 1, AM, GSH, kDump>(codes, d, m, N, K, ks, x, y, out_f32, st);
}

// ---------------------------------------------------------------------------
// ring kernel
// ---------------------------------------------------------------------------

constexpr int kRingWarps = 8;                           // consumers: 16 half-warps, one row each
constexpr int kRingThreads = 32 * (kRingWarps + 1);     // + the producer warp
constexpr int kRowsPerStage = 2 * kRingWarps;           // 16
constexpr int kChunkBytes = 1280;                       // K-chunk of a row per stage
constexpr int kStageBytes = kRowsPerStage * kChunkBytes;  // 20 KB
constexpr int kMaxStages = 4;
constexpr int kSmemPerSm = 227 * 1024;                  // usable per CTA on sm_100
constexpr size_t kRingMaxCodeBytes = (size_t)16 << 20;  // streams below this use the ring

// Shared memory: [stages][16 rows][1280 B] code ring, then the activation
// words xq[M][4][C] (uint4), chunk sums sx[M][C], 1/sigma inv[M][C], and the
// ring's barriers.
struct Layout {
    size_t xq, sx, inv, bars, total;
};

__host__ __device__ inline Layout layout(int M, int C, int stages, int AM) {
    Layout l;
    l.xq = (size_t)stages * kStageBytes;
    l.sx = l.xq + (size_t)M * 4 * C * xword_bytes(AM);
    l.inv = l.sx + (size_t)M * C * 4;
    l.bars = (l.inv + (size_t)M * C * 4 + 7) & ~(size_t)7;
    l.total = l.bars + 2 * kMaxStages * 8 + 16;
    return l;
}

// Resident CTAs per SM the register allocation is sized for (two while the
// per-token accumulators leave room, so that two rings stream per SM).
template <int M>
struct RingMinCtas {
    static constexpr int value = M <= 4 ? 2 : 1;
};

template <int M, int AM, bool kDump = false, int GSH = kG256>
__global__ void __launch_bounds__(kRingThreads, RingMinCtas<M>::value) w4_gemv_ring_kernel(
    const uint8_t* __restrict__ codes, const __half* __restrict__ d, const __half* __restrict__ m,
    int N, int K, int stages, int rows_per_cta, const Act act, void* __restrict__ y, int out_f32,
    int* err) {
    extern __shared__ __align__(128) unsigned char smem[];
    const int C = K >> 5;          // 32-code chunks per row
    const int G = K >> (5 + GSH);  // groups per row
    const int row_bytes = K >> 1;
    const int nkc = (row_bytes + kChunkBytes - 1) / kChunkBytes;  // K-chunks per row
    const Layout L = layout(M, C, stages, AM);
    using XW = typename XWord<AM>::T;
    XW* xq = reinterpret_cast<XW*>(smem + L.xq);
    float* sx = reinterpret_cast<float*>(smem + L.sx);
    float* inv = reinterpret_cast<float*>(smem + L.inv);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + kMaxStages;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(empty + kMaxStages);

    const int warp = threadIdx.x >> 5;
    const int r0 = blockIdx.x * rows_per_cta;
    const int r1 = min(N, r0 + rows_per_cta);
    const int ngrp = (r1 - r0 + kRowsPerStage - 1) / kRowsPerStage;
    const int nstage = ngrp * nkc;  // stages of this CTA, in (row group, K-chunk) order

    if (threadIdx.x == 0) {
        for (int i = 0; i < kMaxStages; ++i) {
            w4::mbar_init(&full[i], 1);
            w4::mbar_init(&empty[i], kRingWarps);
        }
        *abort_flag = 0;
        w4::fence_mbar_init();
    }
    __syncthreads();

    if (warp == kRingWarps) {
        // ---------------- producer: one lane streams the code ring ----------------
        // The producer reads only the weight planes, which do not depend on
        // the preceding kernel in the stream (the caller's contract), so it
        // never waits for that kernel: under programmatic dependent launch the
        // ring fills while the preceding kernel is still running.
        if (w4::elect_one()) {
            int it = 0;
            for (; it < nstage; ++it) {
                const int s = it % stages;
                const uint32_t ph = (uint32_t)(it / stages) & 1u;
                if (!w4::mbar_wait(&empty[s], ph ^ 1u, abort_flag, err)) break;
                const int grp = it / nkc, kc = it - grp * nkc;
                const int rb = r0 + grp * kRowsPerStage;
                const int nr = min(kRowsPerStage, r1 - rb);
                const int off = kc * kChunkBytes;
                const uint32_t bytes = (uint32_t)min(kChunkBytes, row_bytes - off);
                uint8_t* dst = smem + (size_t)s * kStageBytes;
                // the stage's rows and byte range lie inside the codes plane and
                // the ring slot (else, in the debug build, the stage stays unfilled)
                const bool in_range = W4_CHECK(rb + nr <= N && off + (int)bytes <= row_bytes &&
                                                   nr <= kRowsPerStage && (bytes & 15u) == 0,
                                               err);
                w4::mbar_arrive_expect_tx(&full[s], in_range ? bytes * (uint32_t)nr : 0u);
                for (int r = 0; in_range && r < nr; ++r)
                    w4::bulk_load_1d(dst + r * kChunkBytes, codes + (size_t)(rb + r) * row_bytes + off,
                                     bytes, &full[s]);
            }
            // every issued copy lands before the CTA may exit
            for (int k = it - stages < 0 ? 0 : it - stages; k < it; ++k)
                w4::mbar_wait(&full[k % stages], (uint32_t)(k / stages) & 1u, nullptr, err);
        }
        return;
    }

    // ---------------- consumers (warps 0..7) ----------------
    const int h = threadIdx.x >> 4;  // half-warp = row slot of a stage
    const int j = threadIdx.x & 15;  // lane in the half-warp
    // d and m of this lane's chunks in a stage: chunk cl = j + 16 i of K-chunk
    // kc lies in group kc * 10 + 2 i + (j >> 3); loaded one stage ahead
    constexpr int kLaneChunks = kChunkBytes / 16 / 16;  // 5
    auto load_dm = [&](int st, uint32_t (&dm)[kLaneChunks]) {
#pragma unroll
        for (int i = 0; i < kLaneChunks; ++i) dm[i] = 0;
        if (st >= nstage) return;
        const int grp = st / nkc, kc = st - grp * nkc;
        const int row = r0 + grp * kRowsPerStage + h;
        if (row >= r1) return;
        const int nch = min(kChunkBytes, row_bytes - kc * kChunkBytes) >> 4;
#pragma unroll
        for (int i = 0; i < kLaneChunks; ++i) {
            if (j + 16 * i < nch) {
                // chunk j + 16 i of K-chunk kc is chunk kc * 80 + j + 16 i of
                // the row; its group is that index >> GSH
                const size_t gi =
                    (size_t)row * G + ((kc * (kChunkBytes / 16) + j + 16 * i) >> GSH);
                if (W4_CHECK(gi < (size_t)N * G, err))
                    dm[i] = (uint32_t)ld_nc_u16(d + gi) | ((uint32_t)ld_nc_u16(m + gi) << 16);
            }
        }
    };

    // d/m of the next three stages in flight (their loads are plain global
    // loads, so they need more lead than one stage to cover HBM latency); the
    // first three stages' are weights too, so they are requested before the
    // wait for the preceding kernel, like the code ring
    uint32_t dm1[kLaneChunks], dm2[kLaneChunks], dm3[kLaneChunks];
    load_dm(0, dm1);
    load_dm(1, dm2);
    load_dm(2, dm3);
    pdl_wait();

    // activation words, chunk sums and scales, once per CTA; each thread issues
    // up to eight 16-byte loads before converting any
    constexpr int kCons = 32 * kRingWarps;
    if constexpr (AM == kActInt8) {
        for (int v = threadIdx.x; v < M * C; v += kCons)
            stage_block_a8(act, C, v / C, v - (v / C) * C, xq, sx, inv);
    } else if constexpr (AM == kActBf16ToInt8) {
        for (int v = threadIdx.x; v < M * C; v += kCons)
            stage_block_q8x(act, C, v / C, v - (v / C) * C, xq, sx, inv);
    } else {
        const int nq = M * C * 4;  // quarters (8 values) of chunks; a multiple of 4
        for (int base = 0; base < nq; base += 8 * kCons) {
            uint4 raw[8];
#pragma unroll
            for (int p4 = 0; p4 < 8; ++p4) {
                const int v = base + p4 * kCons + threadIdx.x;
                raw[p4] = v < nq ? __ldg(reinterpret_cast<const uint4*>(act.x) + v)
                                 : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int p4 = 0; p4 < 8; ++p4) {
                if (base + p4 * kCons >= nq) break;  // uniform across the consumers
                const int v = base + p4 * kCons + threadIdx.x;
                const bool live = v < nq;
                const int vv = live ? v : 0;
                const int t = vv / (C * 4);
                const int r = vv - t * C * 4;
                const int c = r >> 2, q4 = r & 3;
                if constexpr (AM == kActBf16)
                    stage_quarter(raw[p4], live, &xq[((size_t)t * 4 + q4) * C + c],
                                  &sx[t * C + c], &inv[t * C + c], q4);
            }
        }
    }
    asm volatile("bar.sync 1, %0;" ::"n"(kCons) : "memory");
    pdl_launch_dependents();

    float yacc[M];
#pragma unroll
    for (int t = 0; t < M; ++t) yacc[t] = 0.0f;

    for (int it = 0; it < nstage; ++it) {
        const int s = it % stages;
        const int grp = it / nkc, kc = it - grp * nkc;
        const int row = r0 + grp * kRowsPerStage + h;
        uint32_t dm[kLaneChunks];
#pragma unroll
        for (int i = 0; i < kLaneChunks; ++i) {
            dm[i] = dm1[i];
            dm1[i] = dm2[i];
            dm2[i] = dm3[i];
        }
        load_dm(it + 3, dm3);
        if (!w4::mbar_wait(&full[s], (uint32_t)(it / stages) & 1u, abort_flag, err)) break;
        if (row < r1) {
            const uint8_t* src = smem + (size_t)s * kStageBytes + h * kChunkBytes;
            const int nch = min(kChunkBytes, row_bytes - kc * kChunkBytes) >> 4;
            const int c_base = kc * (kChunkBytes / 16);
#pragma unroll
            for (int i = 0; i < kLaneChunks; ++i) {
                const int cl = j + 16 * i;
                // predicated: chains of live chunks interleave
                const bool live = cl < nch && W4_CHECK(c_base + cl < C, err);
                const int c = c_base + (live ? cl : 0);
                const uint4 wq = live ? *reinterpret_cast<const uint4*>(src + cl * 16)
                                      : make_uint4(0, 0, 0, 0);
                int ah[M], al[M];
#pragma unroll
                for (int t = 0; t < M; ++t) {
                    ah[t] = 0;
                    al[t] = 0;
                }
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    const uint32_t w = wi == 0 ? wq.x : wi == 1 ? wq.y : wi == 2 ? wq.z : wq.w;
                    const uint32_t lo = w & 0x0F0F0F0Fu;         // codes of k = 0, 2, 4, 6
                    const uint32_t hi = (w >> 4) & 0x0F0F0F0Fu;  // codes of k = 1, 3, 5, 7
#pragma unroll
                    for (int t = 0; t < M; ++t) {
                        // this slice's activation word (see XWord)
                        const XW xv = xq[((size_t)t * 4 + wi) * C + c];
                        ah[t] = __dp4a((int)lo, (int)xv.x, ah[t]);
                        ah[t] = __dp4a((int)hi, (int)xv.y, ah[t]);
                        if constexpr (AM == kActBf16) {
                            al[t] = (int)__dp4a(lo, xv.z, (unsigned)al[t]);
                            al[t] = (int)__dp4a(hi, xv.w, (unsigned)al[t]);
                        }
                    }
                }
                if constexpr (kDump) {
                    if (live) {
#pragma unroll
                        for (int t = 0; t < M; ++t)
                            act.dump[((size_t)t * N + row) * C + c] = ah[t];
                    }
                }
                const float dd = __half2float(__ushort_as_half((unsigned short)(dm[i] & 0xFFFFu)));
                const float mm = __half2float(__ushort_as_half((unsigned short)(dm[i] >> 16)));
#pragma unroll
                for (int t = 0; t < M; ++t) {
                    const float qx =
                        (AM != kActBf16 ? (float)ah[t] : (float)(ah[t] * 256 + al[t])) * inv[t * C + c];
                    const float v = fmaf(dd, qx, fmaf(mm, sx[t * C + c], yacc[t]));
                    yacc[t] = live ? v : yacc[t];
                }
            }
        }
        __syncwarp();
        if ((threadIdx.x & 31) == 0) w4::mbar_arrive(&empty[s]);
        if (kc == nkc - 1) {
            // row finished: reduce the 16 lanes (xor < 16 stays in the half-warp)
#pragma unroll
            for (int t = 0; t < M; ++t) {
                float v = yacc[t];
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 2);
                v += __shfl_xor_sync(0xffffffffu, v, 1);
                if (row < r1 && j == t) {
                    if (out_f32)
                        reinterpret_cast<float*>(y)[(size_t)t * N + row] = v;
                    else
                        reinterpret_cast<__nv_bfloat16*>(y)[(size_t)t * N + row] =
                            __float2bfloat16_rn(v);
                }
                yacc[t] = 0.0f;
            }
        }
    }
}

// Stages of the code ring and resident CTAs per SM for M tokens: four stages
// where the activation words leave room, and two CTAs per SM when both fit.
struct Plan {
    int stages, per_sm;
    size_t smem;
};

Plan plan_for(int M, int C, int AM) {
    Plan p{0, 0, 0};
    // (one CTA per SM at M = 1, leaving room beside it for the next kernel's
    // CTAs, was measured slower: 750 against 960 tok/s over the per-token chain)
    for (int st = kMaxStages; st >= 2; --st) {
        const size_t need = layout(M, C, st, AM).total;
        if (need <= (size_t)kSmemPerSm) {
            p.stages = st;
            p.smem = need;
            // 228 KB of shared memory per SM, 1 KB of it reserved per CTA
            p.per_sm = (M <= 4 && 2 * (need + 1024) <= (size_t)228 * 1024) ? 2 : 1;
            return p;
        }
    }
    return p;
}

template <int M, int AM, bool kDump = false, int GSH = kG256>
int launch_ring(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
                const Act& x, void* y, int out_f32, cudaStream_t st) {
    auto kern = w4_gemv_ring_kernel<M, AM, kDump, GSH>;
    const Plan pl = plan_for(M, K / 32, AM);  // per_sm matches RingMinCtas<M>
    if (pl.stages == 0) return W4_ERR_SHAPE;
    static thread_local int attr_dev = -1;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    if (attr_dev != dev) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemPerSm);
        if (e != cudaSuccess) return w4::cuda_fail(e);
        attr_dev = dev;
    }
    // contiguous, balanced row ranges: one per CTA
    int grid = pl.per_sm * w4::sm_count();
    if (grid > N) grid = N;
    const int rows_per_cta = (N + grid - 1) / grid;
    grid = (N + rows_per_cta - 1) / rows_per_cta;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kRingThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, codes, reinterpret_cast<const __half*>(d),
                           reinterpret_cast<const __half*>(m), N, K, pl.stages, rows_per_cta, x,
                           y, out_f32, w4::device_error_word());
    if (e != cudaSuccess) return w4::cuda_fail(e);
    return w4::launch_status();
}


// One launch for M tokens: streams below 16 MB of codes take the ring
// kernel, larger ones the row kernel (both group sizes).
template <int M, int AM, int GSH, bool kDump>
int dispatch_group(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
                   const Act& x, void* y, int out_f32, cudaStream_t st) {
    if ((size_t)N * (size_t)(K / 2) < kRingMaxCodeBytes && plan_for(M, K / 32, AM).stages > 0)
        return launch_ring<M, AM, kDump, GSH>(codes, d, m, N, K, x, y, out_f32, st);
    return dispatch_m<M, AM, GSH, kDump>(codes, d, m, N, K, x, y, out_f32, st);
}

// Most tokens whose staged activation words fit one launch's shared-memory
// budget (0 if not even one token's do).
int tokens_per_pass(int C, int AM) {
    for (int mp = 8; mp >= 1; --mp)
        if (smem_bytes(mp, C, 1, 1, AM) <= (size_t)kSmemBudget) return mp;
    return 0;
}

// The activation form (and dump) of tokens t0, t0 + 1, ...
Act act_from_token(const Act& a, int AM, int t0, int N, int K) {
    Act r = a;
    const size_t C = (size_t)(K / 32);
    if (AM == kActInt8) {
        r.x = static_cast<const int8_t*>(a.x) + (size_t)t0 * K;
        r.dx = a.dx + (size_t)t0 * C;
        r.S = a.S + (size_t)t0 * C;
    } else {
        r.x = static_cast<const uint16_t*>(a.x) + (size_t)t0 * K;
    }
    if (a.dump) r.dump = a.dump + (size_t)t0 * N * C;
    return r;
}

// M tokens in passes of as many as the activation staging holds (each pass
// streams the weights again; one pass for every shape whose M tokens fit).
template <int AM, int GSH = kG256, bool kDump = false>
int dispatch_any_m(const uint8_t* codes, const uint16_t* d, const uint16_t* m, int N, int K,
                   const Act& x, int M, void* y, int out_f32, cudaStream_t st) {
    const int mp = tokens_per_pass(K / 32, AM);
    if (mp == 0) return W4_ERR_SHAPE;
    for (int t0 = 0; t0 < M; t0 += mp) {
        const int mm = M - t0 < mp ? M - t0 : mp;
        const Act xa = act_from_token(x, AM, t0, N, K);
        void* ya = static_cast<uint8_t*>(y) + (size_t)t0 * N * (out_f32 ? 4 : 2);
        int rc;
        switch (mm) {
            case 1: rc = dispatch_group<1, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 2: rc = dispatch_group<2, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 3: rc = dispatch_group<3, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 4: rc = dispatch_group<4, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 5: rc = dispatch_group<5, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 6: rc = dispatch_group<6, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            case 7: rc = dispatch_group<7, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
            default: rc = dispatch_group<8, AM, GSH, kDump>(codes, d, m, N, K, xa, ya, out_f32, st); break;
        }
        if (rc != W4_OK) return rc;
    }
    return W4_OK;
}

// Largest K the decode GEMVs take: one token's staged activation words must
// fit the shared-memory budget in every form.
constexpr int64_t kMaxGemvK = 65536;

// Host validation shared by the entry points; W4_OK if the call may launch.
// K must be a multiple of the group size (256, or 32 for group-32 weights).
int validate(const void* codes, const void* d, const void* m, int64_t N, int64_t K,
             const void* a0, const void* a1, const void* a2, int M, const void* y,
             int out_dtype, int group = 256) {
    if (M < 1 || M > 8 || N < 1 || K < group || K % group != 0) return W4_ERR_SHAPE;
    if (N > (int64_t)1 << 30 || K > kMaxGemvK) return W4_ERR_SHAPE;
    if (out_dtype != W4_OUT_BF16 && out_dtype != W4_OUT_F32) return W4_ERR_SHAPE;
    if (!codes || !d || !m || !a0 || !a1 || !a2 || !y) return W4_ERR_NULL;
    if (!w4::aligned16(codes) || !w4::aligned16(d) || !w4::aligned16(m) ||
        !w4::aligned16(a0) || !w4::aligned16(a1) || !w4::aligned16(a2) || !w4::aligned16(y))
        return W4_ERR_ALIGN;
    return w4::check_device();
}

static_assert(kMaxGemvK / 32 * (16 * 4 + 8) <= kSmemBudget, "one token must fit the staging");

}  // namespace

