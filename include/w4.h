/*
 * w4.h -- C ABI of libw4, the B200 (sm_100a) W4-G256 quantized-matmul library.
 *
 * Format (W4-G256; "HFQ4-G256" in the hipfire MMQ prefill article):
 *   W[N,K], K a multiple of 256, split into groups of 256 consecutive k per
 *   row.  Each group stores 128 bytes of 4-bit codes q in [0,15] plus an fp16
 *   scale d and an fp16 min m; a weight dequantises to w = d*q + m.
 *   Storage is three dense row-major planes:
 *     codes  uint8 [N][K/2]  byte j of a row holds k = 2j in bits 0-3 and
 *                            k = 2j+1 in bits 4-7
 *     d      fp16  [N][K/256] (raw IEEE binary16 bits)
 *     m      fp16  [N][K/256]
 *   Group-32 weights (w4_pack_g32, w4_gemv_g32) use the same codes plane with
 *   d and m planes of [N][K/32], one pair per 32 consecutive k; K % 32 == 0.
 *   Activations are bf16 [M][K] row-major (raw bits).  For the W4A8 product
 *   they are first quantised per 32-element block (the Q8_1-style MMQ layout
 *   the article pre-quantises prefill activations to):
 *     qa  int8  [M][K]      codes in [-127,127]
 *     dx  fp32  [M][K/32]   block scale amax/127 (0 for an all-zero block)
 *     S   int32 [M][K/32]   sum of the block's qa
 *
 * Conventions for every entry point:
 *   - All data pointers are DEVICE pointers to caller-owned memory.  The
 *     library never allocates, frees or synchronises; it only enqueues work on
 *     `stream` (a cudaStream_t passed as void*; NULL is the legacy default
 *     stream) and returns.
 *   - Base pointers must be 16-byte aligned; row strides are the dense ones
 *     implied by the shapes above.
 *   - Arguments are validated on the host before anything is enqueued; a
 *     violation returns its status and enqueues nothing.
 *   - The device must be a compute-capability 10.0 GPU (B200 class); any other
 *     device gives W4_ERR_UNSUPPORTED_DEVICE.  There is no fallback path.
 *   - W4_ERR_CUDA reports a launch error; w4_last_cuda_error() gives the CUDA
 *     error code.  Inputs are assumed finite (not checked).
 *   - Every kernel waits for its own pipeline with bounded spins; a wait that
 *     runs out sets a device-side error word and the kernel returns early.
 *     w4_check_device_error() reads (and clears) that word.
 *   - libw4_debug.so, the same sources built with -DW4_DEBUG, checks the
 *     indices of the kernels' global and shared-memory accesses on the device;
 *     a failed check records W4_ERR_BOUNDS in the same error word and skips
 *     the access (a stand-in for a memory checker; for tests on small shapes).
 *   - Results are bitwise deterministic run to run (fixed reduction orders, no
 *     floating-point atomics).
 *   - The decode GEMVs (w4_gemv, w4a8_gemv, w4a8_gemv_bf16) and the W4A8
 *     product (w4a8_mmq and its variants, when it needs no workspace) are
 *     launched with programmatic dependent launch and read their weight
 *     planes (codes, d, m) without waiting for the kernel launched
 *     immediately before them on the same stream (their activations are read
 *     only after that kernel has completed).  The weight planes must
 *     therefore not be written by that immediately preceding kernel: pack
 *     weights in an earlier launch, or put an event, a synchronisation or any
 *     other launch in between.
 */
#ifndef W4_H
#define W4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define W4_ABI_VERSION 1

typedef enum {
    W4_OK = 0,
    W4_ERR_NULL = 1,               /* a required pointer is NULL            */
    W4_ERR_SHAPE = 2,              /* a size violates the format or range   */
    W4_ERR_ALIGN = 3,              /* a base pointer is not 16-byte aligned */
    W4_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100          */
    W4_ERR_WORKSPACE = 5,          /* workspace missing or too small        */
    W4_ERR_CUDA = 6,               /* a CUDA call or launch failed          */
    W4_ERR_TIMEOUT = 7,            /* a kernel's bounded wait ran out       */
    W4_ERR_BOUNDS = 8              /* debug build only: a device-side index
                                      check failed (the access was skipped) */
} w4_status;

typedef enum {
    W4_OUT_BF16 = 0, /* y stored as bf16, round to nearest even of the fp32 sum */
    W4_OUT_F32 = 1   /* y stored as fp32                                        */
} w4_out_dtype;

/* ABI version of the loaded library (W4_ABI_VERSION at build time). */
int w4_abi_version(void);

/* Static, human-readable name of a status code. */
const char *w4_status_string(int status);

/* CUDA error code (cudaError_t as int) behind the last W4_ERR_CUDA on this
 * host thread, or 0. */
int w4_last_cuda_error(void);

/* Synchronises the current device, then returns W4_ERR_TIMEOUT if any kernel
 * of this library gave up a bounded wait since the last call (and clears the
 * flag), W4_ERR_CUDA if the synchronisation failed, else W4_OK. */
int w4_check_device_error(void);

/* Quantise and pack fp32 weights, min/max per group of 256.
 * Defined by: the format definition above ("groups of 256 ... 4-bit codes
 * plus fp16 d and fp16 m, w = d*q + m"); the rounding rule is the reading
 * adopted where the pages are silent:
 *   per (row, group): mn, mx = min, max (fp32);
 *   d16 = fp16_rn((mx - mn) / 15); m16 = fp16_rn(mn);
 *   q = 0 if d16 == 0 else clamp(rint((w - m16) / d16), 0, 15), ties to even,
 *   all arithmetic IEEE fp32 round-to-nearest.
 * w: fp32 [N][K]; outputs codes [N][K/2], d [N][K/256], m [N][K/256].
 * N >= 0, K >= 0, K % 256 == 0.  N == 0 or K == 0 enqueues nothing. */
int w4_pack(const float *w, int64_t N, int64_t K, uint8_t *codes,
            uint16_t *d_f16, uint16_t *m_f16, void *stream);

/* w4_pack for the group-32 variant of the format: the asymmetric int4,
 * group-32 scheme of the W4A16 checkpoints on the ROCM_OCTAVE page
 * ("Validation": W4A16, int4, group 32; the sparse-attention evaluation's
 * "Setup": asymmetric, g32), read as the same w = d*q + m form with one fp16
 * d and one fp16 m per 32 weights.  Same quantiser rule per group of 32.
 * w: fp32 [N][K]; outputs codes [N][K/2] (nibble order as above), d [N][K/32],
 * m [N][K/32].  N >= 0, K >= 0, K % 32 == 0.  Errors as w4_pack. */
int w4_pack_g32(const float *w, int64_t N, int64_t K, uint8_t *codes,
                uint16_t *d_f16, uint16_t *m_f16, void *stream);

/* Pack one-code-per-byte q [N][K] (values 0..15; higher bits are ignored)
 * into codes [N][K/2] with the nibble order above: the 128-byte packed code
 * block of each group of the HFQ4-G256 format (the hipfire MMQ article's
 * weight format; the nibble order is the reading stated at the top of this
 * file).  K % 2 == 0 and (N*K) % 32 == 0. */
int w4_pack_codes(const uint8_t *q, int64_t N, int64_t K, uint8_t *codes,
                  void *stream);

/* Inverse of w4_pack_codes: codes [N][K/2] -> q [N][K], one code per byte
 * (the 4-bit codes q in [0,15] of the HFQ4-G256 format, hipfire MMQ article).
 * K % 2 == 0 and (N*K) % 32 == 0. */
int w4_unpack(const uint8_t *codes, int64_t N, int64_t K, uint8_t *q,
              void *stream);

/* Decode GEMV, dequantisation fused into the weight stream (the batch-1
 * decode "quant-GEMM bandwidth ladder" of the GFX1100-TG150/TG200 pages):
 *   y[t][n] = sum_g ( d[n][g] * sum_{k in g} q[n][k] * x[t][k]
 *                     + m[n][g] * sum_{k in g} x[t][k] )
 * for t < M, n < N, accumulated in fp32.
 * codes/d/m: the format planes of W[N][K]; x: bf16 [M][K]; y: [M][N] of
 * out_dtype.  1 <= M <= 8, N >= 1, 256 <= K <= 65536, K % 256 == 0; larger
 * sizes give W4_ERR_SHAPE.  Each launch stages its tokens' activations in
 * shared memory (72 bytes per token and 32 k in this bf16 form, 40 bytes in
 * the int8 forms, at most 200 KB): when M tokens do not fit (e.g. M = 8 at
 * K = 12288) they are processed in passes of as many tokens as fit, each pass
 * streaming the weights again. */
int w4_gemv(const uint8_t *codes, const uint16_t *d_f16,
            const uint16_t *m_f16, int64_t N, int64_t K,
            const uint16_t *x_bf16, int M, void *y, int out_dtype,
            void *stream);

/* w4_gemv for group-32 weights (the W4A16 g32 scheme of w4_pack_g32):
 *   y[t][n] = sum_g ( d[n][g] * sum_{k in g} q[n][k] * x[t][k]
 *                     + m[n][g] * sum_{k in g} x[t][k] ),  groups of 32,
 * accumulated in fp32.  codes [N][K/2], d and m [N][K/32] from w4_pack_g32;
 * x: bf16 [M][K]; y: [M][N] of out_dtype.  1 <= M <= 8, N >= 1,
 * 32 <= K <= 65536, K % 32 == 0.  Same validation, errors and token passes
 * as w4_gemv. */
int w4_gemv_g32(const uint8_t *codes, const uint16_t *d_f16,
                const uint16_t *m_f16, int64_t N, int64_t K,
                const uint16_t *x_bf16, int M, void *y, int out_dtype,
                void *stream);

/* Decode GEMV on int8 activation blocks ("keep-quant" decode: the
 * activations stay in the Q8_1-style blocks that q8_quantize_act produces, so
 * the core of every 32-element block is an exact integer dot product, as in
 * the decode arm of the GFX1100-TG200 campaign page that keeps the integer
 * core bit-exact against the CPU).  It computes the W4A8 product of w4a8_mmq
 * for decode batches:
 *   P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]      (exact int32)
 *   y[t][n]    = sum_g ( d[n][g] * sum_{b in g} dx[t][b] * P[t][n][b]
 *                        + m[n][g] * sum_{b in g} dx[t][b] * S[t][b] )
 * scales applied in fp32.  codes/d/m: W[N][K] planes; qa int8 [M][K], dx fp32
 * [M][K/32], bsum int32 [M][K/32]: the output of q8_quantize_act; y: [M][N]
 * of out_dtype.  1 <= M <= 8, N >= 1, 256 <= K <= 65536, K % 256 == 0;
 * every pointer 16-byte aligned.  Same validation, errors and token passes as
 * w4_gemv. */
int w4a8_gemv(const uint8_t *codes, const uint16_t *d_f16,
              const uint16_t *m_f16, int64_t N, int64_t K, const int8_t *qa,
              const float *dx, const int32_t *bsum, int M, void *y,
              int out_dtype, void *stream);

/* w4a8_gemv with the activation quantiser folded in: takes bf16 x [M][K] and
 * quantises each 32-element block inside the GEMV, with the arithmetic of
 * q8_quantize_act, so y is bit-identical to q8_quantize_act followed by
 * w4a8_gemv, without the second launch or the int8 blocks' round trip
 * through memory (the "fold the quantiser into its neighbour" next step of
 * the decode path).  Arguments and errors as w4_gemv. */
int w4a8_gemv_bf16(const uint8_t *codes, const uint16_t *d_f16,
                   const uint16_t *m_f16, int64_t N, int64_t K,
                   const uint16_t *x_bf16, int M, void *y, int out_dtype,
                   void *stream);

/* Quantise bf16 activations to int8 per block of 32 (the article's
 * "pre-quantise prefill activations to the Q8_1 MMQ layout"), with the
 * reading adopted for the unprinted rule:
 *   amax = max |x|;  dx = amax / 127 (IEEE fp32 division);
 *   amax == 0 -> dx = 0, qa = 0, S = 0;
 *   else qa = clamp(rint(x / dx), -127, 127), ties to even;  S = sum(qa).
 * x: bf16 [M][K] -> qa int8 [M][K], dx fp32 [M][K/32], S int32 [M][K/32].
 * M >= 0, K % 32 == 0. */
int q8_quantize_act(const uint16_t *x_bf16, int64_t M, int64_t K, int8_t *qa,
                    float *dx, int32_t *bsum, void *stream);

/* Bytes of device workspace w4a8_mmq needs for this shape (0 means none; the
 * workspace pointer may then be NULL).  The workspace holds the fp32 partial
 * output tiles of a split over K, used when the output tiles do not fill the
 * GPU's SMs in whole waves (all tiles split when they fill less than one wave,
 * otherwise only the tiles of the last, partial wave; the tiled int8
 * matrix-matrix product of the hipfire MMQ article runs here as 128x128
 * tiles; the split is this library's, not the article's): int32 arrival
 * counters for the split tiles, then [split tiles][slices][128][128] fp32.
 * The size depends on the current device's SM count. */
size_t w4a8_mmq_workspace_size(int64_t M, int64_t N, int64_t K);

/* W4A8 prefill product on int8 tensor cores (the article's MMQ path: int8
 * activations, tiled int8 matrix-matrix over the 4-bit weights, scales
 * applied after the integer products):
 *   P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]      (exact int32)
 *   y[t][n]    = sum_g ( d[n][g] * sum_{b in g} dx[t][b] * P[t][n][b]
 *                        + m[n][g] * sum_{b in g} dx[t][b] * S[t][b] )
 * scales applied in fp32.  codes/d/m: W[N][K] planes; qa/dx/bsum: the
 * output of q8_quantize_act for x [M][K]; y: [M][N] of out_dtype.
 * 1 <= M <= 2^24, 1 <= N <= 2^24, 256 <= K <= 131072 (512 groups),
 * K % 256 == 0; larger sizes give W4_ERR_SHAPE.  `workspace` (16-byte
 * aligned) must hold w4a8_mmq_workspace_size(M, N, K) bytes, else
 * W4_ERR_WORKSPACE; it may be NULL when that size is 0. */
int w4a8_mmq(const uint8_t *codes, const uint16_t *d_f16,
             const uint16_t *m_f16, int64_t N, int64_t K, const int8_t *qa,
             const float *dx, const int32_t *bsum, int64_t M, void *y,
             int out_dtype, void *workspace, size_t ws_bytes, void *stream);

/* Size of the library-owned device scratch behind w4a8_mmq_static. */
#define W4A8_MMQ_STATIC_SCRATCH_BYTES (40u * 1024u * 1024u)

/* The W4A8 product of w4a8_mmq for callers that cannot allocate device memory
 * (the pages have no counterpart: this entry point exists for the library's
 * users, not for the method).  Some callers cannot call cudaMalloc or hand out
 * a workspace: plugins whose host framework owns every device allocation and
 * gives the plugin only its inputs and outputs, and deployments whose memory
 * plan is fixed before the first request, where an allocation in the middle
 * of serving is not allowed.  This entry point takes the same inputs and
 * output as w4a8_mmq but no workspace: the split-K scratch is a static device
 * array owned by the library, W4A8_MMQ_STATIC_SCRATCH_BYTES (40 MiB) on every
 * GPU that loads libw4, held until the process exits.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call.
 *   - Arguments are checked exactly as w4a8_mmq checks them, in the same
 *     order; then a shape whose scratch need (w4a8_mmq_workspace_size)
 *     exceeds the static size is rejected with W4_ERR_WORKSPACE before
 *     anything is enqueued (w4a8_mmq with a caller workspace takes it).
 *   - The first call on each device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current) and caches it for the
 *     life of the process: make that first call before any stream capture.
 *     A device reset (cudaDeviceReset, or a reset of the primary context)
 *     invalidates the cached address; do not call this entry point after one.
 *   - Every call on a device shares the one array and it keeps the last call's
 *     contents (the arrival counters it needs at zero are cleared on the call's
 *     stream): calls that can overlap on the GPU -- on different streams, or
 *     from several host threads -- race on it and must be serialised.
 * Arguments, layouts and results are those of w4a8_mmq; for the same inputs
 * the output is bitwise that of w4a8_mmq. */
int w4a8_mmq_static(const uint8_t *codes, const uint16_t *d_f16,
                    const uint16_t *m_f16, int64_t N, int64_t K,
                    const int8_t *qa, const float *dx, const int32_t *bsum,
                    int64_t M, void *y, int out_dtype, void *stream);

/* ------------------------------------------------------------------------ */
/* Test entry points: they check the library's own machinery, not the method */
/* ------------------------------------------------------------------------ */

/* w4a8_mmq that also returns the exact integer block products it formed:
 *   blockdots[t][n][b] = P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]
 * (int32 [M][N][K/32], row-major; bd_bytes >= M*N*(K/32)*4, else
 * W4_ERR_WORKSPACE), read back from the tensor-memory accumulators of the
 * same kernel and tiling that w4a8_mmq runs (the test instantiation of that
 * kernel, which additionally stores every accumulator word it reads), so that
 * the integer core can be compared with the CPU bit for bit, the practice of
 * the GFX1100-TG150 spec ("Design": the keep-quant integer core stays
 * bit-exact against the CPU).  y, workspace and every other argument and error
 * are those of w4a8_mmq.  For tests: the block-product stores make it much
 * slower than w4a8_mmq. */
int w4a8_mmq_blockdots(const uint8_t *codes, const uint16_t *d_f16,
                       const uint16_t *m_f16, int64_t N, int64_t K,
                       const int8_t *qa, const float *dx, const int32_t *bsum,
                       int64_t M, void *y, int out_dtype, int32_t *blockdots,
                       size_t bd_bytes, void *workspace, size_t ws_bytes,
                       void *stream);

/* w4a8_gemv that also returns the exact integer block products its integer
 * core formed:
 *   blockdots[t][n][b] = P[t][n][b] = sum_{k in block b} q[n][k] * qa[t][k]
 * (int32 [M][N][K/32], row-major; bd_bytes >= M*N*(K/32)*4, else
 * W4_ERR_WORKSPACE), stored by the test instantiation of the same kernels,
 * with the same dispatch, that w4a8_gemv runs, so that the decode path's
 * integer core can be compared with the CPU bit for bit (the keep-quant
 * integer core of the GFX1100-TG150 spec, "Design").  y and every other
 * argument and error are those of w4a8_gemv.  For tests. */
int w4a8_gemv_blockdots(const uint8_t *codes, const uint16_t *d_f16,
                        const uint16_t *m_f16, int64_t N, int64_t K,
                        const int8_t *qa, const float *dx, const int32_t *bsum,
                        int M, void *y, int out_dtype, int32_t *blockdots,
                        size_t bd_bytes, void *stream);

/* Runs the bounded-wait routine that every pipelined kernel of this library
 * uses, on a wait that can never complete: one thread waits on an mbarrier
 * phase that nothing completes, for limit_ns nanoseconds of GPU global time,
 * then raises the device error word and returns (no trap, no fault: the
 * context stays usable).  A following w4_check_device_error() returns
 * W4_ERR_TIMEOUT and clears the word.  0 < limit_ns <= 100000000 (0.1 s),
 * else W4_ERR_SHAPE.  Enqueued on `stream`. */
int w4_test_wait_expiry(uint64_t limit_ns, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* W4_H */
