// gemv_blockdots.cu -- the test instantiation of the keep-quant decode GEMV
// (w4a8_gemv) that also stores the exact int32 block products its integer
// core forms.  Kept in its own translation unit so that its kernel
// instantiations compile in parallel with the product's.
#include "gemv_kernels.cuh"

extern "C" int w4a8_gemv_blockdots(const uint8_t* codes, const uint16_t* d_f16,
                                   const uint16_t* m_f16, int64_t N, int64_t K, const int8_t* qa,
                                   const float* dx, const int32_t* bsum, int M, void* y,
                                   int out_dtype, int32_t* blockdots, size_t bd_bytes,
                                   void* stream) {
    int rc = validate(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    if (!blockdots) return W4_ERR_NULL;
    if (!w4::aligned16(blockdots)) return W4_ERR_ALIGN;
    if (bd_bytes < (size_t)M * (size_t)N * (size_t)(K / 32) * 4) return W4_ERR_WORKSPACE;
    const Act act{qa, dx, bsum, blockdots};
    return dispatch_any_m<kActInt8, kG256, true>(codes, d_f16, m_f16, (int)N, (int)K, act, M, y,
                                                 out_dtype == W4_OUT_F32, (cudaStream_t)stream);
}
