// gemv.cu -- entry points of the decode GEMVs (w4_gemv, w4a8_gemv,
// w4a8_gemv_bf16, w4_gemv_g32); the kernels, their dispatch and the host
// validation are in gemv_kernels.cuh.
#include "gemv_kernels.cuh"

extern "C" int w4_gemv(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                       int64_t N, int64_t K, const uint16_t* x_bf16, int M, void* y,
                       int out_dtype, void* stream) {
    const int rc = validate(codes, d_f16, m_f16, N, K, x_bf16, x_bf16, x_bf16, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    const Act act{x_bf16, nullptr, nullptr, nullptr};
    return dispatch_any_m<kActBf16>(codes, d_f16, m_f16, (int)N, (int)K, act, M, y,
                                 out_dtype == W4_OUT_F32, (cudaStream_t)stream);
}

extern "C" int w4a8_gemv(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                         int64_t N, int64_t K, const int8_t* qa, const float* dx,
                         const int32_t* bsum, int M, void* y, int out_dtype, void* stream) {
    const int rc = validate(codes, d_f16, m_f16, N, K, qa, dx, bsum, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    const Act act{qa, dx, bsum, nullptr};
    return dispatch_any_m<kActInt8>(codes, d_f16, m_f16, (int)N, (int)K, act, M, y,
                                out_dtype == W4_OUT_F32, (cudaStream_t)stream);
}

extern "C" int w4a8_gemv_bf16(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                              int64_t N, int64_t K, const uint16_t* x_bf16, int M, void* y,
                              int out_dtype, void* stream) {
    const int rc = validate(codes, d_f16, m_f16, N, K, x_bf16, x_bf16, x_bf16, M, y, out_dtype);
    if (rc != W4_OK) return rc;
    const Act act{x_bf16, nullptr, nullptr, nullptr};
    return dispatch_any_m<kActBf16ToInt8>(codes, d_f16, m_f16, (int)N, (int)K, act, M, y,
                                          out_dtype == W4_OUT_F32, (cudaStream_t)stream);
}

extern "C" int w4_gemv_g32(const uint8_t* codes, const uint16_t* d_f16, const uint16_t* m_f16,
                           int64_t N, int64_t K, const uint16_t* x_bf16, int M, void* y,
                           int out_dtype, void* stream) {
    const int rc =
        validate(codes, d_f16, m_f16, N, K, x_bf16, x_bf16, x_bf16, M, y, out_dtype, 32);
    if (rc != W4_OK) return rc;
    const Act act{x_bf16, nullptr, nullptr, nullptr};
    return dispatch_any_m<kActBf16, kG32>(codes, d_f16, m_f16, (int)N, (int)K, act, M, y,
                                          out_dtype == W4_OUT_F32, (cudaStream_t)stream);
}
