// abi.cu -- library-wide entry points of the C ABI: version, status names,
// the cached device check and the device error word.
#include <cstdio>
#include <mutex>

#include "common.cuh"

namespace {

constexpr int kMaxDevices = 64;
// Longest wait w4_test_wait_expiry accepts (0.1 s).
constexpr uint64_t kMaxTestWaitNs = 100000000ull;

// One error word per device; kernels raise W4_ERR_TIMEOUT here when a bounded
// wait runs out.
__device__ int g_error_word = 0;

thread_local int t_last_cuda_error = 0;

std::mutex g_mu;
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 ok, 2 unsupported
int* g_err_ptr[kMaxDevices];
int g_sms[kMaxDevices];

int current_device(int* dev) {
    cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return w4::cuda_fail(e);
    if (*dev < 0 || *dev >= kMaxDevices) return W4_ERR_UNSUPPORTED_DEVICE;
    return W4_OK;
}

// Test of the bounded-wait path: one thread waits on an mbarrier whose phase
// nothing completes, with the caller's limit, through the same wait routine
// every pipelined kernel uses.  When the limit runs out the routine raises the
// device error word and the kernel returns normally.
__global__ void wait_expiry_kernel(unsigned long long limit_ns, int* err) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    w4::mbar_init(&bar, 1);
    abort_flag = 0;
    w4::fence_mbar_init();
    // phase 0 of `bar` needs one arrival that never comes
    (void)w4::mbar_wait_for(&bar, 0u, &abort_flag, err, limit_ns);
}

}  // namespace

namespace w4 {

int cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return W4_ERR_CUDA;
}

int launch_status() {
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? W4_OK : cuda_fail(e);
}

int check_device() {
    int dev;
    int rc = current_device(&dev);
    if (rc != W4_OK) return rc;
    int cached = __atomic_load_n(&g_arch_ok[dev], __ATOMIC_ACQUIRE);
    if (cached == 1) return W4_OK;
    if (cached == 2) return W4_ERR_UNSUPPORTED_DEVICE;
    int major = 0, minor = 0, sms = 0;
    cudaError_t e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    const bool ok = (major == 10 && minor == 0);
    std::lock_guard<std::mutex> lk(g_mu);
    g_sms[dev] = sms;
    __atomic_store_n(&g_arch_ok[dev], ok ? 1 : 2, __ATOMIC_RELEASE);
    return ok ? W4_OK : W4_ERR_UNSUPPORTED_DEVICE;
}

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
    int s = g_sms[dev];
    return s > 0 ? s : 148;
}

int* device_error_word() {
    int dev;
    if (current_device(&dev) != W4_OK) return nullptr;
    int* p = __atomic_load_n(&g_err_ptr[dev], __ATOMIC_ACQUIRE);
    if (p) return p;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_error_word) != cudaSuccess) return nullptr;
    __atomic_store_n(&g_err_ptr[dev], static_cast<int*>(addr), __ATOMIC_RELEASE);
    return static_cast<int*>(addr);
}

}  // namespace w4

extern "C" {

int w4_abi_version(void) { return W4_ABI_VERSION; }

const char* w4_status_string(int status) {
    switch (status) {
        case W4_OK: return "W4_OK";
        case W4_ERR_NULL: return "W4_ERR_NULL: a required pointer is NULL";
        case W4_ERR_SHAPE: return "W4_ERR_SHAPE: a size violates the format or the supported range";
        case W4_ERR_ALIGN: return "W4_ERR_ALIGN: a base pointer is not 16-byte aligned";
        case W4_ERR_UNSUPPORTED_DEVICE:
            return "W4_ERR_UNSUPPORTED_DEVICE: libw4 runs only on compute capability 10.0 (sm_100a)";
        case W4_ERR_WORKSPACE: return "W4_ERR_WORKSPACE: workspace missing or too small";
        case W4_ERR_CUDA: return "W4_ERR_CUDA: a CUDA call or kernel launch failed";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT: a kernel gave up a bounded wait";
        case W4_ERR_BOUNDS:
            return "W4_ERR_BOUNDS: a device-side index check of the debug build failed";
        default: return "unknown w4 status";
    }
}

int w4_last_cuda_error(void) { return t_last_cuda_error; }

int w4_check_device_error(void) {
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return w4::cuda_fail(e);
    int v = 0;
    e = cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int));
    if (e != cudaSuccess) return w4::cuda_fail(e);
    if (v != 0) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int));
        if (e != cudaSuccess) return w4::cuda_fail(e);
        return v;
    }
    return W4_OK;
}

int w4_test_wait_expiry(uint64_t limit_ns, void* stream) {
    if (limit_ns == 0 || limit_ns > kMaxTestWaitNs) return W4_ERR_SHAPE;
    int rc = w4::check_device();
    if (rc != W4_OK) return rc;
    int* err = w4::device_error_word();
    if (!err) return W4_ERR_CUDA;
    wait_expiry_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((unsigned long long)limit_ns, err);
    return w4::launch_status();
}

}  // extern "C"
