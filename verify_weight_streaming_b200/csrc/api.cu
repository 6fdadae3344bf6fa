// Library-wide entry points: status strings, device queries, the error word
// (mr_poll_errors) and the bounded-wait self test.
#include "common.cuh"

#include <mutex>

namespace mr_host {

mr_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MR_OK : MR_ERR_CUDA; }

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mutex;
int g_sms[kMaxDevices] = {};
int g_optin[kMaxDevices] = {};

bool query(int &dev) {
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
    std::lock_guard<std::mutex> lock(g_mutex);
    if (g_sms[dev] == 0) {
        int sms = 0, optin = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
        if (cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
            return false;
        g_optin[dev] = optin;
        g_sms[dev] = sms;
    }
    return true;
}
}  // namespace

int sm_count() {
    int dev = 0;
    return query(dev) ? g_sms[dev] : 0;
}

int max_smem_optin() {
    int dev = 0;
    return query(dev) ? g_optin[dev] : 0;
}

}  // namespace mr_host

namespace mr {

// Exchange target for mr_poll_errors: the error word is read and cleared in
// one atomic step on the device, then copied back from here.
__device__ uint32_t g_error_mailbox = 0;

__global__ void take_errors_kernel() { g_error_mailbox = atomicExch(&g_error_word, 0u); }

__global__ void selftest_wait_kernel(uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        // Nothing ever arrives on this barrier: the bounded wait must give up.
        mbar_wait_bounded(smem_u32(&bar), 0u, MR_DEVERR_SELFTEST, limit_ns);
    }
}

}  // namespace mr

extern "C" mr_status mr_poll_errors(void *stream, uint32_t *device_flags) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1);
    cfg.stream = s;
    cudaError_t e = cudaLaunchKernelEx(&cfg, mr::take_errors_kernel);
    if (e != cudaSuccess) return MR_ERR_CUDA;
    uint32_t flags = 0;
    e = cudaMemcpyFromSymbolAsync(&flags, mr::g_error_mailbox, sizeof(flags), 0, cudaMemcpyDeviceToHost, s);
    if (e != cudaSuccess) return MR_ERR_CUDA;
    e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return MR_ERR_CUDA;
    if (device_flags) *device_flags = flags;
    return flags ? MR_ERR_TIMEOUT : MR_OK;
}

extern "C" mr_status mr_selftest_wait_timeout(int32_t limit_us, void *stream) {
    if (limit_us < 1 || limit_us > 1000000) return MR_ERR_INVALID_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(32);
    cfg.stream = static_cast<cudaStream_t>(stream);
    return mr_host::cuda_status(
        cudaLaunchKernelEx(&cfg, mr::selftest_wait_kernel, (uint64_t)limit_us * 1000ull));
}

extern "C" const char *mr_status_str(mr_status status) {
    switch (status) {
        case MR_OK: return "MR_OK";
        case MR_ERR_INVALID_ARG: return "MR_ERR_INVALID_ARG";
        case MR_ERR_MISALIGNED: return "MR_ERR_MISALIGNED";
        case MR_ERR_UNSUPPORTED: return "MR_ERR_UNSUPPORTED";
        case MR_ERR_CUDA: return "MR_ERR_CUDA";
        case MR_ERR_TIMEOUT: return "MR_ERR_TIMEOUT";
    }
    return "MR_ERR_UNKNOWN";
}

extern "C" const char *mr_version(void) { return "mrgemm 0.1 (sm_100a)"; }
