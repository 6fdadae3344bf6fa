// Library-wide entry points: status strings, device queries, the error word
// (mr_poll_errors) and the bounded-wait self test.
#include "common.cuh"

#include <condition_variable>
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

// Exchange targets for mr_poll_errors: the error word is read and cleared in
// one atomic step on the device into a mailbox slot, then copied back from
// there.  Polls that run at the same time (other threads, other streams) each
// hold their own slot.
constexpr int kMailboxes = 64;
__device__ uint32_t g_error_mailbox[kMailboxes];

__global__ void take_errors_kernel(int slot) { g_error_mailbox[slot] = atomicExch(&g_error_word, 0u); }

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

namespace mr_host {
namespace {
std::mutex g_mailbox_mutex;
std::condition_variable g_mailbox_free;
uint64_t g_mailbox_busy[kMaxDevices] = {};

// A free mailbox slot of `device` (waits while all are taken), or -1.
int take_mailbox(int device) {
    if (device < 0 || device >= kMaxDevices) return -1;
    std::unique_lock<std::mutex> lock(g_mailbox_mutex);
    g_mailbox_free.wait(lock, [&] { return g_mailbox_busy[device] != ~0ull; });
    const int slot = __builtin_ctzll(~g_mailbox_busy[device]);
    g_mailbox_busy[device] |= 1ull << slot;
    return slot;
}

void give_mailbox(int device, int slot) {
    {
        std::lock_guard<std::mutex> lock(g_mailbox_mutex);
        g_mailbox_busy[device] &= ~(1ull << slot);
    }
    g_mailbox_free.notify_one();
}
}  // namespace
}  // namespace mr_host

extern "C" mr_status mr_poll_errors(void *stream, uint32_t *device_flags) {
    static_assert(mr::kMailboxes == 64, "one bit of the busy mask per mailbox");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return MR_ERR_CUDA;
    const int slot = mr_host::take_mailbox(device);
    if (slot < 0) return MR_ERR_CUDA;
    mr_status st = MR_OK;
    uint32_t flags = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(1);
    cfg.stream = s;
    if (cudaLaunchKernelEx(&cfg, mr::take_errors_kernel, slot) != cudaSuccess ||
        cudaMemcpyFromSymbolAsync(&flags, mr::g_error_mailbox, sizeof(flags), sizeof(uint32_t) * (size_t)slot,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        st = MR_ERR_CUDA;
    mr_host::give_mailbox(device, slot);
    if (st != MR_OK) return st;
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
