// router_topk: per-row top-k (k <= 32) of fp32 logits, one CTA per row.
//
// The multi-row top-10 launch of Strata PR #109 ("What", router bullet: one
// launch for the window's rows, blockIdx.x = token).  Ties go to the lower
// index; -0.0 equals +0.0; a NaN ranks above +inf.
//
// Each element becomes a 64-bit key: the high word maps the float to an
// unsigned integer that increases with its value (sign-magnitude flip, -0.0
// folded onto +0.0, every NaN mapped to the maximum); the low word is
// 0xFFFFFFFF - index, so among equal values the lower index has the larger
// key.  Keys are unique, and "top-k by the total order" is "the k largest
// keys".  Each warp keeps a running top-k spread one entry per lane and
// merges every chunk of 32*P elements into it: a threshold from the lane
// maxima keeps at most 32 candidates, which are ranked with shuffles in one
// pass (k rounds of a warp-wide maximum when ties leave more than 32).  The
// CTA's warps are merged the same way at the end.  Values are re-read from
// the logits at the selected indices so they match bit for bit (a -0.0 stays
// -0.0).  Rows of up to 2048 logits take one warp per row instead.
#include "common.cuh"

#include "topk_core.cuh"

namespace mr {
namespace topk {

constexpr int kWarps = 4;
constexpr int kP = 4;              // elements per lane per chunk (128 per warp)
constexpr int kMaxK = 32;

__global__ void __launch_bounds__(kWarps * 32) topk_kernel(const float *__restrict__ logits, int64_t ldl,
                                                          int n, int K, int32_t *__restrict__ idx,
                                                          float *__restrict__ val, int64_t ldo) {
    __shared__ uint64_t cand[kWarps][32];
    __shared__ uint64_t scratch[kWarps][64];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = blockIdx.x;
    const float *x = logits + row * ldl;
    // Launched with programmatic stream serialization: let the next kernel
    // start its prologue, and read the logits only once the kernel that
    // produced them has completed.
    grid_launch_dependents();
    grid_dependency_wait();

    const uint64_t run = warp_topk_fast<kP>(x, n, K, lane, warp, kWarps, 0ull, scratch[warp]);
    cand[warp][lane] = lane < K ? run : 0ull;
    __syncthreads();
    if (warp == 0) {
        uint64_t keys[kWarps];
#pragma unroll
        for (int w = 0; w < kWarps; ++w) keys[w] = cand[w][lane];
        const uint64_t best = warp_topk_merge<kWarps>(keys, 0ull, K, lane, scratch[0]);
        if (lane < K) {
            const uint32_t j = key_index(best);
            idx[row * ldo + lane] = (int32_t)j;
            if (val) val[row * ldo + lane] = selected_value(best, x);
        }
    }
}

// Rows of up to kWarpRowMax logits: one warp per row (a 32-thread CTA),
// chunks of 512 elements, no cross-warp merge and no block barrier.
constexpr int kWarpRowMax = 2048;

__global__ void __launch_bounds__(32) topk_warp_kernel(const float *__restrict__ logits, int64_t ldl, int n, int K,
                                                       int32_t *__restrict__ idx, float *__restrict__ val,
                                                       int64_t ldo) {
    __shared__ uint64_t scratch[64];
    const int lane = threadIdx.x;
    const int64_t row = blockIdx.x;
    const float *x = logits + row * ldl;
    grid_launch_dependents();
    grid_dependency_wait();
    const uint64_t best = warp_topk_fast<16>(x, n, K, lane, 0, 1, 0ull, scratch);
    if (lane < K) {
        idx[row * ldo + lane] = (int32_t)key_index(best);
        if (val) val[row * ldo + lane] = selected_value(best, x);
    }
}

}  // namespace topk
}  // namespace mr

extern "C" mr_status router_topk(const float *logits, int64_t ldl, int32_t m, int32_t n, int32_t topk,
                                 int32_t *idx, float *val, int64_t ldo, void *stream) {
    if (!logits || !idx) return MR_ERR_INVALID_ARG;
    if (m < 1 || n < 1 || topk < 1 || topk > n) return MR_ERR_INVALID_ARG;
    if (ldl < n || ldo < topk) return MR_ERR_INVALID_ARG;
    if (topk > mr::topk::kMaxK) return MR_ERR_UNSUPPORTED;
    if (((uintptr_t)logits & 3u) || ((uintptr_t)idx & 3u) || ((uintptr_t)val & 3u)) return MR_ERR_MISALIGNED;
    const bool one_warp = n <= mr::topk::kWarpRowMax;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)m);
    cfg.blockDim = dim3(one_warp ? 32 : mr::topk::kWarps * 32);
    cfg.stream = static_cast<cudaStream_t>(stream);
    // Safe for any predecessor: the kernel waits for it before reading input.
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (one_warp)
        return mr_host::cuda_status(
            cudaLaunchKernelEx(&cfg, mr::topk::topk_warp_kernel, logits, ldl, (int)n, (int)topk, idx, val, ldo));
    return mr_host::cuda_status(
        cudaLaunchKernelEx(&cfg, mr::topk::topk_kernel, logits, ldl, (int)n, (int)topk, idx, val, ldo));
}
