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
// maxima keeps at most 32 candidates, which are ranked against each other
// through shared memory in one pass (k rounds of a warp-wide maximum when ties
// leave more than 32).  The CTA's warps are merged the same way at the end.
// Values are decoded from the keys, and re-read from the logits where a key
// does not keep the bits (+-0.0, NaN), so they match bit for bit.  Rows of up
// to 2048 logits take one warp per row instead.
#include "common.cuh"

#include "topk_core.cuh"

namespace mr {
namespace topk {

constexpr int kWarps = 4;
constexpr int kP = 4;              // elements per lane per chunk (128 per warp)
constexpr int kMaxK = 32;
constexpr int64_t kMaxMergeCandidates = 1 << 16;

__global__ void __launch_bounds__(kWarps * 32) topk_kernel(const float *__restrict__ logits, int64_t ldl,
                                                          int n, int K, int32_t *__restrict__ idx,
                                                          float *__restrict__ val, int64_t ldo, int32_t base) {
    __shared__ uint64_t cand[kWarps][32];
    __shared__ __align__(16) uint64_t scratch[kWarps][64];
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
            idx[row * ldo + lane] = (int32_t)j + base;
            if (val) val[row * ldo + lane] = selected_value(best, x);
        }
    }
}

// Rows of up to kWarpRowMax logits: one warp per row, chunks of 512
// elements, no cross-warp merge and no block barrier.  The CTA has a second
// warp that runs the same selection code on synthetic values at once, while
// warp 0 waits for the logits' producer: the selection runs once per launch,
// and fetching its instructions into a cold instruction cache otherwise costs
// more than the selection itself (measured 3.7 us against 1.2 us after a GEMV
// launch).
constexpr int kWarpRowMax = 2048;

__global__ void __launch_bounds__(64) topk_warp_kernel(const float *__restrict__ logits, int64_t ldl, int n, int K,
                                                       int32_t *__restrict__ idx, float *__restrict__ val,
                                                       int64_t ldo, int32_t base) {
    __shared__ __align__(16) uint64_t scratch[2][64];
    const int lane = threadIdx.x & 31;
    const bool warm = (threadIdx.x >> 5) != 0;
    const int64_t row = blockIdx.x;
    const float *x = logits + row * ldl;
    grid_launch_dependents();
    if (!warm) grid_dependency_wait();
    const uint64_t best = warp_topk_fast<16>(x, n, K, lane, 0, 1, 0ull, scratch[warm ? 1 : 0], warm);
    if (warm) return;
    if (lane < K) {
        idx[row * ldo + lane] = (int32_t)key_index(best) + base;
        if (val) val[row * ldo + lane] = selected_value(best, x);
    }
}

// Merge of candidate lists: row r has `groups` lists of `per_group`
// (value, index) pairs, list g at cand + g * ld_group + r * ld_row.  One warp
// per row selects the top K pairs under the same total order, keyed by each
// pair's own index (distinct within a row); an index < 0 marks an empty
// entry.  Chunks of 32 * kMergeP pairs are merged into a running list.
constexpr int kMergeP = 8;

__global__ void __launch_bounds__(64) topk_merge_kernel(const float *__restrict__ cval,
                                                        const int32_t *__restrict__ cidx, int groups,
                                                        int per_group, int64_t ld_row, int64_t ld_group, int K,
                                                        int32_t *__restrict__ idx, float *__restrict__ val,
                                                        int64_t ldo) {
    __shared__ __align__(16) uint64_t scratch[2][64];
    const int lane = threadIdx.x & 31;
    // Warp 1 runs the merge on synthetic pairs to warm the instruction cache
    // (as in topk_warp_kernel).
    const bool warm = (threadIdx.x >> 5) != 0;
    const int64_t row = blockIdx.x;
    grid_launch_dependents();
    if (!warm) grid_dependency_wait();
    const int n = groups * per_group;
    auto at = [&](int p) { return (int64_t)(p / per_group) * ld_group + row * ld_row + p % per_group; };
    uint64_t run = 0ull;
    for (int base = 0; base < n; base += 32 * kMergeP) {
        uint64_t keys[kMergeP];
#pragma unroll
        for (int i = 0; i < kMergeP; ++i) {
            const int p = base + lane + 32 * i;
            keys[i] = 0ull;
            if (p < n) {
                const int32_t j = warm ? p : cidx[at(p)];
                if (j >= 0) keys[i] = make_key(warm ? (float)p : cval[at(p)], (uint32_t)j);
            }
        }
        run = warp_topk_merge<kMergeP>(keys, run, K, lane, scratch[warm ? 1 : 0]);
    }
    if (warm) return;
    if (lane < K) {
        const uint32_t j = key_index(run);
        idx[row * ldo + lane] = run ? (int32_t)j : -1;
        if (val) {
            bool exact;
            float v = key_value(run, exact);
            if (run && !exact) {
                // +-0.0 or NaN: the key does not keep the bits; find the pair.
                for (int p = 0; p < n; ++p)
                    if (cidx[at(p)] == (int32_t)j) {
                        v = cval[at(p)];
                        break;
                    }
            }
            val[row * ldo + lane] = run ? v : __int_as_float(0x7FC00000);
        }
    }
}

}  // namespace topk
}  // namespace mr

namespace mr {
namespace topk {

cudaLaunchConfig_t pdl_config(unsigned grid, unsigned block, void *stream, cudaLaunchAttribute *attr) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.stream = static_cast<cudaStream_t>(stream);
    // Safe for any predecessor: the kernels wait for it before reading input.
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

}  // namespace topk
}  // namespace mr

extern "C" mr_status router_topk_ex(const float *logits, int64_t ldl, int32_t m, int32_t n, int32_t topk,
                                    int32_t *idx, float *val, int64_t ldo, int32_t index_base, void *stream) {
    if (!logits || !idx) return MR_ERR_INVALID_ARG;
    if (m < 1 || n < 1 || topk < 1 || topk > n) return MR_ERR_INVALID_ARG;
    if (ldl < n || ldo < topk) return MR_ERR_INVALID_ARG;
    if (index_base < 0 || (int64_t)index_base + n > (int64_t)INT32_MAX) return MR_ERR_INVALID_ARG;
    if (topk > mr::topk::kMaxK) return MR_ERR_UNSUPPORTED;
    if (((uintptr_t)logits & 3u) || ((uintptr_t)idx & 3u) || ((uintptr_t)val & 3u)) return MR_ERR_MISALIGNED;
    const bool one_warp = n <= mr::topk::kWarpRowMax;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = mr::topk::pdl_config((unsigned)m, one_warp ? 64 : mr::topk::kWarps * 32, stream, attr);
    if (one_warp)
        return mr_host::cuda_status(cudaLaunchKernelEx(&cfg, mr::topk::topk_warp_kernel, logits, ldl, (int)n,
                                                       (int)topk, idx, val, ldo, index_base));
    return mr_host::cuda_status(cudaLaunchKernelEx(&cfg, mr::topk::topk_kernel, logits, ldl, (int)n, (int)topk, idx,
                                                   val, ldo, index_base));
}

extern "C" mr_status router_topk(const float *logits, int64_t ldl, int32_t m, int32_t n, int32_t topk,
                                 int32_t *idx, float *val, int64_t ldo, void *stream) {
    return router_topk_ex(logits, ldl, m, n, topk, idx, val, ldo, 0, stream);
}

extern "C" mr_status router_topk_merge(const float *cand_val, const int32_t *cand_idx, int32_t m, int32_t groups,
                                       int32_t per_group, int64_t ld_row, int64_t ld_group, int32_t topk,
                                       int32_t *idx, float *val, int64_t ldo, void *stream) {
    if (!cand_val || !cand_idx || !idx) return MR_ERR_INVALID_ARG;
    if (m < 1 || groups < 1 || per_group < 1 || topk < 1 || ldo < topk) return MR_ERR_INVALID_ARG;
    if (ld_row < 0 || ld_group < 0) return MR_ERR_INVALID_ARG;
    if ((int64_t)groups * per_group > mr::topk::kMaxMergeCandidates) return MR_ERR_UNSUPPORTED;
    if (topk > mr::topk::kMaxK) return MR_ERR_UNSUPPORTED;
    if (((uintptr_t)cand_val & 3u) || ((uintptr_t)cand_idx & 3u) || ((uintptr_t)idx & 3u) || ((uintptr_t)val & 3u))
        return MR_ERR_MISALIGNED;
    cudaLaunchAttribute attr[1];
    cudaLaunchConfig_t cfg = mr::topk::pdl_config((unsigned)m, 64, stream, attr);
    return mr_host::cuda_status(cudaLaunchKernelEx(&cfg, mr::topk::topk_merge_kernel, cand_val, cand_idx, (int)groups,
                                                   (int)per_group, ld_row, ld_group, (int)topk, idx, val, ldo));
}
