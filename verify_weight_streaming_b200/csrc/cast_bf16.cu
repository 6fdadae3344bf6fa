// cast_f32_bf16: the bf16 cast of a verify window's rows in one call (Strata
// PR #109, "What": the window's rows are contiguous, so one launch casts them
// all), fp32 -> bf16 round to nearest even with CUDA's conversion intrinsic.
// HBM-bound: 6 bytes per element; each thread converts 8 elements per step
// (two 16-byte loads, one 16-byte store) when rows are 16-byte aligned.
#include "common.cuh"

#include <cuda_bf16.h>

namespace mr {
namespace cast {

__global__ void __launch_bounds__(256) cast_kernel(const float *__restrict__ x, int64_t ldx,
                                                   uint16_t *__restrict__ y, int64_t ldy, int rows, int cols,
                                                   int vec) {
    grid_launch_dependents();
    grid_dependency_wait();
    const int64_t per_row = vec ? cols / 8 : cols;
    const int64_t total = per_row * rows;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / per_row, c = e % per_row;
        if (vec) {
            const float4 a = *reinterpret_cast<const float4 *>(x + r * ldx + 8 * c);
            const float4 b = *reinterpret_cast<const float4 *>(x + r * ldx + 8 * c + 4);
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(a.x, a.y), p1 = __floats2bfloat162_rn(a.z, a.w);
            const __nv_bfloat162 p2 = __floats2bfloat162_rn(b.x, b.y), p3 = __floats2bfloat162_rn(b.z, b.w);
            uint4 o;
            o.x = *reinterpret_cast<const uint32_t *>(&p0);
            o.y = *reinterpret_cast<const uint32_t *>(&p1);
            o.z = *reinterpret_cast<const uint32_t *>(&p2);
            o.w = *reinterpret_cast<const uint32_t *>(&p3);
            *reinterpret_cast<uint4 *>(y + r * ldy + 8 * c) = o;
        } else {
            const __nv_bfloat16 h = __float2bfloat16_rn(x[r * ldx + c]);
            y[r * ldy + c] = *reinterpret_cast<const uint16_t *>(&h);
        }
    }
}

}  // namespace cast
}  // namespace mr

extern "C" mr_status cast_f32_bf16(const float *X, int64_t ldx, void *Y, int64_t ldy, int32_t rows, int32_t cols,
                                   void *stream) {
    if (!X || !Y) return MR_ERR_INVALID_ARG;
    if (rows < 1 || cols < 1 || ldx < cols || ldy < cols) return MR_ERR_INVALID_ARG;
    if (((uintptr_t)X & 3u) || ((uintptr_t)Y & 1u)) return MR_ERR_MISALIGNED;
    const int vec = (cols % 8 == 0) && (ldx % 4 == 0) && (ldy % 8 == 0) && (((uintptr_t)X & 15u) == 0) &&
                    (((uintptr_t)Y & 15u) == 0);
    const int64_t work = (vec ? (int64_t)cols / 8 : cols) * rows;
    const int sms = mr_host::sm_count() > 0 ? mr_host::sm_count() : 148;
    const int64_t blocks = std::min<int64_t>((work + 255) / 256, (int64_t)sms * 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::max<int64_t>(1, blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = static_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return mr_host::cuda_status(cudaLaunchKernelEx(&cfg, mr::cast::cast_kernel, X, ldx,
                                                   static_cast<uint16_t *>(Y), ldy, (int)rows, (int)cols, vec));
}
