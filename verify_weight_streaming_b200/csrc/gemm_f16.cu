// gemm_f16: placeholder until the tcgen05 path lands.
#include "common.cuh"

extern "C" int32_t gemm_f16_num_tiles(void) { return 0; }
extern "C" const char *gemm_f16_tile_name(int32_t) { return nullptr; }
extern "C" int32_t gemm_f16_select_tile(int32_t, int32_t, int32_t) { return -1; }
extern "C" mr_status gemm_f16(const void *, int64_t, const void *, int64_t, void *, int64_t, int32_t,
                              int32_t, int32_t, int32_t, int32_t, int32_t, void *) {
    return MR_ERR_UNSUPPORTED;
}
