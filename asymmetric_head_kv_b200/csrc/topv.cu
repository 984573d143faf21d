// topv.cu -- selective-V decode (placeholder until the kernels land).
#include "common.cuh"
#include "internal.h"

namespace diffqkv {
size_t topv_workspace_size(const diffqkv_dims_t *d, int32_t t_max, int32_t topk) {
    (void)d; (void)t_max; (void)topk;
    return 0;
}
diffqkv_status_t topv_launch(const diffqkv_dims_t *, const void *, const void *, const void *, const int32_t *,
                             int32_t, int32_t, int32_t, void *, int32_t *, void *, size_t, cudaStream_t) {
    return DIFFQKV_ERR_UNSUPPORTED;
}
}  // namespace diffqkv
