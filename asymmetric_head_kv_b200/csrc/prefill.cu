// prefill.cu -- causal prefill (placeholder until the kernels land).
#include "common.cuh"
#include "internal.h"

namespace diffqkv {
diffqkv_status_t prefill_launch(const diffqkv_dims_t *, const void *, const void *, const void *, int32_t, void *,
                                cudaStream_t) {
    return DIFFQKV_ERR_UNSUPPORTED;
}
}  // namespace diffqkv
