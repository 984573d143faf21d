// internal.h -- host-side helpers shared by the libdiffqkv translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/diffqkv.h"

namespace diffqkv {

// Per-device cached attributes and the device address of the error word.
struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int max_smem_optin = 0;
    int32_t *status_word = nullptr;  // device address of the error word
};

// Fills `info` for the current device.  Returns DIFFQKV_OK or an error.
diffqkv_status_t current_device_info(DeviceInfo *info);

// Encodes a rank-4 tiled tensor map over a bf16 tensor laid out as
// [dim3][dim2][dim1][dim0] (dim0 innermost, contiguous), box {b0,b1,b2,b3}.
// `promotion`: L2 sector promotion of the loads (256 B by default; 128 B when
// the box rows are 128-byte slices whose neighbours belong to other CTAs).
diffqkv_status_t make_tensor_map_4d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1,
                                    uint64_t dim2, uint64_t dim3, uint32_t box0, uint32_t box1,
                                    uint32_t box2, uint32_t box3, CUtensorMapSwizzle swizzle,
                                    CUtensorMapL2promotion promotion = CU_TENSOR_MAP_L2_PROMOTION_L2_256B);

// Rank-4 tiled tensor map with explicit byte strides of dims 1..3 (a view that need not be dense).
diffqkv_status_t make_tensor_map_4d_strided(CUtensorMap *map, const void *base, const uint64_t dims[4],
                                            const uint64_t strides_bytes[3], const uint32_t box[4],
                                            CUtensorMapSwizzle swizzle);

// Encodes a rank-3 tiled tensor map ([dim2][dim1][dim0], dim0 contiguous).
diffqkv_status_t make_tensor_map_3d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1,
                                    uint64_t dim2, uint64_t stride1_bytes, uint64_t stride2_bytes,
                                    uint32_t box0, uint32_t box1, uint32_t box2,
                                    CUtensorMapSwizzle swizzle);

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Sets a kernel's dynamic shared-memory limit once per (kernel, device).
diffqkv_status_t ensure_dynamic_smem(const void *kernel, int bytes);

// Shape checks common to every entry point.
diffqkv_status_t validate_dims(const diffqkv_dims_t *d);

// decode.cu
// A paged K/V cache: pools [num_pages, page_size, heads, d] for K and for V and
// one block table [batch, max_blocks] (device int32) of pool pages.
struct PagedCache {
    const int32_t *block_table;
    int32_t max_blocks, page_size, num_pages;
};

diffqkv_status_t decode_plan(const diffqkv_dims_t *d, int32_t t_max, int32_t max_seq_len, int32_t num_sms,
                             const diffqkv_decode_tuning_t *tuning, diffqkv_decode_plan_t *plan);
size_t decode_workspace_size(const diffqkv_dims_t *d);
// k_new / v_new given (both or neither): append mode, the caches are written at seq_len.
// paged given: k_cache / v_cache are page pools and t_max = max_blocks * page_size.
diffqkv_status_t decode_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache,
                               const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                               int32_t max_seq_len, void *out, void *workspace, size_t workspace_bytes,
                               const diffqkv_decode_tuning_t *tuning, cudaStream_t stream,
                               const void *k_new = nullptr, const void *v_new = nullptr,
                               const PagedCache *paged = nullptr);

// diffqkv_decode_from_host: all checks of the decode run before the first copy is enqueued.
diffqkv_status_t decode_from_host_launch(const diffqkv_dims_t *d, const void *q_host, const void *k_host,
                                         const void *v_host, const int32_t *seq_lens_host, int32_t t_max,
                                         int32_t max_seq_len, void *out_host, void *q_dev, void *k_dev, void *v_dev,
                                         int32_t *seq_lens_dev, void *out_dev, void *workspace,
                                         size_t workspace_bytes, cudaStream_t stream);

diffqkv_status_t decode_noalloc_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                       int32_t max_seq_len, void *out, cudaStream_t stream);

// topv.cu
size_t topv_workspace_size(const diffqkv_dims_t *d, int32_t t_max, int32_t topk);
// paged given: k_cache / v_cache are page pools and t_max = max_blocks * page_size.
diffqkv_status_t topv_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, int32_t topk,
                             void *out, int32_t *idx_out, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream, int32_t flags = 0, const PagedCache *paged = nullptr);

// prefill.cu
// status: device word the kernel reports into (NULL: the per-device word).
// paged given: k / v are page pools [num_pages, page_size, heads, d] and position j of sequence b
// is row j % page_size of pool page block_table[b][j / page_size].
diffqkv_status_t prefill_launch(const diffqkv_dims_t *d, const void *q, const void *k, const void *v,
                                int32_t seq_len, void *out, cudaStream_t stream, int32_t prefix_len = 0,
                                int32_t *status = nullptr, const PagedCache *paged = nullptr);

// augq.cu
// status: device word the kernels report into (NULL: the per-device word).
diffqkv_status_t augq_launch(const void *x, const void *w_gate, const void *w_up, const void *w_down, int32_t tokens,
                             int32_t d_model, int32_t d_inter, int32_t d_out, void *h_out, void *q_out,
                             int32_t *status, cudaStream_t stream);

// api.cu
diffqkv_status_t wait_timeout_selftest_launch(int64_t timeout_ns, cudaStream_t stream);

// An NVTX range around one C-ABI call, named after it, when the environment variable
// DIFFQKV_NVTX is set (read once); otherwise nothing.  Profilers show each call's
// host-side span next to the kernels it launched.
bool nvtx_enabled();
void nvtx_push(const char *name);
void nvtx_pop();
struct ApiRange {
    const bool on;
    explicit ApiRange(const char *name) : on(nvtx_enabled()) {
        if (on) nvtx_push(name);
    }
    ~ApiRange() {
        if (on) nvtx_pop();
    }
    ApiRange(const ApiRange &) = delete;
    ApiRange &operator=(const ApiRange &) = delete;
};

}  // namespace diffqkv
