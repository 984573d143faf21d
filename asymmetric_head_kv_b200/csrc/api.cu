// api.cu -- the C ABI of libdiffqkv.so (declared in include/diffqkv.h).
//
// Argument checking, device bookkeeping and TMA descriptor encoding.  All
// arithmetic of the attention path lives in the kernels (decode.cu,
// topv.cu, prefill.cu).
#include <cudaTypedefs.h>
#include <math.h>
#include <nvtx3/nvToolsExt.h>
#include <stdio.h>
#include <stdlib.h>

#include <mutex>

#include "common.cuh"
#include "internal.h"

// The per-device error word: first device-side error since the last read.
__device__ int32_t g_diffqkv_status_word[4];

namespace diffqkv {

namespace {

constexpr int kMaxDevices = 64;
DeviceInfo g_devices[kMaxDevices];
std::mutex g_dev_mutex;

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

__global__ void wait_timeout_selftest_kernel(int32_t *status, uint64_t limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        mbar_init(&bar, 1);  // one arrival expected; nothing ever arrives
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, limit_ns, &abort_flag, status);
    __syncthreads();
}

}  // namespace

diffqkv_status_t current_device_info(DeviceInfo *info) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
        cudaGetLastError();
        return DIFFQKV_ERR_NO_DEVICE;
    }
    if (dev >= kMaxDevices) return DIFFQKV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_dev_mutex);
    DeviceInfo &d = g_devices[dev];
    if (d.device != dev) {
        DeviceInfo n;
        n.device = dev;
        int major = 0;
        if (cudaDeviceGetAttribute(&n.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) {
            cudaGetLastError();
            return DIFFQKV_ERR_CUDA;
        }
        if (major != 10) return DIFFQKV_ERR_UNSUPPORTED;
        void *addr = nullptr;
        if (cudaGetSymbolAddress(&addr, g_diffqkv_status_word) != cudaSuccess) {
            cudaGetLastError();
            return DIFFQKV_ERR_CUDA;
        }
        n.status_word = static_cast<int32_t *>(addr);
        d = n;
    }
    *info = d;
    return DIFFQKV_OK;
}

diffqkv_status_t make_tensor_map_4d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1,
                                    uint64_t dim2, uint64_t dim3, uint32_t box0, uint32_t box1, uint32_t box2,
                                    uint32_t box3, CUtensorMapSwizzle swizzle, CUtensorMapL2promotion promotion) {
    auto fn = encode_fn();
    if (!fn) return DIFFQKV_ERR_CUDA;
    const cuuint64_t dims[4] = {dim0, dim1, dim2, dim3};
    const cuuint64_t strides[3] = {dim0 * 2, dim0 * dim1 * 2, dim0 * dim1 * dim2 * 2};
    const cuuint32_t box[4] = {box0, box1, box2, box3};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, promotion, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DIFFQKV_OK : DIFFQKV_ERR_INVALID_ARG;
}

diffqkv_status_t make_tensor_map_4d_strided(CUtensorMap *map, const void *base, const uint64_t dims[4],
                                            const uint64_t strides_bytes[3], const uint32_t box[4],
                                            CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return DIFFQKV_ERR_CUDA;
    const cuuint64_t d[4] = {dims[0], dims[1], dims[2], dims[3]};
    const cuuint64_t st[3] = {strides_bytes[0], strides_bytes[1], strides_bytes[2]};
    const cuuint32_t bx[4] = {box[0], box[1], box[2], box[3]};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), d, st, bx, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DIFFQKV_OK : DIFFQKV_ERR_INVALID_ARG;
}

diffqkv_status_t make_tensor_map_3d(CUtensorMap *map, const void *base, uint64_t dim0, uint64_t dim1,
                                    uint64_t dim2, uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0,
                                    uint32_t box1, uint32_t box2, CUtensorMapSwizzle swizzle) {
    auto fn = encode_fn();
    if (!fn) return DIFFQKV_ERR_CUDA;
    const cuuint64_t dims[3] = {dim0, dim1, dim2};
    const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
    const cuuint32_t box[3] = {box0, box1, box2};
    const cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? DIFFQKV_OK : DIFFQKV_ERR_INVALID_ARG;
}

diffqkv_status_t ensure_dynamic_smem(const void *kernel, int bytes) {
    // cudaFuncSetAttribute costs host time on every call; remember what each
    // (kernel, device) pair has already been given
    struct Entry {
        const void *fn;
        int device;
        int bytes;
    };
    static Entry cache[256];
    static int used = 0;
    static std::mutex m;
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_NO_DEVICE;
    }
    std::lock_guard<std::mutex> lock(m);
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == kernel && cache[i].device == dev && cache[i].bytes >= bytes) return DIFFQKV_OK;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    for (int i = 0; i < used; ++i)
        if (cache[i].fn == kernel && cache[i].device == dev) {
            cache[i].bytes = bytes;
            return DIFFQKV_OK;
        }
    if (used < 256) cache[used++] = Entry{kernel, dev, bytes};
    return DIFFQKV_OK;
}

diffqkv_status_t validate_dims(const diffqkv_dims_t *d) {
    if (!d) return DIFFQKV_ERR_INVALID_ARG;
    if (d->batch < 1 || d->n_q < 1 || d->n_k < 1 || d->n_v < 1 || d->d_k < 1 || d->d_v < 1)
        return DIFFQKV_ERR_INVALID_ARG;
    if (d->n_q % d->n_k != 0 || d->n_q % d->n_v != 0) return DIFFQKV_ERR_INVALID_ARG;
    if (!(d->scale > 0.f) || !isfinite(d->scale)) return DIFFQKV_ERR_INVALID_ARG;
    if (d->d_k % 8 != 0 || d->d_v % 8 != 0) return DIFFQKV_ERR_UNSUPPORTED;
    return DIFFQKV_OK;
}

bool nvtx_enabled() {
    static const bool on = [] {
        const char *e = getenv("DIFFQKV_NVTX");
        return e != nullptr && e[0] != '\0' && !(e[0] == '0' && e[1] == '\0');
    }();
    return on;
}
void nvtx_push(const char *name) { nvtxRangePushA(name); }
void nvtx_pop() { nvtxRangePop(); }

diffqkv_status_t wait_timeout_selftest_launch(int64_t timeout_ns, cudaStream_t stream) {
    if (timeout_ns < 1000 || timeout_ns > 5000000000LL) return DIFFQKV_ERR_INVALID_ARG;
    DeviceInfo dev;
    diffqkv_status_t st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(dev.status_word, (uint64_t)timeout_ns);
    return cudaGetLastError() == cudaSuccess ? DIFFQKV_OK : DIFFQKV_ERR_CUDA;
}

}  // namespace diffqkv

// ====================================================================== C ABI
extern "C" {

const char *diffqkv_status_string(int32_t status) {
    switch (status) {
        case DIFFQKV_OK: return "DIFFQKV_OK";
        case DIFFQKV_ERR_INVALID_ARG: return "DIFFQKV_ERR_INVALID_ARG";
        case DIFFQKV_ERR_UNSUPPORTED: return "DIFFQKV_ERR_UNSUPPORTED";
        case DIFFQKV_ERR_MISALIGNED: return "DIFFQKV_ERR_MISALIGNED";
        case DIFFQKV_ERR_WORKSPACE: return "DIFFQKV_ERR_WORKSPACE";
        case DIFFQKV_ERR_CUDA: return "DIFFQKV_ERR_CUDA";
        case DIFFQKV_ERR_DEVICE_TIMEOUT: return "DIFFQKV_ERR_DEVICE_TIMEOUT";
        case DIFFQKV_ERR_DEVICE_SEQLEN: return "DIFFQKV_ERR_DEVICE_SEQLEN";
        case DIFFQKV_ERR_NO_DEVICE: return "DIFFQKV_ERR_NO_DEVICE";
        case DIFFQKV_ERR_SCRATCH_LIMIT: return "DIFFQKV_ERR_SCRATCH_LIMIT";
        case DIFFQKV_ERR_DEVICE_PAGE: return "DIFFQKV_ERR_DEVICE_PAGE";
        case DIFFQKV_ERR_DEVICE_BOUNDS: return "DIFFQKV_ERR_DEVICE_BOUNDS";
        default: return "DIFFQKV_ERR_UNKNOWN";
    }
}

int32_t diffqkv_version(void) { return 10200; }

size_t diffqkv_decode_workspace_size(const diffqkv_dims_t *dims) { return diffqkv::decode_workspace_size(dims); }

diffqkv_status_t diffqkv_workspace_init(void *workspace, size_t workspace_bytes, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_workspace_init");
    if (!workspace || workspace_bytes == 0) return DIFFQKV_ERR_INVALID_ARG;
    if (cudaMemsetAsync(workspace, 0, workspace_bytes, (cudaStream_t)stream) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    return DIFFQKV_OK;
}

diffqkv_status_t diffqkv_decode(const diffqkv_dims_t *dims, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, void *out,
                                void *workspace, size_t workspace_bytes, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode");
    return diffqkv::decode_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, out, workspace,
                                  workspace_bytes, nullptr, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_decode_append(const diffqkv_dims_t *dims, const void *q, const void *k_new,
                                       const void *v_new, void *k_cache, void *v_cache,
                                       const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len,
                                       void *out, void *workspace, size_t workspace_bytes,
                                       diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_append");
    if (!k_new || !v_new) return DIFFQKV_ERR_INVALID_ARG;
    return diffqkv::decode_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, out, workspace,
                                  workspace_bytes, nullptr, (cudaStream_t)stream, k_new, v_new);
}

diffqkv_status_t diffqkv_decode_paged(const diffqkv_dims_t *dims, const void *q, const void *k_new,
                                      const void *v_new, void *k_pages, void *v_pages,
                                      const int32_t *block_table, int32_t max_blocks, int32_t page_size,
                                      int32_t num_pages, const int32_t *seq_lens, int32_t max_seq_len,
                                      void *out, void *workspace, size_t workspace_bytes,
                                      diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_paged");
    if ((k_new == nullptr) != (v_new == nullptr)) return DIFFQKV_ERR_INVALID_ARG;
    if (max_blocks < 1 || page_size < 1 || (long long)max_blocks * page_size > 0x7fffffffLL)
        return DIFFQKV_ERR_INVALID_ARG;
    const diffqkv::PagedCache paged{block_table, max_blocks, page_size, num_pages};
    return diffqkv::decode_launch(dims, q, k_pages, v_pages, seq_lens, max_blocks * page_size, max_seq_len, out,
                                  workspace, workspace_bytes, nullptr, (cudaStream_t)stream, k_new, v_new, &paged);
}

diffqkv_status_t diffqkv_decode_ex(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                   const void *v_cache, const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len,
                                   void *out, void *workspace, size_t workspace_bytes,
                                   const diffqkv_decode_tuning_t *tuning, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_ex");
    return diffqkv::decode_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, out, workspace,
                                  workspace_bytes, tuning, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_decode_plan(const diffqkv_dims_t *dims, int32_t t_max, int32_t max_seq_len,
                                     int32_t num_sms, const diffqkv_decode_tuning_t *tuning,
                                     diffqkv_decode_plan_t *plan) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_plan");
    return diffqkv::decode_plan(dims, t_max, max_seq_len, num_sms, tuning, plan);
}

diffqkv_status_t diffqkv_decode_from_host(const diffqkv_dims_t *dims, const void *q_host, const void *k_cache_host,
                                          const void *v_cache_host, const int32_t *seq_lens_host, int32_t t_max,
                                          int32_t max_seq_len, void *out_host, void *q_dev, void *k_cache_dev,
                                          void *v_cache_dev, int32_t *seq_lens_dev, void *out_dev,
                                          void *workspace, size_t workspace_bytes, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_from_host");
    return diffqkv::decode_from_host_launch(dims, q_host, k_cache_host, v_cache_host, seq_lens_host, t_max,
                                            max_seq_len, out_host, q_dev, k_cache_dev, v_cache_dev, seq_lens_dev,
                                            out_dev, workspace, workspace_bytes, (cudaStream_t)stream);
}

size_t diffqkv_decode_topv_workspace_size(const diffqkv_dims_t *dims, int32_t t_max, int32_t topk) {
    return diffqkv::topv_workspace_size(dims, t_max, topk);
}

diffqkv_status_t diffqkv_decode_topv(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                     const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                     int32_t max_seq_len, int32_t topk, void *out, int32_t *idx_out,
                                     void *workspace, size_t workspace_bytes, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_topv");
    return diffqkv::topv_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, topk, out, idx_out,
                                workspace, workspace_bytes, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_decode_topv_ex(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                        int32_t max_seq_len, int32_t topk, int32_t flags, void *out,
                                        int32_t *idx_out, void *workspace, size_t workspace_bytes,
                                        diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_topv_ex");
    return diffqkv::topv_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, topk, out, idx_out,
                                workspace, workspace_bytes, (cudaStream_t)stream, flags);
}

diffqkv_status_t diffqkv_decode_topv_paged(const diffqkv_dims_t *dims, const void *q, const void *k_pages,
                                           const void *v_pages, const int32_t *block_table, int32_t max_blocks,
                                           int32_t page_size, int32_t num_pages, const int32_t *seq_lens,
                                           int32_t max_seq_len, int32_t topk, int32_t flags, void *out,
                                           int32_t *idx_out, void *workspace, size_t workspace_bytes,
                                           diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_topv_paged");
    if (max_blocks < 1 || page_size < 1 || (long long)max_blocks * page_size > 0x7fffffffLL)
        return DIFFQKV_ERR_INVALID_ARG;
    const diffqkv::PagedCache paged{block_table, max_blocks, page_size, num_pages};
    return diffqkv::topv_launch(dims, q, k_pages, v_pages, seq_lens, max_blocks * page_size, max_seq_len, topk, out,
                                idx_out, workspace, workspace_bytes, (cudaStream_t)stream, flags, &paged);
}

diffqkv_status_t diffqkv_prefill_causal(const diffqkv_dims_t *dims, const void *q, const void *k, const void *v,
                                        int32_t seq_len, void *out, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_prefill_causal");
    return diffqkv::prefill_launch(dims, q, k, v, seq_len, out, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_prefill_causal_prefix(const diffqkv_dims_t *dims, const void *q, const void *k,
                                               const void *v, int32_t prefix_len, int32_t seq_len, void *out,
                                               diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_prefill_causal_prefix");
    return diffqkv::prefill_launch(dims, q, k, v, seq_len, out, (cudaStream_t)stream, prefix_len);
}

diffqkv_status_t diffqkv_prefill_causal_ex(const diffqkv_dims_t *dims, const void *q, const void *k,
                                           const void *v, int32_t prefix_len, int32_t seq_len, void *out,
                                           int32_t *device_status_word, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_prefill_causal_ex");
    return diffqkv::prefill_launch(dims, q, k, v, seq_len, out, (cudaStream_t)stream, prefix_len,
                                   device_status_word);
}

diffqkv_status_t diffqkv_prefill_causal_paged(const diffqkv_dims_t *dims, const void *q, const void *k_pages,
                                              const void *v_pages, const int32_t *block_table, int32_t max_blocks,
                                              int32_t page_size, int32_t num_pages, int32_t prefix_len,
                                              int32_t seq_len, void *out, int32_t *device_status_word,
                                              diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_prefill_causal_paged");
    const diffqkv::PagedCache paged{block_table, max_blocks, page_size, num_pages};
    return diffqkv::prefill_launch(dims, q, k_pages, v_pages, seq_len, out, (cudaStream_t)stream, prefix_len,
                                   device_status_word, &paged);
}

diffqkv_status_t diffqkv_augq_project(const void *x, const void *w_gate, const void *w_up, const void *w_down,
                                      int32_t tokens, int32_t d_model, int32_t d_inter, int32_t d_out,
                                      void *h_out, void *q_out, int32_t *device_status_word,
                                      diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_augq_project");
    return diffqkv::augq_launch(x, w_gate, w_up, w_down, tokens, d_model, d_inter, d_out, h_out, q_out,
                                device_status_word, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_workspace_status(void *workspace, size_t workspace_bytes, diffqkv_stream_t stream,
                                          int32_t *device_status) {
    diffqkv::ApiRange nvtx_range("diffqkv_workspace_status");
    if (!device_status || !workspace || workspace_bytes < 256) return DIFFQKV_ERR_INVALID_ARG;
    if (!diffqkv::aligned16(workspace)) return DIFFQKV_ERR_MISALIGNED;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(workspace, 0, sizeof v, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    *device_status = v;
    return DIFFQKV_OK;
}

diffqkv_status_t diffqkv_get_device_status(diffqkv_stream_t stream, int32_t *device_status) {
    diffqkv::ApiRange nvtx_range("diffqkv_get_device_status");
    if (!device_status) return DIFFQKV_ERR_INVALID_ARG;
    diffqkv::DeviceInfo dev;
    diffqkv_status_t st = diffqkv::current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    if (cudaStreamSynchronize(s) != cudaSuccess ||
        cudaMemcpyAsync(&v, dev.status_word, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaMemsetAsync(dev.status_word, 0, sizeof v, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    *device_status = v;
    return DIFFQKV_OK;
}

diffqkv_status_t diffqkv_selftest_wait_timeout(int64_t timeout_ns, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_selftest_wait_timeout");
    return diffqkv::wait_timeout_selftest_launch(timeout_ns, (cudaStream_t)stream);
}

diffqkv_status_t diffqkv_decode_noalloc(const diffqkv_dims_t *dims, const void *q, const void *k_cache,
                                        const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                        int32_t max_seq_len, void *out, diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_decode_noalloc");
    return diffqkv::decode_noalloc_launch(dims, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, out,
                                          (cudaStream_t)stream);
}

}  // extern "C"
