// fold.cu -- query and key of different widths: the K up-projection moved onto the query.
//
// Section 3.4 Step 4 of "Sigma: Differential Rescaling of Query, Key and Value
// for Efficient Language Models" (structured summary page, the Attend
// function): when the query head width d_q differs from the K head width d_k,
// every cached K row is first brought to width d_q by a feed-forward layer and
// then dotted with the query.  For a linear layer without bias, k_up = W k
// (W [d_q, d_k]), and <q, W k> = <W^T q, k>: folding W into the query gives a
// d_k-wide query for the ordinary decode and prefill kernels, and no K row is
// ever projected.  This file holds that fold and its C entry point
// (diffqkv_fold_query, declared in include/diffqkv.h).
//
// Design: the fold is a small batched matrix-vector product (rows x d_q x d_k,
// each K head's W read from L2 by the CTAs of its groups), memory/launch bound
// at decode sizes, so it runs on the CUDA cores: one CTA per (row batch b,
// K head g) covers the n_q/n_k query rows of the group.  Lane l of a warp owns
// d_k/32 adjacent output columns, so a warp reads one W row (128 or 256 bytes)
// per step; the 16 warps split the d_q sum into slices that are added in a
// fixed order, so the result does not depend on timing, and each warp keeps
// four steps of loads in flight (the kernel is load-latency bound).  Accumulation is fp32; the
// folded query is rounded to bf16 (round to nearest even), the type of every
// query the attention entry points take.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "../../include/diffqkv.h"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr int kFoldThreads = 512;
constexpr int kFoldWarps = kFoldThreads / 32;

template <int DK>
__global__ void __launch_bounds__(kFoldThreads)
    fold_query_kernel(const __nv_bfloat16 *__restrict__ q_aug, const __nv_bfloat16 *__restrict__ w_up,
                      __nv_bfloat16 *__restrict__ q_out, int n_q, int n_k, int d_q, int w_heads) {
    constexpr int V = DK / 32;  // output columns per lane
    __shared__ float part[kFoldWarps * DK];  // [slice][row of the round][DK]: slices x rows <= warps

    const int qpk = n_q / n_k;
    const int b = blockIdx.x / n_k;
    const int g = blockIdx.x % n_k;
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const __nv_bfloat16 *W = w_up + (size_t)(w_heads == 1 ? 0 : g) * d_q * DK;
    // slices of the d_q sum: warps beyond the group's rows share rows by slicing r
    const int slices = qpk >= kFoldWarps ? 1 : kFoldWarps / qpk;
    const int slice_len = ((d_q + slices - 1) / slices + 7) / 8 * 8;

    // rows are handled in rounds of (kFoldWarps / slices) rows; partials of one round live in part[].
    // When slices does not divide kFoldWarps (n_q / n_k = 3, 5, ...), the last
    // kFoldWarps - slices * rows_per_round warps get no (row, slice) pair: they
    // neither compute nor write part[], whose slots all belong to other warps.
    const int rows_per_round = kFoldWarps / slices;
    const bool has_slot = warp < slices * rows_per_round;
    for (int row0 = 0; row0 < qpk; row0 += rows_per_round) {
        const int j = row0 + warp / slices;  // query row of the group
        const int s = warp % slices;
        float acc[V];
#pragma unroll
        for (int v = 0; v < V; ++v) acc[v] = 0.f;
        if (has_slot && j < qpk) {
            const __nv_bfloat16 *qr = q_aug + ((size_t)b * n_q + g * qpk + j) * d_q;
            const int r0 = s * slice_len;
            const int r1 = min(d_q, r0 + slice_len);
#pragma unroll 4
            for (int r = r0; r < r1; r += 8) {  // d_q and r0 are multiples of 8
                const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(qr + r));
                const __nv_bfloat16 *qe = reinterpret_cast<const __nv_bfloat16 *>(&qv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float qf = __bfloat162float(qe[e]);
                    const __nv_bfloat16 *wr = W + (size_t)(r + e) * DK + lane * V;
                    if constexpr (V == 2) {
                        const __nv_bfloat162 w2 = __ldg(reinterpret_cast<const __nv_bfloat162 *>(wr));
                        acc[0] = fmaf(qf, __low2float(w2), acc[0]);
                        acc[1] = fmaf(qf, __high2float(w2), acc[1]);
                    } else {
                        const uint2 w4 = __ldg(reinterpret_cast<const uint2 *>(wr));
                        const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162 *>(&w4.x);
                        const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162 *>(&w4.y);
                        acc[0] = fmaf(qf, __low2float(lo), acc[0]);
                        acc[1] = fmaf(qf, __high2float(lo), acc[1]);
                        acc[2] = fmaf(qf, __low2float(hi), acc[2]);
                        acc[3] = fmaf(qf, __high2float(hi), acc[3]);
                    }
                }
            }
        }
        // partial of (slice s, row warp / slices) -> part; then sum the slices in order
        if (has_slot) {
            float *dst = part + ((size_t)s * rows_per_round + warp / slices) * DK + lane * V;
#pragma unroll
            for (int v = 0; v < V; ++v) dst[v] = acc[v];
        }
        __syncthreads();
        for (int t = threadIdx.x; t < rows_per_round * DK; t += kFoldThreads) {
            const int jj = row0 + t / DK;
            if (jj >= qpk) continue;
            float sum = 0.f;
            for (int ss = 0; ss < slices; ++ss) sum += part[((size_t)ss * rows_per_round + t / DK) * DK + t % DK];
            q_out[((size_t)b * n_q + g * qpk + jj) * DK + t % DK] = __float2bfloat16_rn(sum);
        }
        __syncthreads();
    }
}

diffqkv_status_t fold_query_launch(const diffqkv_dims_t *d, int32_t d_q, int32_t w_heads, const void *q_aug,
                                   const void *w_up, void *q_out, cudaStream_t stream) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q_aug || !w_up || !q_out || d_q < 8 || d_q % 8 != 0 || !(w_heads == 1 || w_heads == d->n_k))
        return DIFFQKV_ERR_INVALID_ARG;
    if (d->d_k != 64 && d->d_k != 128) return DIFFQKV_ERR_UNSUPPORTED;
    if (!aligned16(q_aug) || !aligned16(w_up) || !aligned16(q_out)) return DIFFQKV_ERR_MISALIGNED;
    const long long ctas = (long long)d->batch * d->n_k;
    if (ctas > 0x7fffffffLL) return DIFFQKV_ERR_UNSUPPORTED;
    const auto *qa = static_cast<const __nv_bfloat16 *>(q_aug);
    const auto *w = static_cast<const __nv_bfloat16 *>(w_up);
    auto *qo = static_cast<__nv_bfloat16 *>(q_out);
    if (d->d_k == 64)
        fold_query_kernel<64><<<(unsigned)ctas, kFoldThreads, 0, stream>>>(qa, w, qo, d->n_q, d->n_k, d_q, w_heads);
    else
        fold_query_kernel<128><<<(unsigned)ctas, kFoldThreads, 0, stream>>>(qa, w, qo, d->n_q, d->n_k, d_q, w_heads);
    return cudaGetLastError() == cudaSuccess ? DIFFQKV_OK : DIFFQKV_ERR_CUDA;
}

}  // namespace

}  // namespace diffqkv

extern "C" diffqkv_status_t diffqkv_fold_query(const diffqkv_dims_t *dims, int32_t d_q, int32_t w_heads,
                                               const void *q_aug, const void *w_up, void *q_out,
                                               diffqkv_stream_t stream) {
    diffqkv::ApiRange nvtx_range("diffqkv_fold_query");
    return diffqkv::fold_query_launch(dims, d_q, w_heads, q_aug, w_up, q_out, (cudaStream_t)stream);
}
