// augq.cu -- augmented query projection for sm_100a: two persistent tcgen05 GEMMs.
//
// "Sigma" structured summary page, section 3.2 "Big-Picture Architecture", item 4:
// the query comes from a gated projection, q = q_down( SiLU(q_gate(x)) * q_up(x) ),
// whose extra parameters are never cached (section 2, Observation 3).  Two launches:
//   1. h = SiLU(x W_gate^T) * (x W_up^T).  A tile is 128 tokens x 128 intermediate
//      features.  The B operand of a K step stacks the tile's 128 rows of W_gate on
//      its 128 rows of W_up, so one M128 x N256 MMA chain accumulates both branches
//      side by side in TMEM, and the epilogue writes bf16(SiLU(gate) * up).
//   2. q = h W_down^T, tiles of 128 tokens x 256 outputs, plain epilogue.
// Weights are [out features][in features] (the linear-layer layout), so both
// operands are K-major and arrive by TMA with the 128-byte swizzle.  One CTA per
// SM walks the tiles (n fastest, so the CTAs in flight share x rows and the weights
// stay in L2); two TMEM accumulators let the epilogue of one tile overlap the MMAs
// of the next.  Every wait is bounded (DIFFQKV_ERR_DEVICE_TIMEOUT).
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr int BM = 128;               // tokens per tile (TMEM lanes)
constexpr int BK = 64;                // reduction elements per stage: one 128-byte swizzle row
constexpr int kMmaN = 256;            // MMA N: gate | up, or 256 outputs
constexpr int kStages = 4;
constexpr int kEpiWarps = 4;          // warps 0-3: thread = TMEM lane = token row of the tile
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;
constexpr int kTmemCols = 2 * kMmaN;  // two accumulators
constexpr int A_BYTES = BM * BK * 2;          // 16 KB
constexpr int B_BYTES = kMmaN * BK * 2;       // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kBarBytes = 1024;
constexpr int kSmemBytes = 1024 + kStages * STAGE_BYTES + kBarBytes;  // alignment slack, ring, barriers

struct GemmArgs {
    __nv_bfloat16 *out;  // [M][ldo]
    int M;               // rows (tokens)
    int n_out;           // valid output columns
    int K;               // reduction length (multiple of BK)
    int ldo;             // output row stride (elements)
    int tiles_n;         // output tiles per row block
    int tiles;           // all tiles
    int32_t *status;
    uint64_t wait_limit_ns;
};

// SiLU(g) * u in fp32 (2^x on the SFU; exp(-g) overflowing to +inf gives -0 for very negative g).
__device__ __forceinline__ float swiglu(float g, float u) {
    return __fdividef(g, 1.0f + fast_exp2(-g * 1.4426950408889634f)) * u;
}

template <bool kSwiGLU>
__global__ void __launch_bounds__(kThreads, 1)
    augq_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b0,
                     const __grid_constant__ CUtensorMap tm_b1, const GemmArgs a) {
    constexpr int BN_OUT = kSwiGLU ? kMmaN / 2 : kMmaN;  // output columns per tile
    extern __shared__ uint8_t dsm_raw[];
    uint8_t *const smem = align_smem_1024(dsm_raw);
    uint64_t *const full_bar = reinterpret_cast<uint64_t *>(smem + kStages * STAGE_BYTES);
    uint64_t *const empty_bar = full_bar + kStages;
    uint64_t *const acc_full = empty_bar + kStages;
    uint64_t *const acc_empty = acc_full + 2;
    uint64_t *const mma_done = acc_empty + 2;
    uint32_t *const tmem_slot = reinterpret_cast<uint32_t *>(mma_done + 1);
    volatile int *const abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int k_steps = a.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(&acc_full[s], 1);
            mbar_init(&acc_empty[s], kEpiWarps);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ======================= TMA producer
        if (lane == 0) {
            prefetch_tensormap(&tm_a);
            prefetch_tensormap(&tm_b0);
            if (kSwiGLU) prefetch_tensormap(&tm_b1);
            int st = 0;
            uint32_t par = 0;
            long long fills = 0;
            for (int tile = blockIdx.x; tile < a.tiles && !*abort_flag; tile += gridDim.x) {
                const int m0 = (tile / a.tiles_n) * BM, n0 = (tile % a.tiles_n) * BN_OUT;
                for (int kb = 0; kb < k_steps; ++kb) {
                    if (fills >= kStages &&
                        !mbar_wait_bounded(&empty_bar[st], par ^ 1u, a.wait_limit_ns, abort_flag, a.status))
                        break;
                    uint8_t *sa = smem + st * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full_bar[st], STAGE_BYTES);
                    tma_load_4d(sa, &tm_a, &full_bar[st], kb * BK, m0, 0, 0);
                    if (kSwiGLU) {
                        tma_load_4d(sb, &tm_b0, &full_bar[st], kb * BK, n0, 0, 0);
                        tma_load_4d(sb + B_BYTES / 2, &tm_b1, &full_bar[st], kb * BK, n0, 0, 0);
                    } else {
                        tma_load_4d(sb, &tm_b0, &full_bar[st], kb * BK, n0, 0, 0);
                    }
                    ++fills;
                    if (++st == kStages) {
                        st = 0;
                        par ^= 1u;
                    }
                }
            }
            // drain: no copy may still be landing when the CTA exits
            for (long long f = (fills > kStages ? fills - kStages : 0); f < fills; ++f)
                mbar_wait_bounded(&full_bar[f % kStages], (uint32_t)((f / kStages) & 1), a.wait_limit_ns, nullptr,
                                  a.status);
        }
    } else if (warp == kMmaWarp) {
        // ======================= MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, kMmaN, false, false);
            int st = 0;
            uint32_t par = 0;
            int lt = 0;  // tiles of this CTA so far
            for (int tile = blockIdx.x; tile < a.tiles && !*abort_flag; tile += gridDim.x, ++lt) {
                const int ab = lt & 1;
                // the accumulator's previous tile (lt - 2) has been read out
                if (lt >= 2 && !mbar_wait_bounded(&acc_empty[ab], (uint32_t)(((lt >> 1) & 1) ^ 1), a.wait_limit_ns,
                                                  abort_flag, a.status))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(ab * kMmaN);
                for (int kb = 0; kb < k_steps; ++kb) {
                    if (!mbar_wait_bounded(&full_bar[st], par, a.wait_limit_ns, abort_flag, a.status)) break;
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + st * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int ks = 0; ks < BK / 16; ++ks) {
                        const uint64_t da = smem_desc_sw128(sa + (uint32_t)ks * 32u, 16, 1024);
                        const uint64_t db = smem_desc_sw128(sb + (uint32_t)ks * 32u, 16, 1024);
                        umma_bf16(d_tmem, da, db, idesc, (kb > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty_bar[st]);
                    if (++st == kStages) {
                        st = 0;
                        par ^= 1u;
                    }
                }
                umma_commit(&acc_full[ab]);
            }
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0, a.wait_limit_ns, nullptr, a.status);
        }
    } else {
        // ======================= epilogue warps 0-3: thread = token row 32 warp + lane of the tile
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        int lt = 0;
        for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x, ++lt) {
            const int ab = lt & 1;
            if (!mbar_wait_bounded(&acc_full[ab], (uint32_t)((lt >> 1) & 1), a.wait_limit_ns, abort_flag, a.status))
                break;
            tc_fence_after();
            const int row = (tile / a.tiles_n) * BM + warp * 32 + lane;
            const int n0 = (tile % a.tiles_n) * BN_OUT;
            const uint32_t t_acc = tmem + lane_base + (uint32_t)(ab * kMmaN);
            __nv_bfloat16 *orow = a.out + (size_t)row * a.ldo + n0;
#pragma unroll 1
            for (int c0 = 0; c0 < BN_OUT; c0 += 32) {
                uint32_t r0[32];
                uint32_t o[16];
                if constexpr (kSwiGLU) {
                    uint32_t r1[32];
                    tmem_ld32(t_acc + (uint32_t)c0, r0);                 // gate
                    tmem_ld32(t_acc + (uint32_t)(kMmaN / 2 + c0), r1);   // up
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = pack_bf16x2(swiglu(__uint_as_float(r0[2 * i]), __uint_as_float(r1[2 * i])),
                                           swiglu(__uint_as_float(r0[2 * i + 1]), __uint_as_float(r1[2 * i + 1])));
                } else {
                    tmem_ld32(t_acc + (uint32_t)c0, r0);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        o[i] = pack_bf16x2(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
                }
                if (row < a.M && n0 + c0 < a.n_out &&
                    in_bounds((long long)row * a.ldo + n0 + c0 + 31, (long long)a.M * a.ldo, a.status)) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c0);
#pragma unroll
                    for (int v = 0; v < 4; ++v) dst[v] = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[ab]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

diffqkv_status_t launch_gemm(bool swiglu, const CUtensorMap &ta, const CUtensorMap &tb0, const CUtensorMap &tb1,
                             const GemmArgs &args, int num_sms, cudaStream_t stream) {
    if (args.tiles == 0) return DIFFQKV_OK;
    const void *fn = swiglu ? reinterpret_cast<const void *>(&augq_gemm_kernel<true>)
                            : reinterpret_cast<const void *>(&augq_gemm_kernel<false>);
    diffqkv_status_t st = ensure_dynamic_smem(fn, kSmemBytes);
    if (st != DIFFQKV_OK) return st;
    const int grid = std::min(args.tiles, num_sms);
    if (swiglu)
        augq_gemm_kernel<true><<<grid, kThreads, kSmemBytes, stream>>>(ta, tb0, tb1, args);
    else
        augq_gemm_kernel<false><<<grid, kThreads, kSmemBytes, stream>>>(ta, tb0, tb1, args);
    return cudaGetLastError() == cudaSuccess ? DIFFQKV_OK : DIFFQKV_ERR_CUDA;
}

}  // namespace

diffqkv_status_t augq_launch(const void *x, const void *w_gate, const void *w_up, const void *w_down, int32_t tokens,
                             int32_t d_model, int32_t d_inter, int32_t d_out, void *h_out, void *q_out,
                             int32_t *status, cudaStream_t stream) {
    // x, h_out and q_out may be null when there are no tokens (an empty tensor has no storage)
    if (!w_gate || !w_up || !w_down || (tokens > 0 && (!x || !h_out || !q_out))) return DIFFQKV_ERR_INVALID_ARG;
    if (tokens < 0 || d_model < BK || d_inter < kMmaN / 2 || d_out < 32) return DIFFQKV_ERR_INVALID_ARG;
    if (d_model % BK || d_inter % (kMmaN / 2) || d_out % 32) return DIFFQKV_ERR_UNSUPPORTED;
    if (!aligned16(x) || !aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down) || !aligned16(h_out) ||
        !aligned16(q_out) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    if ((int64_t)tokens * std::max({d_model, d_inter, d_out}) >= (int64_t)1 << 31 ||
        (int64_t)d_inter * d_model >= (int64_t)1 << 31 || (int64_t)d_out * d_inter >= (int64_t)1 << 31)
        return DIFFQKV_ERR_UNSUPPORTED;
    if (tokens == 0) return DIFFQKV_OK;
    DeviceInfo dev;
    diffqkv_status_t st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    int32_t *const word = status ? status : dev.status_word;  // the caller's word, else the device's

    CUtensorMap t_x, t_wg, t_wu, t_h, t_wd;
    st = make_tensor_map_4d(&t_x, x, d_model, tokens, 1, 1, BK, BM, 1, 1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == DIFFQKV_OK)
        st = make_tensor_map_4d(&t_wg, w_gate, d_model, d_inter, 1, 1, BK, kMmaN / 2, 1, 1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == DIFFQKV_OK)
        st = make_tensor_map_4d(&t_wu, w_up, d_model, d_inter, 1, 1, BK, kMmaN / 2, 1, 1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == DIFFQKV_OK)
        st = make_tensor_map_4d(&t_h, h_out, d_inter, tokens, 1, 1, BK, BM, 1, 1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st == DIFFQKV_OK)
        st = make_tensor_map_4d(&t_wd, w_down, d_inter, d_out, 1, 1, BK, kMmaN, 1, 1, CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DIFFQKV_OK) return st;

    const int tiles_m = (tokens + BM - 1) / BM;
    GemmArgs g1;
    g1.out = static_cast<__nv_bfloat16 *>(h_out);
    g1.M = tokens;
    g1.n_out = d_inter;
    g1.K = d_model;
    g1.ldo = d_inter;
    g1.tiles_n = d_inter / (kMmaN / 2);
    g1.tiles = tiles_m * g1.tiles_n;
    g1.status = word;
    g1.wait_limit_ns = kWaitLimitNs;
    st = launch_gemm(true, t_x, t_wg, t_wu, g1, dev.num_sms, stream);
    if (st != DIFFQKV_OK) return st;
    GemmArgs g2 = g1;
    g2.out = static_cast<__nv_bfloat16 *>(q_out);
    g2.n_out = d_out;
    g2.K = d_inter;
    g2.ldo = d_out;
    g2.tiles_n = (d_out + kMmaN - 1) / kMmaN;
    g2.tiles = tiles_m * g2.tiles_n;
    return launch_gemm(false, t_h, t_wd, t_wd, g2, dev.num_sms, stream);
}

}  // namespace diffqkv
