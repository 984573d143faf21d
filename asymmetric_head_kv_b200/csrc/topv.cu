// topv.cu -- selective V fetch decode for sm_100a.
//
// "Selective V Cache Fetching" (Sigma paper, structured summary page): after
// the scores are computed from the full (thin) K cache, only the V rows of the
// top-k scoring positions are read; positions outside that set contribute nothing.
// The softmax is renormalised over the kept positions, and the positions are
// ranked by the EXACT dot product q.k (ties toward the lower position) so the
// selected set is unique and reproducible.
//
// Four launches:
//  1. topv_score_kernel -- streams K once with TMA (one K row serves all
//     n_q/n_k query heads of its group; four lanes per position, q in
//     registers) and writes fp32 scores s_j = q.k_j (unscaled fp32 FMAs, two
//     per packed f32x2 instruction; every bf16 x bf16 product is exact), a
//     2048-bucket histogram of the top 11 bits of each score's order key per
//     row, and per (batch, K head) the largest |k|.
//  2. topv_filter_kernel -- all SMs: per row, the histogram gives the bucket
//     holding the k-th largest score; every position whose score is at least
//     that bucket's lower end minus 2d (d the rounding bound below) is
//     appended to the row's candidate list.  Everything else is certainly out.
//  3. topv_select_kernel, one CTA per row, on the candidates in shared memory:
//     a. tau = k-th largest fp32 score (radix select on the 21 key bits below
//        the bucket the filter found: 11 bits, then 10);
//     b. d >= |s_j - e_j| for every j, e_j the exact dot product:
//        d = 1.01 gamma_n ||q||_1 max|k| + n 2^-149, gamma_n = n u / (1 - n u), u = 2^-24;
//     c. s_j > tau + 2d: certainly kept; s_j < tau - 2d: certainly not; the
//        rest (usually a handful) get exact keys -- an integer superaccumulator
//        of the products -- and the remaining slots go to the largest exact
//        keys, the lower position first on ties;
//     d. kept positions are marked in a bitmap and written in ascending order.
//  4. topv_gather_kernel, several CTAs per row: the renormalised softmax-weighted
//     sum of exactly the kept V rows; the last CTA of a row adds the parts up.
// Launches 2-4 use programmatic dependent launch: each kernel lets the next one
// be scheduled early and waits (griddepcontrol.wait) before it reads anything
// the previous one wrote.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr int kScoreThreads = 128;      // consumer threads of the score kernel (+1 producer warp)
constexpr int kScoreTile = 128;         // positions per TMA tile (one per consumer thread)
constexpr int kHistBuckets = 2048;      // first radix digit: top 11 bits of the order key
constexpr int kHistWords = kHistBuckets / 2;  // score-kernel histogram: two 16-bit counters per word
constexpr int kScoreMaxTilesPerCta = 511;     // keeps a CTA's positions (and any counter) below 2^16
// Score CTAs per SM: three for d_k = 64; with d_k = 128 the q registers of four heads need two.
constexpr int score_ctas_per_sm(int dk) { return dk == 64 ? 3 : 2; }
constexpr int kRadixBuckets = 256;      // later radix digits: one byte
constexpr int kFilterThreads = 256;
constexpr int kFilterChunk = 8192;      // positions per filter CTA (32 per thread)
constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kPairwiseMax = 64;        // ambiguous sets up to this size are ranked pairwise
constexpr int kKeyWords = 19;           // 18 superaccumulator digits + inverted position
constexpr int kTopvHeader = 256;
constexpr int kCandCap = 12288;         // candidates held in shared memory by the select kernel
constexpr int kTopvMaxContext = 131072; // bitmap of kept positions: 16 KB of shared memory
constexpr int kRowInfoWords = 8;       // per-row words handed from kernel to kernel
enum RowInfo { kRiBucket = 0, kRiAbove = 1, kRiTwoDelta = 2, kRiMax = 3, kRiKept = 4, kRiFullSum = 5 };
constexpr int kMaxFilterChunks = kTopvMaxContext / kFilterChunk;
constexpr int kGatherThreads = 256;
constexpr int kGatherWarps = kGatherThreads / 32;
constexpr int kGatherRows = 128;        // kept V rows per gather CTA and round
constexpr int kGatherMaxSplit = 8;      // gather CTAs of a row: one thread-block cluster

struct TopvArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    const int32_t *seq_lens;
    __nv_bfloat16 *out;
    int32_t *idx_out;
    float *scores;     // [B*n_q][t_pad]
    int32_t *cand_j;   // [B*n_q][t_pad] candidate positions (filter -> select)
    float *cand_s;     // [B*n_q][t_pad] their scores
    int32_t *alist;    // [B*n_q][t_pad] ambiguous positions
    uint8_t *astate;   // [B*n_q][t_pad] exact-select state of ambiguous entries
    uint8_t *adigit;   // [B*n_q][t_pad] current radix digit of ambiguous entries
    uint32_t *kmax;    // [B*n_k] bf16 bit pattern of max |k| (zeroed per call)
    uint32_t *ghist;   // [B*n_q][2048] histogram of the top 11 bits of the score keys (zeroed per call)
    uint32_t *ncand;   // [B*n_q] candidate counts (zeroed per call)
    uint32_t *rowinfo; // [B*n_q][kRowInfoWords]: threshold bucket, count above it, 2 x score error bound
                       // (filter); kept max score, kept count (select)
    int32_t *status;
    int32_t batch, n_q, n_k, n_v, t_max, t_pad, topk, q_per_k, q_per_v;
    int32_t score_stages;
    int32_t full_weights;  // 1: weight the kept rows by the full-softmax alpha_j (no renormalisation)
    float2 *fpart;         // [B*n_q][kMaxFilterChunks] (max score, sum of 2^((s - max) scale log2 e)) per filter chunk
    float scale_log2;
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ int clamp_len(int v, int t_max) { return v < 0 ? 0 : (v > t_max ? t_max : v); }

// Programmatic dependent launch: let the next kernel in the stream be scheduled
// now / wait until the previous kernel has finished and its writes are visible.
// Both are no-ops for a kernel launched without the attribute.  Every chained
// kernel waits before it can exit, so each one finishing implies that all the
// kernels before it have finished too.
__device__ __forceinline__ void pdl_launch_next() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_prev() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// max(a, b, c) in one instruction (three-input form of max.f32, sm_100).
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float r;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
    return r;
}

// All threads of all CTAs of the cluster; shared-memory writes before it are visible after it.
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// 32-bit load from the shared memory of cluster CTA `rank`, at this CTA's shared address `addr`.
__device__ __forceinline__ float ld_dsmem_f32(uint32_t addr, uint32_t rank) {
    uint32_t remote;
    float v;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(addr), "r"(rank));
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(remote) : "memory");
    return v;
}

// Order-preserving map of finite floats onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Rigorous bound of |fp32 FMA-chain score - exact dot| for a row: every product
// is exact, every one of the (at most n = d_k) additions a score sees rounds by
// at most u relative (u = 2^-24) or, in the subnormal range, by 2^-150 absolute;
// sum_c |q_c k_c| <= ||q||_1 max|k|.  1.01 covers the rounding of this formula.
template <int DK>
__device__ __forceinline__ float score_error_bound(float q_l1, float kmax) {
    const double nu = (double)DK * 5.9604644775390625e-08;  // n * 2^-24
    const float gamma = (float)(nu / (1.0 - nu));
    return __fmul_ru(__fmul_ru(__fmul_ru(1.01f, gamma), q_l1), kmax) + (float)DK * 1.4012984643e-45f;
}

// ------------------------------------------------------------------ 1. scores

// Sum over the 4 lanes of a position group of HG per-lane partials, one per
// head; returns the total of head `head_of_lane(r)` to lane r (r = lane % 4).
// For HG = 4 a butterfly leaves head r's total in lane r (3 shuffles).
template <int HG>
__device__ __forceinline__ float reduce_heads(const float (&v)[HG], int r) {
    if constexpr (HG == 4) {
        const bool hi2 = (r & 2) != 0;
        const float a0 = (hi2 ? v[2] : v[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[0] : v[2], 2);
        const float a1 = (hi2 ? v[3] : v[1]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[1] : v[3], 2);
        const bool hi1 = (r & 1) != 0;
        return (hi1 ? a1 : a0) + __shfl_xor_sync(0xffffffffu, hi1 ? a0 : a1, 1);
    } else if constexpr (HG == 2) {
        const bool hi2 = (r & 2) != 0;
        float x = (hi2 ? v[1] : v[0]) + __shfl_xor_sync(0xffffffffu, hi2 ? v[0] : v[1], 2);
        return x + __shfl_xor_sync(0xffffffffu, x, 1);
    } else {
        float x = v[0] + __shfl_xor_sync(0xffffffffu, v[0], 2);
        return x + __shfl_xor_sync(0xffffffffu, x, 1);
    }
}
template <int HG>
__device__ __forceinline__ bool lane_writes(int r) { return HG == 4 ? true : (HG == 2 ? (r & 1) == 0 : r == 0); }
template <int HG>
__device__ __forceinline__ int head_of_lane(int r) { return HG == 4 ? r : (HG == 2 ? r >> 1 : 0); }

// One CTA streams K tiles of one (batch, K head) over an equal share of its
// positions: a producer thread issues TMA loads (128-byte swizzle) into a ring
// of tiles.  Four lanes share a position: lane r reads 16-byte chunks
// (u / 2) * 8 + 2 r + u % 2 of the row, so a quarter warp (two positions, one
// even and one odd) touches eight distinct bank groups, and holds the matching
// elements of q for up to four query heads in registers.  The four partial dot
// products of each head are added across the group, and lane r writes head r.
template <int DK, int QPK>
__global__ void __launch_bounds__(kScoreThreads + 32, score_ctas_per_sm(DK)) topv_score_kernel(const __grid_constant__ CUtensorMap tm_k,
                                                                         const TopvArgs a) {
    constexpr int KB = DK / 64;  // 64-wide swizzle blocks per row
    constexpr int TILE_BYTES = kScoreTile * DK * 2;
    extern __shared__ uint8_t dsm_raw[];
    uint8_t *dsm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(dsm_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *tiles = dsm;                                                                 // [stages][TILE_BYTES]
    uint32_t *hist_s = reinterpret_cast<uint32_t *>(dsm + a.score_stages * TILE_BYTES);  // [QPK][1024]
    float *q_s = reinterpret_cast<float *>(hist_s + QPK * kHistWords);                   // [QPK][DK]
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(q_s + QPK * DK);
    uint64_t *empty_bar = full_bar + a.score_stages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty_bar + a.score_stages);

    const int unit = blockIdx.x;
    const int b = unit / a.n_k;
    const int g = unit % a.n_k;
    const int raw_len = __ldg(a.seq_lens + b);
    const int T = clamp_len(raw_len, a.t_max);
    const int tid = threadIdx.x;
    // a length outside [0, t_max] is clamped (every kernel of the call clamps it the same way) and
    // flagged once per sequence
    if (g == 0 && blockIdx.y == 0 && tid == 0 && raw_len != T) record_error(a.status, DIFFQKV_ERR_DEVICE_SEQLEN);
    const int warp = tid >> 5, lane = tid & 31;
    const int ntiles = (T + kScoreTile - 1) / kScoreTile;
    const int tb = (int)(((long long)ntiles * blockIdx.y) / gridDim.y);
    const int te = (int)(((long long)ntiles * (blockIdx.y + 1)) / gridDim.y);

    if (tid == 0) {
        for (int s = 0; s < a.score_stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], kScoreThreads / 32);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    pdl_launch_next();
    for (int i = tid; i < QPK * kHistWords; i += blockDim.x) hist_s[i] = 0;
    for (int i = tid; i < QPK * DK; i += blockDim.x) {
        const int hh = i / DK, c = i % DK;
        q_s[i] = __bfloat162float(a.q[((size_t)b * a.n_q + g * QPK + hh) * DK + c]);
    }
    __syncthreads();

    if (warp == kScoreThreads / 32) {
        // ---- producer
        if (lane == 0 && te > tb) {
            prefetch_tensormap(&tm_k);
            for (int t = tb, k = 0; t < te; ++t, ++k) {
                const int st = k % a.score_stages;
                if (k >= a.score_stages)
                    mbar_wait_bounded(&empty_bar[st], (uint32_t)(((k / a.score_stages) - 1) & 1), a.wait_limit_ns,
                                      abort_flag, a.status);
                if (*abort_flag) break;
                uint8_t *dst = tiles + st * TILE_BYTES;
                mbar_arrive_expect_tx(&full_bar[st], TILE_BYTES);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_4d(dst + kb * (kScoreTile * 128), &tm_k, &full_bar[st], kb * 64, g, t * kScoreTile, b);
            }
            const int issued = te - tb;
            for (int k = (issued > a.score_stages ? issued - a.score_stages : 0); k < issued; ++k)
                mbar_wait_bounded(&full_bar[k % a.score_stages], (uint32_t)((k / a.score_stages) & 1),
                                  a.wait_limit_ns, nullptr, a.status);
        }
    } else {
        // ---- consumers: warp w takes positions PPW w .. PPW w + PPW - 1 of each tile, 8 at a time
        constexpr int HG = QPK < 4 ? QPK : 4;  // heads per pass (their q in registers)
        constexpr int NPASS = QPK / HG;
        constexpr int CPL = DK / 32;           // 16-byte chunks of a K row per lane
        constexpr int PPW = kScoreTile / (kScoreThreads / 32);  // positions per warp and tile
        static_assert(PPW % 8 == 0, "whole steps of 8 positions");
        const int r = lane & 3, pg = lane >> 2;
        // byte offset of this lane's u-th chunk in a row, swizzle included (row index mod 8 = pg)
        uint32_t coff[CPL];
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
            const int chunk = (u >> 1) * 8 + 2 * r + (u & 1);
            coff[u] = (uint32_t)((chunk >> 3) * (kScoreTile * 128) + (((chunk & 7) ^ pg) << 4));
        }
        float kmf = 0.f;  // largest |k| seen (a bf16 value, so exact in fp32)
        float *sbase = a.scores + ((size_t)b * a.n_q + g * QPK) * a.t_pad;
        f32x2_t qp[HG][CPL][4];  // q[head][chunk elements 2i, 2i + 1]
        auto load_q = [&](int pass) {
#pragma unroll
            for (int hh = 0; hh < HG; ++hh)
#pragma unroll
                for (int u = 0; u < CPL; ++u) {
                    const int chunk = (u >> 1) * 8 + 2 * r + (u & 1);
                    const float *qs = q_s + (pass * HG + hh) * DK + chunk * 8;
                    const float4 x = *reinterpret_cast<const float4 *>(qs);
                    const float4 y = *reinterpret_cast<const float4 *>(qs + 4);
                    qp[hh][u][0] = f2_pack(x.x, x.y);
                    qp[hh][u][1] = f2_pack(x.z, x.w);
                    qp[hh][u][2] = f2_pack(y.x, y.y);
                    qp[hh][u][3] = f2_pack(y.z, y.w);
                }
        };
        if (NPASS == 1) load_q(0);
        for (int t = tb, k = 0; t < te; ++t, ++k) {
            const int st = k % a.score_stages;
            mbar_wait_bounded(&full_bar[st], (uint32_t)((k / a.score_stages) & 1), a.wait_limit_ns, abort_flag,
                              a.status);
            const uint8_t *tile = tiles + st * TILE_BYTES;
#pragma unroll 1
            for (int pass = 0; pass < NPASS; ++pass) {
                if (NPASS > 1) load_q(pass);
#pragma unroll
                for (int step = 0; step < PPW / 8; ++step) {
                    const int pos = warp * PPW + step * 8 + pg;  // row of the tile
                    const int j = t * kScoreTile + pos;
                    const bool cached = pass == 0 && j < T;  // |k| counts for cached positions only
                    // even/odd elements in packed fp32 pairs: every lane of fma.rn.f32x2 is an IEEE
                    // fp32 FMA; a product meets at most 4 CPL + 3 (<= d_k) roundings on its way into the score
                    f32x2_t acc[HG];
#pragma unroll
                    for (int hh = 0; hh < HG; ++hh) acc[hh] = 0ull;
#pragma unroll
                    for (int u = 0; u < CPL; ++u) {
                        const uint4 kv = lds128(tile + pos * 128 + coff[u]);
                        float kf[8];
                        unpack8(kv, kf);
                        if (cached) {
                            kmf = fmax3f(kmf, fabsf(kf[0]), fabsf(kf[1]));
                            kmf = fmax3f(kmf, fabsf(kf[2]), fabsf(kf[3]));
                            kmf = fmax3f(kmf, fabsf(kf[4]), fabsf(kf[5]));
                            kmf = fmax3f(kmf, fabsf(kf[6]), fabsf(kf[7]));
                        }
                        const f32x2_t k01 = f2_pack(kf[0], kf[1]), k23 = f2_pack(kf[2], kf[3]);
                        const f32x2_t k45 = f2_pack(kf[4], kf[5]), k67 = f2_pack(kf[6], kf[7]);
#pragma unroll
                        for (int hh = 0; hh < HG; ++hh) {
                            acc[hh] = f2_fma(qp[hh][u][0], k01, acc[hh]);
                            acc[hh] = f2_fma(qp[hh][u][1], k23, acc[hh]);
                            acc[hh] = f2_fma(qp[hh][u][2], k45, acc[hh]);
                            acc[hh] = f2_fma(qp[hh][u][3], k67, acc[hh]);
                        }
                    }
                    float part[HG];
#pragma unroll
                    for (int hh = 0; hh < HG; ++hh) {
                        float x0, x1;
                        f2_unpack(acc[hh], x0, x1);
                        part[hh] = x0 + x1;
                    }
                    const float score = reduce_heads<HG>(part, r);
                    if (lane_writes<HG>(r) && j < T) {
                        const int hh = pass * HG + head_of_lane<HG>(r);
                        sbase[(size_t)hh * a.t_pad + j] = score;
                        const uint32_t bk = float_key(score) >> 21;
                        atomicAdd(hist_s + hh * kHistWords + (bk >> 1), 1u << ((bk & 1u) << 4));
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty_bar[st]);
        }
        uint32_t kmx = __float_as_uint(kmf) >> 16;  // its bf16 pattern (kmf >= 0: order-preserving)
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, off));
        if (lane == 0) atomicMax(a.kmax + unit, kmx);
    }
    __syncthreads();
    // word i holds buckets 2i (low half) and 2i + 1 of the group's [QPK][2048] histograms
    uint32_t *gh = a.ghist + ((size_t)b * a.n_q + g * QPK) * kHistBuckets;
    for (int i = tid; i < QPK * kHistWords; i += blockDim.x) {
        const uint32_t w = hist_s[i];
        if (w & 0xffffu) atomicAdd(gh + 2 * i, w & 0xffffu);
        if (w >> 16) atomicAdd(gh + 2 * i + 1, w >> 16);
    }
}

// ------------------------------------------------------------------ helpers

// Warp-aggregated shared-memory histogram increment; `bucket` < 0 skips.
__device__ __forceinline__ void hist_add(uint32_t *hist, int bucket) {
    const unsigned peers = __match_any_sync(0xffffffffu, bucket);
    const int leader = __ffs(peers) - 1;
    if (bucket >= 0 && (threadIdx.x & 31) == leader) atomicAdd(hist + bucket, (uint32_t)__popc(peers));
}

// Block-wide exclusive prefix sum of one value per thread (thread order).
// warp_sums needs 33 entries; returns the exclusive prefix and writes the
// block total to *total.
__device__ uint32_t block_exclusive_scan(uint32_t v, uint32_t *warp_sums, uint32_t *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t ws = lane < nw ? warp_sums[lane] : 0u;
        uint32_t wi = ws;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        if (lane < nw) warp_sums[lane] = wi - ws;
        if (lane == 31) warp_sums[32] = wi;
    }
    __syncthreads();
    const uint32_t r = warp_sums[warp] + incl - v;
    *total = warp_sums[32];
    __syncthreads();
    return r;
}

// Block-wide: the bucket d (counting from the top bucket down) that holds the
// kk-th largest element (kk >= 1) of a histogram of nb buckets, and the count
// strictly above it, into *d_out / *above_out (shared).  Thread t scans the
// buckets [nb - (t+1)*span, nb - t*span) from the top down.
__device__ void find_bucket_from_top(const uint32_t *hist, int nb, uint32_t kk, int *d_out, uint32_t *above_out,
                                     uint32_t *warp_sums) {
    const int span = (nb + blockDim.x - 1) / blockDim.x;
    const int top = nb - 1 - (int)threadIdx.x * span;  // first (highest) bucket of this thread
    uint32_t mine = 0;
    for (int i = 0; i < span; ++i)
        if (top - i >= 0) mine += hist[top - i];
    uint32_t total;
    const uint32_t excl = block_exclusive_scan(mine, warp_sums, &total);
    if (mine > 0 && excl < kk && kk <= excl + mine) {
        uint32_t above = excl;
        for (int i = 0; i < span && top - i >= 0; ++i) {
            const uint32_t c = hist[top - i];
            if (above + c >= kk) {
                *d_out = top - i;
                *above_out = above;
                break;
            }
            above += c;
        }
    }
    __syncthreads();
}

// Exact q.k as an ordered key: words 0..17 are the superaccumulator digits
// (most significant first, sign-biased so unsigned comparison orders them),
// word 18 is ~j so that, among equal values, the lower position ranks higher.
//   bf16 value = M * 2^x, M < 256 integer; x = -133 (exponent field 0) or E - 134;
//   product = P * 2^(xq + xk), P < 2^16, accumulated in units of 2^-266 as
//   base-2^32 digits held in int64 slots, then carry-normalised.
template <int DK>
__device__ void exact_key(const uint16_t *qbits, const uint16_t *kbits, int j, uint32_t *out) {
    // digit slots stay in registers: each product is added to its slot by a
    // predicated add over the 16 slots a product can start in (offsets <= 506)
    long long acc[18];
#pragma unroll
    for (int i = 0; i < 18; ++i) acc[i] = 0;
#pragma unroll 1
    for (int c8 = 0; c8 < DK / 8; ++c8) {
        const uint4 kw = *reinterpret_cast<const uint4 *>(kbits + 8 * c8);
        const uint32_t words[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t kb = (e & 1) ? (words[e >> 1] >> 16) : (words[e >> 1] & 0xffffu);
            const uint32_t qb = qbits[8 * c8 + e];
            const int eq = (qb >> 7) & 0xff, ek = (kb >> 7) & 0xff;
            const int mq = (qb & 0x7f) | (eq ? 0x80 : 0), mk = (kb & 0x7f) | (ek ? 0x80 : 0);
            const int off = (eq ? eq - 134 : -133) + (ek ? ek - 134 : -133) + 266;
            long long v = (long long)(mq * mk) << (off & 31);
            if ((qb ^ kb) & 0x8000u) v = -v;
            const int slot = off >> 5;
#pragma unroll
            for (int i = 0; i < 16; ++i) acc[i] += (slot == i) ? v : 0ll;
        }
    }
#pragma unroll
    for (int i = 0; i < 17; ++i) {
        const long long c = acc[i] >> 32;  // floor division by 2^32
        acc[i] -= c * 4294967296LL;
        acc[i + 1] += c;
    }
    out[0] = (uint32_t)acc[17] ^ 0x80000000u;
#pragma unroll
    for (int i = 1; i < 18; ++i) out[i] = (uint32_t)acc[17 - i];
    out[18] = ~(uint32_t)j;
}

// exact_key computed by a whole warp: lane l takes products l, l + 32, ...; the
// per-lane digit slots are integers, so summing them across the warp is exact
// in any order (|slot| < d_k 2^47 <= 2^54).  Only the slots some lane used are
// summed (the range is warp-uniform); lane 0 normalises and writes.  kbits is
// the K row in global memory.
template <int DK>
__device__ void exact_key_warp(const uint16_t *qbits, const uint16_t *kbits, int j, uint32_t *out, int lane) {
    long long acc[18];
#pragma unroll
    for (int i = 0; i < 18; ++i) acc[i] = 0;
    int smin = 15, smax = 0;
#pragma unroll
    for (int u = 0; u < DK / 32; ++u) {
        const int c = lane + 32 * u;
        const uint32_t qb = qbits[c], kb = __ldg(kbits + c);
        const int eq = (qb >> 7) & 0xff, ek = (kb >> 7) & 0xff;
        const int mq = (qb & 0x7f) | (eq ? 0x80 : 0), mk = (kb & 0x7f) | (ek ? 0x80 : 0);
        const int off = (eq ? eq - 134 : -133) + (ek ? ek - 134 : -133) + 266;
        long long v = (long long)(mq * mk) << (off & 31);
        if ((qb ^ kb) & 0x8000u) v = -v;
        const int slot = off >> 5;
        smin = min(smin, slot);
        smax = max(smax, slot);
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] += (slot == i) ? v : 0ll;
    }
    smin = __reduce_min_sync(0xffffffffu, smin);
    smax = __reduce_max_sync(0xffffffffu, smax);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        if (i < smin || i > smax) continue;  // no lane has a product in this slot
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], o);
    }
    if (lane == 0) {
#pragma unroll
        for (int i = 0; i < 17; ++i) {
            const long long c = acc[i] >> 32;  // floor division by 2^32
            acc[i] -= c * 4294967296LL;
            acc[i + 1] += c;
        }
        out[0] = (uint32_t)acc[17] ^ 0x80000000u;
#pragma unroll
        for (int i = 1; i < 18; ++i) out[i] = (uint32_t)acc[17 - i];
        out[18] = ~(uint32_t)j;
    }
}

__device__ __forceinline__ bool key_greater(const uint32_t *x, const uint32_t *y) {
    for (int i = 0; i < kKeyWords; ++i)
        if (x[i] != y[i]) return x[i] > y[i];
    return false;
}

// ||q||_1 of this row's query (every thread gets it; same summation order in all).
template <int DK>
__device__ float row_q_l1(const __nv_bfloat16 *q, float *red) {
    float v = 0.f;
    for (int c = threadIdx.x; c < DK; c += blockDim.x) v += fabsf(__bfloat162float(q[c]));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float t = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += red[w];
    __syncthreads();
    return t;
}

// ------------------------------------------------------------------ 2. filter

template <int DK>
__global__ void __launch_bounds__(kFilterThreads, 4) topv_filter_kernel(const TopvArgs a) {
    __shared__ uint32_t warp_sums[33];
    __shared__ float red[kFilterThreads / 32];
    __shared__ __align__(16) uint32_t hist_s[kHistBuckets];  // filled with 16-byte stores
    __shared__ int sh_d;
    __shared__ uint32_t sh_above;
    const int row = blockIdx.x;
    const int b = row / a.n_q, h = row % a.n_q, g = h / a.q_per_k;
    const int T = clamp_len(__ldg(a.seq_lens + b), a.t_max);
    const int j_begin = blockIdx.y * kFilterChunk;
    pdl_launch_next();
    pdl_wait_prev();  // scores, histograms and max |k| of the score kernel
    if (T <= a.topk || j_begin >= T) return;  // every position kept / nothing here (uniform per CTA)
    const int tid = threadIdx.x, lane = tid & 31;

    // this CTA's scores first (they do not depend on the threshold): lane-interleaved
    // 16-byte loads, each warp load covering 512 contiguous bytes
    const float *s = a.scores + (size_t)row * a.t_pad;
    int32_t *cj = a.cand_j + (size_t)row * a.t_pad;
    float *cs = a.cand_s + (size_t)row * a.t_pad;
    const int j_end = min(T, j_begin + kFilterChunk);
    constexpr int kVec = kFilterChunk / kFilterThreads / 4;  // float4 loads per thread
    static_assert(kVec * 4 <= 32, "a thread's hits fit one 32-bit mask");
    float4 v[kVec];
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const int p = j_begin + (u * kFilterThreads + tid) * 4;
        v[u] = p < j_end ? __ldcg(reinterpret_cast<const float4 *>(s + p)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const uint32_t kmax_bits = __ldcg(a.kmax + b * a.n_k + g);

    if (a.full_weights) {
        // this chunk's share of the full softmax denominator: its max and its sum of exponentials
        float mx = -INFINITY;
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int p = j_begin + (u * kFilterThreads + tid) * 4;
            const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (p + e < j_end) mx = fmaxf(mx, x[e]);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red[tid >> 5] = mx;
        __syncthreads();
        mx = red[0];
        for (int w2 = 1; w2 < kFilterThreads / 32; ++w2) mx = fmaxf(mx, red[w2]);
        __syncthreads();
        float sum = 0.f;
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int p = j_begin + (u * kFilterThreads + tid) * 4;
            const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (p + e < j_end) sum += fast_exp2((x[e] - mx) * a.scale_log2);
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
        if (lane == 0) red[tid >> 5] = sum;
        __syncthreads();
        if (tid == 0) {
            float tot = 0.f;
            for (int w2 = 0; w2 < kFilterThreads / 32; ++w2) tot += red[w2];
            a.fpart[(size_t)row * kMaxFilterChunks + blockIdx.y] = make_float2(mx, tot);
        }
        __syncthreads();
    }

    // bucket of the k-th largest score, and the lower end of the range that can be kept
    {
        const uint4 *src = reinterpret_cast<const uint4 *>(a.ghist + (size_t)row * kHistBuckets);
        uint4 hv[kHistBuckets / 4 / kFilterThreads];
#pragma unroll
        for (int u = 0; u < kHistBuckets / 4 / kFilterThreads; ++u) hv[u] = __ldcg(src + u * kFilterThreads + tid);
#pragma unroll
        for (int u = 0; u < kHistBuckets / 4 / kFilterThreads; ++u)
            reinterpret_cast<uint4 *>(hist_s)[u * kFilterThreads + tid] = hv[u];
    }
    __syncthreads();
    find_bucket_from_top(hist_s, kHistBuckets, (uint32_t)a.topk, &sh_d, &sh_above, warp_sums);
    if (blockIdx.y == 0 && tid == 0) {
        a.rowinfo[kRowInfoWords * row + kRiBucket] = (uint32_t)sh_d;
        a.rowinfo[kRowInfoWords * row + kRiAbove] = sh_above;
    }
    const float q1 = row_q_l1<DK>(a.q + (size_t)row * DK, red);
    const float two_d = __fmul_ru(2.f, score_error_bound<DK>(q1, __uint_as_float(kmax_bits << 16)));
    if (blockIdx.y == 0 && tid == 0) a.rowinfo[kRowInfoWords * row + kRiTwoDelta] = __float_as_uint(two_d);
    // (bucket 0 starts at the NaN patterns: everything in it and above is a candidate)
    const float lower = sh_d == 0 ? -INFINITY : __fsub_rd(key_float((uint32_t)sh_d << 21), two_d);
    // a thread's hits form a bit mask; one block scan gives every thread its slots and
    // one global atomic per CTA reserves them
    uint32_t hits = 0;
#pragma unroll
    for (int u = 0; u < kVec; ++u) {
        const int p = j_begin + (u * kFilterThreads + tid) * 4;
        const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
            if (p + e < j_end && x[e] >= lower) hits |= 1u << (4 * u + e);
    }
    uint32_t total;
    uint32_t slot = block_exclusive_scan((uint32_t)__popc(hits), warp_sums, &total);
    __shared__ uint32_t sh_base;
    if (tid == 0 && total) sh_base = atomicAdd(a.ncand + row, total);
    __syncthreads();
    if (hits) {
        slot += sh_base;
#pragma unroll
        for (int u = 0; u < kVec; ++u) {
            const int p = j_begin + (u * kFilterThreads + tid) * 4;
            const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if ((hits >> (4 * u + e)) & 1u) {
                    cj[slot] = p + e;
                    cs[slot] = x[e];
                    ++slot;
                }
            }
        }
    }
    (void)lane;
}

// ------------------------------------------------------------------ 3. select + gather

template <int DK, int DV>
__global__ void __launch_bounds__(kSelThreads, 1) topv_select_kernel(const TopvArgs a) {
    __shared__ uint32_t hist[kHistBuckets];
    __shared__ uint32_t warp_sums[33];
    __shared__ uint16_t q_s[DK];
    __shared__ uint32_t keys_s[kPairwiseMax][kKeyWords];
    __shared__ int32_t alist_s[kPairwiseMax];  // the first ambiguous positions (the whole list when pairwise)
    __shared__ float red_s[kSelWarps];
    __shared__ int sh_d;
    __shared__ uint32_t sh_above;
    __shared__ int sh_cnt_in, sh_na, sh_done;
    extern __shared__ __align__(16) uint8_t sel_dyn[];
    int32_t *c_j = reinterpret_cast<int32_t *>(sel_dyn);           // [kCandCap]
    float *c_s = reinterpret_cast<float *>(c_j + kCandCap);           // [kCandCap]
    uint32_t *bitmap = reinterpret_cast<uint32_t *>(c_s + kCandCap);  // [kTopvMaxContext / 32]
    uint32_t *wprefix = bitmap + kTopvMaxContext / 32;                               // [kTopvMaxContext / 32]

    const int row = blockIdx.x;
    const int b = row / a.n_q;
    const int h = row % a.n_q;
    const int g = h / a.q_per_k;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = clamp_len(__ldg(a.seq_lens + b), a.t_max);
    const int K = a.topk;
    const float *s = a.scores + (size_t)row * a.t_pad;
    int32_t *alist = a.alist + (size_t)row * a.t_pad;
    uint8_t *ast = a.astate + (size_t)row * a.t_pad;
    uint8_t *adg = a.adigit + (size_t)row * a.t_pad;
    int32_t *idx = a.idx_out + (size_t)row * K;

    pdl_launch_next();
    if (tid < DK) q_s[tid] = reinterpret_cast<const uint16_t *>(a.q)[(size_t)row * DK + tid];
    pdl_wait_prev();  // candidates, bucket and max |k| of the filter and score kernels
    if (T == 0) {
        for (int i = tid; i < K; i += kSelThreads) idx[i] = -1;
        if (tid == 0) {
            a.rowinfo[kRowInfoWords * row + kRiMax] = __float_as_uint(0.f);
            a.rowinfo[kRowInfoWords * row + kRiKept] = 0u;
            a.rowinfo[kRowInfoWords * row + kRiFullSum] = 0u;
        }
        return;
    }
    const int nwords = (T + 31) / 32;
    int nsel;

    if (T <= K) {
        // every cached position is kept: positions 0..T-1, then -1
        for (int i = tid; i < K; i += kSelThreads) idx[i] = i < T ? i : -1;
        float mx = -INFINITY;
        for (int i = tid; i < T; i += kSelThreads) mx = fmaxf(mx, s[i]);
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red_s[warp] = mx;
        nsel = T;
    } else {
        // ---- candidates from the filter (every position that can be kept)
        const uint32_t nc = __ldcg(a.ncand + row);
        const bool in_smem = nc <= (uint32_t)kCandCap;
        const int32_t *cj = in_smem ? c_j : a.cand_j + (size_t)row * a.t_pad;
        const float *cs = in_smem ? c_s : a.cand_s + (size_t)row * a.t_pad;
        if (in_smem) {
            const int32_t *gj = a.cand_j + (size_t)row * a.t_pad;
            const float *gs = a.cand_s + (size_t)row * a.t_pad;
            for (uint32_t base = 0; base < nc; base += 4 * kSelThreads) {
                int32_t jj[4];
                float xx[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t i = base + u * kSelThreads + tid;
                    jj[u] = i < nc ? __ldcg(gj + i) : 0;
                    xx[u] = i < nc ? __ldcg(gs + i) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t i = base + u * kSelThreads + tid;
                    if (i < nc) {
                        c_j[i] = jj[u];
                        c_s[i] = xx[u];
                    }
                }
            }
        }
        for (int i = tid; i < nwords; i += kSelThreads) bitmap[i] = 0u;
        __syncthreads();

        // ---- a. tau = the K-th largest score.  Its top 11 key bits are the filter's bucket,
        //         and `above` positions lie in higher buckets (all of them candidates); a radix
        //         select over the candidates finds the other 21 bits, 11 and then 10 at a time
        uint32_t prefix = __ldcg(a.rowinfo + kRowInfoWords * row + kRiBucket) << 21, pmask = 0xffe00000u;
        uint32_t kk = (uint32_t)K - __ldcg(a.rowinfo + kRowInfoWords * row + kRiAbove);
        for (int pass = 0; pass < 2; ++pass) {
            const int shift = pass == 0 ? 10 : 0;
            const int nb = pass == 0 ? 2048 : 1024;
            for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
            __syncthreads();
            for (uint32_t base = 0; base < nc; base += kSelThreads) {
                const uint32_t i = base + tid;
                int bucket = -1;
                if (i < nc) {
                    const uint32_t key = float_key(cs[i]);
                    if ((key & pmask) == prefix) bucket = (int)((key >> shift) & (uint32_t)(nb - 1));
                }
                hist_add(hist, bucket);
            }
            __syncthreads();
            find_bucket_from_top(hist, nb, kk, &sh_d, &sh_above, warp_sums);
            prefix |= (uint32_t)sh_d << shift;
            pmask |= (uint32_t)(nb - 1) << shift;
            kk -= sh_above;
        }
        const float tau = key_float(prefix);

        // ---- b. rounding bound of every score of this row (the filter's, see score_error_bound)
        const float two_d = __uint_as_float(__ldcg(a.rowinfo + kRowInfoWords * row + kRiTwoDelta));
        const float hi_edge = __fadd_ru(tau, two_d);
        const float lo_edge = __fsub_rd(tau, two_d);
        if (tid == 0) {
            sh_cnt_in = 0;
            sh_na = 0;
        }
        __syncthreads();

        // ---- c. certain / ambiguous classification of the candidates
        int my_in = 0;
        for (uint32_t i = tid; i < nc; i += kSelThreads) {
            const float x = cs[i];
            if (x > hi_edge) {
                const int j = cj[i];
                atomicOr(bitmap + (j >> 5), 1u << (j & 31));
                ++my_in;
            } else if (x >= lo_edge) {
                const int slot = atomicAdd(&sh_na, 1);
                alist[slot] = cj[i];
                if (slot < kPairwiseMax) alist_s[slot] = cj[i];
            }
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) my_in += __shfl_xor_sync(0xffffffffu, my_in, off);
        if (lane == 0 && my_in) atomicAdd(&sh_cnt_in, my_in);
        __syncthreads();
        const int na = sh_na;
        const int need = K - sh_cnt_in;  // 1 <= need <= na when the bound holds
        const __nv_bfloat16 *krow0 = a.k + ((size_t)b * a.t_max * a.n_k + g) * DK;
        const size_t kstride = (size_t)a.n_k * DK;
        auto keep = [&](int j) { atomicOr(bitmap + (j >> 5), 1u << (j & 31)); };

        if (need <= 0) {
            // nothing left to choose (cannot happen when the bound holds)
        } else if (need >= na) {
            for (int i = tid; i < na; i += kSelThreads) keep(alist[i]);
        } else if (na <= kPairwiseMax) {
            // rank the few ambiguous positions pairwise by exact key (a warp per key)
            for (int r = warp; r < na; r += kSelWarps) {
                const int j = alist_s[r];
                exact_key_warp<DK>(q_s, reinterpret_cast<const uint16_t *>(krow0 + (size_t)j * kstride), j,
                                   keys_s[r], lane);
            }
            __syncthreads();
            if (tid < na) {
                int better = 0;
                for (int u = 0; u < na; ++u) better += key_greater(keys_s[u], keys_s[tid]) ? 1 : 0;
                if (better < need) keep(alist[tid]);
            }
        } else {
            // radix select over the exact keys, one byte per pass (keys are unique)
            for (int i = tid; i < na; i += kSelThreads) ast[i] = 0;
            if (tid == 0) sh_done = 0;
            uint32_t kk2 = (uint32_t)need;
            __syncthreads();
            for (int p = 0; p < kKeyWords * 4 && !sh_done; ++p) {
                for (int i = tid; i < kRadixBuckets; i += kSelThreads) hist[i] = 0;
                __syncthreads();
                for (int base = 0; base < na; base += kSelThreads) {
                    const int i = base + tid;
                    int bucket = -1;
                    if (i < na && ast[i] == 0) {
                        uint32_t key[kKeyWords];
                        const int j = alist[i];
                        exact_key<DK>(q_s, reinterpret_cast<const uint16_t *>(krow0 + (size_t)j * kstride), j, key);
                        bucket = (int)((key[p >> 2] >> (24 - 8 * (p & 3))) & 0xffu);
                        adg[i] = (uint8_t)bucket;
                    }
                    hist_add(hist, bucket);
                }
                __syncthreads();
                find_bucket_from_top(hist, kRadixBuckets, kk2, &sh_d, &sh_above, warp_sums);
                const int d = sh_d;
                kk2 -= sh_above;
                const bool finish = hist[d] == kk2;
                for (int i = tid; i < na; i += kSelThreads) {
                    if (ast[i] != 0) continue;
                    const int dig = adg[i];
                    if (dig > d || (finish && dig == d)) ast[i] = 1;
                    else if (dig < d) ast[i] = 2;
                }
                if (tid == 0 && finish) sh_done = 1;
                __syncthreads();
            }
            for (int i = tid; i < na; i += kSelThreads)
                if (ast[i] == 1) keep(alist[i]);
        }
        __syncthreads();

        // ---- d. ascending order: a kept position's slot is the number of kept
        //         positions before it, from per-word prefix counts of the bitmap
        const int wper = (nwords + kSelThreads - 1) / kSelThreads;
        const int w0 = min(nwords, tid * wper), w1 = min(nwords, w0 + wper);
        uint32_t cnt = 0;
        for (int w = w0; w < w1; ++w) cnt += __popc(bitmap[w]);
        uint32_t total;
        uint32_t run = block_exclusive_scan(cnt, warp_sums, &total);
        for (int w = w0; w < w1; ++w) {
            wprefix[w] = run;
            run += __popc(bitmap[w]);
        }
        nsel = (int)total;
        __syncthreads();
        float mx = -INFINITY;
        for (uint32_t i = tid; i < nc; i += kSelThreads) {
            const int j = cj[i];
            const uint32_t word = bitmap[j >> 5];
            if ((word >> (j & 31)) & 1u) {
                const uint32_t slot = wprefix[j >> 5] + __popc(word & ((1u << (j & 31)) - 1u));
                idx[slot] = j;
                mx = fmaxf(mx, cs[i]);
            }
        }
        if (tid == 0 && nsel != K) record_error(a.status, DIFFQKV_ERR_INVALID_ARG);
        for (int i = nsel + tid; i < K; i += kSelThreads) idx[i] = -1;
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if (lane == 0) red_s[warp] = mx;
    }
    __syncthreads();
    if (tid == 0) {
        float m = red_s[0];
        for (int w = 1; w < kSelWarps; ++w) m = fmaxf(m, red_s[w]);
        float full_sum = 0.f;  // 0: renormalise over the kept set
        if (a.full_weights && T > K) {
            // the full softmax denominator from the filter's chunk partials, relative to the row max
            const int nch = (T + kFilterChunk - 1) / kFilterChunk;
            float M = -INFINITY;
            for (int ch = 0; ch < nch; ++ch) M = fmaxf(M, __ldcg(&a.fpart[(size_t)row * kMaxFilterChunks + ch].x));
            for (int ch = 0; ch < nch; ++ch) {
                const float2 pc = __ldcg(&a.fpart[(size_t)row * kMaxFilterChunks + ch]);
                full_sum += pc.y * fast_exp2((pc.x - M) * a.scale_log2);
            }
            m = M;
        }
        a.rowinfo[kRowInfoWords * row + kRiMax] = __float_as_uint(m);
        a.rowinfo[kRowInfoWords * row + kRiKept] = (uint32_t)nsel;
        a.rowinfo[kRowInfoWords * row + kRiFullSum] = __float_as_uint(full_sum);
    }
}

// ------------------------------------------------------------------ 4. gather

// CTA (row, part) sums its share of the kept positions (in ascending order):
// sum_j 2^((s_j - m) scale log2 e) v_j and the weight sum, with m the largest
// kept score.  The parts of a row form one thread-block cluster: each leaves its
// sums in its own shared memory, and rank 0 adds them in rank order through
// distributed shared memory and writes the normalised output.  No CTA returns
// early, so every thread reaches both cluster barriers.
template <int DV>
__global__ void __launch_bounds__(kGatherThreads) topv_gather_kernel(const TopvArgs a) {
    __shared__ float o_s[kGatherWarps][DV];
    __shared__ float l_s[kGatherWarps];
    __shared__ float part_s[DV + 1];  // this CTA's sums: o[0..DV-1], then the weight sum
    const int row = blockIdx.x, part = blockIdx.y, nparts = gridDim.y;
    const int b = row / a.n_q, h = row % a.n_q, vh = h / a.q_per_v;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    pdl_wait_prev();  // kept positions and their maximum from the select kernel
    const float m = __uint_as_float(__ldcg(a.rowinfo + kRowInfoWords * row + kRiMax));
    const int nsel = (int)__ldcg(a.rowinfo + kRowInfoWords * row + kRiKept);
    const int i_begin = (int)(((long long)nsel * part) / nparts);
    const int i_end = (int)(((long long)nsel * (part + 1)) / nparts);
    const int32_t *idx = a.idx_out + (size_t)row * a.topk;
    const float *s = a.scores + (size_t)row * a.t_pad;

    constexpr int CPV = DV / 8;      // lanes per V row
    constexpr int RPW = 32 / CPV;    // V rows per warp step
    constexpr int GU = 8;            // V rows in flight per lane: a CTA's 128 rows in one round
    const int vc = lane % CPV, vs = lane / CPV;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = 0.f;
    float l = 0.f;
    const __nv_bfloat16 *vbase = a.v + ((size_t)b * a.t_max * a.n_v + vh) * DV + vc * 8;
    const size_t vstride = (size_t)a.n_v * DV;
    for (int i0 = i_begin + warp * RPW; i0 < i_end; i0 += kGatherWarps * RPW * GU) {
        // every position first, then every score and V row: two dependent rounds of loads
        int jj[GU];
#pragma unroll
        for (int u = 0; u < GU; ++u) {
            const int i = i0 + u * kGatherWarps * RPW + vs;
            jj[u] = i < i_end ? __ldcg(idx + i) : -1;
        }
        uint4 vv[GU];
        float sx[GU];
#pragma unroll
        for (int u = 0; u < GU; ++u) {
            if (jj[u] >= 0) {
                sx[u] = __ldcg(s + jj[u]);
                vv[u] = __ldg(reinterpret_cast<const uint4 *>(vbase + (size_t)jj[u] * vstride));
            } else {
                sx[u] = -INFINITY;
                vv[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < GU; ++u) {
            const float w = jj[u] >= 0 ? fast_exp2((sx[u] - m) * a.scale_log2) : 0.f;
            float vf[8];
            unpack8(vv[u], vf);
            l += w;
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = fmaf(w, vf[e], o[e]);
        }
    }
    // reduce over the RPW row slots of the warp, then over warps
#pragma unroll
    for (int off = CPV; off < 32; off <<= 1) {
        l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
    }
    if (vs == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) o_s[warp][vc * 8 + e] = o[e];
    }
    if (lane == 0) l_s[warp] = l;
    __syncthreads();
    for (int c = tid; c <= DV; c += kGatherThreads) {
        float acc = 0.f;
        for (int w = 0; w < kGatherWarps; ++w) acc += c < DV ? o_s[w][c] : l_s[w];
        part_s[c] = acc;
    }
    cluster_sync();  // every part of the row is in its CTA's shared memory
    if (part == 0) {
        const uint32_t base = smem_addr(part_s);
        float lt = 0.f;
        for (int p = 0; p < nparts; ++p) lt += ld_dsmem_f32(base + DV * 4u, (uint32_t)p);
        // full-softmax weights: divide by the sum over every cached position instead
        const float full_sum = __uint_as_float(__ldcg(a.rowinfo + kRowInfoWords * row + kRiFullSum));
        if (full_sum > 0.f) lt = full_sum;
        for (int c = tid; c < DV; c += kGatherThreads) {
            float acc = 0.f;
            for (int p = 0; p < nparts; ++p) acc += ld_dsmem_f32(base + (uint32_t)c * 4u, (uint32_t)p);
            a.out[(size_t)row * DV + c] = __float2bfloat16(lt > 0.f ? acc / lt : 0.f);
        }
    }
    cluster_sync();  // no CTA leaves while rank 0 still reads its shared memory
}

size_t align_up(size_t x, size_t al) { return (x + al - 1) / al * al; }

using ScoreFn = void (*)(CUtensorMap, TopvArgs);
using RowFn = void (*)(TopvArgs);

template <int DK>
ScoreFn pick_score_qpk(int qpk) {
    switch (qpk) {
        case 1: return topv_score_kernel<DK, 1>;
        case 2: return topv_score_kernel<DK, 2>;
        case 4: return topv_score_kernel<DK, 4>;
        case 8: return topv_score_kernel<DK, 8>;
        case 16: return topv_score_kernel<DK, 16>;
        default: return nullptr;
    }
}

ScoreFn pick_score(int dk, int qpk) {
    if (dk == 64) return pick_score_qpk<64>(qpk);
    if (dk == 128) return pick_score_qpk<128>(qpk);
    return nullptr;
}

RowFn pick_filter(int dk) {
    if (dk == 64) return topv_filter_kernel<64>;
    if (dk == 128) return topv_filter_kernel<128>;
    return nullptr;
}

RowFn pick_select(int dk, int dv) {
    if (dk == 64 && dv == 64) return topv_select_kernel<64, 64>;
    if (dk == 64 && dv == 128) return topv_select_kernel<64, 128>;
    if (dk == 128 && dv == 64) return topv_select_kernel<128, 64>;
    if (dk == 128 && dv == 128) return topv_select_kernel<128, 128>;
    return nullptr;
}

RowFn pick_gather(int dv) {
    if (dv == 64) return topv_gather_kernel<64>;
    if (dv == 128) return topv_gather_kernel<128>;
    return nullptr;
}

size_t padded_len(int32_t t_max) { return align_up((size_t)t_max, 64); }

// kmax entries, rounded up so the histograms after them start 16-byte aligned.
size_t kmax_slots(const diffqkv_dims_t *d) { return align_up((size_t)d->batch * d->n_k, 4); }

// Zero-filled per call: kmax [B*n_k, padded], histograms [rows][2048], candidate counts [rows].
size_t zeroed_bytes(const diffqkv_dims_t *d) {
    const size_t rows = (size_t)d->batch * d->n_q;
    return kmax_slots(d) * 4 + rows * kHistBuckets * 4 + rows * 4;
}

// Gather CTAs per row (one cluster): a round of kGatherRows kept rows each, at most kGatherMaxSplit.
int gather_split(int32_t topk) { return std::max(1, std::min(kGatherMaxSplit, (topk + kGatherRows - 1) / kGatherRows)); }

// rowinfo [rows][kRowInfoWords], then the filter's softmax partials [rows][kMaxFilterChunks]
size_t rowinfo_bytes(const diffqkv_dims_t *d) { return align_up((size_t)d->batch * d->n_q * kRowInfoWords * 4, 256); }
size_t row_bytes(const diffqkv_dims_t *d) {
    return rowinfo_bytes(d) + align_up((size_t)d->batch * d->n_q * kMaxFilterChunks * sizeof(float2), 256);
}

// Launch after the previous kernel of the stream with programmatic dependent launch;
// cluster_y > 1 groups that many consecutive CTAs along y into one cluster.
template <typename... P, typename... A>
cudaError_t launch_after_prev(void (*kernel)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              int cluster_y, A... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 1;
    if (cluster_y > 1) {
        attr[1].id = cudaLaunchAttributeClusterDimension;
        attr[1].val.clusterDim.x = 1;
        attr[1].val.clusterDim.y = (unsigned)cluster_y;
        attr[1].val.clusterDim.z = 1;
        cfg.numAttrs = 2;
    }
    cfg.attrs = attr;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace

size_t topv_workspace_size(const diffqkv_dims_t *d, int32_t t_max, int32_t topk) {
    if (validate_dims(d) != DIFFQKV_OK || t_max < 1 || topk < 1) return 0;
    const size_t rows = (size_t)d->batch * d->n_q;
    const size_t per = padded_len(t_max);
    return kTopvHeader + align_up(zeroed_bytes(d), 256) + row_bytes(d) + align_up(rows * per * 4, 256) * 4 +
           align_up(rows * per, 256) * 2;
}

diffqkv_status_t topv_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, int32_t topk, void *out,
                             int32_t *idx_out, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                             int32_t flags) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !idx_out || t_max < 1 || topk < 1)
        return DIFFQKV_ERR_INVALID_ARG;
    if (t_max > kTopvMaxContext) return DIFFQKV_ERR_UNSUPPORTED;
    if (flags & ~DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS) return DIFFQKV_ERR_INVALID_ARG;
    const int qpk = d->n_q / d->n_k;
    ScoreFn score = pick_score(d->d_k, qpk);
    RowFn filter = pick_filter(d->d_k);
    RowFn select = pick_select(d->d_k, d->d_v);
    RowFn gather = pick_gather(d->d_v);
    if (!score || !filter || !select || !gather) return DIFFQKV_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(idx_out) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    const size_t need = topv_workspace_size(d, t_max, topk);
    if (!workspace || workspace_bytes < need) return DIFFQKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return DIFFQKV_ERR_MISALIGNED;
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;

    const size_t rows = (size_t)d->batch * d->n_q;
    const size_t t_pad = padded_len(t_max);
    uint8_t *ws = static_cast<uint8_t *>(workspace) + kTopvHeader;
    TopvArgs a;
    a.kmax = reinterpret_cast<uint32_t *>(ws);
    a.ghist = a.kmax + kmax_slots(d);  // 16-byte aligned (read with 16-byte loads)
    a.ncand = a.ghist + rows * kHistBuckets;
    ws += align_up(zeroed_bytes(d), 256);
    a.rowinfo = reinterpret_cast<uint32_t *>(ws);
    a.fpart = reinterpret_cast<float2 *>(ws + rowinfo_bytes(d));
    a.full_weights = (flags & DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS) ? 1 : 0;
    ws += row_bytes(d);
    a.scores = reinterpret_cast<float *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.cand_j = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.cand_s = reinterpret_cast<float *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.alist = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.astate = ws;
    ws += align_up(rows * t_pad, 256);
    a.adigit = ws;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.idx_out = idx_out;
    a.status = reinterpret_cast<int32_t *>(workspace);  // the workspace's own error word (header word 0)
    a.batch = d->batch;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.t_max = t_max;
    a.t_pad = (int32_t)t_pad;
    a.topk = topk;
    a.q_per_k = qpk;
    a.q_per_v = d->n_q / d->n_v;
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);
    a.wait_limit_ns = kWaitLimitNs;
    (void)max_seq_len;  // every grid adapts to the device lengths by itself

    if (cudaMemsetAsync(a.kmax, 0, zeroed_bytes(d), stream) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    // 1. scores: TMA tiles of K {d_k, n_k, t_max, B}, box {64, 1, 128, 1}, 128-byte swizzle
    CUtensorMap tm_k;
    st = make_tensor_map_4d(&tm_k, k_cache, d->d_k, d->n_k, t_max, d->batch, 64, 1, kScoreTile, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DIFFQKV_OK) return st;
    const int tile_bytes = kScoreTile * d->d_k * 2;
    const int fixed = qpk * kHistWords * 4 + qpk * d->d_k * 4 + 16 * 8 + 16 + 1024;
    // the deepest ring (2..8 tiles) that still lets score_ctas_per_sm CTAs share an SM (228 KB, 1 KB
    // reserved per CTA): occupancy hides more of the consumers' latency than a deeper ring does
    const int want = score_ctas_per_sm(d->d_k);
    int stages = 8;
    while (stages > 2 && want * (stages * tile_bytes + fixed + 1024) > 228 * 1024) --stages;
    a.score_stages = stages;
    const int score_smem = stages * tile_bytes + fixed;
    const int per_sm = std::max(1, std::min(want, (228 * 1024) / (score_smem + 1024)));
    const int units = d->batch * d->n_k;
    const int ntiles = (t_max + kScoreTile - 1) / kScoreTile;
    const int ygrid = std::max({1, (dev.num_sms * per_sm) / units,
                                (ntiles + kScoreMaxTilesPerCta - 1) / kScoreMaxTilesPerCta});
    const int select_smem = kCandCap * 8 + 2 * (kTopvMaxContext / 8);
    if (ensure_dynamic_smem((const void *)score, score_smem) != DIFFQKV_OK ||
        ensure_dynamic_smem((const void *)select, select_smem) != DIFFQKV_OK)
        return DIFFQKV_ERR_CUDA;
    score<<<dim3(units, ygrid), kScoreThreads + 32, score_smem, stream>>>(tm_k, a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    // 2. filter: every row, in chunks of kFilterChunk positions (chunks past a row's length return at once)
    if (launch_after_prev(filter, dim3((unsigned)rows, (t_max + kFilterChunk - 1) / kFilterChunk),
                          dim3(kFilterThreads), 0, stream, 1, a) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    // 3. select: one CTA per row
    if (launch_after_prev(select, dim3((unsigned)rows), dim3(kSelThreads), select_smem, stream, 1, a) !=
        cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    // 4. gather: one cluster of gather_split CTAs per row
    const int split = gather_split(topk);
    if (launch_after_prev(gather, dim3((unsigned)rows, (unsigned)split), dim3(kGatherThreads), 0, stream, split, a) !=
        cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    return DIFFQKV_OK;
}

}  // namespace diffqkv
