// topv.cu -- selective V fetch decode for sm_100a.
//
// "Selective V Cache Fetching" (Sigma paper, structured summary page): after
// the scores are computed from the full (thin) K cache, only the V rows of the
// top-k scoring positions are read; the other positions are treated as zero.
// The softmax is renormalised over the kept positions, and the positions are
// ranked by the EXACT dot product q.k (ties toward the lower position) so the
// selected set is unique and reproducible.
//
// Two launches:
//  1. topv_score_kernel: streams K once (16-byte loads, one K row serves all
//     n_q/n_k query heads of its group) and writes fp32 scores s_j = q.k_j
//     (unscaled, fp32 FMA chain: every bf16 x bf16 product is exact) plus, per
//     (batch, K head), the largest |k| element for the rounding bound.
//  2. topv_select_kernel, one CTA per (batch, query head):
//     a. tau = k-th largest fp32 score (3-pass radix select over the
//        order-preserving integer image of the floats);
//     b. rigorous bound d >= |s_j - e_j| for every j (e_j the exact dot):
//        d = gamma_n * ||q||_1 * max|k| (gamma_n = n u / (1 - n u), u = 2^-24)
//        plus n * 2^-149 for subnormal roundings;
//     c. s_j > tau + 2d: certainly selected; s_j < tau - 2d: certainly not;
//        the rest (usually a handful) get exact keys -- an integer
//        superaccumulator of the products -- and the remaining slots go to the
//        largest exact keys, lower position first on ties;
//     d. selected positions are compacted in ascending order, and the
//        renormalised softmax-weighted sum of exactly those V rows is written.
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr int kScoreThreads = 256;
constexpr int kScoreChunk = 2048;     // positions per score CTA iteration
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kPairwiseMax = 64;      // ambiguous sets up to this size are ranked pairwise
constexpr int kKeyWords = 19;         // 18 superaccumulator digits + inverted position
constexpr int kTopvHeader = 256;

struct TopvArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    const int32_t *seq_lens;
    __nv_bfloat16 *out;
    int32_t *idx_out;
    float *scores;     // [B*n_q][t_max]
    int32_t *alist;    // [B*n_q][t_max] ambiguous positions
    uint8_t *flags;    // [B*n_q][t_max] 1 = selected
    uint8_t *astate;   // [B*n_q][t_max] exact-select state of ambiguous entries
    uint8_t *adigit;   // [B*n_q][t_max] current radix digit of ambiguous entries
    uint32_t *kmax;    // [B*n_k] bf16 bit pattern of max |k|
    int32_t *status;
    int32_t batch, n_q, n_k, n_v, t_max, topk, q_per_k, q_per_v;
    float scale_log2;
};

__device__ __forceinline__ int clamp_len(int v, int t_max) { return v < 0 ? 0 : (v > t_max ? t_max : v); }

// ------------------------------------------------------------------ scores

template <int DK, int QPK>
__global__ void __launch_bounds__(kScoreThreads) topv_score_kernel(const TopvArgs a) {
    constexpr int LPT = DK / 8;           // lanes per K row (16 bytes each)
    constexpr int TPW = 32 / LPT;         // rows per warp per step
    constexpr int NW = kScoreThreads / 32;
    constexpr int UNROLL = 4;
    const int unit = blockIdx.x;
    const int b = unit / a.n_k;
    const int g = unit % a.n_k;
    const int T = clamp_len(__ldg(a.seq_lens + b), a.t_max);
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int kc = lane % LPT;
    const int kt = lane / LPT;

    float qf[QPK][8];
#pragma unroll
    for (int h = 0; h < QPK; ++h) {
        const uint4 qv = __ldg(reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.n_q + g * QPK + h) * DK) + kc);
        unpack8(qv, qf[h]);
    }
    uint32_t kmx = 0;
    const __nv_bfloat16 *kbase = a.k + (size_t)b * a.t_max * a.n_k * DK + (size_t)g * DK + kc * 8;
    const size_t krow = (size_t)a.n_k * DK;
    float *sbase = a.scores + ((size_t)b * a.n_q + g * QPK) * a.t_max;

    for (int c0 = blockIdx.y * kScoreChunk; c0 < T; c0 += gridDim.y * kScoreChunk) {
        const int c1 = min(T, c0 + kScoreChunk);
        for (int base = c0 + warp * TPW; base < c1; base += NW * TPW * UNROLL) {
            uint4 kv[UNROLL];
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int j = base + u * NW * TPW + kt;
                kv[u] = j < c1 ? __ldg(reinterpret_cast<const uint4 *>(kbase + (size_t)j * krow))
                               : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < UNROLL; ++u) {
                const int j = base + u * NW * TPW + kt;
                const uint32_t w[4] = {kv[u].x, kv[u].y, kv[u].z, kv[u].w};
#pragma unroll
                for (int e = 0; e < 4; ++e) kmx = max(kmx, max(w[e] & 0x7fffu, (w[e] >> 16) & 0x7fffu));
                float kf[8];
                unpack8(kv[u], kf);
                float acc[QPK];
#pragma unroll
                for (int h = 0; h < QPK; ++h) {
                    float s = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) s = fmaf(qf[h][e], kf[e], s);
#pragma unroll
                    for (int off = LPT / 2; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
                    acc[h] = s;
                }
                if (j < c1) {
#pragma unroll
                    for (int h = 0; h < QPK; ++h)
                        if (h % LPT == kc) sbase[(size_t)h * a.t_max + j] = acc[h];
                }
            }
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, off));
    if (lane == 0) atomicMax(a.kmax + unit, kmx);
}

// ------------------------------------------------------------------ selection helpers

// Order-preserving map of finite floats onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Warp-aggregated shared-memory histogram increment; `bucket` < 0 skips.
__device__ __forceinline__ void hist_add(uint32_t *hist, int bucket) {
    const unsigned peers = __match_any_sync(0xffffffffu, bucket);
    const int leader = __ffs(peers) - 1;
    if (bucket >= 0 && (threadIdx.x & 31) == leader) atomicAdd(hist + bucket, (uint32_t)__popc(peers));
}

// Block-wide: find the bucket d (counting from the highest bucket down) that
// holds the kk-th largest element (kk >= 1), and the count strictly above it.
// nb <= 2 * kSelThreads.  Results in *d_out / *above_out (shared).
__device__ void find_bucket_from_top(const uint32_t *hist, int nb, uint32_t kk, int *d_out, uint32_t *above_out,
                                     uint32_t *warp_sums) {
    const int t = threadIdx.x;
    const int hi = nb - 1 - 2 * t;
    const int lo = hi - 1;
    const uint32_t chi = hi >= 0 ? hist[hi] : 0u;
    const uint32_t clo = lo >= 0 ? hist[lo] : 0u;
    const uint32_t mine = chi + clo;
    // exclusive scan over threads (thread 0 owns the top buckets)
    uint32_t incl = mine;
    const int lane = t & 31, warp = t >> 5;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t ws = warp_sums[lane];
        uint32_t wi = ws;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        warp_sums[lane] = wi - ws;  // exclusive prefix of warps
    }
    __syncthreads();
    const uint32_t excl = warp_sums[warp] + incl - mine;
    if (mine > 0 && excl < kk && kk <= excl + mine) {
        if (excl + chi >= kk) {
            *d_out = hi;
            *above_out = excl;
        } else {
            *d_out = lo;
            *above_out = excl + chi;
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
    long long acc[18];
#pragma unroll
    for (int i = 0; i < 18; ++i) acc[i] = 0;
    for (int c = 0; c < DK; ++c) {
        const uint32_t qb = qbits[c], kb = kbits[c];
        const int eq = (qb >> 7) & 0xff, ek = (kb >> 7) & 0xff;
        const int mq = (qb & 0x7f) | (eq ? 0x80 : 0), mk = (kb & 0x7f) | (ek ? 0x80 : 0);
        const long long P = (long long)(mq * mk);
        if (P == 0) continue;
        const int off = (eq ? eq - 134 : -133) + (ek ? ek - 134 : -133) + 266;
        const long long v = P << (off & 31);
        if ((qb ^ kb) & 0x8000u) acc[off >> 5] -= v;
        else acc[off >> 5] += v;
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

__device__ __forceinline__ bool key_greater(const uint32_t *x, const uint32_t *y) {
    for (int i = 0; i < kKeyWords; ++i)
        if (x[i] != y[i]) return x[i] > y[i];
    return false;
}

// ------------------------------------------------------------------ select + gather

template <int DK, int DV>
__global__ void __launch_bounds__(kSelThreads, 1) topv_select_kernel(const TopvArgs a) {
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t warp_sums[32];
    __shared__ uint16_t q_s[DK];
    __shared__ uint32_t keys_s[kPairwiseMax][kKeyWords];
    __shared__ float red_s[kSelWarps];
    __shared__ float o_s[kSelWarps][DV];
    __shared__ int sh_d;
    __shared__ uint32_t sh_above;
    __shared__ int sh_cnt_in, sh_na, sh_done;

    const int row = blockIdx.x;
    const int b = row / a.n_q;
    const int h = row % a.n_q;
    const int g = h / a.q_per_k;
    const int vh = h / a.q_per_v;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = clamp_len(__ldg(a.seq_lens + b), a.t_max);
    const int K = a.topk;
    const float *s = a.scores + (size_t)row * a.t_max;
    uint8_t *fl = a.flags + (size_t)row * a.t_max;
    int32_t *alist = a.alist + (size_t)row * a.t_max;
    uint8_t *ast = a.astate + (size_t)row * a.t_max;
    uint8_t *adg = a.adigit + (size_t)row * a.t_max;
    int32_t *idx = a.idx_out + (size_t)row * K;
    __nv_bfloat16 *outp = a.out + (size_t)row * DV;

    if (tid < DK) q_s[tid] = reinterpret_cast<const uint16_t *>(a.q)[(size_t)row * DK + tid];
    if (T == 0) {
        for (int i = tid; i < K; i += kSelThreads) idx[i] = -1;
        for (int i = tid; i < DV; i += kSelThreads) outp[i] = __float2bfloat16(0.f);
        return;
    }

    if (T <= K) {
        for (int j = tid; j < T; j += kSelThreads) fl[j] = 1;
    } else {
        // ---- a. tau: the K-th largest fp32 score (radix digits 11, 11, 10 bits)
        uint32_t prefix = 0, pmask = 0, kk = (uint32_t)K;
        const int shifts[3] = {21, 10, 0};
        const int widths[3] = {11, 11, 10};
        for (int pass = 0; pass < 3; ++pass) {
            const int nb = 1 << widths[pass];
            for (int i = tid; i < nb; i += kSelThreads) hist[i] = 0;
            __syncthreads();
            for (int base = 0; base < T; base += kSelThreads) {
                const int j = base + tid;
                int bucket = -1;
                if (j < T) {
                    const uint32_t key = float_key(s[j]);
                    if ((key & pmask) == prefix) bucket = (int)((key >> shifts[pass]) & (uint32_t)(nb - 1));
                }
                hist_add(hist, bucket);
            }
            __syncthreads();
            find_bucket_from_top(hist, nb, kk, &sh_d, &sh_above, warp_sums);
            prefix |= (uint32_t)sh_d << shifts[pass];
            pmask |= (uint32_t)(nb - 1) << shifts[pass];
            kk -= sh_above;
            __syncthreads();
        }
        const float tau = key_float(prefix);

        // ---- b. rounding bound of every fp32 score
        float q1 = 0.f;
        if (warp == 0) {
            for (int c = lane; c < DK; c += 32) q1 += fabsf(__uint_as_float((uint32_t)q_s[c] << 16));
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) q1 += __shfl_xor_sync(0xffffffffu, q1, off);
            if (lane == 0) red_s[0] = q1;
        }
        if (tid == 0) {
            sh_cnt_in = 0;
            sh_na = 0;
        }
        __syncthreads();
        q1 = red_s[0];
        const float kmax = __uint_as_float(__ldcg(a.kmax + b * a.n_k + g) << 16);
        const double nu = (double)DK * 5.9604644775390625e-08;  // n * 2^-24
        const float gamma = (float)(nu / (1.0 - nu));
        const float delta = __fmul_ru(__fmul_ru(__fmul_ru(1.01f, gamma), q1), kmax) + (float)DK * 1.4012984643e-45f;
        const float two_d = __fmul_ru(2.f, delta);
        const float hi_edge = __fadd_ru(tau, two_d);
        const float lo_edge = __fsub_rd(tau, two_d);

        // ---- c. certain / ambiguous classification
        int my_in = 0;
        for (int j = tid; j < T; j += kSelThreads) {
            const float x = s[j];
            uint8_t f = 0;
            if (x > hi_edge) {
                f = 1;
                ++my_in;
            } else if (x >= lo_edge) {
                const int slot = atomicAdd(&sh_na, 1);
                alist[slot] = j;
            }
            fl[j] = f;
        }
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) my_in += __shfl_xor_sync(0xffffffffu, my_in, off);
        if (lane == 0 && my_in) atomicAdd(&sh_cnt_in, my_in);
        __syncthreads();
        const int na = sh_na;
        const int need = K - sh_cnt_in;  // 1 <= need <= na
        const __nv_bfloat16 *krow0 = a.k + ((size_t)b * a.t_max * a.n_k + g) * DK;
        const size_t kstride = (size_t)a.n_k * DK;

        if (need <= 0) {
            // nothing left to choose (cannot happen when the bound holds)
        } else if (need >= na) {
            for (int i = tid; i < na; i += kSelThreads) fl[alist[i]] = 1;
        } else if (na <= kPairwiseMax) {
            // rank the few ambiguous positions pairwise by exact key
            if (tid < na) {
                const int j = alist[tid];
                exact_key<DK>(q_s, reinterpret_cast<const uint16_t *>(krow0 + (size_t)j * kstride), j, keys_s[tid]);
            }
            __syncthreads();
            if (tid < na) {
                int better = 0;
                for (int u = 0; u < na; ++u) better += key_greater(keys_s[u], keys_s[tid]) ? 1 : 0;
                if (better < need) fl[alist[tid]] = 1;
            }
        } else {
            // radix select over the exact keys, one byte per pass (keys are unique)
            for (int i = tid; i < na; i += kSelThreads) ast[i] = 0;
            if (tid == 0) sh_done = 0;
            uint32_t kk2 = (uint32_t)need;
            __syncthreads();
            for (int p = 0; p < kKeyWords * 4 && !sh_done; ++p) {
                for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
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
                find_bucket_from_top(hist, 256, kk2, &sh_d, &sh_above, warp_sums);
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
                if (ast[i] == 1) fl[alist[i]] = 1;
        }
    }
    __syncthreads();

    // ---- d. compaction in ascending position order
    const int per = (T + kSelThreads - 1) / kSelThreads;
    const int j0 = min(T, tid * per), j1 = min(T, j0 + per);
    int cnt = 0;
    for (int j = j0; j < j1; ++j) cnt += fl[j];
    int incl = cnt;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    if (lane == 31) warp_sums[warp] = (uint32_t)incl;
    __syncthreads();
    if (warp == 0) {
        const uint32_t ws = warp_sums[lane];
        uint32_t wi = ws;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, wi, off);
            if (lane >= off) wi += y;
        }
        warp_sums[lane] = wi - ws;
        if (lane == 31) sh_cnt_in = (int)wi;  // total selected
    }
    __syncthreads();
    int pos = (int)warp_sums[warp] + incl - cnt;
    for (int j = j0; j < j1; ++j)
        if (fl[j]) idx[pos++] = j;
    const int nsel = sh_cnt_in;
    if (tid == 0 && nsel != min(K, T)) record_error(a.status, DIFFQKV_ERR_INVALID_ARG);
    for (int i = nsel + tid; i < K; i += kSelThreads) idx[i] = -1;
    __syncthreads();

    // ---- e. renormalised softmax over the selected rows; only their V rows are read
    float m = -INFINITY;
    for (int i = tid; i < nsel; i += kSelThreads) m = fmaxf(m, s[idx[i]]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    if (lane == 0) red_s[warp] = m;
    __syncthreads();
    m = red_s[0];
#pragma unroll 1
    for (int w = 1; w < kSelWarps; ++w) m = fmaxf(m, red_s[w]);
    __syncthreads();

    constexpr int CPV = DV / 8;      // lanes per V row
    constexpr int RPW = 32 / CPV;    // V rows per warp step
    const int vc = lane % CPV, vs = lane / CPV;
    float o[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = 0.f;
    float l = 0.f;
    const __nv_bfloat16 *vbase = a.v + ((size_t)b * a.t_max * a.n_v + vh) * DV + vc * 8;
    const size_t vstride = (size_t)a.n_v * DV;
    for (int i0 = warp * RPW; i0 < nsel; i0 += kSelWarps * RPW * 2) {
        uint4 vv[2];
        float w[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int i = i0 + u * kSelWarps * RPW + vs;
            if (i < nsel) {
                const int j = idx[i];
                w[u] = fast_exp2((s[j] - m) * a.scale_log2);
                vv[u] = __ldg(reinterpret_cast<const uint4 *>(vbase + (size_t)j * vstride));
            } else {
                w[u] = 0.f;
                vv[u] = make_uint4(0, 0, 0, 0);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            float vf[8];
            unpack8(vv[u], vf);
            l += w[u];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = fmaf(w[u], vf[e], o[e]);
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
    if (lane == 0) red_s[warp] = l;
    __syncthreads();
    if (tid < DV) {
        float acc = 0.f, lt = 0.f;
#pragma unroll 1
        for (int w = 0; w < kSelWarps; ++w) {
            acc += o_s[w][tid];
            lt += red_s[w];
        }
        outp[tid] = __float2bfloat16(lt > 0.f ? acc / lt : 0.f);
    }
}

size_t align_up(size_t x, size_t al) { return (x + al - 1) / al * al; }

using ScoreFn = void (*)(TopvArgs);
using SelectFn = void (*)(TopvArgs);

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

SelectFn pick_select(int dk, int dv) {
    if (dk == 64 && dv == 64) return topv_select_kernel<64, 64>;
    if (dk == 64 && dv == 128) return topv_select_kernel<64, 128>;
    if (dk == 128 && dv == 64) return topv_select_kernel<128, 64>;
    if (dk == 128 && dv == 128) return topv_select_kernel<128, 128>;
    return nullptr;
}

}  // namespace

size_t topv_workspace_size(const diffqkv_dims_t *d, int32_t t_max, int32_t topk) {
    if (validate_dims(d) != DIFFQKV_OK || t_max < 1 || topk < 1) return 0;
    const size_t rows = (size_t)d->batch * d->n_q;
    const size_t per = (size_t)t_max;
    return kTopvHeader + align_up((size_t)d->batch * d->n_k * 4, 256) + align_up(rows * per * 4, 256) * 2 +
           align_up(rows * per, 256) * 3;
}

diffqkv_status_t topv_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, int32_t topk, void *out,
                             int32_t *idx_out, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !idx_out || t_max < 1 || topk < 1)
        return DIFFQKV_ERR_INVALID_ARG;
    const int qpk = d->n_q / d->n_k;
    ScoreFn score = pick_score(d->d_k, qpk);
    SelectFn select = pick_select(d->d_k, d->d_v);
    if (!score || !select) return DIFFQKV_ERR_UNSUPPORTED;
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
    uint8_t *ws = static_cast<uint8_t *>(workspace) + kTopvHeader;
    TopvArgs a;
    a.kmax = reinterpret_cast<uint32_t *>(ws);
    ws += align_up((size_t)d->batch * d->n_k * 4, 256);
    a.scores = reinterpret_cast<float *>(ws);
    ws += align_up(rows * t_max * 4, 256);
    a.alist = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * t_max * 4, 256);
    a.flags = ws;
    ws += align_up(rows * t_max, 256);
    a.astate = ws;
    ws += align_up(rows * t_max, 256);
    a.adigit = ws;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.idx_out = idx_out;
    a.status = dev.status_word;
    a.batch = d->batch;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.t_max = t_max;
    a.topk = topk;
    a.q_per_k = qpk;
    a.q_per_v = d->n_q / d->n_v;
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);

    if (cudaMemsetAsync(a.kmax, 0, (size_t)d->batch * d->n_k * 4, stream) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    const int msl = (max_seq_len >= 1 && max_seq_len <= t_max) ? max_seq_len : t_max;
    const int units = d->batch * d->n_k;
    int chunks = (msl + kScoreChunk - 1) / kScoreChunk;
    const int want = dev.num_sms * 8;  // resident score CTAs
    chunks = std::max(1, std::min(chunks, (want + units - 1) / units));
    dim3 grid_s(units, chunks);
    score<<<grid_s, kScoreThreads, 0, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    select<<<(unsigned)rows, kSelThreads, 0, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    return DIFFQKV_OK;
}

}  // namespace diffqkv
