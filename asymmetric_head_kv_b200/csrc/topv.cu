// topv.cu -- selective V fetch decode for sm_100a, one cooperative launch.
//
// "Selective V Cache Fetching" (Sigma paper, structured summary page): after
// the scores are computed from the full (thin) K cache, only the V rows of the
// top-k scoring positions are read; positions outside that set contribute nothing.
// The softmax is renormalised over the kept positions (or, on request, the kept
// rows take the full-softmax weights of the pages' formula), and positions are
// ranked by the EXACT dot product q.k (ties toward the lower position) so the
// selected set is unique and reproducible.  The pages note that the V fetch
// depends on the whole K pass; here that dependency is a wait inside one kernel
// instead of a chain of launches.
//
// One persistent CTA per SM (a cooperative launch, so every CTA is resident).
// Work unit u = (batch b, K head g): the n_q/n_k query rows ("rows") of the
// group share one pass over K head g.  Each unit is cut into Y equal tile ranges
// ("parts"), one per CTA; with more units than fit, CTAs take them in rounds.
// Per unit:
//  1. Scores.  A producer warp streams the part's K tiles (128 positions) with
//     TMA into a ring; one thread issues tcgen05 MMAs S = K_tile q^T (M = 128
//     positions, N = 16 rows of q, zero-padded past the group's, K = d_k) into
//     a ring of TMEM buffers; three consumer warpgroups take the tiles in turn,
//     read one position's scores per thread out of TMEM, keep the group's rows
//     of them in TMEM (the whole part's scores stay there, so shared memory is
//     all ring), add them to a 2048-bucket histogram of the top 11 bits of each
//     score's order key, and fold the position's K row into the largest |k|.
//     Histograms go to global memory; the CTA arrives on the unit's counter H.
//  2. Candidates.  Once H counts all Y parts, each CTA finds in every row's
//     histogram the bucket holding the k-th largest score and emits every own
//     score at or above that bucket's lower end minus 2d (d the rounding bound
//     below) to the row's candidate list.  It arrives on the unit's counter C.
//  3. Select (one CTA per row).  Once C counts all Y parts: tau = the k-th
//     largest fp32 score (its top 11 bits are the bucket; two radix passes over
//     the candidates find the next 11 and the last 10); with d >= |s_j - e_j|
//     for every j (e_j the exact dot),
//        d = 1.01 gamma ||q||_1 max|k| + n 2^-126, gamma = nu / (1 - nu), nu = n (17/16) 2^-23,
//     scores above tau + 2d are certainly kept, below tau - 2d certainly not,
//     and the rest (usually a handful) get exact keys -- an integer
//     superaccumulator of the products -- and the remaining slots go to the
//     largest exact keys, the lower position first.  Kept positions are written
//     in ascending order with their scores.
//  4. Gather, by the same CTA: the weighted sum of the row's kept V rows and of
//     the weights, the warps' sums added in warp order (so the result does not
//     depend on timing), and the output.
// Every wait on another CTA is bounded (globaltimer): a wait that runs out
// records DIFFQKV_ERR_DEVICE_TIMEOUT and the CTA returns.  The counters and
// histograms clean themselves up (the last user of each resets it), so the
// workspace needs zero-filling only before its first use.
#include <math.h>

#include <string.h>

#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

// 16 warps.  Scores: warps 0-11 are three consumer warpgroups, warp 12 the TMA producer, warp 13
// the MMA issuer (and TMEM owner); warps 14 and 15 join from the candidates on.
constexpr int kTile = 128;                 // positions per K tile: the MMA's M (TMEM lanes)
constexpr int kConsumerGroups = 3;         // warpgroups reading scores out of TMEM, tiles dealt in turn
constexpr int kConsumerWarps = 4 * kConsumerGroups;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kMmaWarp = kConsumerWarps + 1;
constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kQRows = 16;                 // rows of q in the MMA's B operand (its N), zero past the group's
constexpr int kTmemBufs = 8;               // TMEM buffers of kQRows columns the MMAs write
constexpr int kTmemCols = 512;             // allocation: the MMA buffers, then the part's scores
constexpr int kScoreCol0 = kTmemBufs * kQRows;      // first column of the part's scores
constexpr int kScoreCols = kTmemCols - kScoreCol0;  // tile i's row hh at column kScoreCol0 + i QPK + hh
constexpr int kHistBuckets = 2048;       // both histogram levels: 11 bits of the order key
constexpr int kHistWords = kHistBuckets / 2;  // shared histogram: two 16-bit counters per word
constexpr int kRadixBuckets = 1024;      // last 10 key bits
constexpr int kByteBuckets = 256;        // radix select over exact keys: one byte per pass
constexpr int kPairwiseMax = 64;         // ambiguous sets up to this size are ranked pairwise
constexpr int kKeyWords = 19;            // 18 superaccumulator digits + inverted position
constexpr int kTopvHeader = 256;
constexpr int kTopvMaxContext = 131072;  // bitmap of kept positions
constexpr int kMaxParts = 256;           // CTAs per unit (sizes the per-part records)
constexpr int kMaxStages = 12;
constexpr int kTableWin = 512;           // paged producer: block-table entries held in shared memory
constexpr int kRowInfoWords = 8;
enum RowInfo { kRiBucket = 0, kRiAbove = 1, kRiTwoDelta = 2 };
enum UnitSync { kUsHist = 0, kUsCand = 1, kUsDone = 2, kUsKmax = 3 };
enum RowSync { kRsCand = 2 };  // (words 0, 1 and 3 of a row's four are unused)
constexpr int kDynSmemCap = 218 * 1024;  // dynamic shared memory (the static part needs the rest of 227 KB)

struct TopvArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k;
    const __nv_bfloat16 *v;
    const int32_t *seq_lens;
    __nv_bfloat16 *out;
    int32_t *idx_out;
    int32_t *status;
    // zero before the first call, left zero by every call that completes
    uint32_t *unit_sync;  // [units][4]: H arrivals, C arrivals, -, max |k| (bf16 bits)
    uint32_t *row_sync;   // [rows][4]: selected flag, parts gathered, candidate count, -
    uint32_t *hist1;      // [rows][2048]: top 11 key bits of every score
    // written and read within a call
    uint32_t *rowinfo;    // [rows][8]
    float2 *chunk_part;   // [rows][kMaxParts]: (max score, sum of 2^((s - max) scale log2 e)) of a part
    int32_t *cand_j;      // [rows][t_pad]
    float *cand_s;        // [rows][t_pad]
    float *kept_s;        // [rows][k_pad]: scores of the kept positions, in idx_out order
    int32_t *kept_row;    // [rows][k_pad]: their cache rows (sequence b position j: b t_max + j, or the
                          // pool row of a paged cache)
    int32_t *alist;       // [rows][t_pad]: ambiguous positions
    uint8_t *astate;      // [rows][t_pad]
    uint8_t *adigit;      // [rows][t_pad]
    int32_t batch, n_q, n_k, n_v, t_max, t_pad, topk, k_pad, q_per_v;
    int32_t parts;        // Y: CTAs per unit
    int32_t units_per_round, rounds, stages;
    int32_t cand_cap;     // candidates the select keeps in shared memory
    int32_t full_weights;
    // paged caches: block_table == null means contiguous [B, t_max, heads, d] caches; else K and V
    // are pools [num_pages, page_size, heads, d] and position j of sequence b is row j % page_size
    // of pool page block_table[b][j / page_size]
    const int32_t *block_table;
    int32_t max_blocks, page_size, num_pages;
    int32_t max_box_log;  // paged: boxes of 8 << i rows, i <= max_box_log, divide the page size
    int32_t tile_box;     // paged, page size a multiple of kTile: one kTile-row box per tile (m[0])
    int32_t page_shift;   // paged: log2(page_size) when it is a power of two, else -1
    long long cache_rows; // rows of the K / V caches or pools
    float scale_log2;
    uint64_t wait_limit_ns;
};

__device__ __forceinline__ int clamp_len(int v, int t_max) { return v < 0 ? 0 : (v > t_max ? t_max : v); }

// Pool page of logical page pi of sequence b; an entry outside [0, num_pages) is flagged
// DIFFQKV_ERR_DEVICE_PAGE and page 0 used in its place, so no access leaves the pools.
__device__ __forceinline__ int paged_page(const TopvArgs &a, int b, int pi) {
    const int e = __ldg(a.block_table + (size_t)b * a.max_blocks + pi);
    if (e >= 0 && e < a.num_pages) return e;
    record_error(a.status, DIFFQKV_ERR_DEVICE_PAGE);
    return 0;
}

// Cache row of position j of sequence b: [row][heads][d] indexing of the K and V caches or pools.
__device__ __forceinline__ long long cache_row(const TopvArgs &a, int b, int j) {
    if (!a.block_table) return (long long)b * a.t_max + j;
    return (long long)paged_page(a, b, j / a.page_size) * a.page_size + j % a.page_size;
}

// Order-preserving map of finite floats onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
    const uint32_t u = __float_as_uint(f);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float key_float(uint32_t k) {
    return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Bound of |tensor-core score - exact dot| for a row.  Every bf16 x bf16 product is exact in
// fp32 (or, below the normal range, flushed: at most 2^-126 each).  The MMA adds the products
// (16 per instruction, then the fp32 accumulator) in an order and with a rounding the PTX
// documentation leaves open.  The bound is that of the truncating block-addition model that
// published measurements found on earlier tensor cores: each block of 16 products and the
// accumulator is aligned to its largest operand and truncated, which loses less than one fp32 ulp
// (2^-23 relative) per operand, so n products lose less than gamma with nu = n (1 + 1/16) 2^-23,
// times sum_c |q_c k_c| <= ||q||_1 max|k|.  1.01 covers the rounding of this formula.  A GPU test
// measures the scores' error against it (worst seen: 0.05 of it).
template <int DK>
__device__ __forceinline__ float score_error_bound(float q_l1, float kmax) {
    const double nu = (double)DK * (17.0 / 16.0) * 1.1920928955078125e-07;  // n (1 + 1/16) 2^-23
    const float gamma = (float)(nu / (1.0 - nu));
    return __fmul_ru(__fmul_ru(__fmul_ru(1.01f, gamma), q_l1), kmax) + (float)DK * 1.1754943508e-38f;
}

// ------------------------------------------------------------------ waits between CTAs

__device__ __forceinline__ uint32_t ld_acquire(const uint32_t *p) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Release add at GPU scope.  After a __syncthreads, one by thread 0 publishes every write the CTA
// made before it (release is cumulative over the writes the barrier ordered before it); a
// reader's ld.acquire of the value, a __syncthreads, and L2 loads see them all.
__device__ __forceinline__ void red_release_add(uint32_t *p, uint32_t v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Thread 0 waits, for at most limit_ns, until *ctr >= target; false when the wait ran out
// (DIFFQKV_ERR_DEVICE_TIMEOUT recorded).
__device__ bool wait_at_least(const uint32_t *ctr, uint32_t target, const TopvArgs &a) {
    if (ld_acquire(ctr) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire(ctr) < target) {
        __nanosleep(64);
        if (globaltimer_ns() - t0 > a.wait_limit_ns) {
            record_error(a.status, DIFFQKV_ERR_DEVICE_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Every thread of the CTA calls this; thread 0 waits (bounded) until *ctr >= target.  Returns
// false for the whole CTA when the wait ran out.  Data the arriving CTAs wrote is read
// afterwards with L2 loads (__ldcg).
__device__ bool cta_wait_at_least(const uint32_t *ctr, uint32_t target, const TopvArgs &a, volatile int *flag) {
    __syncthreads();
    if (threadIdx.x == 0) *flag = wait_at_least(ctr, target, a) ? 1 : 0;
    __syncthreads();
    const bool ok = *flag != 0;
    __syncthreads();
    return ok;
}

// Every thread calls this after its global writes: they become visible before *ctr grows by one.
__device__ __forceinline__ void cta_arrive(uint32_t *ctr) {
    __syncthreads();
    if (threadIdx.x == 0) red_release_add(ctr, 1u);
}

// ------------------------------------------------------------------ block helpers

// Warp-aggregated shared-memory histogram increment; `bucket` < 0 skips.
__device__ __forceinline__ void hist_add(uint32_t *hist, int bucket) {
    const unsigned peers = __match_any_sync(0xffffffffu, bucket);
    const int leader = __ffs(peers) - 1;
    if (bucket >= 0 && (threadIdx.x & 31) == leader) atomicAdd(hist + bucket, (uint32_t)__popc(peers));
}

// Block-wide exclusive prefix sum of one value per thread (thread order).
// warp_sums needs 33 entries; returns the exclusive prefix and the block total.
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

// Block-wide: the bucket d that holds the kk-th largest element (kk >= 1) of a
// shared histogram of nb buckets, and the count strictly above it, into
// *d_out / *above_out (shared).  Thread t scans a span of buckets from the top.
__device__ void find_bucket_from_top(const uint32_t *hist, int nb, uint32_t kk, int *d_out, uint32_t *above_out,
                                     uint32_t *warp_sums) {
    const int span = (nb + blockDim.x - 1) / blockDim.x;
    const int top = nb - 1 - (int)threadIdx.x * span;
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

// Warp-wide version on a global histogram of 2048 buckets (L2 loads): lane l
// holds buckets [2048 - 64 (l + 1), 2048 - 64 l).  Every lane gets the bucket
// holding the kk-th largest element and the count above it.
__device__ void warp_find_bucket_2048(const uint32_t *hist, uint32_t kk, int *d_out, uint32_t *above_out) {
    const int lane = threadIdx.x & 31;
    const int lo = kHistBuckets - 64 * (lane + 1);
    uint4 w[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) w[i] = __ldcg(reinterpret_cast<const uint4 *>(hist + lo) + i);
    uint32_t mine = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) mine += w[i].x + w[i].y + w[i].z + w[i].w;
    uint32_t incl = mine;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const uint32_t excl = incl - mine;
    const bool hit = mine > 0 && excl < kk && kk <= incl;
    int d = 0;
    uint32_t above = 0;
    if (hit) {
        // from the lane's top bucket down; constant indices keep w in registers
        above = excl;
        bool found = false;
#pragma unroll
        for (int i = 15; i >= 0; --i) {
            const uint32_t c4[4] = {w[i].w, w[i].z, w[i].y, w[i].x};  // buckets lo + 4i + 3 .. lo + 4i
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                if (!found) {
                    if (above + c4[e] >= kk) {
                        d = lo + 4 * i + 3 - e;
                        found = true;
                    } else {
                        above += c4[e];
                    }
                }
            }
        }
    }
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    const int src = m ? __ffs(m) - 1 : 0;
    *d_out = __shfl_sync(0xffffffffu, d, src);
    *above_out = __shfl_sync(0xffffffffu, above, src);
}

// ------------------------------------------------------------------ exact keys

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
#pragma unroll 1
    for (int c8 = 0; c8 < DK / 8; ++c8) {
        const uint4 kw = __ldg(reinterpret_cast<const uint4 *>(kbits + 8 * c8));
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
// summed (the range is warp-uniform); lane 0 normalises and writes.  Out of line, so that the one
// copy of its code can be fetched ahead of the select (see the warm-up in phase 1).
template <int DK>
__device__ __noinline__ void exact_key_warp(const uint16_t *qbits, const uint16_t *kbits, int j, uint32_t *out, int lane) {
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
            const long long c = acc[i] >> 32;
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

// ------------------------------------------------------------------ the kernel

// mbarriers: ring full / empty, TMEM buffer full / empty, and the MMA drain
constexpr int kBarBytes = (2 * kMaxStages + 2 * kTmemBufs + 1) * 8;
// Bytes before the ring: q as the MMA's B operand (128-byte swizzled, 1024-byte aligned), barriers,
// q in fp32, histograms, rounded up to the ring's 1024-byte alignment.
__host__ __device__ constexpr int head_bytes(int dk, int qpk) {
    return (kQRows * dk * 2 + kBarBytes + qpk * dk * 4 + qpk * kHistWords * 4 + 1023) / 1024 * 1024;
}

// Two bf16 per word: the result's halves have the larger magnitude of each pair (their signs are
// the XOR of the inputs' signs, which the caller masks off).
__device__ __forceinline__ uint32_t bf16x2_absmax(uint32_t a, uint32_t b) {
    uint32_t r;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
    return r;
}

// Small shared state of the kernel (statically allocated).
struct Shared {
    int flag;               // broadcast of a wait's outcome
    int abort_flag;         // the mbarrier waits' CTA-wide abort
    int sh_d;
    uint32_t sh_above;
    int sh_cnt_in, sh_na, sh_done;
    float lower[16];        // per row of the group: candidates are scores >= lower
    float red[kWarps];
    uint32_t warp_sums[33];
    uint16_t qbits[128];
    uint32_t keys[kPairwiseMax][kKeyWords];
    int32_t alist[kPairwiseMax];
    uint32_t emit_total[16];
    uint32_t emit_base[16];
    int32_t table[kTableWin];       // paged producer: block-table entries of pages tbl0 .. tbl0 + kTableWin - 1
    float sel_m, sel_full;          // the selected row's weight maximum and full softmax sum (0: renormalise)
    int small_n;                    // select: candidates left after the first radix pass (when few)
    uint32_t small_keys[32], small_tau;
    int sel_n;                      // its kept positions
    uint32_t tmem_base;             // the score buffers' TMEM address
};

// K tensor maps: m[0] has kTile-row boxes over a contiguous cache; over a paged pool m[i] has
// (8 << i)-row boxes, for the heights that divide the page size (i <= TopvArgs::max_box_log).
struct KMaps {
    CUtensorMap m[4];
};

template <int DK, int DV, int QPK>
__global__ void __launch_bounds__(kThreads, 1)
    topv_fused_kernel(const __grid_constant__ KMaps maps, const TopvArgs a) {
    constexpr int TILE_BYTES = kTile * DK * 2;
    constexpr int KB = DK / 64;            // 64-element (128-byte) column blocks of a K row
    static_assert(kTile == 128 && kTile <= 256, "the MMA's M and the TMA box height");
    static_assert(QPK <= kQRows && DK <= 128 && DK % 64 == 0, "shape");
    static_assert(kProducerWarp < kWarps && kMmaWarp < kWarps, "warp roles");

    // dynamic shared memory: q_b [KB][kQRows][128 B] (bf16, 128-byte swizzled) | barriers |
    // q [QPK][DK] fp32 | histograms [QPK][kHistWords] | ring [stages][TILE_BYTES] (1024-byte
    // aligned for the 128-byte swizzle).  The select and the gather reuse the ring ("overlay");
    // what sits before it is never overwritten.  The part's scores live in TMEM.
    extern __shared__ uint8_t dsm_raw[];
    uint8_t *const base = align_smem_1024(dsm_raw);
    uint8_t *const q_b = base;
    uint64_t *const full_bar = reinterpret_cast<uint64_t *>(base + kQRows * DK * 2);
    uint64_t *const empty_bar = full_bar + kMaxStages;
    uint64_t *const tfull_bar = empty_bar + kMaxStages;
    uint64_t *const tempty_bar = tfull_bar + kTmemBufs;
    uint64_t *const mma_done = tempty_bar + kTmemBufs;
    float *const q_s = reinterpret_cast<float *>(base + kQRows * DK * 2 + kBarBytes);
    uint32_t *const hist_s = reinterpret_cast<uint32_t *>(q_s + QPK * DK);
    uint8_t *const ring = base + head_bytes(DK, QPK);
    uint8_t *const overlay = ring;
    __shared__ Shared sh;
    volatile int *const abort_flag = &sh.abort_flag;
    volatile int *const flag = &sh.flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int Y = a.parts;
    const int units = a.batch * a.n_k;
    const int K = a.topk;

    if (tid == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1 + 4);  // the MMAs' commit and the consuming warpgroup
        }
        for (int s = 0; s < kTmemBufs; ++s) {
            mbar_init(&tfull_bar[s], 1);
            mbar_init(&tempty_bar[s], 4);
        }
        mbar_init(mma_done, 1);
        sh.abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&sh.tmem_base, kTmemCols);
        tmem_relinquish();
    }
    if (warp == kProducerWarp && lane == 0) {
        prefetch_tensormap(&maps.m[0]);
        if (a.block_table) {
            prefetch_tensormap(&maps.m[1]);
            prefetch_tensormap(&maps.m[2]);
            prefetch_tensormap(&maps.m[3]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    long long ring_k = 0;  // tiles this CTA has put through its ring (all rounds): barrier phases
    for (int round = 0; round < a.rounds; ++round) {
        const int u = round * a.units_per_round + (int)blockIdx.x / Y;
        const int j = (int)blockIdx.x % Y;
        if (u >= units) break;
        const int b = u / a.n_k, g = u % a.n_k;
        const int raw_len = __ldg(a.seq_lens + b);
        const int T = clamp_len(raw_len, a.t_max);
        const int nt = (T + kTile - 1) / kTile;
        const int tb = (int)(((long long)nt * j) / Y), te = (int)(((long long)nt * (j + 1)) / Y);
        const int p0 = tb * kTile;                       // first position of this part
        const int np = max(0, min(T, te * kTile) - p0);  // positions of this part
        const int row0 = b * a.n_q + g * QPK;            // first row of the group
        uint32_t *const usync = a.unit_sync + (size_t)u * 4;
        // a length outside [0, t_max] is clamped and flagged once per sequence
        if (j == 0 && g == 0 && tid == 0 && raw_len != T) record_error(a.status, DIFFQKV_ERR_DEVICE_SEQLEN);

        // =============================================================== 1. scores
        for (int i = tid; i < QPK * kHistWords; i += kThreads) hist_s[i] = 0;
        for (int i = tid; i < QPK * DK; i += kThreads) {
            const int hh = i / DK, c = i % DK;
            q_s[i] = __bfloat162float(a.q[((size_t)row0 + hh) * DK + c]);
        }
        // q as the MMA's B operand: row n (n < QPK; zero beyond) of 64-element block kb at
        // kb * kQRows * 128 + n * 128, 16-byte chunk c at chunk position c ^ (n % 8) (128-byte swizzle)
        for (int i = tid; i < kQRows * DK / 2; i += kThreads) {
            const int n = i / (DK / 2), c2 = i % (DK / 2);  // elements 2 c2 and 2 c2 + 1 of row n
            uint32_t w = 0u;
            if (n < QPK) w = __ldg(reinterpret_cast<const uint32_t *>(a.q + ((size_t)row0 + n) * DK) + c2);
            const int c = 2 * c2, kb = c / 64, chunk = (c % 64) / 8;
            *reinterpret_cast<uint32_t *>(q_b + kb * (kQRows * 128) + n * 128 + ((chunk ^ (n & 7)) << 4) +
                                          (c % 8) * 2) = w;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // q_b is read by the tensor core
        __syncthreads();
        if (warp == kProducerWarp && a.block_table) {
            // ---- producer, paged caches (the whole warp).  A tile's rows are covered greedily by
            //      aligned boxes of 8, 16, 32 or 64 rows (heights that divide the page, so a box never
            //      leaves its page), or by one whole-tile box when the page size is a multiple of the
            //      tile; lane f issues box f, so a tile's boxes leave as one warp instruction (one lane
            //      issuing them all measured slower).  The block-table entries sit in shared memory, a
            //      window of kTableWin pages loaded at once; an entry is checked when a box uses it.
            //      Only pages holding cached positions are read (later entries may hold anything);
            //      rows past the sequence inside a loaded box are harmless.
            if (te > tb) {
                if (lane == 0) asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                __syncwarp();
                const long long k0 = ring_k;
                auto covered = [&](int t) { return (min(kTile, T - t * kTile) + 7) & ~7; };  // rows loaded
                // position -> page and row: shifts for power-of-two pages (a runtime division is dozens
                // of instructions, and this warp shares its sub-partition with consumer warps)
                const int ps = a.page_shift;
                auto pdiv = [&](int x) { return ps >= 0 ? x >> ps : x / a.page_size; };
                auto pmod = [&](int x) { return ps >= 0 ? x & (a.page_size - 1) : x % a.page_size; };
                auto first_page = [&](int t) { return pdiv(t * kTile); };
                // the part's block-table entries, a window of kTableWin pages at a time, loaded into
                // shared memory by the whole warp in one round trip (per-tile copies of a few entries
                // cost this warp more than they saved); entries for pages past the sequence's are
                // never loaded
                const int pages_seq = T > 0 ? pdiv(((T + 7) & ~7) - 1) + 1 : 0;
                int tbl0 = -kTableWin;
                int st = (int)(k0 % a.stages);
                uint32_t par = (uint32_t)((k0 / a.stages) & 1);
                bool wrapped = k0 >= a.stages;
                long long issued_end = k0;
                for (int t = tb; t < te; ++t) {
                    const int last_page = pdiv(t * kTile + covered(t) - 1);
                    if (last_page >= tbl0 + kTableWin) {  // (the same decision in every lane)
                        tbl0 = first_page(t);
                        const int cnt = min(kTableWin, pages_seq - tbl0);
                        __syncwarp();
                        for (int i = lane; i < cnt; i += 32)
                            sh.table[i] = __ldg(a.block_table + (size_t)b * a.max_blocks + tbl0 + i);
                        __syncwarp();
                    }
                    if (wrapped) mbar_wait_bounded(&empty_bar[st], par ^ 1u, a.wait_limit_ns, abort_flag, a.status);
                    if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
                    const int start = t * kTile, end = start + (a.tile_box ? kTile : covered(t));
                    int cur = a.tile_box ? end : start, f = 0, my_cur = -1, my_hi = 0;
                    if (a.tile_box && lane == 0) my_cur = start;
                    if (!a.tile_box && ps >= 0 && end - start == kTile) {
                        // a full tile over power-of-two pages: every box is 8 << max_box_log rows
                        const int rows = 8 << a.max_box_log;
                        if (lane < kTile / rows) {
                            my_cur = start + lane * rows;
                            my_hi = a.max_box_log;
                        }
                        cur = end;
                    }
                    // otherwise every lane walks the same greedy decomposition and keeps box `lane`
                    while (cur < end) {
                        int hi = a.max_box_log;
                        while (hi > 0 && ((cur & ((8 << hi) - 1)) != 0 || cur + (8 << hi) > end)) --hi;
                        if (f == lane) {
                            my_cur = cur;
                            my_hi = hi;
                        }
                        cur += 8 << hi;
                        ++f;
                    }
                    uint8_t *dst = ring + (size_t)st * TILE_BYTES;
                    if (lane == 0) mbar_arrive_expect_tx(&full_bar[st], (uint32_t)((end - start) * DK * 2));
                    __syncwarp();
                    if (my_cur >= 0) {
                        int page = sh.table[pdiv(my_cur) - tbl0];
                        if (page < 0 || page >= a.num_pages) {  // flagged; pool page 0 read in its place
                            record_error(a.status, DIFFQKV_ERR_DEVICE_PAGE);
                            page = 0;
                        }
                        // constant indices keep the descriptors in the kernel's parameter space
                        const CUtensorMap *tm = my_hi == 0 ? &maps.m[0]
                                                : my_hi == 1 ? &maps.m[1]
                                                : my_hi == 2 ? &maps.m[2]
                                                             : &maps.m[3];
#pragma unroll
                        for (int kb = 0; kb < DK / 64; ++kb)
                            tma_load_4d(dst + kb * (kTile * 128) + (my_cur - start) * 128, tm, &full_bar[st], kb * 64,
                                        g, pmod(my_cur), page);
                    }
                    issued_end = k0 + (t - tb) + 1;
                    if (++st == a.stages) {
                        st = 0;
                        par ^= 1u;
                        wrapped = true;
                    }
                }
                if (lane == 0)
                    for (long long kk = (issued_end - a.stages > k0 ? issued_end - a.stages : k0); kk < issued_end; ++kk)
                        mbar_wait_bounded(&full_bar[kk % a.stages], (uint32_t)((kk / a.stages) & 1), a.wait_limit_ns,
                                          nullptr, a.status);
            }
        } else if (warp == kProducerWarp) {
            // ---- producer: one lane issues the TMA loads of this part's tiles into the ring
            if (lane == 0 && te > tb) {
                // the ring may hold the previous round's select and gather data, written by the generic proxy
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                const long long k0 = ring_k;
                long long issued_end = k0;
                // ring position of tile kk: stage kk mod stages, fill round kk / stages (its parity);
                // kept incrementally (a 64-bit division per tile costs dozens of instructions)
                int st = (int)(k0 % a.stages);
                uint32_t par = (uint32_t)((k0 / a.stages) & 1);
                bool wrapped = k0 >= a.stages;
                for (int t = tb; t < te; ++t) {
                    const long long kk = k0 + (t - tb);
                    // the slot's previous fill (round - 1) must have been consumed
                    if (wrapped)
                        mbar_wait_bounded(&empty_bar[st], par ^ 1u, a.wait_limit_ns, abort_flag, a.status);
                    if (*abort_flag) break;
                    uint8_t *dst = ring + (size_t)st * TILE_BYTES;
                    mbar_arrive_expect_tx(&full_bar[st], TILE_BYTES);
#pragma unroll
                    for (int kb = 0; kb < DK / 64; ++kb)
                        tma_load_4d(dst + kb * (kTile * 128), &maps.m[0], &full_bar[st], kb * 64, g, t * kTile, b);
                    issued_end = kk + 1;
                    if (++st == a.stages) {
                        st = 0;
                        par ^= 1u;
                        wrapped = true;
                    }
                }
                // drain: every copy into the ring has landed before the CTA moves on
                for (long long kk = (issued_end - a.stages > k0 ? issued_end - a.stages : k0); kk < issued_end; ++kk)
                    mbar_wait_bounded(&full_bar[kk % a.stages], (uint32_t)((kk / a.stages) & 1), a.wait_limit_ns,
                                      nullptr, a.status);
            }
        } else if (warp == kMmaWarp) {
            // ---- MMA issuer: S(tile) = K_tile q^T into TMEM buffer k % kTmemBufs (lane = position of
            //      the tile, column = row of the group).  The commits free the ring slot (together with
            //      the consuming warpgroup, which reads the slot's K rows for max |k|) and hand the
            //      buffer to the consumers.
            if (lane == 0 && te > tb) {
                constexpr uint32_t idesc = umma_idesc_bf16(kTile, kQRows, false, false);
                const uint32_t qb_addr = smem_addr(q_b);
                const long long k0 = ring_k;
                int st = (int)(k0 % a.stages);
                uint32_t par = (uint32_t)((k0 / a.stages) & 1);
                for (int t = tb; t < te; ++t) {
                    const long long kk = k0 + (t - tb);
                    const int tb_i = (int)(kk & (kTmemBufs - 1));
                    if (!mbar_wait_bounded(&full_bar[st], par, a.wait_limit_ns, abort_flag, a.status)) break;
                    // the buffer's previous tile (kk - kTmemBufs) has been read out
                    if (kk >= kTmemBufs &&
                        !mbar_wait_bounded(&tempty_bar[tb_i], (uint32_t)(((kk >> 3) & 1) ^ 1), a.wait_limit_ns,
                                           abort_flag, a.status))
                        break;
                    tc_fence_after();
                    const uint32_t k_addr = smem_addr(ring + (size_t)st * TILE_BYTES);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks) {
                        const uint32_t blk = (uint32_t)(ks >> 2), sub = (uint32_t)(ks & 3) * 32u;
                        const uint64_t da = smem_desc_sw128(k_addr + blk * (kTile * 128) + sub, 16, 1024);
                        const uint64_t db = smem_desc_sw128(qb_addr + blk * (kQRows * 128) + sub, 16, 1024);
                        umma_bf16(tmem + (uint32_t)(tb_i * kQRows), da, db, idesc, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&tfull_bar[tb_i]);
                    umma_commit(&empty_bar[st]);
                    if (++st == a.stages) {
                        st = 0;
                        par ^= 1u;
                    }
                }
            }
            __syncwarp();
        } else if (warp < kConsumerWarps) {
            // ---- consumers: warpgroup cg takes the part's tiles cg, cg + 3, ...; thread (warp % 4,
            //      lane) owns position 32 (warp % 4) + lane of a tile: its scores (TMEM lane = position)
            //      and its K row (for max |k|)
            const int cg = warp >> 2, quarter = warp & 3;
            const int pos = quarter * 32 + lane;                      // row of the tile
            const uint32_t t_lane = tmem + ((uint32_t)(quarter * 32) << 16);
            uint32_t kacc = 0u;  // two bf16 whose magnitudes bound every |k| seen
            long long kk = ring_k + cg;
            int st = (int)(kk % a.stages);
            uint32_t par = (uint32_t)((kk / a.stages) & 1);
            for (int t = tb + cg; t < te; t += kConsumerGroups) {
                const int tb_i = (int)(kk & (kTmemBufs - 1));
                if (!mbar_wait_bounded(&tfull_bar[tb_i], (uint32_t)((kk >> 3) & 1), a.wait_limit_ns, abort_flag,
                                       a.status))
                    break;
                tc_fence_after();
                uint32_t sr[QPK];
                tmem_ld_cols<QPK>(t_lane + (uint32_t)(tb_i * kQRows), sr);
                tmem_wait_ld();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty_bar[tb_i]);
                const int lp = (t - tb) * kTile + pos;  // position within this part
                const bool valid = lp < np;
                // this position's K row: every 16-byte chunk once, in an order that spreads the
                // warp's loads over all banks (the max does not depend on the order)
                mbar_wait_bounded(&full_bar[st], par, a.wait_limit_ns, abort_flag, a.status);
                const uint8_t *krow = ring + (size_t)st * TILE_BYTES + pos * 128;
                uint4 kv[8 * KB];
#pragma unroll
                for (int c = 0; c < 8 * KB; ++c)
                    kv[c] = lds128(krow + (c / 8) * (kTile * 128) + (((c + lane) & 7) << 4));
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty_bar[st]);
                if (valid) {
#pragma unroll
                    for (int c = 0; c < 8 * KB; ++c) {
                        kacc = bf16x2_absmax(kacc, kv[c].x);
                        kacc = bf16x2_absmax(kacc, kv[c].y);
                        kacc = bf16x2_absmax(kacc, kv[c].z);
                        kacc = bf16x2_absmax(kacc, kv[c].w);
                    }
#pragma unroll
                    for (int hh = 0; hh < QPK; ++hh) {
                        const uint32_t bk = float_key(__uint_as_float(sr[hh])) >> 21;
                        atomicAdd(hist_s + hh * kHistWords + (bk >> 1), 1u << ((bk & 1u) << 4));
                    }
                }
                // the part keeps its scores in TMEM: tile t's rows at columns kScoreCol0 + (t - tb) QPK
                const int col = kScoreCol0 + (t - tb) * QPK;
                if (in_bounds(col + QPK - 1, kTmemCols, a.status))
                    tmem_st_cols<QPK>(t_lane + (uint32_t)col, sr);
                kk += kConsumerGroups;
                st += kConsumerGroups;
                while (st >= a.stages) {
                    st -= a.stages;
                    par ^= 1u;
                }
            }
            tmem_wait_st();
            tc_fence_before();  // the scores' stores, before the barrier that ends the phase
            // largest |k| as a bf16 magnitude pattern (order-preserving for non-negative values)
            uint32_t kmx = max(kacc & 0x7fffu, (kacc >> 16) & 0x7fffu);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) kmx = max(kmx, __shfl_xor_sync(0xffffffffu, kmx, off));
            if (lane == 0 && kmx) atomicMax(usync + kUsKmax, kmx);
        } else if (warp == kWarps - 1 && j < QPK && T > K) {
            // idle in phase 1: run the exact-key code once on a scratch key (the cache's first K row
            // against itself), so that a select CTA finds it in the instruction caches instead of
            // fetching it on the critical path
            const uint16_t *k0 = reinterpret_cast<const uint16_t *>(a.k);
            exact_key_warp<DK>(k0, k0, 0, sh.keys[kPairwiseMax - 1], lane);
        }
        ring_k += te - tb;
        __syncthreads();
        if (*abort_flag) goto finish;  // a ring wait ran out (recorded); the producer has drained
        // the part's histograms (word i: buckets 2i and 2i + 1) into the rows' global histograms
        for (int i = tid; i < QPK * kHistWords; i += kThreads) {
            const uint32_t w = hist_s[i];
            uint32_t *gh = a.hist1 + ((size_t)row0 + i / kHistWords) * kHistBuckets + 2 * (i % kHistWords);
            if (w & 0xffffu) atomicAdd(gh, w & 0xffffu);
            if (w >> 16) atomicAdd(gh + 1, w >> 16);
        }
        cta_arrive(usync + kUsHist);

        // =============================================================== 2. candidates
        if (!cta_wait_at_least(usync + kUsHist, (uint32_t)Y, a, flag)) goto finish;
        if (warp < QPK) {
            const int row = row0 + warp;
            float lower = -INFINITY;
            int d = -1;
            uint32_t above = 0;
            float two_d = 0.f;
            if (T > K) {
                warp_find_bucket_2048(a.hist1 + (size_t)row * kHistBuckets, (uint32_t)K, &d, &above);
                float q1 = 0.f;
                for (int c = lane; c < DK; c += 32) q1 += fabsf(q_s[warp * DK + c]);
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) q1 += __shfl_xor_sync(0xffffffffu, q1, off);
                const uint32_t kmax_bits = __ldcg(usync + kUsKmax);
                two_d = __fmul_ru(2.f, score_error_bound<DK>(q1, __uint_as_float(kmax_bits << 16)));
                // (bucket 0 starts at the NaN patterns: everything in it and above is a candidate)
                lower = d == 0 ? -INFINITY : __fsub_rd(key_float((uint32_t)d << 21), two_d);
            }
            if (lane == 0) {
                sh.lower[warp] = lower;
                if (j == 0) {
                    a.rowinfo[kRowInfoWords * row + kRiBucket] = (uint32_t)d;
                    a.rowinfo[kRowInfoWords * row + kRiAbove] = above;
                    a.rowinfo[kRowInfoWords * row + kRiTwoDelta] = __float_as_uint(two_d);
                }
            }
        }
        __syncthreads();
        tc_fence_after();  // the scores the consumers stored to TMEM in phase 1
        // The part's scores, read back out of TMEM: warp w reads TMEM lanes 32 (w % 4) .. + 31 (the
        // positions 32 (w % 4) + lane of a tile), 16 columns = TPL consecutive tiles per load, the
        // blocks of TPL tiles dealt to the four warps of a lane quarter in turn; f(lp, valid, s)
        // sees position lp of the part and its QPK scores s[0 .. QPK).  (A part has at most
        // kScoreCols / QPK tiles, a multiple of TPL, so no load reaches past the allocation.)
        constexpr int TPL = 16 / QPK;
        auto for_each_score = [&](auto &&f) {
            const uint32_t t_lane = tmem + ((uint32_t)((warp & 3) * 32) << 16);
            const int ntl = te - tb;
            for (int i0 = (warp >> 2) * TPL; i0 < ntl; i0 += (kWarps / 4) * TPL) {
                uint32_t sr[16];
                tmem_ld_cols<16>(t_lane + (uint32_t)(kScoreCol0 + i0 * QPK), sr);
                tmem_wait_ld();
#pragma unroll
                for (int k = 0; k < TPL; ++k) {
                    const int lp = (i0 + k) * kTile + (warp & 3) * 32 + lane;
                    f(lp, i0 + k < ntl && lp < np, sr + k * QPK);
                }
            }
        };
        if (a.full_weights && T > K) {
            // this part's share of each row's full softmax denominator: its max and its sum of exponentials
            float mx[QPK], sum[QPK];
#pragma unroll
            for (int hh = 0; hh < QPK; ++hh) mx[hh] = -INFINITY, sum[hh] = 0.f;
            for_each_score([&](int, bool valid, const uint32_t *sr) {
                if (valid)
#pragma unroll
                    for (int hh = 0; hh < QPK; ++hh) mx[hh] = fmaxf(mx[hh], __uint_as_float(sr[hh]));
            });
            for (int hh = 0; hh < QPK; ++hh) {
                float m = mx[hh];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
                if (lane == 0) sh.red[warp] = m;
                __syncthreads();
                m = sh.red[0];
                for (int w = 1; w < kWarps; ++w) m = fmaxf(m, sh.red[w]);
                __syncthreads();
                mx[hh] = m;
            }
            for_each_score([&](int, bool valid, const uint32_t *sr) {
                if (valid)
#pragma unroll
                    for (int hh = 0; hh < QPK; ++hh)
                        if (mx[hh] != -INFINITY)
                            sum[hh] += fast_exp2((__uint_as_float(sr[hh]) - mx[hh]) * a.scale_log2);
            });
            for (int hh = 0; hh < QPK; ++hh) {
                float v = sum[hh];
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) sh.red[warp] = v;
                __syncthreads();
                if (tid == 0) {
                    float tot = 0.f;
                    for (int w = 0; w < kWarps; ++w) tot += sh.red[w];
                    a.chunk_part[(size_t)(row0 + hh) * kMaxParts + j] = make_float2(mx[hh], tot);
                }
                __syncthreads();
            }
        }
        // emit candidates: each thread counts its hits per row (first pass over its scores), one
        // block scan of the counts plus one atomic per (CTA, row) gives every hit its slot in the
        // row's candidate list, and the second pass writes them
        {
            uint32_t cnt[QPK];
#pragma unroll
            for (int hh = 0; hh < QPK; ++hh) cnt[hh] = 0u;
            for_each_score([&](int, bool valid, const uint32_t *sr) {
#pragma unroll
                for (int hh = 0; hh < QPK; ++hh) cnt[hh] += (valid && __uint_as_float(sr[hh]) >= sh.lower[hh]) ? 1u : 0u;
            });
            // exclusive prefix of every row's hit count, two rows per scan (16-bit fields: a part holds
            // at most kScoreCols / QPK * kTile <= 49152 positions)
            uint32_t slot[QPK];
#pragma unroll
            for (int hh = 0; hh < QPK; hh += 2) {
                const uint32_t packed = cnt[hh] | (hh + 1 < QPK ? cnt[hh + 1 < QPK ? hh + 1 : hh] << 16 : 0u);
                uint32_t total;
                const uint32_t ex = block_exclusive_scan(packed, sh.warp_sums, &total);
                slot[hh] = ex & 0xffffu;
                if (hh + 1 < QPK) slot[hh + 1 < QPK ? hh + 1 : hh] = ex >> 16;
                if (tid == 0) {
                    sh.emit_total[hh] = total & 0xffffu;
                    if (hh + 1 < QPK) sh.emit_total[hh + 1] = total >> 16;
                }
            }
            __syncthreads();
            if (tid < QPK)
                sh.emit_base[tid] = sh.emit_total[tid]
                                        ? atomicAdd(a.row_sync + (size_t)(row0 + tid) * 4 + kRsCand, sh.emit_total[tid])
                                        : 0u;
            __syncthreads();
#pragma unroll
            for (int hh = 0; hh < QPK; ++hh) slot[hh] += sh.emit_base[hh];
            for_each_score([&](int lp, bool valid, const uint32_t *sr) {
#pragma unroll
                for (int hh = 0; hh < QPK; ++hh) {
                    const float x = __uint_as_float(sr[hh]);
                    if (valid && x >= sh.lower[hh]) {
                        if (slot[hh] < (uint32_t)a.t_pad) {  // (a count left over by an aborted call stays in bounds)
                            a.cand_j[(size_t)(row0 + hh) * a.t_pad + slot[hh]] = p0 + lp;
                            a.cand_s[(size_t)(row0 + hh) * a.t_pad + slot[hh]] = x;
                        }
                        ++slot[hh];
                    }
                }
            });
        }
        tc_fence_before();  // the score loads, before the barriers that let the next round's MMAs in
        cta_arrive(usync + kUsCand);

        // =============================================================== 3. select
        for (int hh = j; hh < QPK; hh += Y) {
            if (!cta_wait_at_least(usync + kUsCand, (uint32_t)Y, a, flag)) goto finish;
            const int row = row0 + hh;
            int32_t *idx = a.idx_out + (size_t)row * K;
            float *ks = a.kept_s + (size_t)row * a.k_pad;
            int32_t *kr = a.kept_row + (size_t)row * a.k_pad;
            const uint32_t nc = min(__ldcg(a.row_sync + (size_t)row * 4 + kRsCand), (uint32_t)T);
            const int nwords = (T + 31) / 32;
            // overlay: bitmap | word prefixes | histogram | candidate positions | candidate scores
            uint32_t *bitmap = reinterpret_cast<uint32_t *>(overlay);
            uint32_t *wprefix = bitmap + (a.t_pad >> 5);
            uint32_t *hist = wprefix + (a.t_pad >> 5);
            int32_t *c_j = reinterpret_cast<int32_t *>(hist + kHistBuckets);
            float *c_s = reinterpret_cast<float *>(c_j + a.cand_cap);
            const bool in_smem = nc <= (uint32_t)a.cand_cap;
            const int32_t *cj = in_smem ? c_j : a.cand_j + (size_t)row * a.t_pad;
            const float *cs = in_smem ? c_s : a.cand_s + (size_t)row * a.t_pad;
            if (tid < DK) sh.qbits[tid] = reinterpret_cast<const uint16_t *>(a.q)[(size_t)row * DK + tid];
            if (in_smem) {
                const int32_t *gj = a.cand_j + (size_t)row * a.t_pad;
                const float *gs = a.cand_s + (size_t)row * a.t_pad;
                for (uint32_t i = tid; i < nc; i += kThreads) {
                    c_j[i] = __ldcg(gj + i);
                    c_s[i] = __ldcg(gs + i);
                }
            }
            for (int i = tid; i < nwords; i += kThreads) bitmap[i] = 0u;
            __syncthreads();
            float mx = -INFINITY;
            int nsel = 0;
            if (T == 0) {
                for (int i = tid; i < K; i += kThreads) idx[i] = -1;
            } else if (T <= K) {
                // every cached position is kept: the candidate list holds them all
                for (uint32_t i = tid; i < nc; i += kThreads) {
                    const int jj = cj[i];
                    if (!in_bounds(jj, K, a.status)) continue;
                    idx[jj] = jj;
                    ks[jj] = cs[i];
                    kr[jj] = (int32_t)cache_row(a, b, jj);
                    mx = fmaxf(mx, cs[i]);
                }
                for (int i = T + tid; i < K; i += kThreads) idx[i] = -1;
                nsel = T;
            } else {
                // ---- a. tau = the K-th largest score.  Its top 11 key bits are the bucket, and `above`
                //         scores lie in higher buckets (all of them candidates); a radix select over the
                //         candidates finds the other 21 bits, 11 and then 10 at a time
                uint32_t prefix = __ldcg(a.rowinfo + kRowInfoWords * row + kRiBucket) << 21, pmask = 0xffe00000u;
                uint32_t kk = (uint32_t)K - __ldcg(a.rowinfo + kRowInfoWords * row + kRiAbove);
                for (int pass = 0; pass < 2; ++pass) {
                    const int shift = pass == 0 ? 10 : 0;
                    const int nb = pass == 0 ? kHistBuckets : kRadixBuckets;
                    if (pass == 1 && hist[sh.sh_d] <= 32u) {
                        // at most 32 candidates share the first 22 key bits: warp 0 ranks their keys
                        // directly (the kk-th largest, ties counted in slot order) instead of a
                        // block-wide histogram pass over the last 10 bits
                        if (tid == 0) sh.small_n = 0;
                        __syncthreads();
                        for (uint32_t i = tid; i < nc; i += kThreads) {
                            const uint32_t key = float_key(cs[i]);
                            if ((key & pmask) == prefix) {
                                const int sl = atomicAdd(&sh.small_n, 1);
                                if (sl < 32) sh.small_keys[sl] = key;
                            }
                        }
                        __syncthreads();
                        if (warp == 0) {
                            const int n = min(sh.small_n, 32);
                            const uint32_t my = lane < n ? sh.small_keys[lane] : 0u;
                            int greater = 0;
                            for (int jl = 0; jl < n; ++jl) {
                                const uint32_t kj = __shfl_sync(0xffffffffu, my, jl);
                                greater += (kj > my || (kj == my && jl < lane)) ? 1 : 0;
                            }
                            const unsigned hit = __ballot_sync(0xffffffffu, lane < n && greater == (int)kk - 1);
                            const uint32_t tkey = __shfl_sync(0xffffffffu, my, hit ? __ffs(hit) - 1 : 0);
                            if (lane == 0) sh.small_tau = hit ? tkey : prefix;
                        }
                        __syncthreads();
                        prefix = sh.small_tau;
                        break;
                    }
                    for (int i = tid; i < nb; i += kThreads) hist[i] = 0;
                    __syncthreads();
                    for (uint32_t base_i = 0; base_i < nc; base_i += kThreads) {
                        const uint32_t i = base_i + tid;
                        int bkt = -1;
                        if (i < nc) {
                            const uint32_t key = float_key(cs[i]);
                            if ((key & pmask) == prefix) bkt = (int)((key >> shift) & (uint32_t)(nb - 1));
                        }
                        hist_add(hist, bkt);
                    }
                    __syncthreads();
                    find_bucket_from_top(hist, nb, kk, &sh.sh_d, &sh.sh_above, sh.warp_sums);
                    prefix |= (uint32_t)sh.sh_d << shift;
                    pmask |= (uint32_t)(nb - 1) << shift;
                    kk -= sh.sh_above;
                }
                const float tau = key_float(prefix);

                // ---- b./c. the rounding bound; certain and ambiguous candidates
                const float two_d = __uint_as_float(__ldcg(a.rowinfo + kRowInfoWords * row + kRiTwoDelta));
                const float hi_edge = __fadd_ru(tau, two_d);
                const float lo_edge = __fsub_rd(tau, two_d);
                if (tid == 0) {
                    sh.sh_cnt_in = 0;
                    sh.sh_na = 0;
                }
                __syncthreads();
                int32_t *alist = a.alist + (size_t)row * a.t_pad;
                int my_in = 0;
                for (uint32_t i = tid; i < nc; i += kThreads) {
                    const float x = cs[i];
                    if (x > hi_edge) {
                        const int jj = cj[i];
                        atomicOr(bitmap + (jj >> 5), 1u << (jj & 31));
                        ++my_in;
                    } else if (x >= lo_edge) {
                        const int slot = atomicAdd(&sh.sh_na, 1);
                        alist[slot] = cj[i];
                        if (slot < kPairwiseMax) sh.alist[slot] = cj[i];
                    }
                }
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) my_in += __shfl_xor_sync(0xffffffffu, my_in, off);
                if (lane == 0 && my_in) atomicAdd(&sh.sh_cnt_in, my_in);
                __syncthreads();
                const int na = sh.sh_na;
                const int need = K - sh.sh_cnt_in;  // 1 <= need <= na when the bound holds
                // K row of position jj (exact keys of the ambiguous positions)
                auto krow = [&](int jj) {
                    long long r = cache_row(a, b, jj);
                    if (!in_bounds(r, a.cache_rows, a.status)) r = 0;
                    return reinterpret_cast<const uint16_t *>(a.k + ((size_t)r * a.n_k + g) * DK);
                };
                auto keep = [&](int jj) { atomicOr(bitmap + (jj >> 5), 1u << (jj & 31)); };
                if (need <= 0) {
                    // nothing left to choose (cannot happen when the bound holds)
                } else if (need >= na) {
                    for (int i = tid; i < na; i += kThreads) keep(__ldcg(alist + i));
                } else if (na <= kPairwiseMax) {
                    // rank the few ambiguous positions pairwise by exact key (a warp per key)
                    for (int rr = warp; rr < na; rr += kWarps) {
                        const int jj = sh.alist[rr];
                        exact_key_warp<DK>(sh.qbits, krow(jj), jj, sh.keys[rr], lane);
                    }
                    __syncthreads();
                    if (tid < na) {
                        int better = 0;
                        for (int uu = 0; uu < na; ++uu) better += key_greater(sh.keys[uu], sh.keys[tid]) ? 1 : 0;
                        if (better < need) keep(sh.alist[tid]);
                    }
                } else {
                    // radix select over the exact keys, one byte per pass (keys are unique)
                    uint8_t *ast = a.astate + (size_t)row * a.t_pad;
                    uint8_t *adg = a.adigit + (size_t)row * a.t_pad;
                    for (int i = tid; i < na; i += kThreads) ast[i] = 0;
                    if (tid == 0) sh.sh_done = 0;
                    uint32_t kk2 = (uint32_t)need;
                    __syncthreads();
                    for (int p = 0; p < kKeyWords * 4 && !sh.sh_done; ++p) {
                        for (int i = tid; i < kByteBuckets; i += kThreads) hist[i] = 0;
                        __syncthreads();
                        for (int base_i = 0; base_i < na; base_i += kThreads) {
                            const int i = base_i + tid;
                            int bkt = -1;
                            if (i < na && ast[i] == 0) {
                                uint32_t key[kKeyWords];
                                const int jj = alist[i];
                                exact_key<DK>(sh.qbits, krow(jj), jj, key);
                                bkt = (int)((key[p >> 2] >> (24 - 8 * (p & 3))) & 0xffu);
                                adg[i] = (uint8_t)bkt;
                            }
                            hist_add(hist, bkt);
                        }
                        __syncthreads();
                        find_bucket_from_top(hist, kByteBuckets, kk2, &sh.sh_d, &sh.sh_above, sh.warp_sums);
                        const int d = sh.sh_d;
                        kk2 -= sh.sh_above;
                        const bool finish = hist[d] == kk2;
                        for (int i = tid; i < na; i += kThreads) {
                            if (ast[i] != 0) continue;
                            const int dig = adg[i];
                            if (dig > d || (finish && dig == d)) ast[i] = 1;
                            else if (dig < d) ast[i] = 2;
                        }
                        if (tid == 0 && finish) sh.sh_done = 1;
                        __syncthreads();
                    }
                    for (int i = tid; i < na; i += kThreads)
                        if (ast[i] == 1) keep(alist[i]);
                }
                __syncthreads();

                // ---- d. ascending order: a kept position's slot is the number of kept
                //         positions before it, from per-word prefix counts of the bitmap
                const int wper = (nwords + kThreads - 1) / kThreads;
                const int w0 = min(nwords, tid * wper), w1 = min(nwords, w0 + wper);
                uint32_t cnt = 0;
                for (int w = w0; w < w1; ++w) cnt += __popc(bitmap[w]);
                uint32_t total;
                uint32_t run = block_exclusive_scan(cnt, sh.warp_sums, &total);
                for (int w = w0; w < w1; ++w) {
                    wprefix[w] = run;
                    run += __popc(bitmap[w]);
                }
                nsel = (int)total;
                __syncthreads();
                for (uint32_t i = tid; i < nc; i += kThreads) {
                    const int jj = cj[i];
                    const uint32_t word = bitmap[jj >> 5];
                    if ((word >> (jj & 31)) & 1u) {
                        const uint32_t slot = wprefix[jj >> 5] + __popc(word & ((1u << (jj & 31)) - 1u));
                        if (slot < (uint32_t)K) {  // more than K kept only if the bound failed (flagged below)
                            idx[slot] = jj;
                            ks[slot] = cs[i];
                            kr[slot] = (int32_t)cache_row(a, b, jj);
                            mx = fmaxf(mx, cs[i]);
                        }
                    }
                }
                if (tid == 0 && nsel != K) record_error(a.status, DIFFQKV_ERR_INVALID_ARG);
                nsel = min(nsel, K);
                for (int i = nsel + tid; i < K; i += kThreads) idx[i] = -1;
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            if (lane == 0) sh.red[warp] = mx;
            // the row's histogram returns to zero for the next call (every part of the unit read it
            // before it arrived on C)
            uint32_t *h1 = a.hist1 + (size_t)row * kHistBuckets;
            for (int i = tid; i < kHistBuckets; i += kThreads) h1[i] = 0u;
            __syncthreads();
            if (tid == 0) {
                float m = sh.red[0];
                for (int w = 1; w < kWarps; ++w) m = fmaxf(m, sh.red[w]);
                float full_sum = 0.f;  // 0: renormalise over the kept set
                if (a.full_weights && T > K) {
                    // the full softmax denominator from the parts' partials, relative to the row max
                    float M = -INFINITY;
                    for (int p = 0; p < Y; ++p) M = fmaxf(M, __ldcg(&a.chunk_part[(size_t)row * kMaxParts + p].x));
                    for (int p = 0; p < Y; ++p) {
                        const float2 pc = __ldcg(&a.chunk_part[(size_t)row * kMaxParts + p]);
                        if (pc.y > 0.f) full_sum += pc.y * fast_exp2((pc.x - M) * a.scale_log2);
                    }
                    m = M;
                }
                if (T == 0) m = 0.f;
                sh.sel_m = m;
                sh.sel_n = nsel;
                sh.sel_full = full_sum;
                a.row_sync[(size_t)row * 4 + kRsCand] = 0u;
            }
            __syncthreads();

            // ---- e. gather: this CTA sums the row's kept V rows itself (16 in flight per lane), the
            //         weights 2^((s_j - m) scale log2 e), and writes the output.  The warps' sums are
            //         added in warp order, so the result does not depend on timing.
            {
                constexpr int CPV = DV / 8;  // lanes per V row
                constexpr int RPW = 32 / CPV;  // V rows per warp step
                constexpr int GU = 16;         // V rows in flight per lane
                const int vc = lane % CPV, vs = lane / CPV;
                const int vh = (g * QPK + hh) / a.q_per_v;
                const float m = sh.sel_m;
                const int ns = sh.sel_n;
                const __nv_bfloat16 *vbase = a.v + (size_t)vh * DV + vc * 8;
                // the kept list (cache rows, scores) into shared memory in one round trip, past the
                // warps' partial sums, when it fits (the V loads below then wait on nothing else)
                float *o_s = reinterpret_cast<float *>(overlay);  // [kWarps][DV + 4] (the select is done with it)
                int32_t *kr_s = reinterpret_cast<int32_t *>(o_s + kWarps * (DV + 4));
                float *ks_s = reinterpret_cast<float *>(kr_s + ns);
                const bool kept_in_smem =
                    (size_t)kWarps * (DV + 4) * 4 + (size_t)ns * 8 <= (size_t)a.stages * kTile * DK * 2;
                if (kept_in_smem) {
                    for (int i = tid; i < ns; i += kThreads) {
                        kr_s[i] = __ldcg(kr + i);
                        ks_s[i] = __ldcg(ks + i);
                    }
                    __syncthreads();
                }
                const int32_t *krp = kept_in_smem ? kr_s : kr;
                const float *ksp = kept_in_smem ? ks_s : ks;
                const size_t vstride = (size_t)a.n_v * DV;
                float o[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] = 0.f;
                float l = 0.f;
                for (int i0 = warp * RPW + vs; i0 < ns; i0 += kWarps * RPW * GU) {
                    int jj[GU];
                    float sx[GU];
#pragma unroll
                    for (int uu = 0; uu < GU; ++uu) {
                        const int i = i0 + uu * kWarps * RPW;
                        jj[uu] = i < ns ? (kept_in_smem ? krp[i] : __ldcg(krp + i)) : -1;  // the cache row
                        if (jj[uu] >= 0 && !in_bounds(jj[uu], a.cache_rows, a.status)) jj[uu] = -1;
                        sx[uu] = i < ns ? (kept_in_smem ? ksp[i] : __ldcg(ksp + i)) : -INFINITY;
                    }
                    uint4 vv[GU];
#pragma unroll
                    for (int uu = 0; uu < GU; ++uu)
                        vv[uu] = jj[uu] >= 0 ? __ldg(reinterpret_cast<const uint4 *>(vbase + (size_t)jj[uu] * vstride))
                                             : make_uint4(0, 0, 0, 0);
#pragma unroll
                    for (int uu = 0; uu < GU; ++uu) {
                        const float w = jj[uu] >= 0 ? fast_exp2((sx[uu] - m) * a.scale_log2) : 0.f;
                        float vf[8];
                        unpack8(vv[uu], vf);
                        l += w;
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = fmaf(w, vf[e], o[e]);
                    }
                }
#pragma unroll
                for (int off = CPV; off < 32; off <<= 1) {
                    l += __shfl_xor_sync(0xffffffffu, l, off);
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
                }
                float *dst = o_s + warp * (DV + 4);
                if (vs == 0) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) dst[vc * 8 + e] = o[e];
                }
                if (lane == 0) dst[DV] = l;
                __syncthreads();
                for (int c = tid; c < DV; c += kThreads) {
                    float acc = 0.f, lt = 0.f;
                    for (int w = 0; w < kWarps; ++w) {
                        acc += o_s[w * (DV + 4) + c];
                        lt += o_s[w * (DV + 4) + DV];
                    }
                    if (sh.sel_full > 0.f) lt = sh.sel_full;
                    if (in_bounds(row, (long long)a.batch * a.n_q, a.status))
                        a.out[(size_t)row * DV + c] = __float2bfloat16(lt > 0.f ? acc / lt : 0.f);
                }
                if (tid == 0) {
                    // every select of the unit has passed its wait on C once all of them counted
                    // themselves here, and every part read H and max |k| before it arrived on C: the
                    // last one resets the unit's counters for the next call
                    if (atomicAdd(usync + kUsDone, 1u) == (uint32_t)QPK - 1) {
                        usync[kUsHist] = 0u;
                        usync[kUsCand] = 0u;
                        usync[kUsKmax] = 0u;
                        usync[kUsDone] = 0u;
                    }
                }
                __syncthreads();  // o_s and the smem state are reused by the next row
            }
        }

    }
finish:
    // the tensor memory goes back once no MMA is in flight (every exit of the loop above is taken by
    // the whole CTA)
    if (warp == kMmaWarp) {
        if (lane == 0) {
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0, a.wait_limit_ns, nullptr, a.status);
        }
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ------------------------------------------------------------------ host side

size_t align_up(size_t x, size_t al) { return (x + al - 1) / al * al; }

using TopvFn = void (*)(KMaps, TopvArgs);

template <int DK, int DV>
TopvFn pick_qpk(int qpk) {
    switch (qpk) {
        case 1: return topv_fused_kernel<DK, DV, 1>;
        case 2: return topv_fused_kernel<DK, DV, 2>;
        case 4: return topv_fused_kernel<DK, DV, 4>;
        case 8: return topv_fused_kernel<DK, DV, 8>;
        case 16: return topv_fused_kernel<DK, DV, 16>;
        default: return nullptr;
    }
}

TopvFn pick_kernel(int dk, int dv, int qpk) {
    if (dk == 64 && dv == 64) return pick_qpk<64, 64>(qpk);
    if (dk == 64 && dv == 128) return pick_qpk<64, 128>(qpk);
    if (dk == 128 && dv == 64) return pick_qpk<128, 64>(qpk);
    if (dk == 128 && dv == 128) return pick_qpk<128, 128>(qpk);
    return nullptr;
}

size_t padded_len(int32_t t_max) { return align_up((size_t)t_max, 64); }
size_t padded_k(int32_t topk) { return align_up((size_t)topk, 4); }

// Zero before the first call, left zero by every call: per unit and per row sync words, the histograms.
size_t unit_sync_bytes(const diffqkv_dims_t *d) { return align_up((size_t)d->batch * d->n_k * 16, 256); }
size_t row_sync_bytes(const diffqkv_dims_t *d) { return align_up((size_t)d->batch * d->n_q * 16, 256); }
size_t zeroed_bytes(const diffqkv_dims_t *d) {
    return unit_sync_bytes(d) + row_sync_bytes(d) + (size_t)d->batch * d->n_q * kHistBuckets * 4;
}

// Launch plan: parts per unit (Y), rounds, ring depth, shared memory.
struct Plan {
    int parts, units_per_round, rounds, stages, cand_cap, grid;
    size_t smem;
};

// Y = G / units (one round) unless a part's scores would not fit in TMEM; the ring takes as many
// stages as shared memory holds.
bool make_plan(const diffqkv_dims_t *d, int32_t t_max, int num_sms, Plan *p) {
    const int qpk = d->n_q / d->n_k;
    const int units = d->batch * d->n_k;
    const int nt_max = (t_max + kTile - 1) / kTile;
    const int G = std::min(num_sms, kMaxParts);  // one CTA per SM
    const size_t t_pad = padded_len(t_max);
    // the select's overlay: bitmap and word prefixes, a histogram, then candidates (at least 1024)
    const size_t sel_fixed = 2 * (t_pad / 8) + (size_t)kHistBuckets * 4;
    const size_t gather_bytes = (size_t)kWarps * (d->d_v + 4) * 4;
    // a part's scores stay in TMEM: at most kScoreCols / qpk tiles per part (a multiple of the
    // 16 / qpk tiles one phase-2 load reads)
    const int max_tiles = kScoreCols / qpk;
    int Y = std::max(1, std::min(G / std::max(1, units), nt_max));
    Y = std::max(Y, (nt_max + max_tiles - 1) / max_tiles);
    if (Y > G) return false;
    // dynamic bytes: 1 KB of alignment slack, the head, then the overlay (the ring, at least what the
    // select and the gather need)
    auto layout = [&](int stages, size_t *smem, int *cap) {
        const size_t ring = (size_t)stages * kTile * d->d_k * 2;
        const size_t overlay = std::max({ring, sel_fixed + 8 * 1024, gather_bytes});
        *smem = 1024 + head_bytes(d->d_k, qpk) + overlay;
        *cap = (int)std::min<size_t>((overlay - sel_fixed) / 8, t_pad);
        return *smem <= (size_t)kDynSmemCap;
    };
    size_t smem = 0;
    int cap = 0;
    int stages = 2;
    if (!layout(stages, &smem, &cap)) return false;
    while (stages < kMaxStages && layout(stages + 1, &smem, &cap)) ++stages;
    layout(stages, &smem, &cap);
    p->parts = Y;
    p->units_per_round = std::max(1, G / Y);
    p->rounds = (units + p->units_per_round - 1) / p->units_per_round;
    p->grid = std::min(units, p->units_per_round) * Y;
    p->stages = stages;
    p->cand_cap = cap;
    p->smem = smem;
    return true;
}

}  // namespace

size_t topv_workspace_size(const diffqkv_dims_t *d, int32_t t_max, int32_t topk) {
    if (validate_dims(d) != DIFFQKV_OK || t_max < 1 || topk < 1) return 0;
    const size_t rows = (size_t)d->batch * d->n_q;
    const size_t per = padded_len(t_max);
    return kTopvHeader + align_up(zeroed_bytes(d), 256) + align_up(rows * kRowInfoWords * 4, 256) +
           align_up(rows * kMaxParts * sizeof(float2), 256) +
           align_up(rows * per * 4, 256) * 3 + align_up(rows * padded_k(topk) * 4, 256) * 2 +
           align_up(rows * per, 256) * 2;
}

diffqkv_status_t topv_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, int32_t topk, void *out,
                             int32_t *idx_out, void *workspace, size_t workspace_bytes, cudaStream_t stream,
                             int32_t flags, const PagedCache *paged) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || !idx_out || t_max < 1 || topk < 1)
        return DIFFQKV_ERR_INVALID_ARG;
    if (t_max > kTopvMaxContext) return DIFFQKV_ERR_UNSUPPORTED;
    if (flags & ~DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS) return DIFFQKV_ERR_INVALID_ARG;
    int max_box_log = 0;
    if (paged) {
        if (!paged->block_table || paged->max_blocks < 1 || paged->page_size < 1 || paged->num_pages < 1 ||
            (long long)paged->max_blocks * paged->page_size != t_max)
            return DIFFQKV_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(paged->block_table) & 3u) return DIFFQKV_ERR_MISALIGNED;
        // a tile is loaded as boxes of 8, 16, 32 or 64 rows that divide the page (so each lies in one
        // page); with the 128-byte swizzle every box must start on an 8-row boundary
        if (paged->page_size % 8 != 0) return DIFFQKV_ERR_UNSUPPORTED;
        while (max_box_log < 3 && paged->page_size % (16 << max_box_log) == 0) ++max_box_log;
        if ((long long)paged->num_pages * paged->page_size > 0x7fffffffLL) return DIFFQKV_ERR_UNSUPPORTED;
    } else if ((long long)d->batch * t_max > 0x7fffffffLL) {
        return DIFFQKV_ERR_UNSUPPORTED;  // kept positions' cache rows are int32
    }
    const int qpk = d->n_q / d->n_k;
    TopvFn fn = pick_kernel(d->d_k, d->d_v, qpk);
    if (!fn) return DIFFQKV_ERR_UNSUPPORTED;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(idx_out) & 3u) || (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    const size_t need = topv_workspace_size(d, t_max, topk);
    if (!workspace || workspace_bytes < need) return DIFFQKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return DIFFQKV_ERR_MISALIGNED;
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    Plan plan;
    if (!make_plan(d, t_max, dev.num_sms, &plan)) return DIFFQKV_ERR_UNSUPPORTED;

    const size_t rows = (size_t)d->batch * d->n_q;
    const size_t t_pad = padded_len(t_max);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    TopvArgs a;
    a.status = reinterpret_cast<int32_t *>(ws);  // the workspace's own error word (header word 0)
    ws += kTopvHeader;
    a.unit_sync = reinterpret_cast<uint32_t *>(ws);
    a.row_sync = reinterpret_cast<uint32_t *>(ws + unit_sync_bytes(d));
    a.hist1 = reinterpret_cast<uint32_t *>(ws + unit_sync_bytes(d) + row_sync_bytes(d));
    ws += align_up(zeroed_bytes(d), 256);
    a.rowinfo = reinterpret_cast<uint32_t *>(ws);
    ws += align_up(rows * kRowInfoWords * 4, 256);
    a.chunk_part = reinterpret_cast<float2 *>(ws);
    ws += align_up(rows * kMaxParts * sizeof(float2), 256);
    a.cand_j = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.cand_s = reinterpret_cast<float *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.alist = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * t_pad * 4, 256);
    a.kept_s = reinterpret_cast<float *>(ws);
    ws += align_up(rows * padded_k(topk) * 4, 256);
    a.kept_row = reinterpret_cast<int32_t *>(ws);
    ws += align_up(rows * padded_k(topk) * 4, 256);
    a.astate = ws;
    ws += align_up(rows * t_pad, 256);
    a.adigit = ws;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.k = static_cast<const __nv_bfloat16 *>(k_cache);
    a.v = static_cast<const __nv_bfloat16 *>(v_cache);
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.idx_out = idx_out;
    a.batch = d->batch;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.t_max = t_max;
    a.t_pad = (int32_t)t_pad;
    a.topk = topk;
    a.k_pad = (int32_t)padded_k(topk);
    a.q_per_v = d->n_q / d->n_v;
    a.parts = plan.parts;
    a.units_per_round = plan.units_per_round;
    a.rounds = plan.rounds;
    a.stages = plan.stages;
    a.cand_cap = plan.cand_cap;
    a.full_weights = (flags & DIFFQKV_TOPV_FULL_SOFTMAX_WEIGHTS) ? 1 : 0;
    a.block_table = paged ? paged->block_table : nullptr;
    a.max_blocks = paged ? paged->max_blocks : 0;
    a.page_size = paged ? paged->page_size : 0;
    a.num_pages = paged ? paged->num_pages : 0;
    a.max_box_log = max_box_log;
    a.cache_rows = paged ? (long long)paged->num_pages * paged->page_size : (long long)d->batch * t_max;
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);
    a.wait_limit_ns = kWaitLimitNs;
    (void)max_seq_len;  // the parts adapt to the device lengths by themselves

    // K tiles {64 elements, 1 head, kTile positions, 1 sequence} of [B, t_max, n_k, d_k], or boxes
    // {64, 1, 8 << i, 1} of the pool [num_pages, page_size, n_k, d_k]; 128-byte swizzle
    KMaps maps;
    memset(&maps, 0, sizeof maps);
    const bool tile_box = paged && paged->page_size % kTile == 0;
    a.tile_box = tile_box ? 1 : 0;
    a.page_shift = -1;
    if (paged && (paged->page_size & (paged->page_size - 1)) == 0) {
        a.page_shift = 0;
        while ((1 << a.page_shift) < paged->page_size) ++a.page_shift;
    }
    if (tile_box) {
        st = make_tensor_map_4d(&maps.m[0], k_cache, d->d_k, d->n_k, paged->page_size, paged->num_pages, 64, 1,
                                kTile, 1, CU_TENSOR_MAP_SWIZZLE_128B);
        for (int i = 1; i < 4; ++i) maps.m[i] = maps.m[0];
    } else if (paged) {
        for (int i = 0; i <= max_box_log && st == DIFFQKV_OK; ++i)
            st = make_tensor_map_4d(&maps.m[i], k_cache, d->d_k, d->n_k, paged->page_size, paged->num_pages, 64, 1,
                                    8u << i, 1, CU_TENSOR_MAP_SWIZZLE_128B);
        for (int i = max_box_log + 1; i < 4; ++i) maps.m[i] = maps.m[0];
    } else {
        st = make_tensor_map_4d(&maps.m[0], k_cache, d->d_k, d->n_k, t_max, d->batch, 64, 1, kTile, 1,
                                CU_TENSOR_MAP_SWIZZLE_128B);
        for (int i = 1; i < 4; ++i) maps.m[i] = maps.m[0];
    }
    if (st != DIFFQKV_OK) return st;
    if (ensure_dynamic_smem((const void *)fn, (int)plan.smem) != DIFFQKV_OK) return DIFFQKV_ERR_CUDA;
    // parts of a unit wait on one another: the whole grid must be resident at once (cooperative launch)
    int per_sm = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kThreads, plan.smem) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    if (per_sm < 1 || plan.grid > per_sm * dev.num_sms) return DIFFQKV_ERR_UNSUPPORTED;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)plan.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = plan.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, fn, maps, a) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    return DIFFQKV_OK;
}

}  // namespace diffqkv
