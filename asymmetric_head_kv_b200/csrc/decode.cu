// decode.cu -- split/combine DiffQKV decode attention for sm_100a.
//
// Follows the split kernel + combine kernel structure of FlexHeadFA ("Sigma:
// Differential Rescaling of Query, Key and Value for Efficient Language
// Models", structured summary page, "FlexHeadFA Kernel and Deployment
// Infrastructure"): every KV chunk yields (running max, sum of exp,
// unnormalised output) and a combine step merges the chunks.  The K and V
// head of a query head are addressed separately (GroupSharing, section 3.4
// Step 3): K head h/(n_q/n_k), V head h/(n_q/n_v).
//
// B200 design (one launch, memory-bound):
//  * Work unit = (batch b, K-head group g): the n_q/n_k query heads that
//    share K head g.  One K tile in shared memory serves all of them; each
//    query head reads its own V head.
//  * The K/V token range of all units is concatenated into one tile list and
//    cut into equal contiguous ranges, one per CTA (grid = SMs x resident
//    CTAs), so ragged batches and short contexts keep every SM equally busy.
//    A CTA range may start or end inside a unit: each (unit, CTA) piece is one
//    split.
//  * One producer warp streams K and V tiles with TMA (cp.async.bulk.tensor,
//    no multicast) into a multi-stage shared-memory ring guarded by
//    mbarriers; consumer warps compute scores with 16-byte shared loads and
//    warp-shuffle reductions, keep the online softmax in the log2 domain and
//    accumulate P.V in fp32 registers.
//  * The combine is fused: the last CTA to finish a unit (atomic counter in
//    the workspace, reset afterwards) merges that unit's split partials and
//    writes bf16 output.  No CTA ever waits on another.
//  * Append mode (k_new, v_new given): the step's new token joins the cache at
//    position p = seq_len and the output attends over positions 0..p.  The
//    tiles still cover the p cached positions only; the combining CTA adds the
//    new token as one more partial (m = its score, l = 1, o = v_new) and writes
//    k_new / v_new into the cache at p, which no CTA of this launch reads.
//  * Paged caches (block table given): K and V live in two page pools
//    [num_pages, page_size, heads, d] that share one block table [B, max_blocks]
//    (position j of sequence b is row j % page_size of pool page
//    table[b][j / page_size]).  The tiles, splits and combine are unchanged;
//    the producer fills a tile with sub-boxes of gcd(tile, page_size)
//    positions, each inside one page, so the consumers see the same shared
//    memory layout as with contiguous caches.
#include <math.h>

#include <algorithm>
#include <mutex>
#include <numeric>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr int kGridMax = 2048;        // upper bound of split-kernel CTAs (sizes the workspace)
constexpr int kWorkspaceHeader = 256; // reserved
constexpr int kPartialPad = 4;        // per-head partial record: o[d_v], m, l, pad, pad

struct DecodeArgs {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_new = nullptr;  // [B, n_k, d_k] (append mode) or null
    const __nv_bfloat16 *v_new = nullptr;  // [B, n_v, d_v] (append mode) or null
    __nv_bfloat16 *k_store = nullptr;      // the K cache, written at position seq_len (append mode)
    __nv_bfloat16 *v_store = nullptr;      // the V cache, likewise
    const int32_t *seq_lens;
    __nv_bfloat16 *out;
    float *partials;
    uint32_t *counters;
    int32_t *status;
    int32_t batch, n_q, n_k, n_v, t_max;
    int32_t vpg;      // V heads carried by one tile
    int32_t q_per_v;  // n_q / n_v
    int32_t stages;
    int32_t grid;
    uint32_t stage_bytes;   // bytes TMA lands per stage (K box + V box)
    uint32_t k_tile_bytes;  // offset of the V box inside a stage
    uint32_t stage_stride;  // bytes between stages
    float scale_log2;       // scale * log2(e)
    uint64_t wait_limit_ns;
    // paged caches; block_table == null means contiguous [B, t_max, heads, d] caches
    const int32_t *block_table = nullptr;  // [B, max_blocks] pool page of each logical page
    int32_t max_blocks = 0, page_size = 0, num_pages = 0;
    int32_t sub_rows = 0;                  // positions per sub-box (divides the tile and the page)
    int32_t sub_shift = -1, page_shift = -1;  // log2 of sub_rows / page_size when powers of two, else -1
    long long partial_slots = 0;           // split-partial records the scratch holds
    long long store_rows = 0;              // rows of the K / V caches or pools (append stores)
    uint32_t sub_k_bytes = 0, sub_v_bytes = 0;
};


// Position of the tile walk: unit (b, g), tile i of nt, first global tile P.
struct Walker {
    int b, g, i, nt, T;
    long long P;
};

__device__ __forceinline__ int clamp_len(int v, int t_max) { return v < 0 ? 0 : (v > t_max ? t_max : v); }

// Block-table entry of logical page pi of sequence b, unchecked.
__device__ __forceinline__ int page_entry(const DecodeArgs &a, int b, int pi) {
    return __ldg(a.block_table + (size_t)b * a.max_blocks + pi);
}

// A block-table entry checked against the pool: an entry outside
// [0, num_pages) is flagged DIFFQKV_ERR_DEVICE_PAGE and -1 returned.
__device__ __forceinline__ int checked_page(const DecodeArgs &a, int page) {
    if (page >= 0 && page < a.num_pages) return page;
    record_error(a.status, DIFFQKV_ERR_DEVICE_PAGE);
    return -1;
}

// Pool page holding logical page pi of sequence b (checked).
__device__ __forceinline__ int paged_page(const DecodeArgs &a, int b, int pi) {
    return checked_page(a, page_entry(a, b, pi));
}

// Storage row (one position's heads) of position p of sequence b, or -1 when
// its page-table entry is out of range.
__device__ __forceinline__ long long cache_row(const DecodeArgs &a, int b, int p) {
    if (!a.block_table) return (long long)b * a.t_max + p;
    const int page = paged_page(a, b, p / a.page_size);
    return page < 0 ? -1 : (long long)page * a.page_size + p % a.page_size;
}

template <int TT>
__device__ __forceinline__ void walker_advance(Walker &w, const DecodeArgs &a) {
    if (++w.i < w.nt) return;
    w.P += w.nt;
    w.i = 0;
    if (++w.g < a.n_k) return;
    w.g = 0;
    for (;;) {
        if (++w.b >= a.batch) { w.nt = 0; return; }
        w.T = clamp_len(__ldg(a.seq_lens + w.b), a.t_max);
        w.nt = (w.T + TT - 1) / TT;
        if (w.nt > 0) return;
    }
}

// CTA that owns global tile t when N tiles are cut into G equal ranges
// [floor(c N / G), floor((c+1) N / G)).
__device__ __forceinline__ long long cta_of_tile(long long t, long long N, long long G) {
    return ((t + 1) * G - 1) / N;
}

// x / sub_rows, x / page_size and x % page_size: shifts when they are powers of two (the producer
// warp shares its sub-partition with consumers, and a runtime division is dozens of instructions).
__device__ __forceinline__ int div_sub(const DecodeArgs &a, int x) {
    return a.sub_shift >= 0 ? x >> a.sub_shift : x / a.sub_rows;
}
__device__ __forceinline__ int div_page(const DecodeArgs &a, int x) {
    return a.page_shift >= 0 ? x >> a.page_shift : x / a.page_size;
}
__device__ __forceinline__ int mod_page(const DecodeArgs &a, int x) {
    return a.page_shift >= 0 ? x & (a.page_size - 1) : x % a.page_size;
}

// Sub-boxes holding the valid positions of the walker's current tile (paged caches).
template <int TT>
__device__ __forceinline__ int sub_boxes(const DecodeArgs &a, const Walker &w) {
    return div_sub(a, min(TT, w.T - w.i * TT) + a.sub_rows - 1);
}

// Block-table entry of sub-box f of the walker's current tile, 0 when f is past its sub-boxes.
template <int TT>
__device__ __forceinline__ int sub_box_entry(const DecodeArgs &a, const Walker &w, int f) {
    return f < sub_boxes<TT>(a, w) ? page_entry(a, w.b, div_page(a, w.i * TT + f * a.sub_rows)) : 0;
}

// Producer for paged caches, run by the whole producer warp.  Lane f issues the K and V loads of
// sub-boxes f, f + 32, ... of a tile, so a tile's sub-boxes leave as one warp instruction each;
// every lane reads its block-table entry for the next tile one full iteration ahead.  Returns the
// number of tiles issued.
template <int TT, int QPK>
__device__ long long produce_paged(const CUtensorMap *tm_k, const CUtensorMap *tm_v, const DecodeArgs &a, Walker w,
                                   long long t_begin, long long t_end, uint8_t *smem, uint64_t *full_bar,
                                   uint64_t *empty_bar, volatile int *abort_flag, int lane) {
    int cur = sub_box_entry<TT>(a, w, lane);
    long long k = 0;
    int stage = 0;        // k mod stages, kept incrementally
    uint32_t par = 0;     // parity of k / stages
    for (long long t = t_begin; t < t_end; ++t, ++k) {
        const int n_sub = sub_boxes<TT>(a, w);
        Walker wn = w;
        if (t + 1 < t_end) walker_advance<TT>(wn, a);
        const int nxt = (t + 1 < t_end) ? sub_box_entry<TT>(a, wn, lane) : 0;
        if (k >= a.stages) mbar_wait_bounded(&empty_bar[stage], par ^ 1u, a.wait_limit_ns, abort_flag, a.status);
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        uint8_t *sb = smem + (size_t)stage * a.stage_stride;
        if (lane == 0) mbar_arrive_expect_tx(&full_bar[stage], (uint32_t)n_sub * (a.sub_k_bytes + a.sub_v_bytes));
        __syncwarp();
        const int v0 = (w.g * QPK) / a.q_per_v;
        for (int f = lane; f < n_sub; f += 32) {
            // a bad entry (flagged) loads pool page 0 instead: the loads stay in bounds
            const int entry = f == lane ? cur : page_entry(a, w.b, div_page(a, w.i * TT + f * a.sub_rows));
            const int page = max(checked_page(a, entry), 0);
            const int row = mod_page(a, w.i * TT + f * a.sub_rows);
            tma_load_4d(sb + (size_t)f * a.sub_k_bytes, tm_k, &full_bar[stage], 0, w.g, row, page);
            tma_load_4d(sb + a.k_tile_bytes + (size_t)f * a.sub_v_bytes, tm_v, &full_bar[stage], 0, v0, row, page);
        }
        cur = nxt;
        w = wn;
        if (++stage == a.stages) {
            stage = 0;
            par ^= 1u;
        }
    }
    return k;
}

template <int DK, int DV, int QPK, int TT, int NCW>
__global__ void __launch_bounds__((NCW + 1) * 32, 1)
    decode_split_combine_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                                const DecodeArgs a) {
    constexpr int LPT = DK / 8;      // lanes per token in the score pass (8 bf16 per lane)
    constexpr int TPP = 32 / LPT;    // tokens per score pass
    constexpr int R = NCW / QPK;     // warps per query head (token split inside a tile)
    constexpr int TPW = TT / R;      // tokens per warp per tile
    constexpr int NPASS = TPW / TPP; // score passes per tile
    constexpr int CPV = DV / 8;      // lanes per V row (8 bf16 per lane)
    constexpr int NSL = 32 / CPV;    // token slots in the P.V pass
    static_assert(NCW % QPK == 0 && TT % R == 0, "bad warp split");
    static_assert(TPW % TPP == 0 && TPW % NSL == 0 && NPASS >= 1, "bad tile split");
    static_assert(DK % 64 == 0 && DV % 64 == 0, "head dims");

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full_bar = reinterpret_cast<uint64_t *>(smem + a.stages * a.stage_stride);
    uint64_t *empty_bar = full_bar + a.stages;
    float *p_s = reinterpret_cast<float *>(empty_bar + a.stages);  // [NCW][TPW]
    float *merge_s = p_s + NCW * TPW;                               // [NCW][DV + 4]
    int *flags = reinterpret_cast<int *>(merge_s + NCW * (DV + kPartialPad));
    volatile int *abort_flag = flags;      // flags[0]
    volatile int *last_flag = flags + 1;   // flags[1]
    long long *scan_s = reinterpret_cast<long long *>(flags + 4);  // [0]=N, [1]=P0, [2]=b0|g0, [3]=i0

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const long long G = a.grid;
    const long long c = blockIdx.x;

    if (tid == 0) {
        for (int s = 0; s < a.stages; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], NCW);
        }
        flags[0] = 0;
        flags[1] = 0;
        fence_barrier_init();
    }
    if (warp == NCW && lane == 0) {
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
    }

    // ---- prologue (warp 0): total tile count N, then the unit holding this CTA's first tile
    if (warp == 0) {
        long long acc = 0;
        for (int base = 0; base < a.batch; base += 32) {
            const int b = base + lane;
            int nt = 0;
            if (b < a.batch) {
                const int raw = __ldg(a.seq_lens + b);
                if (c == 0 && (raw < 0 || raw > a.t_max)) record_error(a.status, DIFFQKV_ERR_DEVICE_SEQLEN);
                nt = (clamp_len(raw, a.t_max) + TT - 1) / TT;
            }
            long long incl = (long long)nt * a.n_k;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            acc += __shfl_sync(0xffffffffu, incl, 31);
        }
        const long long N = acc;
        // never more CTAs than tiles: every CTA range is then non-empty
        const long long Ge = N < G ? N : G;
        const long long t_begin = (c < Ge) ? (c * N) / Ge : N;
        long long P0 = 0;
        int b0 = a.batch, g0 = 0, i0 = 0;
        acc = 0;
        bool found = false;
        for (int base = 0; base < a.batch && !found && N > 0; base += 32) {
            const int b = base + lane;
            const int nt = b < a.batch ? (clamp_len(__ldg(a.seq_lens + b), a.t_max) + TT - 1) / TT : 0;
            const long long w = (long long)nt * a.n_k;
            long long incl = w;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const long long y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const long long excl = incl - w;
            const bool hit = b < a.batch && nt > 0 && acc + excl <= t_begin && t_begin < acc + incl;
            const unsigned m = __ballot_sync(0xffffffffu, hit);
            if (m) {
                const int L = __ffs(m) - 1;
                const long long start = __shfl_sync(0xffffffffu, acc + excl, L);
                const int ntL = __shfl_sync(0xffffffffu, nt, L);
                const long long within = t_begin - start;
                b0 = base + L;
                g0 = (int)(within / ntL);
                i0 = (int)(within % ntL);
                P0 = start + (long long)g0 * ntL;
                found = true;
            }
            acc += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            scan_s[0] = N;
            scan_s[1] = P0;
            scan_s[2] = ((long long)b0 << 32) | (unsigned)g0;
            scan_s[3] = i0;
        }
    }
    __syncthreads();

    const long long N = scan_s[0];
    // sequences with no cached positions produce zero rows (distributed over CTAs); in
    // append mode their output is the new token's V row, and the new token fills position 0
    for (int b = (int)c; b < a.batch; b += (int)G) {
        if (clamp_len(__ldg(a.seq_lens + b), a.t_max) == 0) {
            __nv_bfloat16 *o = a.out + (size_t)b * a.n_q * DV;
            if (a.k_new) {
                for (int e = tid; e < a.n_q * DV; e += blockDim.x) {
                    const int h = e / DV;
                    o[e] = a.v_new[((size_t)b * a.n_v + h / a.q_per_v) * DV + e % DV];
                }
                const long long row0 = cache_row(a, b, 0);
                if (row0 >= 0) {
                    for (int e = tid; e < a.n_k * DK; e += blockDim.x)
                        a.k_store[(size_t)row0 * a.n_k * DK + e] = a.k_new[(size_t)b * a.n_k * DK + e];
                    for (int e = tid; e < a.n_v * DV; e += blockDim.x)
                        a.v_store[(size_t)row0 * a.n_v * DV + e] = a.v_new[(size_t)b * a.n_v * DV + e];
                }
            } else {
                for (int e = tid; e < a.n_q * DV; e += blockDim.x) o[e] = __float2bfloat16(0.f);
            }
        }
    }
    const long long Ge = N < G ? N : G;  // CTAs that own tiles
    if (c >= Ge) return;
    const long long t_begin = (c * N) / Ge;
    const long long t_end = ((c + 1) * N) / Ge;

    Walker w0;
    w0.b = (int)(scan_s[2] >> 32);
    w0.g = (int)(scan_s[2] & 0xffffffff);
    w0.i = (int)scan_s[3];
    w0.P = scan_s[1];
    w0.T = clamp_len(__ldg(a.seq_lens + w0.b), a.t_max);
    w0.nt = (w0.T + TT - 1) / TT;

    if (warp == NCW) {
        // ================= producer: one elected lane issues the TMA loads of contiguous caches;
        // the whole warp runs the paged producer
        long long k = 0;
        if (a.block_table) {
            k = produce_paged<TT, QPK>(&tm_k, &tm_v, a, w0, t_begin, t_end, smem, full_bar, empty_bar, abort_flag,
                                       lane);
        } else if (lane == 0) {
            Walker w = w0;
            int stage = 0;     // k mod stages, kept incrementally
            uint32_t par = 0;  // parity of k / stages
            for (long long t = t_begin; t < t_end; ++t, ++k) {
                if (k >= a.stages) mbar_wait_bounded(&empty_bar[stage], par ^ 1u, a.wait_limit_ns, abort_flag, a.status);
                if (*abort_flag) break;
                uint8_t *sb = smem + (size_t)stage * a.stage_stride;
                mbar_arrive_expect_tx(&full_bar[stage], a.stage_bytes);
                const int v0 = (w.g * QPK) / a.q_per_v;
                tma_load_4d(sb, &tm_k, &full_bar[stage], 0, w.g, w.i * TT, w.b);
                tma_load_4d(sb + a.k_tile_bytes, &tm_v, &full_bar[stage], 0, v0, w.i * TT, w.b);
                walker_advance<TT>(w, a);
                if (++stage == a.stages) {
                    stage = 0;
                    par ^= 1u;
                }
            }
        }
        if (lane == 0) {
            // drain: never leave the CTA with copies still landing in its shared memory
            const long long issued = k;
            for (long long j = (issued > a.stages ? issued - a.stages : 0); j < issued; ++j) {
                const int stage = (int)(j % a.stages);
                mbar_wait_bounded(&full_bar[stage], (uint32_t)((j / a.stages) & 1), a.wait_limit_ns, nullptr,
                                  a.status);
            }
        }
        return;
    }

    // ================= consumers: warp = (head slot hs, token slice r)
    const int hs = warp / R;
    const int r = warp % R;
    float *my_p = p_s + warp * TPW;
    float *my_merge = merge_s + warp * (DV + kPartialPad);
    const int kc = lane % LPT;   // K chunk (8 dims)
    const int kt = lane / LPT;   // token within a score pass
    const int vc = lane % CPV;   // V chunk (8 dims)
    const int vs = lane / CPV;   // token slot in the P.V pass

    f32x2_t q2[4];  // this lane's 8 query values (scaled), as packed pairs
    f32x2_t o2[4];  // this lane's 8 output accumulators, as packed pairs
    float m_run = -INFINITY, l_run = 0.f;
    int v_local = 0;

    Walker w = w0;
    int stage = 0;     // tile index mod stages, kept incrementally
    uint32_t par = 0;  // parity of tile index / stages
    for (long long t = t_begin; t < t_end; ++t) {
        const int h = w.g * QPK + hs;
        if (t == t_begin || w.i == 0) {
            // new split: this warp's query chunk, pre-scaled into the log2 domain
            const uint4 qv = in_bounds((long long)w.b * a.n_q + h, (long long)a.batch * a.n_q, a.status)
                                 ? __ldg(reinterpret_cast<const uint4 *>(a.q + ((size_t)w.b * a.n_q + h) * DK) + kc)
                                 : make_uint4(0, 0, 0, 0);
            const f32x2_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
            q2[0] = f2_mul(bf16x2_to_f2(qv.x), sc2);
            q2[1] = f2_mul(bf16x2_to_f2(qv.y), sc2);
            q2[2] = f2_mul(bf16x2_to_f2(qv.z), sc2);
            q2[3] = f2_mul(bf16x2_to_f2(qv.w), sc2);
#pragma unroll
            for (int e = 0; e < 4; ++e) o2[e] = 0ull;
            m_run = -INFINITY;
            l_run = 0.f;
            v_local = h / a.q_per_v - (w.g * QPK) / a.q_per_v;
        }
        mbar_wait_bounded(&full_bar[stage], par, a.wait_limit_ns, abort_flag, a.status);
        const uint8_t *sb = smem + (size_t)stage * a.stage_stride;
        const __nv_bfloat16 *Ks = reinterpret_cast<const __nv_bfloat16 *>(sb);
        const __nv_bfloat16 *Vs = reinterpret_cast<const __nv_bfloat16 *>(sb + a.k_tile_bytes);

        const int valid = min(TT, w.T - w.i * TT);
        const int my_valid = max(0, min(TPW, valid - r * TPW));

        // ---- scores s = (q . k) * scale * log2(e) for this warp's TPW tokens
        float s[NPASS];
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
            const int tw = ps * TPP + kt;
            const uint4 kv = lds128(Ks + (size_t)(r * TPW + tw) * DK + kc * 8);
            f32x2_t acc2 = f2_mul(q2[0], bf16x2_to_f2(kv.x));
            acc2 = f2_fma(q2[1], bf16x2_to_f2(kv.y), acc2);
            acc2 = f2_fma(q2[2], bf16x2_to_f2(kv.z), acc2);
            acc2 = f2_fma(q2[3], bf16x2_to_f2(kv.w), acc2);
            float acc, acc_hi;
            f2_unpack(acc2, acc, acc_hi);
            acc += acc_hi;
#pragma unroll
            for (int off = LPT / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
            s[ps] = tw < my_valid ? acc : -INFINITY;
        }
        // ---- online softmax update (log2 domain)
        float mx = s[0];
#pragma unroll
        for (int ps = 1; ps < NPASS; ++ps) mx = fmaxf(mx, s[ps]);
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_run, mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = fast_exp2(m_run - m_use);
        float psum = 0.f;
#pragma unroll
        for (int ps = 0; ps < NPASS; ++ps) {
            s[ps] = fast_exp2(s[ps] - m_use);
            psum += s[ps];
        }
#pragma unroll
        for (int off = LPT; off < 32; off <<= 1) psum += __shfl_xor_sync(0xffffffffu, psum, off);
        l_run = l_run * alpha + psum;
        m_run = m_new;
        if (kc == 0) {
#pragma unroll
            for (int ps = 0; ps < NPASS; ++ps) my_p[ps * TPP + kt] = s[ps];
        }
        __syncwarp();

        // ---- o = o * alpha + sum_j p_j V[j, vh]
        const f32x2_t alpha2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int e = 0; e < 4; ++e) o2[e] = f2_mul(o2[e], alpha2);
        const __nv_bfloat16 *vrow = Vs + ((size_t)(r * TPW) * a.vpg + v_local) * DV + vc * 8;
        const size_t vstride = (size_t)a.vpg * DV;
        if (my_valid == TPW) {
#pragma unroll
            for (int tt = vs; tt < TPW; tt += NSL) {
                const float pv = my_p[tt];
                const uint4 vv = lds128(vrow + tt * vstride);
                const f32x2_t p2 = f2_pack(pv, pv);
                o2[0] = f2_fma(p2, bf16x2_to_f2(vv.x), o2[0]);
                o2[1] = f2_fma(p2, bf16x2_to_f2(vv.y), o2[1]);
                o2[2] = f2_fma(p2, bf16x2_to_f2(vv.z), o2[2]);
                o2[3] = f2_fma(p2, bf16x2_to_f2(vv.w), o2[3]);
            }
        } else {
            for (int tt = vs; tt < my_valid; tt += NSL) {
                const float pv = my_p[tt];
                const uint4 vv = lds128(vrow + tt * vstride);
                const f32x2_t p2 = f2_pack(pv, pv);
                o2[0] = f2_fma(p2, bf16x2_to_f2(vv.x), o2[0]);
                o2[1] = f2_fma(p2, bf16x2_to_f2(vv.y), o2[1]);
                o2[2] = f2_fma(p2, bf16x2_to_f2(vv.z), o2[2]);
                o2[3] = f2_fma(p2, bf16x2_to_f2(vv.w), o2[3]);
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty_bar[stage]);
        if (++stage == a.stages) {
            stage = 0;
            par ^= 1u;
        }

        // ---- end of this CTA's piece of the unit: write the split partial, maybe combine
        if (w.i == w.nt - 1 || t == t_end - 1) {
            float o[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) f2_unpack(o2[e], o[2 * e], o[2 * e + 1]);
#pragma unroll
            for (int off = CPV; off < 32; off <<= 1) {
#pragma unroll
                for (int e = 0; e < 8; ++e) o[e] += __shfl_xor_sync(0xffffffffu, o[e], off);
            }
            if (R > 1) {
                if (vs == 0) {
                    *reinterpret_cast<float4 *>(my_merge + vc * 8) = make_float4(o[0], o[1], o[2], o[3]);
                    *reinterpret_cast<float4 *>(my_merge + vc * 8 + 4) = make_float4(o[4], o[5], o[6], o[7]);
                }
                if (lane == 0) {
                    my_merge[DV] = m_run;
                    my_merge[DV + 1] = l_run;
                }
            }
            named_barrier(1, NCW * 32);
            const long long u = (long long)w.b * a.n_k + w.g;
            const long long first = cta_of_tile(w.P, N, Ge);
            const long long last = cta_of_tile(w.P + w.nt - 1, N, Ge);
            if (r == 0) {
                float M = m_run, L = l_run;
                float O[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) O[e] = o[e];
                if (R > 1) {
                    M = -INFINITY;
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) M = fmaxf(M, merge_s[(warp + rr) * (DV + kPartialPad) + DV]);
                    const float Mu = (M == -INFINITY) ? 0.f : M;
                    L = 0.f;
#pragma unroll
                    for (int e = 0; e < 8; ++e) O[e] = 0.f;
#pragma unroll
                    for (int rr = 0; rr < R; ++rr) {
                        const float *src = merge_s + (warp + rr) * (DV + kPartialPad);
                        const float f = fast_exp2(src[DV] - Mu);
                        L += f * src[DV + 1];
#pragma unroll
                        for (int e = 0; e < 8; ++e) O[e] = fmaf(f, src[vc * 8 + e], O[e]);
                    }
                }
                float *dst = a.partials + ((size_t)(u + c) * QPK + hs) * (DV + kPartialPad);
                if (vs == 0 && in_bounds(u + c, a.partial_slots, a.status)) {
                    __stcg(reinterpret_cast<float4 *>(dst + vc * 8), make_float4(O[0], O[1], O[2], O[3]));
                    __stcg(reinterpret_cast<float4 *>(dst + vc * 8 + 4), make_float4(O[4], O[5], O[6], O[7]));
                }
                if (lane == 0) {
                    __stcg(dst + DV, M);
                    __stcg(dst + DV + 1, L);
                }
            }
            __threadfence();
            named_barrier(1, NCW * 32);
            if (tid == 0) {
                const unsigned old =
                    in_bounds(u, (long long)a.batch * a.n_k, a.status) ? atomicAdd(a.counters + u, 1u) : 0u;
                *last_flag = (old == (unsigned)(last - first)) ? 1 : 0;
            }
            named_barrier(1, NCW * 32);
            if (*last_flag) {
                __threadfence();
                // append mode: the new token's score for each query head of the group (merge_s is
                // free again here), and its K / V rows into the cache at position p
                const bool append = a.k_new != nullptr && w.T < a.t_max;
                if (a.k_new != nullptr && !append && tid == 0) record_error(a.status, DIFFQKV_ERR_DEVICE_SEQLEN);
                if (append) {
                    const int p = w.T;
                    if (warp < QPK) {
                        const int h = w.g * QPK + warp;
                        const __nv_bfloat16 *qh = a.q + ((size_t)w.b * a.n_q + h) * DK;
                        const __nv_bfloat16 *kn = a.k_new + ((size_t)w.b * a.n_k + w.g) * DK;
                        float dot = 0.f;
                        for (int e = lane; e < DK; e += 32)
                            dot = fmaf(__bfloat162float(qh[e]), __bfloat162float(kn[e]), dot);
#pragma unroll
                        for (int off = 16; off >= 1; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
                        if (lane == 0) merge_s[warp] = dot * a.scale_log2;
                    }
                    long long row = cache_row(a, w.b, p);  // -1: bad page entry, nothing written
                    if (row >= 0 && !in_bounds(row, a.store_rows, a.status)) row = -1;
                    const size_t kdst = ((size_t)row * a.n_k + w.g) * DK;
                    const size_t ksrc = ((size_t)w.b * a.n_k + w.g) * DK;
                    for (int e = tid; e < DK / 8 && row >= 0; e += NCW * 32)
                        reinterpret_cast<uint4 *>(a.k_store + kdst)[e] = reinterpret_cast<const uint4 *>(a.k_new + ksrc)[e];
                    for (int e = tid; e < QPK * (DV / 8) && row >= 0; e += NCW * 32) {
                        const int h = w.g * QPK + e / (DV / 8);
                        if (h % a.q_per_v != 0) continue;  // one writer per V head: its first query head
                        const int vh = h / a.q_per_v;
                        const size_t vdst = ((size_t)row * a.n_v + vh) * DV;
                        const size_t vsrc = ((size_t)w.b * a.n_v + vh) * DV;
                        reinterpret_cast<uint4 *>(a.v_store + vdst)[e % (DV / 8)] =
                            reinterpret_cast<const uint4 *>(a.v_new + vsrc)[e % (DV / 8)];
                    }
                    named_barrier(1, NCW * 32);
                }
                constexpr int ITEMS = QPK * (DV / 4);
                constexpr int kBatch = QPK >= 16 ? 1 : 4;  // partials loaded together (one L2 round trip per batch)
                // (checked build: a combine whose partial records would fall outside the scratch is skipped)
                const bool parts_ok = in_bounds(u + last, a.partial_slots, a.status);
                for (int it = tid; it < ITEMS && parts_ok; it += NCW * 32) {
                    const int h2 = it / (DV / 4);
                    const int d4 = it % (DV / 4);
                    constexpr int kBatchM = QPK >= 16 ? 4 : 16;  // maxima only: wider batches
                    float M = -INFINITY;
                    for (long long c0 = first; c0 <= last; c0 += kBatchM) {
                        float mv[kBatchM];
#pragma unroll
                        for (int e = 0; e < kBatchM; ++e)
                            mv[e] = c0 + e <= last
                                        ? __ldcg(a.partials + ((size_t)(u + c0 + e) * QPK + h2) * (DV + kPartialPad) + DV)
                                        : -INFINITY;
#pragma unroll
                        for (int e = 0; e < kBatchM; ++e) M = fmaxf(M, mv[e]);
                    }
                    const float s_new = append ? merge_s[h2] : -INFINITY;
                    M = fmaxf(M, s_new);
                    const float Mu = (M == -INFINITY) ? 0.f : M;
                    float L = 0.f;
                    float4 O = make_float4(0.f, 0.f, 0.f, 0.f);
                    for (long long c0 = first; c0 <= last; c0 += kBatch) {
                        float mv[kBatch], lv[kBatch];
                        float4 xv[kBatch];
#pragma unroll
                        for (int e = 0; e < kBatch; ++e) {
                            if (c0 + e <= last) {
                                const float *src = a.partials + ((size_t)(u + c0 + e) * QPK + h2) * (DV + kPartialPad);
                                mv[e] = __ldcg(src + DV);
                                lv[e] = __ldcg(src + DV + 1);
                                xv[e] = __ldcg(reinterpret_cast<const float4 *>(src) + d4);
                            }
                        }
                        // the same fixed order over the partials as one at a time
#pragma unroll
                        for (int e = 0; e < kBatch; ++e) {
                            if (c0 + e > last) break;
                            const float f = fast_exp2(mv[e] - Mu);
                            L = fmaf(f, lv[e], L);
                            O.x = fmaf(f, xv[e].x, O.x);
                            O.y = fmaf(f, xv[e].y, O.y);
                            O.z = fmaf(f, xv[e].z, O.z);
                            O.w = fmaf(f, xv[e].w, O.w);
                        }
                    }
                    if (append) {  // the new token: m = s_new, l = 1, o = v_new
                        const float f = fast_exp2(s_new - Mu);
                        L += f;
                        const int vh = (w.g * QPK + h2) / a.q_per_v;
                        const __nv_bfloat16 *vn = a.v_new + ((size_t)w.b * a.n_v + vh) * DV + d4 * 4;
                        O.x = fmaf(f, __bfloat162float(vn[0]), O.x);
                        O.y = fmaf(f, __bfloat162float(vn[1]), O.y);
                        O.z = fmaf(f, __bfloat162float(vn[2]), O.z);
                        O.w = fmaf(f, __bfloat162float(vn[3]), O.w);
                    }
                    const float inv = L > 0.f ? 1.f / L : 0.f;
                    __nv_bfloat162 lo = __floats2bfloat162_rn(O.x * inv, O.y * inv);
                    __nv_bfloat162 hi = __floats2bfloat162_rn(O.z * inv, O.w * inv);
                    uint2 packed;
                    packed.x = *reinterpret_cast<uint32_t *>(&lo);
                    packed.y = *reinterpret_cast<uint32_t *>(&hi);
                    if (in_bounds((long long)w.b * a.n_q + w.g * QPK + h2, (long long)a.batch * a.n_q, a.status))
                        *reinterpret_cast<uint2 *>(a.out + ((size_t)w.b * a.n_q + w.g * QPK + h2) * DV + d4 * 4) = packed;
                }
                if (tid == 0) a.counters[u] = 0u;
            }
            named_barrier(1, NCW * 32);
        }
        walker_advance<TT>(w, a);
    }
}

// ------------------------------------------------------------------ host side

constexpr int ncw_for(int qpk) { return qpk > 8 ? qpk : 8; }

// Smallest legal tile height: the R warps of a head split the tile, and each
// warp's share must be whole score passes and whole P.V slot rounds.
constexpr int tile_granule(int dk, int dv, int qpk) {
    const int r = ncw_for(qpk) / qpk;
    const int tpp = 32 / (dk / 8), nsl = 32 / (dv / 8);
    return r * (tpp > nsl ? tpp : nsl);
}

// Tile height: about 56 KiB of K+V per stage (V side sized for the widest group),
// at most 128 positions.  Measured on B200 at 32k context: per-tile overheads
// (barrier, softmax reductions, rescale) make small tiles slow, while more than
// ~170 KiB in flight per SM reads more slowly (16 x 32768 DiffQKV: 32-position
// tiles 6074 GB/s, 48 x 3 stages 6836, 64 x 3 stages 6487).
constexpr int tt_for(int dk, int dv, int qpk) {
    const int g = tile_granule(dk, dv, qpk);
    const int bytes_per_token = 2 * dk + 2 * qpk * dv;
    int tt = (56 * 1024 / bytes_per_token) / g * g;
    if (tt < g) tt = g;
    if (tt > 128) tt = 128 / g * g;
    return tt;
}

int v_heads_per_tile(const diffqkv_dims_t *d) {
    const int qpk = d->n_q / d->n_k;
    const int qpv = d->n_q / d->n_v;
    int span = 1;
    for (int g = 0; g < d->n_k; ++g) {
        const int v0 = (g * qpk) / qpv;
        const int v1 = ((g + 1) * qpk - 1) / qpv;
        span = std::max(span, v1 - v0 + 1);
    }
    return span;
}

bool supported_qpk(int qpk) { return qpk == 1 || qpk == 2 || qpk == 4 || qpk == 8 || qpk == 16; }

using KernelFn = void (*)(CUtensorMap, CUtensorMap, DecodeArgs);

template <int DK, int DV, int QPK>
KernelFn kernel_for() {
    return decode_split_combine_kernel<DK, DV, QPK, tt_for(DK, DV, QPK), ncw_for(QPK)>;
}

template <int DK, int DV>
KernelFn pick_kernel_qpk(int qpk) {
    switch (qpk) {
        case 1: return kernel_for<DK, DV, 1>();
        case 2: return kernel_for<DK, DV, 2>();
        case 4: return kernel_for<DK, DV, 4>();
        case 8: return kernel_for<DK, DV, 8>();
        case 16: return kernel_for<DK, DV, 16>();
        default: return nullptr;
    }
}

KernelFn pick_kernel(int dk, int dv, int qpk) {
    if (dk == 64 && dv == 64) return pick_kernel_qpk<64, 64>(qpk);
    if (dk == 64 && dv == 128) return pick_kernel_qpk<64, 128>(qpk);
    if (dk == 128 && dv == 64) return pick_kernel_qpk<128, 64>(qpk);
    if (dk == 128 && dv == 128) return pick_kernel_qpk<128, 128>(qpk);
    return nullptr;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// A K tile row is one head's d_k slice of a position; the other K heads of the
// position sit beside it and are read by other CTAs, usually much later.  With
// 128-byte rows, 256-byte L2 promotion would fetch a neighbour's row for nothing.
CUtensorMapL2promotion k_promotion(const diffqkv_dims_t *d) {
    return (d->n_k > 1 && d->d_k * 2 <= 128) ? CU_TENSOR_MAP_L2_PROMOTION_L2_128B : CU_TENSOR_MAP_L2_PROMOTION_L2_256B;
}

}  // namespace

size_t decode_workspace_size(const diffqkv_dims_t *d) {
    if (validate_dims(d) != DIFFQKV_OK) return 0;
    const size_t units = (size_t)d->batch * d->n_k;
    const size_t qpk = d->n_q / d->n_k;
    const size_t counters = align_up(units * sizeof(uint32_t), 256);
    const size_t partials = (units + kGridMax) * qpk * (d->d_v + kPartialPad) * sizeof(float);
    return kWorkspaceHeader + counters + partials;
}

diffqkv_status_t decode_plan(const diffqkv_dims_t *d, int32_t t_max, int32_t max_seq_len, int32_t num_sms,
                             const diffqkv_decode_tuning_t *tuning, diffqkv_decode_plan_t *plan) {
    if (!plan) return DIFFQKV_ERR_INVALID_ARG;
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (t_max < 1 || num_sms < 1) return DIFFQKV_ERR_INVALID_ARG;
    const int qpk = d->n_q / d->n_k;
    if (!supported_qpk(qpk) || (d->d_k != 64 && d->d_k != 128) || (d->d_v != 64 && d->d_v != 128))
        return DIFFQKV_ERR_UNSUPPORTED;
    struct { int tt, ncw; } ks = {tt_for(d->d_k, d->d_v, qpk), ncw_for(qpk)};
    const int vpg = v_heads_per_tile(d);
    const size_t k_tile = (size_t)ks.tt * d->d_k * 2;
    const size_t v_tile = (size_t)ks.tt * vpg * d->d_v * 2;
    const size_t stage_stride = align_up(k_tile + v_tile, 1024);
    const size_t extra = 16 * 8 /*barriers*/ + (size_t)ks.ncw * (ks.tt / (ks.ncw / qpk)) * 4 +
                         (size_t)ks.ncw * (d->d_v + kPartialPad) * 4 + 64 + 1024 /*alignment slack*/;
    const size_t smem_cap = 227 * 1024;
    int stages = (tuning && tuning->stages) ? tuning->stages : 0;
    if (stages == 0) {
        // three ~56 KiB stages (see tt_for): deeper rings read more slowly on B200
        stages = 3;
        while (stages > 2 && stages * stage_stride + extra > smem_cap) --stages;
    }
    if (stages < 2 || stages > 8 || stages * stage_stride + extra > smem_cap) return DIFFQKV_ERR_UNSUPPORTED;
    int cps = (tuning && tuning->ctas_per_sm) ? tuning->ctas_per_sm : 1;
    if (cps < 1 || cps > 4) return DIFFQKV_ERR_INVALID_ARG;
    const int msl = (max_seq_len >= 1 && max_seq_len <= t_max) ? max_seq_len : t_max;
    const long long n_est = (long long)d->batch * d->n_k * ((msl + ks.tt - 1) / ks.tt);
    long long grid = (long long)num_sms * cps;
    if (grid > n_est) grid = n_est;
    if (tuning && tuning->grid_ctas) grid = tuning->grid_ctas;
    if (grid < 1 || grid > kGridMax) return DIFFQKV_ERR_INVALID_ARG;
    plan->tile_tokens = ks.tt;
    plan->stages = stages;
    plan->grid_ctas = (int32_t)grid;
    plan->threads = (ks.ncw + 1) * 32;
    plan->v_heads_per_tile = vpg;
    plan->smem_bytes = (int64_t)(stages * stage_stride + extra);
    plan->workspace_bytes = (int64_t)decode_workspace_size(d);
    return DIFFQKV_OK;
}

namespace {

// A checked, fully encoded decode launch: everything decode_launch needs except the stream.
struct DecodeLaunch {
    KernelFn fn = nullptr;
    CUtensorMap tm_k, tm_v;
    DecodeArgs a;
    int grid = 0, threads = 0;
    size_t smem = 0;
};

// Every host-side check of a decode call (dims, pointers, alignment, workspace, device, plan) and
// the tensor-map encoding; nothing is enqueued.  The device status word is the workspace's first
// 32-bit word (inside its 256-byte header), so every workspace reports its own calls' errors.
diffqkv_status_t decode_prepare(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, void *out,
                                void *workspace, size_t workspace_bytes, const diffqkv_decode_tuning_t *tuning,
                                const void *k_new, const void *v_new, const PagedCache *paged, DecodeLaunch *L) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || t_max < 1) return DIFFQKV_ERR_INVALID_ARG;
    L->fn = pick_kernel(d->d_k, d->d_v, d->n_q / d->n_k);
    if (!L->fn) return DIFFQKV_ERR_UNSUPPORTED;
    if (paged) {
        if (!paged->block_table || paged->max_blocks < 1 || paged->page_size < 1 || paged->num_pages < 1 ||
            (long long)paged->max_blocks * paged->page_size != t_max)
            return DIFFQKV_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(paged->block_table) & 3u) return DIFFQKV_ERR_MISALIGNED;
    }
    if ((k_new == nullptr) != (v_new == nullptr)) return DIFFQKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    if (k_new && (!aligned16(k_new) || !aligned16(v_new))) return DIFFQKV_ERR_MISALIGNED;
    const size_t need = decode_workspace_size(d);
    if (!workspace || workspace_bytes < need) return DIFFQKV_ERR_WORKSPACE;
    if (!aligned16(workspace)) return DIFFQKV_ERR_MISALIGNED;

    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    diffqkv_decode_plan_t plan;
    st = decode_plan(d, t_max, max_seq_len, dev.num_sms, tuning, &plan);
    if (st != DIFFQKV_OK) return st;

    // contiguous caches: one box per tile over [B, t_max, heads, d]; paged: sub-boxes over
    // [num_pages, page_size, heads, d], each gcd(tile, page_size) positions inside one page
    const int sub_rows = paged ? std::gcd(plan.tile_tokens, paged->page_size) : plan.tile_tokens;
    const uint64_t rows_dim = paged ? (uint64_t)paged->page_size : (uint64_t)t_max;
    const uint64_t outer_dim = paged ? (uint64_t)paged->num_pages : (uint64_t)d->batch;
    st = make_tensor_map_4d(&L->tm_k, k_cache, d->d_k, d->n_k, rows_dim, outer_dim, d->d_k, 1, sub_rows, 1,
                            CU_TENSOR_MAP_SWIZZLE_NONE, k_promotion(d));
    if (st != DIFFQKV_OK) return st;
    st = make_tensor_map_4d(&L->tm_v, v_cache, d->d_v, d->n_v, rows_dim, outer_dim, d->d_v, plan.v_heads_per_tile,
                            sub_rows, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != DIFFQKV_OK) return st;

    DecodeArgs &a = L->a;
    if (paged) {
        a.block_table = paged->block_table;
        a.max_blocks = paged->max_blocks;
        a.page_size = paged->page_size;
        a.num_pages = paged->num_pages;
        a.sub_rows = sub_rows;
        auto log2_or = [](int v) {
            if (v <= 0 || (v & (v - 1))) return -1;
            int l = 0;
            while ((1 << l) < v) ++l;
            return l;
        };
        a.sub_shift = log2_or(sub_rows);
        a.page_shift = log2_or(paged->page_size);
        a.sub_k_bytes = (uint32_t)sub_rows * d->d_k * 2;
        a.sub_v_bytes = (uint32_t)sub_rows * plan.v_heads_per_tile * d->d_v * 2;
    }
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const size_t units = (size_t)d->batch * d->n_k;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    if (k_new) {
        a.k_new = static_cast<const __nv_bfloat16 *>(k_new);
        a.v_new = static_cast<const __nv_bfloat16 *>(v_new);
        a.k_store = static_cast<__nv_bfloat16 *>(const_cast<void *>(k_cache));
        a.v_store = static_cast<__nv_bfloat16 *>(const_cast<void *>(v_cache));
    }
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.counters = reinterpret_cast<uint32_t *>(ws + kWorkspaceHeader);
    a.partials = reinterpret_cast<float *>(ws + kWorkspaceHeader + align_up(units * sizeof(uint32_t), 256));
    a.status = reinterpret_cast<int32_t *>(ws);  // the workspace's own error word
    a.partial_slots = (long long)units + kGridMax;
    a.store_rows = paged ? (long long)paged->num_pages * paged->page_size : (long long)d->batch * t_max;
    a.batch = d->batch;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.t_max = t_max;
    a.vpg = plan.v_heads_per_tile;
    a.q_per_v = d->n_q / d->n_v;
    a.stages = plan.stages;
    a.grid = plan.grid_ctas;
    a.k_tile_bytes = (uint32_t)plan.tile_tokens * d->d_k * 2;
    a.stage_bytes = a.k_tile_bytes + (uint32_t)plan.tile_tokens * plan.v_heads_per_tile * d->d_v * 2;
    a.stage_stride = (uint32_t)align_up(a.stage_bytes, 1024);
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);
    a.wait_limit_ns = kWaitLimitNs;
    L->grid = plan.grid_ctas;
    L->threads = plan.threads;
    L->smem = (size_t)plan.smem_bytes;
    if (ensure_dynamic_smem((const void *)L->fn, (int)plan.smem_bytes) != DIFFQKV_OK) return DIFFQKV_ERR_CUDA;
    return DIFFQKV_OK;
}

diffqkv_status_t decode_enqueue(const DecodeLaunch &L, cudaStream_t stream) {
    L.fn<<<L.grid, L.threads, L.smem, stream>>>(L.tm_k, L.tm_v, L.a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    return DIFFQKV_OK;
}

}  // namespace

diffqkv_status_t decode_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache, const void *v_cache,
                               const int32_t *seq_lens, int32_t t_max, int32_t max_seq_len, void *out,
                               void *workspace, size_t workspace_bytes, const diffqkv_decode_tuning_t *tuning,
                               cudaStream_t stream, const void *k_new, const void *v_new, const PagedCache *paged) {
    DecodeLaunch L;
    const diffqkv_status_t st = decode_prepare(d, q, k_cache, v_cache, seq_lens, t_max, max_seq_len, out, workspace,
                                               workspace_bytes, tuning, k_new, v_new, paged, &L);
    if (st != DIFFQKV_OK) return st;
    return decode_enqueue(L, stream);
}

diffqkv_status_t decode_from_host_launch(const diffqkv_dims_t *d, const void *q_host, const void *k_host,
                                         const void *v_host, const int32_t *seq_lens_host, int32_t t_max,
                                         int32_t max_seq_len, void *out_host, void *q_dev, void *k_dev, void *v_dev,
                                         int32_t *seq_lens_dev, void *out_dev, void *workspace,
                                         size_t workspace_bytes, cudaStream_t stream) {
    if (!q_host || !k_host || !v_host || !seq_lens_host || !out_host) return DIFFQKV_ERR_INVALID_ARG;
    // every argument check of the decode runs before the first copy is enqueued
    DecodeLaunch L;
    diffqkv_status_t st = decode_prepare(d, q_dev, k_dev, v_dev, seq_lens_dev, t_max, max_seq_len, out_dev,
                                         workspace, workspace_bytes, nullptr, nullptr, nullptr, nullptr, &L);
    if (st != DIFFQKV_OK) return st;
    const size_t B = d->batch;
    const size_t q_bytes = B * d->n_q * d->d_k * 2;
    const size_t k_bytes = B * (size_t)t_max * d->n_k * d->d_k * 2;
    const size_t v_bytes = B * (size_t)t_max * d->n_v * d->d_v * 2;
    const size_t o_bytes = B * d->n_q * d->d_v * 2;
    // one plain async copy per buffer
    if (cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(k_dev, k_host, k_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(v_dev, v_host, v_bytes, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaMemcpyAsync(seq_lens_dev, seq_lens_host, B * sizeof(int32_t), cudaMemcpyHostToDevice, stream) !=
            cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    st = decode_enqueue(L, stream);
    if (st != DIFFQKV_OK) return st;
    if (cudaMemcpyAsync(out_host, out_dev, o_bytes, cudaMemcpyDeviceToHost, stream) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    return DIFFQKV_OK;
}

// ------------------------------------------------------------------ allocation-free variant
//
// The same split/combine kernel, with its scratch (split partials and per-unit
// counters) in a file-scope device array instead of a caller workspace.

static __device__ __align__(256) uint8_t g_decode_noalloc_scratch[DIFFQKV_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoAllocMaxDevices = 64;
void *g_noalloc_scratch_ptr[kNoAllocMaxDevices];
std::mutex g_noalloc_mutex;

// Device address of the scratch array on the current device (looked up once per device).
diffqkv_status_t noalloc_scratch(int device, uint8_t **ptr) {
    if (device < 0 || device >= kNoAllocMaxDevices) return DIFFQKV_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_scratch_ptr[device]) {
        void *p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress((void **)&p, g_decode_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            cudaGetLastError();
            return DIFFQKV_ERR_CUDA;
        }
        g_noalloc_scratch_ptr[device] = p;
    }
    *ptr = static_cast<uint8_t *>(g_noalloc_scratch_ptr[device]);
    return DIFFQKV_OK;
}

}  // namespace

diffqkv_status_t decode_noalloc_launch(const diffqkv_dims_t *d, const void *q, const void *k_cache,
                                       const void *v_cache, const int32_t *seq_lens, int32_t t_max,
                                       int32_t max_seq_len, void *out, cudaStream_t stream) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k_cache || !v_cache || !seq_lens || !out || t_max < 1) return DIFFQKV_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(seq_lens) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;
    diffqkv_decode_plan_t plan;
    st = decode_plan(d, t_max, max_seq_len, dev.num_sms, nullptr, &plan);
    if (st != DIFFQKV_OK) return st;
    const int qpk = d->n_q / d->n_k;
    KernelFn fn = pick_kernel(d->d_k, d->d_v, qpk);
    if (!fn) return DIFFQKV_ERR_UNSUPPORTED;

    // scratch: header, one counter per unit, then partial slots u + c < units + grid
    const size_t units = (size_t)d->batch * d->n_k;
    const size_t counter_bytes = align_up(units * sizeof(uint32_t), 256);
    const size_t need = kWorkspaceHeader + counter_bytes +
                        (units + (size_t)plan.grid_ctas) * qpk * (d->d_v + kPartialPad) * sizeof(float);
    if (need > (size_t)DIFFQKV_NOALLOC_SCRATCH_BYTES) return DIFFQKV_ERR_SCRATCH_LIMIT;
    uint8_t *scratch = nullptr;
    st = noalloc_scratch(dev.device, &scratch);
    if (st != DIFFQKV_OK) return st;

    CUtensorMap tm_k, tm_v;
    st = make_tensor_map_4d(&tm_k, k_cache, d->d_k, d->n_k, t_max, d->batch, d->d_k, 1, plan.tile_tokens, 1,
                            CU_TENSOR_MAP_SWIZZLE_NONE, k_promotion(d));
    if (st != DIFFQKV_OK) return st;
    st = make_tensor_map_4d(&tm_v, v_cache, d->d_v, d->n_v, t_max, d->batch, d->d_v, plan.v_heads_per_tile,
                            plan.tile_tokens, 1, CU_TENSOR_MAP_SWIZZLE_NONE);
    if (st != DIFFQKV_OK) return st;

    DecodeArgs a;
    a.q = static_cast<const __nv_bfloat16 *>(q);
    a.seq_lens = seq_lens;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.counters = reinterpret_cast<uint32_t *>(scratch + kWorkspaceHeader);
    a.partial_slots = (long long)units + plan.grid_ctas;
    a.store_rows = (long long)d->batch * t_max;
    a.partials = reinterpret_cast<float *>(scratch + kWorkspaceHeader + counter_bytes);
    a.status = dev.status_word;
    a.batch = d->batch;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.t_max = t_max;
    a.vpg = plan.v_heads_per_tile;
    a.q_per_v = d->n_q / d->n_v;
    a.stages = plan.stages;
    a.grid = plan.grid_ctas;
    a.k_tile_bytes = (uint32_t)plan.tile_tokens * d->d_k * 2;
    a.stage_bytes = a.k_tile_bytes + (uint32_t)plan.tile_tokens * plan.v_heads_per_tile * d->d_v * 2;
    a.stage_stride = (uint32_t)align_up(a.stage_bytes, 1024);
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);
    a.wait_limit_ns = kWaitLimitNs;

    // the counters must start at zero whatever an earlier call left behind
    if (cudaMemsetAsync(a.counters, 0, units * sizeof(uint32_t), stream) != cudaSuccess) {
        cudaGetLastError();
        return DIFFQKV_ERR_CUDA;
    }
    if (ensure_dynamic_smem((const void *)fn, (int)plan.smem_bytes) != DIFFQKV_OK) return DIFFQKV_ERR_CUDA;
    fn<<<plan.grid_ctas, plan.threads, plan.smem_bytes, stream>>>(tm_k, tm_v, a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    return DIFFQKV_OK;
}

}  // namespace diffqkv
