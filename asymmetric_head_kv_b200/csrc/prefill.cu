// prefill.cu -- causal DiffQKV prefill on the sm_100a tensor cores.
//
// out[b,i,h] = sum_{j<=i} softmax_j(scale q[b,i,h].k[b,j,kh]) v[b,j,vh],
// kh = h/(n_q/n_k), vh = h/(n_q/n_v)  (Sigma paper, structured summary page,
// section 3.4 Steps 3-5, with the causal lower-triangular mask of the prefix
// phase).  Unlike decode this is a dense contraction, so it runs on tcgen05.
//
// Two tilings, chosen by d_k:
//  * d_k = 64 (the DiffQKV key width): `tile64` -- one 128-row query tile per
//    CTA, 64-position K/V tiles, two S buffers in TMEM so that S(n+1) = Q K^T
//    runs while the softmax works on S(n), two CTAs per SM.  With d_k = 64 the
//    exponentials (64 per row and tile) outweigh the MMAs, and this overlap
//    within a tile is what keeps the SFU busy.
//  * d_k = 128: `pair128` -- two 128-row query tiles per CTA sharing each
//    128-position K/V tile, one CTA per SM (512 TMEM columns), the MMA thread
//    alternating between the tiles.  A Q K^T MMA with N = 64 would read its
//    Q operand from shared memory faster than shared memory delivers it once
//    d_k = 128 makes that product the larger one; N = 128 halves those reads.
// In both, P goes back to TMEM (bf16 pairs over the first columns of its S)
// and the P.V MMA reads it as its A operand; tcgen05.mma operations from one
// thread run in issue order, so S is overwritten only after the P.V that reads
// P from the same columns.  O is rescaled in TMEM only when a row maximum grows
// by more than 2^8 (the stale maximum is used consistently for O and the row
// sum, so the result is exact up to rounding).  Every mbarrier wait is bounded;
// CTAs are ordered heaviest (most K/V tiles) first.
//
// K and V may also come from page pools [num_pages, page_size, heads, d] with a
// block table (position j of sequence b is row j % page_size of pool page
// table[b][j / page_size]); only the producer differs (paged_kv_producer).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"

namespace diffqkv {

namespace {

constexpr float kRescaleLog2 = 8.f;  // lazy O rescale threshold (log2 domain)

struct PrefillArgs {
    __nv_bfloat16 *out;
    int32_t *status;
    int32_t batch, seq, n_q, n_k, n_v, q_per_k, q_per_v, n_ctas_per_head;
    int32_t prefix;  // cached positions before the first query row (query row r sits at position prefix + r)
    int32_t kv_len;  // prefix + seq: positions in K and V
    float scale_log2;
    uint64_t wait_limit_ns;
    // paged pools (block_table NULL: contiguous [B, kv_len, heads, d] caches)
    const int32_t *block_table;  // [batch][max_blocks]
    int32_t max_blocks, page_size, num_pages;
    int32_t n_pages;      // pages a sequence uses: ceil(kv_len / page_size)
    int32_t max_box_log;  // paged boxes are 8 << i rows, i <= max_box_log (heights that divide the page)
    int32_t page_shift;   // log2(page_size) when it is a power of two, else -1
};

constexpr int kPgTableWin = 512;  // paged producer: block-table entries held in shared memory

// K and V tensor maps of paged pools: k[i] / v[i] have (8 << i)-row boxes over the whole pool;
// k_tail[i] / v_tail[i] the same boxes over a view of the pool whose pages hold only the rows of
// a sequence's last page that carry positions, so that rows past the sequence read as zeros, as
// the contiguous maps' rows past kv_len do (the P.V MMA multiplies them by P = 0, and 0 times a
// stale NaN would not be 0).
struct PagedMaps {
    CUtensorMap k[4], v[4], k_tail[4], v_tail[4];
};

// Paged K/V producer of both tilings (all 32 lanes of the producer warp).  Tile n holds positions
// [n BN, n BN + BN) of sequence b in stage n % STAGES of the ring (K: KB 64-column blocks of BN
// rows, then V: VB blocks).  The tile's rows are covered greedily by aligned boxes of 8 << i rows
// that stay inside one page; lane f issues box f.  Boxes in the sequence's last page use the tail
// maps; boxes past it use a tail map at a row past its extent (all zeros).  The block-table
// entries sit in shared memory, a window of kPgTableWin pages loaded by the warp in one round
// trip; an entry outside [0, num_pages) is flagged DIFFQKV_ERR_DEVICE_PAGE and pool page 0 read
// instead.
template <int BN, int KB, int VB, int STAGES, int STAGE_BYTES, int K_BYTES>
__device__ __noinline__ void paged_kv_producer(const PagedMaps &pm, const PrefillArgs &a, int b, int kh, int vh, int n_kv,
                                  uint8_t *kv_base, uint64_t *kv_full, uint64_t *kv_empty,
                                  int32_t *table, volatile int *abort_flag, int lane) {
    const int P = a.page_size;
    const int pend = a.n_pages * P;  // positions the sequence's pages hold
    // position -> page and row in page: shifts for power-of-two pages (a runtime division is dozens
    // of instructions, and this warp shares its sub-partition with softmax warps)
    const int ps = a.page_shift;
    auto pdiv = [&](int x) { return ps >= 0 ? x >> ps : x / P; };
    auto pmod = [&](int x) { return ps >= 0 ? x & (P - 1) : x % P; };
    auto first_page = [&](int t) { return pdiv(t * BN); };
    int tbl0 = -kPgTableWin;  // pages tbl0 .. tbl0 + kPgTableWin - 1 are in `table`
    int issued = 0;
    for (int n = 0; n < n_kv; ++n) {
        const int last = min(a.n_pages - 1, pdiv(n * BN + BN - 1));
        if (last >= tbl0 + kPgTableWin) {  // (the same decision in every lane)
            tbl0 = first_page(n);
            const int cnt = min(kPgTableWin, a.n_pages - tbl0);
            __syncwarp();
            for (int i = lane; i < cnt; i += 32)
                if (in_bounds(tbl0 + i, a.max_blocks, a.status))
                    table[i] = __ldg(a.block_table + (size_t)b * a.max_blocks + tbl0 + i);
            __syncwarp();
        }
        const int st = n % STAGES;
        if (n >= STAGES)
            mbar_wait_bounded(&kv_empty[st], (uint32_t)(((n / STAGES) - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
        if (__any_sync(0xffffffffu, *abort_flag != 0)) break;
        const int start = n * BN, end = start + BN;
        int my_cur = -1, my_hi = a.max_box_log;
        if (ps >= 0) {
            // power-of-two pages: every box is 8 << max_box_log rows (the page, or 64 rows of it)
            const int rows = 8 << a.max_box_log;
            if (lane < BN / rows) my_cur = start + lane * rows;
        } else {
            // every lane walks the same greedy decomposition and keeps box `lane`
            int cur = start, f = 0;
            while (cur < end) {
                const int seg_end = cur < pend ? min(end, (pdiv(cur) + 1) * P) : end;
                int hi = a.max_box_log;
                while (hi > 0 && ((cur & ((8 << hi) - 1)) != 0 || cur + (8 << hi) > seg_end)) --hi;
                if (f == lane) {
                    my_cur = cur;
                    my_hi = hi;
                }
                cur += 8 << hi;
                ++f;
            }
        }
        uint8_t *kdst = kv_base + st * STAGE_BYTES;
        uint8_t *vdst = kdst + K_BYTES;
        if (lane == 0) mbar_arrive_expect_tx(&kv_full[st], STAGE_BYTES);
        __syncwarp();
        const bool in_seq = my_cur >= 0 && my_cur < pend;
        const int pidx = in_seq ? pdiv(my_cur) : 0;
        if (my_cur >= 0) {
            int page = in_seq ? table[pidx - tbl0] : 0;
            int row = P;        // past the sequence's pages: a row past the tail view's extent
            bool tail = true;
            if (in_seq) {
                if (page < 0 || page >= a.num_pages) {
                    record_error(a.status, DIFFQKV_ERR_DEVICE_PAGE);
                    page = 0;
                }
                row = pmod(my_cur);
                tail = pidx == a.n_pages - 1;
            } else {
                page = 0;
            }
            // constant indices keep the descriptors in the kernel's parameter space
            const CUtensorMap *km, *vm;
            if (tail) {
                km = my_hi == 0 ? &pm.k_tail[0] : my_hi == 1 ? &pm.k_tail[1] : my_hi == 2 ? &pm.k_tail[2] : &pm.k_tail[3];
                vm = my_hi == 0 ? &pm.v_tail[0] : my_hi == 1 ? &pm.v_tail[1] : my_hi == 2 ? &pm.v_tail[2] : &pm.v_tail[3];
            } else {
                km = my_hi == 0 ? &pm.k[0] : my_hi == 1 ? &pm.k[1] : my_hi == 2 ? &pm.k[2] : &pm.k[3];
                vm = my_hi == 0 ? &pm.v[0] : my_hi == 1 ? &pm.v[1] : my_hi == 2 ? &pm.v[2] : &pm.v[3];
            }
            const int off = (my_cur - start) * 128;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) tma_load_4d(kdst + kb * (BN * 128) + off, km, &kv_full[st], kb * 64, kh, row, page);
#pragma unroll
            for (int vb = 0; vb < VB; ++vb) tma_load_4d(vdst + vb * (BN * 128) + off, vm, &kv_full[st], vb * 64, vh, row, page);
        }
        issued = n + 1;
    }
    // drain: no copy may still be landing when the CTA exits
    if (lane == 0)
        for (int n = (issued > STAGES ? issued - STAGES : 0); n < issued; ++n)
            mbar_wait_bounded(&kv_full[n % STAGES], (uint32_t)((n / STAGES) & 1), a.wait_limit_ns, nullptr, a.status);
}

// ---------------------------------------------------------------- d_k = 64
// warps 0-3 softmax (thread t owns query row t = TMEM lane t), warp 4 TMA
// producer (Q once, K/V ring), warp 5 TMEM allocation and MMA issue.  S(n) goes
// to one of two 64-column S buffers; P(n) over the first 32 columns of it.
namespace tile64 {

constexpr int BM = 128;             // query rows per CTA
constexpr int BN = 64;              // K/V positions per tile
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarp = 4;
constexpr int kMmaWarp = 5;
constexpr int kThreads = 192;       // 4 softmax warps, producer, MMA
constexpr int kTmemCols = 256;      // S0 | S1 | O
template <int DK, int DV>
struct Cfg {
    static constexpr int KB = DK / 64;                 // 64-wide swizzle blocks along d_k
    static constexpr int VB = DV / 64;                 // ... along d_v
    static constexpr int Q_BYTES = BM * DK * 2;
    static constexpr int K_BYTES = BN * DK * 2;
    static constexpr int V_BYTES = BN * DV * 2;
    static constexpr int STAGES = DK == 64 ? 3 : 2;
    static constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers/flags + alignment slack
};

template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 2)
    prefill_causal_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PagedMaps pm,
                          const PrefillArgs a) {
    using C = Cfg<DK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kv_full = bars;                 // [STAGES]
    uint64_t *kv_empty = bars + 4;            // [STAGES]
    uint64_t *q_full = bars + 8;
    uint64_t *s_full = bars + 9;              // [2]
    uint64_t *p_full = bars + 13;
    uint64_t *pv_done = bars + 14;
    uint64_t *mma_done = bars + 15;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 17);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // heaviest tiles first: query tile index descends with blockIdx
    const int bh_count = a.batch * a.n_q;
    const int qt = a.n_ctas_per_head - 1 - (int)(blockIdx.x / bh_count);
    const int bh = (int)(blockIdx.x % bh_count);
    const int b = bh / a.n_q;
    const int h = bh % a.n_q;
    const int kh = h / a.q_per_k;
    const int vh = h / a.q_per_v;
    const int row0 = qt * BM;               // first query row of the tile (Q and out rows)
    const int pos0 = a.prefix + row0;       // its position among the keys
    const int kv_tiles_total = (a.kv_len + BN - 1) / BN;
    const int n_kv = min(kv_tiles_total, (pos0 + BM + BN - 1) / BN);

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(q_full, 1);
        mbar_init(&s_full[0], 1);
        mbar_init(&s_full[1], 1);
        mbar_init(p_full, kSoftmaxWarps);
        mbar_init(pv_done, 1);
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
    const uint32_t t_o = tmem + 2 * BN;  // S buffer sb (and P over its first BN/2 columns) at tmem + sb * BN

    if (warp == kProducerWarp) {
        // ======================= TMA producer
        __shared__ int32_t pg_table[kPgTableWin];  // paged: a window of block-table entries
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
                tma_load_4d(smem + C::OFF_Q + kb * (BM * 128), &tm_q, q_full, kb * 64, h, row0, b);
        }
        if (a.block_table) {
            __syncwarp();
            paged_kv_producer<BN, C::KB, C::VB, C::STAGES, C::STAGE_BYTES, C::K_BYTES>(
                pm, a, b, kh, vh, n_kv, smem + C::OFF_KV, kv_full, kv_empty, pg_table, abort_flag, lane);
            if (lane == 0) mbar_wait_bounded(q_full, 0, a.wait_limit_ns, nullptr, a.status);
        } else if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            for (int n = 0; n < n_kv; ++n) {
                const int st = n % C::STAGES;
                if (n >= C::STAGES)
                    mbar_wait_bounded(&kv_empty[st], (uint32_t)(((n / C::STAGES) - 1) & 1), a.wait_limit_ns,
                                      abort_flag, a.status);
                if (*abort_flag) break;
                uint8_t *kdst = smem + C::OFF_KV + st * C::STAGE_BYTES;
                uint8_t *vdst = kdst + C::K_BYTES;
                mbar_arrive_expect_tx(&kv_full[st], C::STAGE_BYTES);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_4d(kdst + kb * (BN * 128), &tm_k, &kv_full[st], kb * 64, kh, n * BN, b);
#pragma unroll
                for (int vb = 0; vb < C::VB; ++vb)
                    tma_load_4d(vdst + vb * (BN * 128), &tm_v, &kv_full[st], vb * 64, vh, n * BN, b);
            }
            // drain: no copy may still be landing when the CTA exits
            mbar_wait_bounded(q_full, 0, a.wait_limit_ns, nullptr, a.status);
            for (int n = (n_kv > C::STAGES ? n_kv - C::STAGES : 0); n < n_kv; ++n)
                mbar_wait_bounded(&kv_full[n % C::STAGES], (uint32_t)((n / C::STAGES) & 1), a.wait_limit_ns,
                                  nullptr, a.status);
        }
    } else if (warp == kMmaWarp) {
        // ======================= MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(BM, DV, false, true);
            const uint32_t q_addr = smem_addr(smem + C::OFF_Q);
            mbar_wait_bounded(q_full, 0, a.wait_limit_ns, abort_flag, a.status);
            for (int n = 0; n <= n_kv; ++n) {
                if (n < n_kv) {
                    // S[n%2] = Q K_n^T
                    const int st = n % C::STAGES;
                    const int sb = n & 1;
                    // S buffer sb last held S(n-2) and P(n-2): the softmax was done with it before
                    // p_full(n-2), and P(n-2) V(n-2) was issued ahead of this MMA
                    mbar_wait_bounded(&kv_full[st], (uint32_t)((n / C::STAGES) & 1), a.wait_limit_ns, abort_flag,
                                      a.status);
                    tc_fence_after();
                    const uint32_t k_addr = smem_addr(smem + C::OFF_KV + st * C::STAGE_BYTES);
#pragma unroll
                    for (int ks = 0; ks < DK / 16; ++ks) {
                        const uint32_t blk = (uint32_t)(ks >> 2), sub = (uint32_t)(ks & 3) * 32u;
                        const uint64_t da = smem_desc_sw128(q_addr + blk * (BM * 128) + sub, 16, 1024);
                        const uint64_t db = smem_desc_sw128(k_addr + blk * (BN * 128) + sub, 16, 1024);
                        umma_bf16(tmem + (uint32_t)(sb * BN), da, db, idesc_qk, ks > 0 ? 1u : 0u);
                    }
                    umma_commit(&s_full[sb]);
                }
                if (n >= 1) {
                    // O += P_{n-1} V_{n-1}
                    const int m = n - 1;
                    const int st = m % C::STAGES;
                    mbar_wait_bounded(p_full, (uint32_t)(m & 1), a.wait_limit_ns, abort_flag, a.status);
                    tc_fence_after();
                    const uint32_t v_addr = smem_addr(smem + C::OFF_KV + st * C::STAGE_BYTES + C::K_BYTES);
                    const uint32_t p_tmem = tmem + (uint32_t)((m & 1) * BN);
#pragma unroll
                    for (int ks = 0; ks < BN / 16; ++ks) {
                        // A = P(m) columns [8 ks, 8 ks + 8): 16 bf16 keys per row
                        const uint64_t db = smem_desc_sw128(v_addr + (uint32_t)ks * (16 * 128), BN * 128, 1024);
                        umma_bf16_tmem_a(t_o, p_tmem + (uint32_t)ks * 8u, db, idesc_pv, (m > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(pv_done);
                    umma_commit(&kv_empty[st]);
                }
            }
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0, a.wait_limit_ns, nullptr, a.status);
        }
    } else {
        // ======================= softmax warps 0-3: thread tid owns query row row0 + tid
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        const int i = pos0 + tid;     // key position of this thread's query row
        const int qrow = row0 + tid;  // its row in q and out
        float m_used = -INFINITY;  // log2-domain maximum the stored O and l are relative to
        float l = 0.f;
        for (int n = 0; n < n_kv; ++n) {
            const int sb = n & 1;
            const uint32_t t_sb = tmem + (uint32_t)(sb * BN) + lane_base;
            mbar_wait_bounded(&s_full[sb], (uint32_t)((n >> 1) & 1), a.wait_limit_ns, abort_flag, a.status);
            tc_fence_after();
            float s[BN];
            {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_sb, r0);
                tmem_ld32(t_sb + 32, r1);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    s[c] = __uint_as_float(r0[c]);
                    s[32 + c] = __uint_as_float(r1[c]);
                }
            }

            // causal mask on tiles that reach past this row
            const int j0 = n * BN;
            if (j0 + BN - 1 > pos0) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (j0 + c > i) s[c] = -INFINITY;
            }
            // row max as 8 independent chains of three-input maxima (a single 64-long chain is
            // latency-bound; the three-input form halves the instructions)
            float mx8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(s[e], s[8 + e]);
#pragma unroll
            for (int c = 16; c < BN; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = fmax3f(mx8[e], s[c + e], s[c + 8 + e]);
            const float mx = fmax3f(fmax3f(mx8[0], mx8[1], mx8[2]), fmax3f(mx8[3], mx8[4], mx8[5]),
                                    fmaxf(mx8[6], mx8[7]));
            const float m_new = mx * a.scale_log2;
            bool waited_pv = false;
            if (n == 0) {
                m_used = m_new;
            } else {
                const bool need = m_new > m_used + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    // O must be final for tile n-1 before it is rescaled in TMEM
                    mbar_wait_bounded(pv_done, (uint32_t)((n - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
                    waited_pv = true;
                    tc_fence_after();
                    const float alpha = need ? fast_exp2(m_used - m_new) : 1.f;
#pragma unroll 1
                    for (int c = 0; c < DV; c += 32) {
                        uint32_t r[32];
                        tmem_ld32(t_o + lane_base + c, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                        tmem_st32(t_o + lane_base + c, r);
                    }
                    tmem_wait_st();
                    if (need) {
                        l *= alpha;
                        m_used = m_new;
                    }
                }
            }
            // p = 2^(s * scale * log2 e - m): packed fp32 pairs, row sum as 4 pair-chains
            const f32x2_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
            const f32x2_t nm2 = f2_pack(-m_used, -m_used);
            uint32_t pk[BN / 2];
            f32x2_t l2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c = 0; c < BN; c += 2) {
                float t0, t1;
                f2_unpack(f2_fma(f2_pack(s[c], s[c + 1]), sc2, nm2), t0, t1);
                const float p0 = fast_exp2(t0);
                const float p1 = fast_exp2(t1);
                l2[(c >> 1) & 3] = f2_add(l2[(c >> 1) & 3], f2_pack(p0, p1));
                pk[c >> 1] = pack_bf16x2(p0, p1);
            }
            float la, lb;
            f2_unpack(f2_add(f2_add(l2[0], l2[1]), f2_add(l2[2], l2[3])), la, lb);
            l += la + lb;
            // P(n) over the first 32 columns of S(n): key 2c in the low half of column c
            tmem_st32(t_sb, pk);
            tmem_wait_st();
            if (n >= 1 && !waited_pv) {
                // keeps this warp at most one P.V behind, so every pv_done phase is waited in turn
                mbar_wait_bounded(pv_done, (uint32_t)((n - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        // epilogue: O / l -> bf16
        mbar_wait_bounded(pv_done, (uint32_t)((n_kv - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
        tc_fence_after();
        const float inv_l = l > 0.f ? 1.f / l : 0.f;
        __nv_bfloat16 *orow = a.out + (((size_t)b * a.seq + qrow) * a.n_q + h) * DV;
#pragma unroll 1
        for (int c = 0; c < DV; c += 32) {
            uint32_t r[32];
            tmem_ld32(t_o + lane_base + c, r);
            tmem_wait_ld();
            if (qrow < a.seq &&
                in_bounds(((long long)b * a.seq + qrow) * a.n_q + h, (long long)a.batch * a.seq * a.n_q, a.status)) {
#pragma unroll
                for (int e = 0; e < 32; e += 8) {
                    uint4 v;
                    v.x = pack_bf16x2(__uint_as_float(r[e]) * inv_l, __uint_as_float(r[e + 1]) * inv_l);
                    v.y = pack_bf16x2(__uint_as_float(r[e + 2]) * inv_l, __uint_as_float(r[e + 3]) * inv_l);
                    v.z = pack_bf16x2(__uint_as_float(r[e + 4]) * inv_l, __uint_as_float(r[e + 5]) * inv_l);
                    v.w = pack_bf16x2(__uint_as_float(r[e + 6]) * inv_l, __uint_as_float(r[e + 7]) * inv_l);
                    *reinterpret_cast<uint4 *>(orow + c + e) = v;
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace tile64

// ---------------------------------------------------------------- d_k = 128
// warps 0-3 softmax of query tile 0 and warps 4-7 of query tile 1 (thread r of a
// group owns row r = TMEM lane r), warp 8 TMA producer (both Q tiles once, K/V
// ring), warp 9 TMEM allocation and MMA issue: P_0(n) V(n), Q_0 K(n+1)^T,
// P_1(n) V(n), Q_1 K(n+1)^T, ... so one tile's softmax overlaps the other's MMAs.
// S_t is one 128-column buffer per tile; P_t(n) over its first 64 columns.
namespace pair128 {

constexpr int BM = 128;              // query rows per tile (TMEM lanes)
constexpr int QT = 2;                // query tiles per CTA
constexpr int BN = 128;              // K/V positions per tile
constexpr int kSoftmaxWarps = 4 * QT;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
constexpr int kTmemCols = 512;       // S_0 | S_1 | O_0 | O_1

template <int DK, int DV>
struct Cfg {
    static constexpr int KB = DK / 64;  // 64-wide swizzle blocks along d_k
    static constexpr int VB = DV / 64;  // ... along d_v
    static constexpr int Q_BYTES = BM * DK * 2;  // one query tile
    static constexpr int K_BYTES = BN * DK * 2;
    static constexpr int V_BYTES = BN * DV * 2;
    static constexpr int STAGE_BYTES = K_BYTES + V_BYTES;
    static constexpr int RING = 220 * 1024 - QT * Q_BYTES;
    static constexpr int STAGES = RING / STAGE_BYTES > 4 ? 4 : RING / STAGE_BYTES;
    static_assert(STAGES >= 2, "at least two K/V stages");
    static constexpr int OFF_Q = 0;
    static constexpr int OFF_KV = QT * Q_BYTES;
    static constexpr int OFF_BAR = OFF_KV + STAGES * STAGE_BYTES;
    static constexpr int SMEM = OFF_BAR + 256 + 1024;  // barriers/flags + alignment slack
    static constexpr uint32_t T_O = QT * BN;            // first O column
};


template <int DK, int DV>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_causal_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ PagedMaps pm,
                          const PrefillArgs a) {
    using C = Cfg<DK, DV>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *kv_full = bars;        // [STAGES]
    uint64_t *kv_empty = bars + 4;   // [STAGES]
    uint64_t *q_full = bars + 8;
    uint64_t *s_full = bars + 9;     // [QT]
    uint64_t *p_full = bars + 11;    // [QT]
    uint64_t *pv_done = bars + 13;   // [QT]
    uint64_t *mma_done = bars + 15;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 16);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(bars + 17);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    // heaviest tile pairs first: the pair index descends with blockIdx
    const int bh_count = a.batch * a.n_q;
    const int qp = a.n_ctas_per_head - 1 - (int)(blockIdx.x / bh_count);
    const int bh = (int)(blockIdx.x % bh_count);
    const int b = bh / a.n_q;
    const int h = bh % a.n_q;
    const int kh = h / a.q_per_k;
    const int vh = h / a.q_per_v;
    const int row0 = qp * QT * BM;          // first query row of the pair (Q and out rows)
    const int pos0 = a.prefix + row0;       // its position among the keys
    const int kv_tiles_total = (a.kv_len + BN - 1) / BN;
    int n_kv[QT];
#pragma unroll
    for (int t = 0; t < QT; ++t) n_kv[t] = min(kv_tiles_total, (pos0 + (t + 1) * BM + BN - 1) / BN);
    const int n_kv_all = n_kv[QT - 1];

    if (tid == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&kv_full[s], 1);
            mbar_init(&kv_empty[s], 1);
        }
        mbar_init(q_full, 1);
        for (int t = 0; t < QT; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&p_full[t], 4);
            mbar_init(&pv_done[t], 1);
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
        __shared__ int32_t pg_table[kPgTableWin];  // paged: a window of block-table entries
        if (lane == 0) {
            prefetch_tensormap(&tm_q);
            mbar_arrive_expect_tx(q_full, QT * C::Q_BYTES);
#pragma unroll
            for (int t = 0; t < QT; ++t)
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_4d(smem + C::OFF_Q + t * C::Q_BYTES + kb * (BM * 128), &tm_q, q_full, kb * 64, h,
                                row0 + t * BM, b);
        }
        if (a.block_table) {
            __syncwarp();
            paged_kv_producer<BN, C::KB, C::VB, C::STAGES, C::STAGE_BYTES, C::K_BYTES>(
                pm, a, b, kh, vh, n_kv_all, smem + C::OFF_KV, kv_full, kv_empty, pg_table, abort_flag, lane);
            if (lane == 0) mbar_wait_bounded(q_full, 0, a.wait_limit_ns, nullptr, a.status);
        } else if (lane == 0) {
            prefetch_tensormap(&tm_k);
            prefetch_tensormap(&tm_v);
            for (int n = 0; n < n_kv_all; ++n) {
                const int st = n % C::STAGES;
                if (n >= C::STAGES)
                    mbar_wait_bounded(&kv_empty[st], (uint32_t)(((n / C::STAGES) - 1) & 1), a.wait_limit_ns,
                                      abort_flag, a.status);
                if (*abort_flag) break;
                uint8_t *kdst = smem + C::OFF_KV + st * C::STAGE_BYTES;
                uint8_t *vdst = kdst + C::K_BYTES;
                mbar_arrive_expect_tx(&kv_full[st], C::STAGE_BYTES);
#pragma unroll
                for (int kb = 0; kb < C::KB; ++kb)
                    tma_load_4d(kdst + kb * (BN * 128), &tm_k, &kv_full[st], kb * 64, kh, n * BN, b);
#pragma unroll
                for (int vb = 0; vb < C::VB; ++vb)
                    tma_load_4d(vdst + vb * (BN * 128), &tm_v, &kv_full[st], vb * 64, vh, n * BN, b);
            }
            // drain: no copy may still be landing when the CTA exits
            mbar_wait_bounded(q_full, 0, a.wait_limit_ns, nullptr, a.status);
            for (int n = (n_kv_all > C::STAGES ? n_kv_all - C::STAGES : 0); n < n_kv_all; ++n)
                mbar_wait_bounded(&kv_full[n % C::STAGES], (uint32_t)((n / C::STAGES) & 1), a.wait_limit_ns,
                                  nullptr, a.status);
        }
    } else if (warp == kMmaWarp) {
        // ======================= MMA issuer (one thread)
        if (lane == 0) {
            constexpr uint32_t idesc_qk = umma_idesc_bf16(BM, BN, false, false);
            constexpr uint32_t idesc_pv = umma_idesc_bf16(BM, DV, false, true);
            const uint32_t q_addr = smem_addr(smem + C::OFF_Q);
            int kv_waited = -1;  // highest K/V stage fill waited for
            // S_t(n) = Q_t K(n)^T into the tile's S columns
            auto issue_qk = [&](int t, int n) {
                if (n > kv_waited) {
                    mbar_wait_bounded(&kv_full[n % C::STAGES], (uint32_t)((n / C::STAGES) & 1), a.wait_limit_ns,
                                      abort_flag, a.status);
                    kv_waited = n;
                }
                tc_fence_after();
                const uint32_t k_addr = smem_addr(smem + C::OFF_KV + (n % C::STAGES) * C::STAGE_BYTES);
                const uint32_t qa = q_addr + (uint32_t)(t * C::Q_BYTES);
#pragma unroll
                for (int ks = 0; ks < DK / 16; ++ks) {
                    const uint32_t blk = (uint32_t)(ks >> 2), sub = (uint32_t)(ks & 3) * 32u;
                    const uint64_t da = smem_desc_sw128(qa + blk * (BM * 128) + sub, 16, 1024);
                    const uint64_t db = smem_desc_sw128(k_addr + blk * (BN * 128) + sub, 16, 1024);
                    umma_bf16(tmem + (uint32_t)(t * BN), da, db, idesc_qk, ks > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[t]);
            };
            mbar_wait_bounded(q_full, 0, a.wait_limit_ns, abort_flag, a.status);
#pragma unroll
            for (int t = 0; t < QT; ++t)
                if (n_kv[t] > 0) issue_qk(t, 0);
            for (int n = 0; n < n_kv_all; ++n) {
                const uint32_t v_addr =
                    smem_addr(smem + C::OFF_KV + (n % C::STAGES) * C::STAGE_BYTES + C::K_BYTES);
#pragma unroll
                for (int t = 0; t < QT; ++t) {
                    if (n >= n_kv[t]) continue;
                    // O_t += P_t(n) V(n), P_t(n) in the first 64 columns of S_t
                    mbar_wait_bounded(&p_full[t], (uint32_t)(n & 1), a.wait_limit_ns, abort_flag, a.status);
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < BN / 16; ++ks) {
                        const uint64_t db = smem_desc_sw128(v_addr + (uint32_t)ks * (16 * 128), BN * 128, 1024);
                        umma_bf16_tmem_a(tmem + C::T_O + (uint32_t)(t * DV), tmem + (uint32_t)(t * BN + ks * 8), db,
                                         idesc_pv, (n > 0 || ks > 0) ? 1u : 0u);
                    }
                    umma_commit(&pv_done[t]);
                    if (n + 1 < n_kv[t]) issue_qk(t, n + 1);
                }
                umma_commit(&kv_empty[n % C::STAGES]);  // every MMA reading stage n has been issued
            }
            umma_commit(mma_done);
            mbar_wait_bounded(mma_done, 0, a.wait_limit_ns, nullptr, a.status);
        }
    } else {
        // ======================= softmax: warps 4t .. 4t+3 for query tile t, thread r owns row r
        const int t = warp >> 2;
        const int r = tid & (BM - 1);
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t t_s = tmem + (uint32_t)(t * BN) + lane_base;
        const uint32_t t_o = tmem + C::T_O + (uint32_t)(t * DV) + lane_base;
        const int tile_row0 = pos0 + t * BM;  // key position of the tile's first query row
        const int i = tile_row0 + r;          // key position of this thread's query row
        const int qrow = row0 + t * BM + r;   // its row in q and out
        const int nk = n_kv[t];
        float m_used = -INFINITY;     // log2-domain maximum the stored O and l are relative to
        float l = 0.f;
        for (int n = 0; n < nk; ++n) {
            mbar_wait_bounded(&s_full[t], (uint32_t)(n & 1), a.wait_limit_ns, abort_flag, a.status);
            tc_fence_after();
            float s[BN];
#pragma unroll
            for (int c = 0; c < BN; c += 32) {
                uint32_t rr[32];
                tmem_ld32(t_s + (uint32_t)c, rr);
#pragma unroll
                for (int e = 0; e < 32; ++e) s[c + e] = __uint_as_float(rr[e]);
            }
            tmem_wait_ld();

            // causal mask on tiles that reach past this tile's first row
            const int j0 = n * BN;
            if (j0 + BN - 1 > tile_row0) {
#pragma unroll
                for (int c = 0; c < BN; ++c)
                    if (j0 + c > i) s[c] = -INFINITY;
            }
            // row max as 8 independent chains
            float mx8[8];  // three-input maxima, as in the d_k = 64 tiling
#pragma unroll
            for (int e = 0; e < 8; ++e) mx8[e] = fmaxf(s[e], s[8 + e]);
#pragma unroll
            for (int c = 16; c < BN; c += 16)
#pragma unroll
                for (int e = 0; e < 8; ++e) mx8[e] = fmax3f(mx8[e], s[c + e], s[c + 8 + e]);
            const float mx = fmax3f(fmax3f(mx8[0], mx8[1], mx8[2]), fmax3f(mx8[3], mx8[4], mx8[5]),
                                    fmaxf(mx8[6], mx8[7]));
            const float m_new = mx * a.scale_log2;
            // the lazy O rescale is decided here and done after P is stored (the row's 128 scores are
            // dead by then; loading O next to them overran the 168 registers ten warps leave a thread)
            bool rescale = false;
            float alpha = 1.f;
            if (n == 0) {
                m_used = m_new;
            } else {
                const bool need = m_new > m_used + kRescaleLog2;
                if (__any_sync(0xffffffffu, need)) {
                    rescale = true;
                    if (need) {
                        alpha = fast_exp2(m_used - m_new);
                        l *= alpha;
                        m_used = m_new;
                    }
                }
            }
            // p = 2^(s * scale * log2 e - m): packed fp32 pairs, row sum as 4 pair-chains;
            // P in bf16 pairs over the first 64 columns of S (key 2c in the low half of column c)
            const f32x2_t sc2 = f2_pack(a.scale_log2, a.scale_log2);
            const f32x2_t nm2 = f2_pack(-m_used, -m_used);
            f32x2_t l2[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
            for (int c0 = 0; c0 < BN; c0 += 32) {  // 32 keys (16 packed columns) per store
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    float t0, t1;
                    f2_unpack(f2_fma(f2_pack(s[c0 + c], s[c0 + c + 1]), sc2, nm2), t0, t1);
                    const float p0 = fast_exp2(t0);
                    const float p1 = fast_exp2(t1);
                    l2[(c >> 1) & 3] = f2_add(l2[(c >> 1) & 3], f2_pack(p0, p1));
                    pk[c >> 1] = pack_bf16x2(p0, p1);
                }
                tmem_st_cols<16>(t_s + (uint32_t)(c0 / 2), pk);
            }
            float la, lb;
            f2_unpack(f2_add(f2_add(l2[0], l2[1]), f2_add(l2[2], l2[3])), la, lb);
            l += la + lb;
            tmem_wait_st();
            if (n >= 1) {
                // O is final for tile n-1 (and this group stays at most one P.V behind, so every pv_done
                // phase is waited in turn); then the rescale, before P(n) is handed to the MMA
                mbar_wait_bounded(&pv_done[t], (uint32_t)((n - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
                if (rescale) {
                    tc_fence_after();
#pragma unroll 1
                    for (int c = 0; c < DV; c += 32) {
                        uint32_t rr[32];
                        tmem_ld32(t_o + (uint32_t)c, rr);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) rr[e] = __float_as_uint(__uint_as_float(rr[e]) * alpha);
                        tmem_st32(t_o + (uint32_t)c, rr);
                    }
                    tmem_wait_st();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&p_full[t]);
        }
        // epilogue: O / l -> bf16
        if (nk > 0) {
            mbar_wait_bounded(&pv_done[t], (uint32_t)((nk - 1) & 1), a.wait_limit_ns, abort_flag, a.status);
            tc_fence_after();
            const float inv_l = l > 0.f ? 1.f / l : 0.f;
            __nv_bfloat16 *orow = a.out + (((size_t)b * a.seq + qrow) * a.n_q + h) * DV;
#pragma unroll 1
            for (int c = 0; c < DV; c += 32) {
                uint32_t rr[32];
                tmem_ld32(t_o + (uint32_t)c, rr);
                tmem_wait_ld();
                if (qrow < a.seq &&
                    in_bounds(((long long)b * a.seq + qrow) * a.n_q + h, (long long)a.batch * a.seq * a.n_q, a.status)) {
#pragma unroll
                    for (int e = 0; e < 32; e += 8) {
                        uint4 v;
                        v.x = pack_bf16x2(__uint_as_float(rr[e]) * inv_l, __uint_as_float(rr[e + 1]) * inv_l);
                        v.y = pack_bf16x2(__uint_as_float(rr[e + 2]) * inv_l, __uint_as_float(rr[e + 3]) * inv_l);
                        v.z = pack_bf16x2(__uint_as_float(rr[e + 4]) * inv_l, __uint_as_float(rr[e + 5]) * inv_l);
                        v.w = pack_bf16x2(__uint_as_float(rr[e + 6]) * inv_l, __uint_as_float(rr[e + 7]) * inv_l);
                        *reinterpret_cast<uint4 *>(orow + c + e) = v;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

}  // namespace pair128

using PrefillFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, PagedMaps, PrefillArgs);

struct Plan {
    PrefillFn fn;
    int smem, threads, rows_per_cta, q_box, kv_box;
};

bool pick(int dk, int dv, Plan *p) {
    if (dk == 64) {
        using namespace tile64;
        p->threads = kThreads;
        p->rows_per_cta = BM;
        p->q_box = BM;
        p->kv_box = BN;
        if (dv == 64) { p->smem = Cfg<64, 64>::SMEM; p->fn = prefill_causal_kernel<64, 64>; return true; }
        if (dv == 128) { p->smem = Cfg<64, 128>::SMEM; p->fn = prefill_causal_kernel<64, 128>; return true; }
    } else if (dk == 128) {
        using namespace pair128;
        p->threads = kThreads;
        p->rows_per_cta = QT * BM;
        p->q_box = BM;
        p->kv_box = BN;
        if (dv == 64) { p->smem = Cfg<128, 64>::SMEM; p->fn = prefill_causal_kernel<128, 64>; return true; }
        if (dv == 128) { p->smem = Cfg<128, 128>::SMEM; p->fn = prefill_causal_kernel<128, 128>; return true; }
    }
    return false;
}

}  // namespace

diffqkv_status_t prefill_launch(const diffqkv_dims_t *d, const void *q, const void *k, const void *v, int32_t seq_len,
                                void *out, cudaStream_t stream, int32_t prefix_len, int32_t *status,
                                const PagedCache *paged) {
    diffqkv_status_t st = validate_dims(d);
    if (st != DIFFQKV_OK) return st;
    if (!q || !k || !v || !out || seq_len < 1 || prefix_len < 0) return DIFFQKV_ERR_INVALID_ARG;
    if ((long long)prefix_len + seq_len > 0x7fffffffLL) return DIFFQKV_ERR_UNSUPPORTED;
    const int32_t kv_len = prefix_len + seq_len;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(status) & 3u))
        return DIFFQKV_ERR_MISALIGNED;
    Plan plan;
    if (!pick(d->d_k, d->d_v, &plan)) return DIFFQKV_ERR_UNSUPPORTED;
    int32_t n_pages = 0, max_box_log = 0;
    if (paged) {
        const long long P = paged->page_size;
        if (!paged->block_table || paged->max_blocks < 1 || P < 1 || paged->num_pages < 1)
            return DIFFQKV_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(paged->block_table) & 3u) return DIFFQKV_ERR_MISALIGNED;
        // boxes of at least 8 rows keep every box on a 1024-byte swizzle atom of the tile
        if (P % 8 != 0) return DIFFQKV_ERR_UNSUPPORTED;
        n_pages = (int32_t)((kv_len + P - 1) / P);
        if (n_pages > paged->max_blocks) return DIFFQKV_ERR_INVALID_ARG;
        if ((long long)paged->num_pages * P > 0x7fffffffLL ||
            (long long)d->batch * paged->max_blocks > 0x7fffffffLL)
            return DIFFQKV_ERR_UNSUPPORTED;
        while (max_box_log < 3 && P % (8 << (max_box_log + 1)) == 0 && (8 << (max_box_log + 1)) <= plan.kv_box)
            ++max_box_log;
    }
    DeviceInfo dev;
    st = current_device_info(&dev);
    if (st != DIFFQKV_OK) return st;

    CUtensorMap tm_q, tm_k, tm_v;
    PagedMaps pm;
    memset(&pm, 0, sizeof(pm));
    st = make_tensor_map_4d(&tm_q, q, d->d_k, d->n_q, seq_len, d->batch, 64, 1, plan.q_box, 1,
                            CU_TENSOR_MAP_SWIZZLE_128B);
    if (st != DIFFQKV_OK) return st;
    if (!paged) {
        st = make_tensor_map_4d(&tm_k, k, d->d_k, d->n_k, kv_len, d->batch, 64, 1, plan.kv_box, 1,
                                CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != DIFFQKV_OK) return st;
        st = make_tensor_map_4d(&tm_v, v, d->d_v, d->n_v, kv_len, d->batch, 64, 1, plan.kv_box, 1,
                                CU_TENSOR_MAP_SWIZZLE_128B);
        if (st != DIFFQKV_OK) return st;
    } else {
        // whole-pool maps with boxes of 8 << i rows, and the tail views: the same pages with only the
        // rows of the last page that hold positions (the rest of a box there reads as zeros)
        const uint64_t P = (uint64_t)paged->page_size;
        const uint64_t last_rows = (uint64_t)kv_len - (uint64_t)(n_pages - 1) * P;
        for (int i = 0; i < 4; ++i) {
            const int hi = i <= max_box_log ? i : 0;
            const uint32_t rows = 8u << hi;
            st = make_tensor_map_4d(&pm.k[i], k, d->d_k, d->n_k, P, paged->num_pages, 64, 1, rows, 1,
                                    CU_TENSOR_MAP_SWIZZLE_128B);
            if (st == DIFFQKV_OK)
                st = make_tensor_map_4d(&pm.v[i], v, d->d_v, d->n_v, P, paged->num_pages, 64, 1, rows, 1,
                                        CU_TENSOR_MAP_SWIZZLE_128B);
            const uint64_t kd[4] = {(uint64_t)d->d_k, (uint64_t)d->n_k, last_rows, (uint64_t)paged->num_pages};
            const uint64_t ks[3] = {(uint64_t)d->d_k * 2, (uint64_t)d->d_k * d->n_k * 2, (uint64_t)d->d_k * d->n_k * P * 2};
            const uint64_t vd[4] = {(uint64_t)d->d_v, (uint64_t)d->n_v, last_rows, (uint64_t)paged->num_pages};
            const uint64_t vs[3] = {(uint64_t)d->d_v * 2, (uint64_t)d->d_v * d->n_v * 2, (uint64_t)d->d_v * d->n_v * P * 2};
            const uint32_t box[4] = {64, 1, rows, 1};
            if (st == DIFFQKV_OK) st = make_tensor_map_4d_strided(&pm.k_tail[i], k, kd, ks, box, CU_TENSOR_MAP_SWIZZLE_128B);
            if (st == DIFFQKV_OK) st = make_tensor_map_4d_strided(&pm.v_tail[i], v, vd, vs, box, CU_TENSOR_MAP_SWIZZLE_128B);
            if (st != DIFFQKV_OK) return st;
        }
        tm_k = pm.k[0];
        tm_v = pm.v[0];
    }

    PrefillArgs a;
    a.out = static_cast<__nv_bfloat16 *>(out);
    a.status = status ? status : dev.status_word;  // the caller's word, else the device's
    a.batch = d->batch;
    a.seq = seq_len;
    a.prefix = prefix_len;
    a.kv_len = kv_len;
    a.n_q = d->n_q;
    a.n_k = d->n_k;
    a.n_v = d->n_v;
    a.q_per_k = d->n_q / d->n_k;
    a.q_per_v = d->n_q / d->n_v;
    a.n_ctas_per_head = (seq_len + plan.rows_per_cta - 1) / plan.rows_per_cta;
    a.scale_log2 = (float)((double)d->scale * 1.4426950408889634);
    a.wait_limit_ns = kWaitLimitNs;
    a.block_table = paged ? paged->block_table : nullptr;
    a.max_blocks = paged ? paged->max_blocks : 0;
    a.page_size = paged ? paged->page_size : 0;
    a.num_pages = paged ? paged->num_pages : 0;
    a.n_pages = n_pages;
    a.max_box_log = max_box_log;
    a.page_shift = -1;
    if (paged && (paged->page_size & (paged->page_size - 1)) == 0) {
        a.page_shift = 0;
        while ((1 << a.page_shift) < paged->page_size) ++a.page_shift;
    }
    const long long grid = (long long)a.n_ctas_per_head * d->batch * d->n_q;
    if (grid > 0x7fffffffLL) return DIFFQKV_ERR_UNSUPPORTED;
    if (ensure_dynamic_smem((const void *)plan.fn, plan.smem) != DIFFQKV_OK) return DIFFQKV_ERR_CUDA;
    plan.fn<<<(unsigned)grid, plan.threads, plan.smem, stream>>>(tm_q, tm_k, tm_v, pm, a);
    if (cudaGetLastError() != cudaSuccess) return DIFFQKV_ERR_CUDA;
    return DIFFQKV_OK;
}

}  // namespace diffqkv
