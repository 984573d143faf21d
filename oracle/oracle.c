/*
 * oracle.c -- plain, slow, fp64 CPU oracle for DiffQKV attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file; only tests/, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the
 * CUDA library under asymmetric_head_kv_b200/.
 *
 * What it computes (source: "Sigma: Differential Rescaling of Query, Key and
 * Value for Efficient Language Models", structured summary page, section 3.4
 * "DiffQKV Attention: Generalized Formulation", Steps 2-5; "Selective V Cache
 * Fetching"; "FlexHeadFA Kernel and Deployment Infrastructure"):
 *
 *   head map     idx_i = floor(idx_q * n_i / n_q), i in {k, v}     (Step 3)
 *   scores       s_j   = scale * <q_h, K[j, idx_k]>                 (Step 4)
 *   weights      alpha = softmax_j(s)                               (Step 4)
 *   output       o_h   = sum_j alpha_j V[j, idx_v]                  (Step 5)
 *   split/combine   per KV chunk: (max, sum of exp, unnormalised o); the
 *                combine pass rescales each chunk by exp(m_c - M)   (FlexHeadFA)
 *   selective V  o_h  ~= sum over the top-k positions of the weights,
 *                renormalised over that set                         (Selective V)
 *   paged cache  position j of sequence b is row j % P of pool page
 *                table[b][j / P]; K and V keep separate pools  ("Where
 *                Existing Approaches Fall Short", system-level optimisations)
 *   d_q != d_k   each cached K row is projected up to the query width,
 *                k_up = W k, before the dot product         (Step 4, Attend)
 *   augmented Q  q = q_down( SiLU(q_gate(x)) * q_up(x) ), SiLU(g) = g / (1 + e^-g),
 *                three bias-free linear maps (section 3.2 "Big-Picture
 *                Architecture", item 4: augmented Q with SwiGLU gating)
 *
 * All arithmetic is fp64.  bf16 inputs arrive as raw 16-bit patterns and are
 * widened exactly.  The top-k selection ranks positions by the EXACT dot
 * product (a fixed-point superaccumulator, every bf16 x bf16 product is an
 * integer times a power of two), ties broken toward the lower position.
 *
 * Status codes: 0 ok, -1 bad argument, -2 non-finite bf16 input where an
 * exact key is needed, -3 out of memory.
 *
 * Parity pins: every function here is pinned by tests in tests/test_oracle_*.py
 * (closed forms, library SDPA in fp64, brute force, Fraction arithmetic).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

/* ------------------------------------------------------------------ */
/* bf16 widening                                                       */
/* ------------------------------------------------------------------ */

/* bf16 is the upper half of an IEEE binary32 pattern: widening is exact. */
static double bf16_to_f64(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------ */
/* GroupSharing head map (section 3.4, Step 3; FlexHeadFA address calc) */
/* ------------------------------------------------------------------ */

/* Query head h reads K (or V) head floor(h * n_kv / n_q). */
int oracle_head_map(int n_q, int n_kv, int h) {
    if (n_q <= 0 || n_kv <= 0 || h < 0 || h >= n_q) return -1;
    return (int)(((int64_t)h * n_kv) / n_q);
}

/* ------------------------------------------------------------------ */
/* simple pthread fan-out over independent rows                        */
/* ------------------------------------------------------------------ */

typedef void (*row_fn)(void *ctx, int64_t row);

typedef struct {
    row_fn fn;
    void *ctx;
    int64_t n_rows;
    int64_t next;
    pthread_mutex_t lock;
} pool_t;

static void *pool_worker(void *arg) {
    pool_t *p = (pool_t *)arg;
    for (;;) {
        pthread_mutex_lock(&p->lock);
        int64_t r = p->next++;
        pthread_mutex_unlock(&p->lock);
        if (r >= p->n_rows) break;
        p->fn(p->ctx, r);
    }
    return NULL;
}

static void run_rows(row_fn fn, void *ctx, int64_t n_rows, int n_threads) {
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > 256) n_threads = 256;
    if ((int64_t)n_threads > n_rows) n_threads = (int)(n_rows > 0 ? n_rows : 1);
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n_rows = n_rows;
    p.next = 0;
    pthread_mutex_init(&p.lock, NULL);
    if (n_threads == 1) {
        pool_worker(&p);
    } else {
        pthread_t th[256];
        int started = 0;
        for (int i = 0; i < n_threads; ++i) {
            if (pthread_create(&th[i], NULL, pool_worker, &p) != 0) break;
            ++started;
        }
        if (started == 0) pool_worker(&p);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    }
    pthread_mutex_destroy(&p.lock);
}

/* ------------------------------------------------------------------ */
/* Decode over a KV cache (section 3.4, Steps 2-5)                     */
/* ------------------------------------------------------------------ */

typedef struct {
    int batch, n_q, n_k, n_v, d_k, d_v, t_max;
    double scale;
    int num_splits;            /* 0: plain two-pass softmax; >0: split/combine */
    const uint16_t *q;         /* [B, n_q, d_k]        */
    const uint16_t *k;         /* [B, t_max, n_k, d_k] */
    const uint16_t *v;         /* [B, t_max, n_v, d_v] */
    const int32_t *seq_lens;   /* [B]                  */
    const int32_t *rows;       /* n_rows pairs (b, h), or NULL for all */
    double *out;               /* [n_rows, d_v]        */
    int status;
} decode_ctx;

/* s_j = scale * sum_c q[c] * K[b, j, kh, c], for 0 <= j < T */
static void decode_scores(const decode_ctx *c, int b, int h, int T, double *s) {
    const int kh = oracle_head_map(c->n_q, c->n_k, h);
    const uint16_t *q = c->q + ((int64_t)b * c->n_q + h) * c->d_k;
    for (int j = 0; j < T; ++j) {
        const uint16_t *kr = c->k + (((int64_t)b * c->t_max + j) * c->n_k + kh) * c->d_k;
        double acc = 0.0;
        for (int e = 0; e < c->d_k; ++e) acc += bf16_to_f64(q[e]) * bf16_to_f64(kr[e]);
        s[j] = c->scale * acc;
    }
}

static const uint16_t *v_row(const decode_ctx *c, int b, int j, int vh) {
    return c->v + (((int64_t)b * c->t_max + j) * c->n_v + vh) * c->d_v;
}

static void decode_row(void *vctx, int64_t r) {
    decode_ctx *c = (decode_ctx *)vctx;
    int b, h;
    if (c->rows) { b = c->rows[2 * r]; h = c->rows[2 * r + 1]; }
    else { b = (int)(r / c->n_q); h = (int)(r % c->n_q); }
    double *o = c->out + r * c->d_v;
    for (int e = 0; e < c->d_v; ++e) o[e] = 0.0;
    int T = c->seq_lens[b];
    if (T > c->t_max) T = c->t_max;
    if (T <= 0) return; /* empty context: the output row is zero */
    const int vh = oracle_head_map(c->n_q, c->n_v, h);
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    if (!s) { c->status = -3; return; }
    decode_scores(c, b, h, T, s);

    if (c->num_splits <= 0) {
        /* two-pass full softmax: m = max s; w = exp(s - m); o = sum w V / sum w */
        double m = -INFINITY;
        for (int j = 0; j < T; ++j) if (s[j] > m) m = s[j];
        double den = 0.0;
        for (int j = 0; j < T; ++j) {
            const double w = exp(s[j] - m);
            den += w;
            const uint16_t *vr = v_row(c, b, j, vh);
            for (int e = 0; e < c->d_v; ++e) o[e] += w * bf16_to_f64(vr[e]);
        }
        for (int e = 0; e < c->d_v; ++e) o[e] /= den;
    } else {
        /* split/combine: chunk i covers [i*L, min(T, (i+1)*L)), L = ceil(T/splits).
         * Each chunk keeps (m_i, l_i, o_i) with o_i unnormalised; the combine
         * pass merges them with weights exp(m_i - M), M = max_i m_i. */
        const int ns = c->num_splits;
        const int L = (T + ns - 1) / ns;
        double *mi = (double *)malloc(sizeof(double) * (size_t)ns);
        double *li = (double *)malloc(sizeof(double) * (size_t)ns);
        double *oi = (double *)calloc((size_t)ns * (size_t)c->d_v, sizeof(double));
        int *used = (int *)calloc((size_t)ns, sizeof(int));
        if (!mi || !li || !oi || !used) { c->status = -3; free(mi); free(li); free(oi); free(used); free(s); return; }
        for (int i = 0; i < ns; ++i) {
            const int j0 = i * L, j1 = (j0 + L < T) ? j0 + L : T;
            if (j0 >= j1) continue;
            used[i] = 1;
            double m = -INFINITY;
            for (int j = j0; j < j1; ++j) if (s[j] > m) m = s[j];
            double l = 0.0;
            for (int j = j0; j < j1; ++j) {
                const double w = exp(s[j] - m);
                l += w;
                const uint16_t *vr = v_row(c, b, j, vh);
                for (int e = 0; e < c->d_v; ++e) oi[(int64_t)i * c->d_v + e] += w * bf16_to_f64(vr[e]);
            }
            mi[i] = m;
            li[i] = l;
        }
        double M = -INFINITY;
        for (int i = 0; i < ns; ++i) if (used[i] && mi[i] > M) M = mi[i];
        double den = 0.0;
        for (int i = 0; i < ns; ++i) {
            if (!used[i]) continue;
            const double f = exp(mi[i] - M);
            den += f * li[i];
            for (int e = 0; e < c->d_v; ++e) o[e] += f * oi[(int64_t)i * c->d_v + e];
        }
        for (int e = 0; e < c->d_v; ++e) o[e] /= den;
        free(mi); free(li); free(oi); free(used);
    }
    free(s);
}

static int check_dims(int batch, int n_q, int n_k, int n_v, int d_k, int d_v) {
    if (batch < 0 || n_q <= 0 || n_k <= 0 || n_v <= 0 || d_k <= 0 || d_v <= 0) return -1;
    if (n_k > n_q || n_v > n_q) return -1;
    return 0;
}

/* Decode for n_rows (b, h) pairs (rows == NULL: all B*n_q rows in order).
 * out: fp64 [n_rows, d_v]. */
int oracle_decode(int batch, int n_q, int n_k, int n_v, int d_k, int d_v, double scale,
                  const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *seq_lens, int t_max, int num_splits,
                  const int32_t *rows, int64_t n_rows, double *out, int n_threads) {
    if (check_dims(batch, n_q, n_k, n_v, d_k, d_v) || t_max < 0 || !q || !k_cache || !v_cache ||
        !seq_lens || !out)
        return -1;
    if (!rows) n_rows = (int64_t)batch * n_q;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[2 * r] < 0 || rows[2 * r] >= batch || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= n_q)
            return -1;
    decode_ctx c = {batch, n_q, n_k, n_v, d_k, d_v, t_max, scale, num_splits,
                    q, k_cache, v_cache, seq_lens, rows, out, 0};
    run_rows(decode_row, &c, n_rows, n_threads);
    return c.status;
}

/* ------------------------------------------------------------------ */
/* Causal prefill: row i attends to positions j <= i (same arithmetic) */
/* ------------------------------------------------------------------ */

typedef struct {
    int batch, seq, n_q, n_k, n_v, d_k, d_v;
    double scale;
    const uint16_t *q;   /* [B, S, n_q, d_k] */
    const uint16_t *k;   /* [B, S, n_k, d_k] */
    const uint16_t *v;   /* [B, S, n_v, d_v] */
    const int32_t *rows; /* n_rows triples (b, i, h), or NULL for all */
    double *out;         /* [n_rows, d_v] */
    int status;
} prefill_ctx;

static void prefill_row(void *vctx, int64_t r) {
    prefill_ctx *c = (prefill_ctx *)vctx;
    int b, i, h;
    if (c->rows) { b = c->rows[3 * r]; i = c->rows[3 * r + 1]; h = c->rows[3 * r + 2]; }
    else {
        b = (int)(r / ((int64_t)c->seq * c->n_q));
        const int64_t rem = r % ((int64_t)c->seq * c->n_q);
        i = (int)(rem / c->n_q);
        h = (int)(rem % c->n_q);
    }
    const int kh = oracle_head_map(c->n_q, c->n_k, h);
    const int vh = oracle_head_map(c->n_q, c->n_v, h);
    const int T = i + 1;
    double *o = c->out + r * c->d_v;
    for (int e = 0; e < c->d_v; ++e) o[e] = 0.0;
    double *s = (double *)malloc(sizeof(double) * (size_t)T);
    if (!s) { c->status = -3; return; }
    const uint16_t *qr = c->q + (((int64_t)b * c->seq + i) * c->n_q + h) * c->d_k;
    double m = -INFINITY;
    for (int j = 0; j < T; ++j) {
        const uint16_t *kr = c->k + (((int64_t)b * c->seq + j) * c->n_k + kh) * c->d_k;
        double acc = 0.0;
        for (int e = 0; e < c->d_k; ++e) acc += bf16_to_f64(qr[e]) * bf16_to_f64(kr[e]);
        s[j] = c->scale * acc;
        if (s[j] > m) m = s[j];
    }
    double den = 0.0;
    for (int j = 0; j < T; ++j) {
        const double w = exp(s[j] - m);
        den += w;
        const uint16_t *vr = c->v + (((int64_t)b * c->seq + j) * c->n_v + vh) * c->d_v;
        for (int e = 0; e < c->d_v; ++e) o[e] += w * bf16_to_f64(vr[e]);
    }
    for (int e = 0; e < c->d_v; ++e) o[e] /= den;
    free(s);
}

int oracle_prefill_causal(int batch, int seq, int n_q, int n_k, int n_v, int d_k, int d_v,
                          double scale, const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *rows, int64_t n_rows, double *out, int n_threads) {
    if (check_dims(batch, n_q, n_k, n_v, d_k, d_v) || seq < 0 || !q || !k || !v || !out) return -1;
    if (!rows) n_rows = (int64_t)batch * seq * n_q;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[3 * r] < 0 || rows[3 * r] >= batch || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= seq ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= n_q)
            return -1;
    prefill_ctx c = {batch, seq, n_q, n_k, n_v, d_k, d_v, scale, q, k, v, rows, out, 0};
    run_rows(prefill_row, &c, n_rows, n_threads);
    return c.status;
}

/* ------------------------------------------------------------------ */
/* Exact dot products of bf16 vectors (fixed-point superaccumulator)   */
/* ------------------------------------------------------------------ */
/*
 * A finite bf16 value is M * 2^x with integer 0 <= M < 256:
 *   exponent field E = 0  (zero/subnormal): M = mantissa,       x = -133
 *   1 <= E <= 254         (normal):         M = 128 + mantissa, x = E - 134
 * so a product is P * 2^(xa + xb) with 0 <= P < 2^16 and xa + xb >= -266.
 * The accumulator is an integer in units of 2^-266, held as SA_DIGITS
 * base-2^32 digits in int64 slots (room for carries while summing).
 * After normalisation digits 0..SA_DIGITS-2 lie in [0, 2^32) and the top
 * digit is signed: the value is sum_i d_i * 2^(32 i - 266).
 */
#define SA_DIGITS 18
#define SA_LSB_EXP 266

typedef struct { int64_t d[SA_DIGITS]; } sacc_t;

static int bf16_decompose(uint16_t bits, int *neg, int *mant, int *expo) {
    const int E = (bits >> 7) & 0xff;
    const int m = bits & 0x7f;
    if (E == 0xff) return -2; /* inf / nan */
    *neg = (bits >> 15) & 1;
    if (E == 0) { *mant = m; *expo = -133; }
    else { *mant = 128 + m; *expo = E - 134; }
    return 0;
}

static int sa_add_product(sacc_t *a, uint16_t x, uint16_t y) {
    int nx, mx, ex, ny, my, ey;
    if (bf16_decompose(x, &nx, &mx, &ex) || bf16_decompose(y, &ny, &my, &ey)) return -2;
    const int64_t P = (int64_t)mx * my;
    if (P == 0) return 0;
    const int off = ex + ey + SA_LSB_EXP; /* >= 0 */
    const int64_t v = P * ((int64_t)1 << (off % 32)); /* < 2^47 */
    a->d[off / 32] += (nx ^ ny) ? -v : v;
    return 0;
}

static void sa_normalize(sacc_t *a) {
    for (int i = 0; i + 1 < SA_DIGITS; ++i) {
        /* floor division by 2^32 (works for negative digits too) */
        int64_t c = a->d[i] / 4294967296LL;
        if (a->d[i] - c * 4294967296LL < 0) c -= 1;
        a->d[i] -= c * 4294967296LL;
        a->d[i + 1] += c;
    }
}

/* Compare two normalised accumulators: -1, 0, +1. */
static int sa_compare(const sacc_t *a, const sacc_t *b) {
    for (int i = SA_DIGITS - 1; i >= 0; --i) {
        if (a->d[i] < b->d[i]) return -1;
        if (a->d[i] > b->d[i]) return 1;
    }
    return 0;
}

static int sa_dot(const uint16_t *a, const uint16_t *b, int n, sacc_t *out) {
    memset(out, 0, sizeof *out);
    for (int i = 0; i < n; ++i)
        if (sa_add_product(out, a[i], b[i])) return -2;
    sa_normalize(out);
    return 0;
}

/* Exact dot product; digits_out[SA_DIGITS] receives the normalised digits.
 * Returns the number of digits (SA_DIGITS) and writes the weight exponent of
 * digit 0 (-266) to *lsb_exp, or a negative status. */
int oracle_exact_dot(const uint16_t *a, const uint16_t *b, int n, int64_t *digits_out, int *lsb_exp) {
    if (!a || !b || !digits_out || n < 0) return -1;
    sacc_t s;
    if (sa_dot(a, b, n, &s)) return -2;
    memcpy(digits_out, s.d, sizeof s.d);
    if (lsb_exp) *lsb_exp = -SA_LSB_EXP;
    return SA_DIGITS;
}

/* ------------------------------------------------------------------ */
/* Selective V fetch (top-k positions per query head), renormalised    */
/* ------------------------------------------------------------------ */

typedef struct {
    decode_ctx base;
    int topk;
    int full_weights; /* 0: renormalise over the kept set; 1: full-softmax weights alpha_j */
    int32_t *idx_out; /* [n_rows, topk], ascending, -1 padded */
} topv_ctx;

typedef struct { sacc_t key; int j; } keyed_pos;

/* order: larger exact key first; equal keys -> lower position first */
static int keyed_cmp(const void *pa, const void *pb) {
    const keyed_pos *a = (const keyed_pos *)pa, *b = (const keyed_pos *)pb;
    const int c = sa_compare(&a->key, &b->key);
    if (c != 0) return -c;
    return (a->j > b->j) - (a->j < b->j);
}

static int int_cmp(const void *pa, const void *pb) {
    const int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

static void topv_row(void *vctx, int64_t r) {
    topv_ctx *tc = (topv_ctx *)vctx;
    decode_ctx *c = &tc->base;
    int b, h;
    if (c->rows) { b = c->rows[2 * r]; h = c->rows[2 * r + 1]; }
    else { b = (int)(r / c->n_q); h = (int)(r % c->n_q); }
    double *o = c->out + r * c->d_v;
    int32_t *idx = tc->idx_out + r * tc->topk;
    for (int e = 0; e < c->d_v; ++e) o[e] = 0.0;
    for (int e = 0; e < tc->topk; ++e) idx[e] = -1;
    int T = c->seq_lens[b];
    if (T > c->t_max) T = c->t_max;
    if (T <= 0 || tc->topk <= 0) return;
    const int kh = oracle_head_map(c->n_q, c->n_k, h);
    const int vh = oracle_head_map(c->n_q, c->n_v, h);
    const uint16_t *q = c->q + ((int64_t)b * c->n_q + h) * c->d_k;

    /* 1. exact key e_j = <q, K_j> for every cached position */
    keyed_pos *kp = (keyed_pos *)malloc(sizeof(keyed_pos) * (size_t)T);
    if (!kp) { c->status = -3; return; }
    for (int j = 0; j < T; ++j) {
        const uint16_t *kr = c->k + (((int64_t)b * c->t_max + j) * c->n_k + kh) * c->d_k;
        if (sa_dot(q, kr, c->d_k, &kp[j].key)) { c->status = -2; free(kp); return; }
        kp[j].j = j;
    }
    /* 2. the k largest, ties toward the lower position */
    qsort(kp, (size_t)T, sizeof(keyed_pos), keyed_cmp);
    const int ksel = tc->topk < T ? tc->topk : T;
    int *sel = (int *)malloc(sizeof(int) * (size_t)ksel);
    if (!sel) { c->status = -3; free(kp); return; }
    for (int e = 0; e < ksel; ++e) sel[e] = kp[e].j;
    free(kp);
    qsort(sel, (size_t)ksel, sizeof(int), int_cmp);
    for (int e = 0; e < ksel; ++e) idx[e] = sel[e];

    /* 3. weighted V rows of the selected set: the softmax renormalised over the set
     *    ("Selective V Cache Fetching" as the workload asks), or the full-softmax
     *    weights alpha_j of the pages' formula, the other positions counting as zero */
    double *s = (double *)malloc(sizeof(double) * (size_t)ksel);
    if (!s) { c->status = -3; free(sel); return; }
    double m = -INFINITY;
    for (int e = 0; e < ksel; ++e) {
        const uint16_t *kr = c->k + (((int64_t)b * c->t_max + sel[e]) * c->n_k + kh) * c->d_k;
        double acc = 0.0;
        for (int d = 0; d < c->d_k; ++d) acc += bf16_to_f64(q[d]) * bf16_to_f64(kr[d]);
        s[e] = c->scale * acc;
        if (s[e] > m) m = s[e];
    }
    double den = 0.0;
    if (tc->full_weights) {
        /* alpha_j = exp(s_j - M) / sum over every cached position of exp(s_i - M) */
        double *all = (double *)malloc(sizeof(double) * (size_t)T);
        if (!all) { c->status = -3; free(s); free(sel); return; }
        double mall = -INFINITY;
        for (int j = 0; j < T; ++j) {
            const uint16_t *kr = c->k + (((int64_t)b * c->t_max + j) * c->n_k + kh) * c->d_k;
            double acc = 0.0;
            for (int d = 0; d < c->d_k; ++d) acc += bf16_to_f64(q[d]) * bf16_to_f64(kr[d]);
            all[j] = c->scale * acc;
            if (all[j] > mall) mall = all[j];
        }
        for (int j = 0; j < T; ++j) den += exp(all[j] - mall);
        free(all);
        m = mall;
    }
    double kept = 0.0;
    for (int e = 0; e < ksel; ++e) {
        const double w = exp(s[e] - m);
        kept += w;
        const uint16_t *vr = v_row(c, b, sel[e], vh);
        for (int d = 0; d < c->d_v; ++d) o[d] += w * bf16_to_f64(vr[d]);
    }
    if (!tc->full_weights) den = kept;
    for (int d = 0; d < c->d_v; ++d) o[d] /= den;
    free(s);
    free(sel);
}

int oracle_decode_topv_ex(int batch, int n_q, int n_k, int n_v, int d_k, int d_v, double scale,
                          const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                          const int32_t *seq_lens, int t_max, int topk, int full_weights,
                          const int32_t *rows, int64_t n_rows, double *out, int32_t *idx_out,
                          int n_threads) {
    if (check_dims(batch, n_q, n_k, n_v, d_k, d_v) || t_max < 0 || topk < 0 || !q || !k_cache ||
        !v_cache || !seq_lens || !out || !idx_out)
        return -1;
    if (!rows) n_rows = (int64_t)batch * n_q;
    for (int64_t r = 0; rows && r < n_rows; ++r)
        if (rows[2 * r] < 0 || rows[2 * r] >= batch || rows[2 * r + 1] < 0 || rows[2 * r + 1] >= n_q)
            return -1;
    topv_ctx c;
    decode_ctx base = {batch, n_q, n_k, n_v, d_k, d_v, t_max, scale, 0,
                       q, k_cache, v_cache, seq_lens, rows, out, 0};
    c.base = base;
    c.topk = topk;
    c.full_weights = full_weights ? 1 : 0;
    c.idx_out = idx_out;
    run_rows(topv_row, &c, n_rows, n_threads);
    return c.base.status;
}

int oracle_decode_topv(int batch, int n_q, int n_k, int n_v, int d_k, int d_v, double scale,
                       const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                       const int32_t *seq_lens, int t_max, int topk,
                       const int32_t *rows, int64_t n_rows, double *out, int32_t *idx_out,
                       int n_threads) {
    return oracle_decode_topv_ex(batch, n_q, n_k, n_v, d_k, d_v, scale, q, k_cache, v_cache, seq_lens, t_max,
                                 topk, 0, rows, n_rows, out, idx_out, n_threads);
}

/* ------------------------------------------------------------------ */
/* Paged caches ("Where Existing Approaches Fall Short", item 4: paged */
/* KV memory management; the per-position K and V caches of the       */
/* deployment section kept as two pools of fixed-size pages)           */
/* ------------------------------------------------------------------ */

/* Copies the first seq_lens[b] positions of every sequence out of a page pool
 * [num_pages, page_size, heads, d] into a contiguous cache
 * [batch, max_blocks * page_size, heads, d]: position j of sequence b is row
 * j % page_size of pool page table[b * max_blocks + j / page_size].  Positions
 * at or past seq_lens[b] are zero.  Returns -1 on a bad argument, a seq_len
 * outside [0, max_blocks * page_size] or a used table entry outside
 * [0, num_pages). */
int oracle_gather_paged(int batch, int heads, int d, int page_size, int max_blocks, int num_pages,
                        const uint16_t *pool, const int32_t *table, const int32_t *seq_lens, uint16_t *out) {
    if (batch < 0 || heads < 1 || d < 1 || page_size < 1 || max_blocks < 1 || num_pages < 1) return -1;
    const int64_t t_max = (int64_t)max_blocks * page_size;
    const int64_t row = (int64_t)heads * d; /* elements of one position */
    memset(out, 0, sizeof(uint16_t) * (size_t)(batch * t_max * row));
    for (int b = 0; b < batch; ++b) {
        if (seq_lens[b] < 0 || seq_lens[b] > t_max) return -1;
        for (int64_t j = 0; j < seq_lens[b]; ++j) {
            const int32_t page = table[(int64_t)b * max_blocks + j / page_size];
            if (page < 0 || page >= num_pages) return -1;
            const uint16_t *src = pool + ((int64_t)page * page_size + j % page_size) * row;
            memcpy(out + ((int64_t)b * t_max + j) * row, src, sizeof(uint16_t) * (size_t)row);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Query and key of different widths (section 3.4, Step 4: the Attend  */
/* function; K is brought to the query's width by a feed-forward layer */
/* before the dot product, read here as a linear map without bias)     */
/* ------------------------------------------------------------------ */

/* Decode with up-projected keys, in the pages' order: every cached K row of
 * head g is mapped to the query width, k_up[r] = sum_c W[m][r][c] * K[j][g][c]
 * (W [w_heads, d_q, d_k], m = g when w_heads == n_k, 0 when w_heads == 1), the
 * score is s_j = scale * <q_aug[b][h], k_up>, and the output is the softmax-
 * weighted sum of the V rows.  q_aug [B, n_q, d_q]; caches as in oracle_decode.
 * out [B, n_q, d_v].  Single-threaded; meant for test sizes. */
int oracle_decode_up_projected(int batch, int n_q, int n_k, int n_v, int d_q, int d_k, int d_v, int w_heads,
                               double scale, const uint16_t *q_aug, const uint16_t *w_up,
                               const uint16_t *k_cache, const uint16_t *v_cache, const int32_t *seq_lens,
                               int t_max, double *out) {
    if (check_dims(batch, n_q, n_k, n_v, d_k, d_v) || d_q < 1 || t_max < 0 || !(w_heads == 1 || w_heads == n_k))
        return -1;
    double *kup = (double *)malloc(sizeof(double) * (size_t)d_q);
    double *s = (double *)malloc(sizeof(double) * (size_t)(t_max > 0 ? t_max : 1));
    if (!kup || !s) { free(kup); free(s); return -3; }
    for (int b = 0; b < batch; ++b) {
        const int T = seq_lens[b];
        if (T < 0 || T > t_max) { free(kup); free(s); return -1; }
        for (int h = 0; h < n_q; ++h) {
            const int g = oracle_head_map(n_q, n_k, h);
            const int vh = oracle_head_map(n_q, n_v, h);
            const uint16_t *W = w_up + (int64_t)(w_heads == 1 ? 0 : g) * d_q * d_k;
            const uint16_t *qa = q_aug + ((int64_t)b * n_q + h) * d_q;
            double *o = out + ((int64_t)b * n_q + h) * d_v;
            for (int e = 0; e < d_v; ++e) o[e] = 0.0;
            if (T == 0) continue;
            double m = -INFINITY;
            for (int j = 0; j < T; ++j) {
                const uint16_t *kr = k_cache + (((int64_t)b * t_max + j) * n_k + g) * d_k;
                for (int r = 0; r < d_q; ++r) {
                    double acc = 0.0;
                    for (int c = 0; c < d_k; ++c) acc += bf16_to_f64(W[(int64_t)r * d_k + c]) * bf16_to_f64(kr[c]);
                    kup[r] = acc;
                }
                double dot = 0.0;
                for (int r = 0; r < d_q; ++r) dot += bf16_to_f64(qa[r]) * kup[r];
                s[j] = scale * dot;
                if (s[j] > m) m = s[j];
            }
            double den = 0.0;
            for (int j = 0; j < T; ++j) {
                const double w = exp(s[j] - m);
                den += w;
                const uint16_t *vr = v_cache + (((int64_t)b * t_max + j) * n_v + vh) * d_v;
                for (int e = 0; e < d_v; ++e) o[e] += w * bf16_to_f64(vr[e]);
            }
            for (int e = 0; e < d_v; ++e) o[e] /= den;
        }
    }
    free(kup);
    free(s);
    return 0;
}

/* The same up-projection moved onto the query: <q, W k> = <W^T q, k>, so
 * q_fold[b][h][c] = sum_r q_aug[b][h][r] * W[m][r][c] (m as above) is a query
 * of width d_k for the ordinary decode.  out [B, n_q, d_k] in fp64. */
int oracle_fold_query(int batch, int n_q, int n_k, int d_q, int d_k, int w_heads, const uint16_t *q_aug,
                      const uint16_t *w_up, double *out) {
    if (batch < 0 || n_q < 1 || n_k < 1 || n_q % n_k || d_q < 1 || d_k < 1 || !(w_heads == 1 || w_heads == n_k))
        return -1;
    for (int b = 0; b < batch; ++b)
        for (int h = 0; h < n_q; ++h) {
            const int g = oracle_head_map(n_q, n_k, h);
            const uint16_t *W = w_up + (int64_t)(w_heads == 1 ? 0 : g) * d_q * d_k;
            const uint16_t *qa = q_aug + ((int64_t)b * n_q + h) * d_q;
            double *o = out + ((int64_t)b * n_q + h) * d_k;
            for (int c = 0; c < d_k; ++c) {
                double acc = 0.0;
                for (int r = 0; r < d_q; ++r) acc += bf16_to_f64(qa[r]) * bf16_to_f64(W[(int64_t)r * d_k + c]);
                o[c] = acc;
            }
        }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Augmented query projection (section 3.2, item 4)                     */
/* ------------------------------------------------------------------ */
/* The hidden state x passes through two parallel bias-free linear maps, q_gate
 * and q_up; the gate's output goes through SiLU (the Swish of SwiGLU) and
 * multiplies the up branch element by element; q_down maps the product to the
 * query width.  Weights follow the linear-layer layout: W[o][i] is the weight
 * of input feature i in output feature o.
 *
 * oracle_augq_hidden: h[r][o] = SiLU(sum_i x[t][i] Wg[o][i]) * sum_i x[t][i] Wu[o][i]
 *   for the token rows t = rows[r] (all tokens when rows is NULL; n_rows of them).
 *   x [tokens, d_model], Wg and Wu [d_inter, d_model] bf16; h [n_rows, d_inter] fp64.
 * oracle_augq_down: q[r][o] = sum_i h[r][i] Wd[o][i]; h [n_rows, d_inter] fp64 (any
 *   source, e.g. the GPU's rounded hidden state), Wd [d_out, d_inter] bf16, q fp64. */

typedef struct {
    int d_in, d_out;
    const uint16_t *x;      /* bf16 rows of width d_in (hidden stage) */
    const double *xd;       /* fp64 rows of width d_in (down stage)   */
    const uint16_t *w0, *w1;
    const int32_t *rows;
    double *out;
} augq_ctx;

static double silu(double g) { return g / (1.0 + exp(-g)); }

static void augq_hidden_row(void *vctx, int64_t r) {
    const augq_ctx *c = (const augq_ctx *)vctx;
    const int64_t t = c->rows ? c->rows[r] : r;
    const uint16_t *xr = c->x + t * c->d_in;
    for (int o = 0; o < c->d_out; ++o) {
        const uint16_t *wg = c->w0 + (int64_t)o * c->d_in, *wu = c->w1 + (int64_t)o * c->d_in;
        double g = 0.0, u = 0.0;
        for (int i = 0; i < c->d_in; ++i) {
            const double xi = bf16_to_f64(xr[i]);
            g += xi * bf16_to_f64(wg[i]);
            u += xi * bf16_to_f64(wu[i]);
        }
        c->out[r * c->d_out + o] = silu(g) * u;
    }
}

static void augq_down_row(void *vctx, int64_t r) {
    const augq_ctx *c = (const augq_ctx *)vctx;
    const double *hr = c->xd + r * c->d_in;
    for (int o = 0; o < c->d_out; ++o) {
        const uint16_t *wd = c->w0 + (int64_t)o * c->d_in;
        double acc = 0.0;
        for (int i = 0; i < c->d_in; ++i) acc += hr[i] * bf16_to_f64(wd[i]);
        c->out[r * c->d_out + o] = acc;
    }
}

int oracle_augq_hidden(int tokens, int d_model, int d_inter, const uint16_t *x, const uint16_t *w_gate,
                       const uint16_t *w_up, const int32_t *rows, int n_rows, double *h, int n_threads) {
    if (tokens < 0 || d_model < 1 || d_inter < 1 || n_rows < 0 || !x || !w_gate || !w_up || !h) return -1;
    if (!rows && n_rows != tokens) return -1;
    for (int r = 0; rows && r < n_rows; ++r)
        if (rows[r] < 0 || rows[r] >= tokens) return -1;
    augq_ctx c = {d_model, d_inter, x, NULL, w_gate, w_up, rows, h};
    run_rows(augq_hidden_row, &c, n_rows, n_threads);
    return 0;
}

int oracle_augq_down(int n_rows, int d_inter, int d_out, const double *h, const uint16_t *w_down, double *q,
                     int n_threads) {
    if (n_rows < 0 || d_inter < 1 || d_out < 1 || !h || !w_down || !q) return -1;
    augq_ctx c = {d_inter, d_out, NULL, h, w_down, NULL, NULL, q};
    run_rows(augq_down_row, &c, n_rows, n_threads);
    return 0;
}
