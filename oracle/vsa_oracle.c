/*
 * CPU oracle for block-sparse 3D-video attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the test suite, the package smoke check and the benchmark's CPU
 * baseline leg may load this library.  The product path never calls it.
 * It shares no code with the CUDA library: no headers, helpers or tables.
 *
 * Everything is plain fp64 / integer C, written as the straightforward
 * definition, with no blocking or reordering beyond what the definition states:
 *
 *  - orc_tile_major_order: tokens of the (T,H,W) latent grid, padded per axis
 *    to a multiple of the 3D unit (bt,bh,bw), listed unit by unit (units in
 *    (t,h,w) row-major order) and inside a unit in (t,h,w) row-major order.
 *    "Parameterized Stripe Attention for Efficient Video Generation", key
 *    design 2 (hierarchical (T',H',W',bt,bh,bw) layout, T' = ceil(T/bt)*bt);
 *    "Fast Video Generation with Sliding Tile Attention", section 3 (tokens of
 *    a tile numbered contiguously).  Padding slots map to -1.
 *
 *  - orc_frame0_first_order: the layout for temporal heads ("Sparse VideoGen:
 *    accelerating video diffusion attention on TPU", "arranging tokens for
 *    efficient temporal access"; "Video diffusion long-sequence attention and
 *    sparsity", section 7.2: tokens of one spatial position across frames made
 *    contiguous, so a temporal head's diagonal stripe becomes contiguous
 *    bands).  Reading: the frame-0 sink would otherwise put one kept key in
 *    every tile, so frame 0 is listed first, in (h,w) row-major order, then
 *    each (h,w) position in row-major order with its frames 1..T-1 in order.
 *    No padding inside; slots past T*H*W map to -1.
 *
 *  - orc_keep: the element predicate of each mask family on real coordinates.
 *      spatial / temporal heads + frame-0 sink: "Sparse VideoGen: accelerating
 *        video diffusion attention on TPU", section on SVG heads (figure 3);
 *      STA: "Fast Video Generation with Sliding Tile Attention", section 3
 *        (tile-level window; clamped at the grid edge, the reading Eq. 4 and
 *        Table 2's sparsities force);
 *      stripe M(Tw,To,Ts,Sw,So,Ss): "Parameterized Stripe Attention", key
 *        design 1 (inter/intra conditions).
 *
 *  - orc_attention_rows: dense softmax(q k^T * scale + M) v with the mask
 *    applied before the softmax ("Fast Video Generation with Sliding Tile
 *    Attention", section 2, Eq. 1), for a list of query rows, in fp64, with
 *    lse = log sum exp over kept keys.
 *
 *  - orc_tile_counts: for q tiles of Bq slots and kv tiles of Bk slots in
 *    the head's order, the number of kept (real query, key slot) pairs, by
 *    brute force.  The three-class map (empty / boundary / full) is read off
 *    those counts ("Sparse VideoGen ... on TPU", section "logical sparsity is
 *    not physical sparsity").
 *
 *  - orc_kept_pairs: total kept pairs of one head over real x real tokens.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int32_t kind, sink, rt, rh, rw, kt, kh, kw, Tw, To, Ts, Sw, So, Ss;
    int32_t layout;   /* token order of the head: 0 tile-major, 1 frame 0 first */
    int32_t tile_round;  /* unused here: the rounded mask is built in Python from the counts */
} orc_mask;

typedef struct {
    int32_t T, H, W, bt, bh, bw;
} orc_grid;

enum { ORC_FULL = 0, ORC_SPATIAL = 1, ORC_TEMPORAL = 2, ORC_STA = 3, ORC_STRIPE = 4 };

static int ceil_to(int x, int m) { return ((x + m - 1) / m) * m; }
static int iabs(int x) { return x < 0 ? -x : x; }

/* ------------------------------------------------------------------------ */
/* layout                                                                    */

int64_t orc_padded_tokens(const orc_grid* g)
{
    return (int64_t)ceil_to(g->T, g->bt) * ceil_to(g->H, g->bh) * ceil_to(g->W, g->bw);
}

/* perm[slot] = natural token index (t*H + h)*W + w, or -1 for padding.
   Slots past the padded grid (up to n_slots) are padding too.  Returns the
   padded-grid token count, or -1 if n_slots is too small. */
int64_t orc_tile_major_order(const orc_grid* g, int64_t n_slots, int32_t* perm)
{
    const int Tp = ceil_to(g->T, g->bt), Hp = ceil_to(g->H, g->bh), Wp = ceil_to(g->W, g->bw);
    const int64_t npad = (int64_t)Tp * Hp * Wp;
    if (n_slots < npad) return -1;
    int64_t slot = 0;
    for (int tt = 0; tt < Tp / g->bt; ++tt)
        for (int th = 0; th < Hp / g->bh; ++th)
            for (int tw = 0; tw < Wp / g->bw; ++tw)
                for (int ot = 0; ot < g->bt; ++ot)
                    for (int oh = 0; oh < g->bh; ++oh)
                        for (int ow = 0; ow < g->bw; ++ow) {
                            const int t = tt * g->bt + ot, h = th * g->bh + oh, w = tw * g->bw + ow;
                            const int real = t < g->T && h < g->H && w < g->W;
                            perm[slot++] = real ? (int32_t)(((int64_t)t * g->H + h) * g->W + w) : -1;
                        }
    while (slot < n_slots) perm[slot++] = -1;
    return npad;
}

/* perm[slot] = natural token index: frame 0 in (h,w) order, then every (h,w)
   position with its frames 1..T-1.  Returns T*H*W, or -1 if n_slots is too
   small. */
int64_t orc_frame0_first_order(const orc_grid* g, int64_t n_slots, int32_t* perm)
{
    const int64_t n = (int64_t)g->T * g->H * g->W;
    if (n_slots < n) return -1;
    int64_t slot = 0;
    for (int h = 0; h < g->H; ++h)
        for (int w = 0; w < g->W; ++w) perm[slot++] = (int32_t)((int64_t)h * g->W + w);
    for (int h = 0; h < g->H; ++h)
        for (int w = 0; w < g->W; ++w)
            for (int t = 1; t < g->T; ++t) perm[slot++] = (int32_t)(((int64_t)t * g->H + h) * g->W + w);
    while (slot < n_slots) perm[slot++] = -1;
    return n;
}

/* The order of a head, by its layout field. */
static int64_t head_order(const orc_mask* m, const orc_grid* g, int64_t n_slots, int32_t* perm)
{
    if (m->layout == 1) return orc_frame0_first_order(g, n_slots, perm);
    return orc_tile_major_order(g, n_slots, perm);
}

/* ------------------------------------------------------------------------ */
/* predicate                                                                 */

/* STA along one axis: the query's unit sees k consecutive units (k clamped to
   the number of units n), centred on its own unit and shifted inward at the
   edges so that it always sees exactly k units. */
static int sta_axis(int cq, int ck, int b, int n, int k)
{
    const int uq = cq / b, uk = ck / b;
    const int kk = k < n ? k : n;
    int start = uq - kk / 2;
    if (start < 0) start = 0;
    if (start > n - kk) start = n - kk;
    return uk >= start && uk < start + kk;
}

static int keep_coords(const orc_mask* m, const orc_grid* g,
                       int tq, int hq, int wq, int tk, int hk, int wk)
{
    if (m->sink && tk == 0) return 1;
    switch (m->kind) {
    case ORC_FULL:
        return 1;
    case ORC_SPATIAL:
        return iabs(tk - tq) <= m->rt;
    case ORC_TEMPORAL:
        return iabs(hk - hq) <= m->rh && iabs(wk - wq) <= m->rw;
    case ORC_STA: {
        const int nt = ceil_to(g->T, g->bt) / g->bt;
        const int nh = ceil_to(g->H, g->bh) / g->bh;
        const int nw = ceil_to(g->W, g->bw) / g->bw;
        return sta_axis(tq, tk, g->bt, nt, m->kt) && sta_axis(hq, hk, g->bh, nh, m->kh) &&
               sta_axis(wq, wk, g->bw, nw, m->kw);
    }
    case ORC_STRIPE: {
        const int sq = hq * g->W + wq, sk = hk * g->W + wk;
        const int inter = (iabs(tk - tq - m->To) % m->Ts) <= m->Tw - 1;
        const int intra = (iabs(sk - sq - m->So) % m->Ss) <= m->Sw - 1;
        return inter && intra;
    }
    default:
        return 0;
    }
}

/* keep(q, k) for natural token indices of real tokens. */
int orc_keep(const orc_mask* m, const orc_grid* g, int64_t nq, int64_t nk)
{
    const int64_t HW = (int64_t)g->H * g->W;
    const int tq = (int)(nq / HW), hq = (int)((nq % HW) / g->W), wq = (int)(nq % g->W);
    const int tk = (int)(nk / HW), hk = (int)((nk % HW) / g->W), wk = (int)(nk % g->W);
    return keep_coords(m, g, tq, hq, wq, tk, hk, wk);
}

/* ------------------------------------------------------------------------ */
/* threading helper: run fn(i, ctx) for i in [0, n) over nthreads threads    */

typedef void (*orc_item_fn)(int64_t i, void* ctx);
typedef struct {
    orc_item_fn fn;
    void* ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
} orc_pool;

static void* orc_worker(void* arg)
{
    orc_pool* p = (orc_pool*)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        const int64_t i = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (i >= p->n) break;
        p->fn(i, p->ctx);
    }
    return NULL;
}

static void orc_parallel(int64_t n, int nthreads, orc_item_fn fn, void* ctx)
{
    orc_pool p;
    p.fn = fn; p.ctx = ctx; p.n = n; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0;
    for (int i = 1; i < nthreads; ++i)
        if (pthread_create(&th[started], NULL, orc_worker, &p) == 0) ++started;
    orc_worker(&p);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------------ */
/* dense masked attention, fp64                                              */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

typedef struct {
    const orc_mask* m;
    const orc_grid* g;
    int D;
    double scale;
    const uint16_t* q;           /* [N, D] natural order, bf16 bits */
    const double *k, *v;         /* [N, D] natural order, widened to fp64 */
    const int64_t* rows;
    double* out_o;               /* [nrows, D] */
    double* out_lse;             /* [nrows] */
    int64_t N;
} orc_attn_ctx;

static void orc_attn_row(int64_t r, void* vctx)
{
    orc_attn_ctx* c = (orc_attn_ctx*)vctx;
    const int D = c->D;
    const int64_t nq = c->rows[r];
    const int64_t HW = (int64_t)c->g->H * c->g->W;
    const int tq = (int)(nq / HW), hq = (int)((nq % HW) / c->g->W), wq = (int)(nq % c->g->W);
    double* qd = (double*)malloc(sizeof(double) * D);
    double* s = (double*)malloc(sizeof(double) * c->N);
    double* o = c->out_o + r * D;
    for (int d = 0; d < D; ++d) qd[d] = bf16_to_double(c->q[nq * D + d]);
    /* scores over every real key, -inf where the mask drops the pair */
    double mx = -INFINITY;
    for (int64_t nk = 0; nk < c->N; ++nk) {
        const int tk = (int)(nk / HW), hk = (int)((nk % HW) / c->g->W), wk = (int)(nk % c->g->W);
        if (!keep_coords(c->m, c->g, tq, hq, wq, tk, hk, wk)) { s[nk] = -INFINITY; continue; }
        double acc = 0.0;
        const double* kr = c->k + nk * D;
        for (int d = 0; d < D; ++d) acc += qd[d] * kr[d];
        s[nk] = acc * c->scale;
        if (s[nk] > mx) mx = s[nk];
    }
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (mx == -INFINITY) {           /* no kept key: o = 0, lse = -inf */
        c->out_lse[r] = -INFINITY;
        free(qd); free(s);
        return;
    }
    double l = 0.0;
    for (int64_t nk = 0; nk < c->N; ++nk) {
        if (s[nk] == -INFINITY) continue;
        const double p = exp(s[nk] - mx);
        l += p;
        const double* vr = c->v + nk * D;
        for (int d = 0; d < D; ++d) o[d] += p * vr[d];
    }
    for (int d = 0; d < D; ++d) o[d] /= l;
    c->out_lse[r] = mx + log(l);
    free(qd); free(s);
}

/* q, k, v: one (batch, head) slice, [N, D] natural order, bf16 bits. */
int orc_attention_rows(const orc_mask* m, const orc_grid* g, int D, double scale,
                       const uint16_t* q, const uint16_t* k, const uint16_t* v,
                       int64_t nrows, const int64_t* rows,
                       double* out_o, double* out_lse, int nthreads)
{
    if (!m || !g || !q || !k || !v || !rows || !out_o || !out_lse || D <= 0) return -1;
    orc_attn_ctx c;
    c.m = m; c.g = g; c.D = D; c.scale = scale; c.q = q;
    c.rows = rows; c.out_o = out_o; c.out_lse = out_lse;
    c.N = (int64_t)g->T * g->H * g->W;
    for (int64_t r = 0; r < nrows; ++r)
        if (rows[r] < 0 || rows[r] >= c.N) return -1;
    /* bf16 -> fp64 is exact; widen k and v once */
    double* kd = (double*)malloc(sizeof(double) * (size_t)c.N * D);
    double* vd = (double*)malloc(sizeof(double) * (size_t)c.N * D);
    if (!kd || !vd) { free(kd); free(vd); return -2; }
    for (int64_t i = 0; i < c.N * D; ++i) { kd[i] = bf16_to_double(k[i]); vd[i] = bf16_to_double(v[i]); }
    c.k = kd; c.v = vd;
    orc_parallel(nrows, nthreads, orc_attn_row, &c);
    free(kd); free(vd);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* brute-force tile pair counts                                              */

typedef struct {
    const orc_mask* m;
    const orc_grid* g;
    const int32_t* perm;
    const int32_t *ct, *ch, *cw;   /* coordinates of each slot (ct = -1: padding) */
    int64_t n_slots;
    int Bq, Bk;
    const int64_t* qtiles;
    int64_t* counts;       /* [nqt, n_slots / Bk] */
    int64_t* real_q;       /* [nqt] */
} orc_tc_ctx;

static void orc_tile_row(int64_t i, void* vctx)
{
    orc_tc_ctx* c = (orc_tc_ctx*)vctx;
    const int64_t nk_tiles = c->n_slots / c->Bk;
    int64_t* row = c->counts + i * nk_tiles;
    const int64_t HW = (int64_t)c->g->H * c->g->W;
    memset(row, 0, sizeof(int64_t) * nk_tiles);
    int64_t nreal = 0;
    for (int a = 0; a < c->Bq; ++a) {
        const int64_t pq = c->qtiles[i] * c->Bq + a;
        const int32_t nq = c->perm[pq];
        if (nq < 0) continue;
        ++nreal;
        const int tq = (int)(nq / HW), hq = (int)((nq % HW) / c->g->W), wq = (int)(nq % c->g->W);
        for (int64_t pk = 0; pk < c->n_slots; ++pk) {
            if (c->ct[pk] < 0) continue;   /* padding keys are never kept */
            if (keep_coords(c->m, c->g, tq, hq, wq, c->ct[pk], c->ch[pk], c->cw[pk]))
                row[pk / c->Bk] += 1;
        }
    }
    c->real_q[i] = nreal;
}

/* counts[i][j] = kept (real query, key slot) pairs between q tile qtiles[i]
   (slots [qtiles[i]*Bq, +Bq)) and kv tile j; real_q[i] = real queries in it. */
int orc_tile_counts(const orc_mask* m, const orc_grid* g, int64_t n_slots, int Bq, int Bk,
                    int64_t nqt, const int64_t* qtiles, int64_t* counts, int64_t* real_q,
                    int nthreads)
{
    if (!m || !g || Bq <= 0 || Bk <= 0 || n_slots % Bq || n_slots % Bk) return -1;
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * n_slots);
    if (!perm) return -2;
    if (head_order(m, g, n_slots, perm) < 0) { free(perm); return -1; }
    for (int64_t i = 0; i < nqt; ++i)
        if (qtiles[i] < 0 || qtiles[i] >= n_slots / Bq) { free(perm); return -1; }
    int32_t* coords = (int32_t*)malloc(sizeof(int32_t) * 3 * n_slots);
    if (!coords) { free(perm); return -2; }
    const int64_t HW = (int64_t)g->H * g->W;
    for (int64_t p = 0; p < n_slots; ++p) {
        const int32_t n = perm[p];
        coords[p] = n < 0 ? -1 : (int32_t)(n / HW);
        coords[n_slots + p] = n < 0 ? -1 : (int32_t)((n % HW) / g->W);
        coords[2 * n_slots + p] = n < 0 ? -1 : (int32_t)(n % g->W);
    }
    orc_tc_ctx c;
    c.m = m; c.g = g; c.perm = perm; c.n_slots = n_slots; c.Bq = Bq; c.Bk = Bk;
    c.ct = coords; c.ch = coords + n_slots; c.cw = coords + 2 * n_slots;
    c.qtiles = qtiles; c.counts = counts; c.real_q = real_q;
    orc_parallel(nqt, nthreads, orc_tile_row, &c);
    free(coords);
    free(perm);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* kept pairs over real x real                                               */

typedef struct {
    const orc_mask* m;
    const orc_grid* g;
    int64_t* per_q;        /* per query frame-row partial sums: [T*H] */
} orc_kp_ctx;

static void orc_kept_slab(int64_t i, void* vctx)
{
    orc_kp_ctx* c = (orc_kp_ctx*)vctx;
    const orc_grid* g = c->g;
    const int tq = (int)(i / g->H), hq = (int)(i % g->H);
    int64_t acc = 0;
    for (int wq = 0; wq < g->W; ++wq)
        for (int tk = 0; tk < g->T; ++tk)
            for (int hk = 0; hk < g->H; ++hk)
                for (int wk = 0; wk < g->W; ++wk)
                    acc += keep_coords(c->m, g, tq, hq, wq, tk, hk, wk);
    c->per_q[i] = acc;
}

int64_t orc_kept_pairs(const orc_mask* m, const orc_grid* g, int nthreads)
{
    const int64_t n = (int64_t)g->T * g->H;
    int64_t* per = (int64_t*)calloc((size_t)n, sizeof(int64_t));
    if (!per) return -1;
    orc_kp_ctx c;
    c.m = m; c.g = g; c.per_q = per;
    orc_parallel(n, nthreads, orc_kept_slab, &c);
    int64_t total = 0;
    for (int64_t i = 0; i < n; ++i) total += per[i];
    free(per);
    return total;
}

/* ------------------------------------------------------------------------ */
/* full predicate matrix for small grids: out[nq * N + nk] = keep(nq, nk)    */

int orc_keep_matrix(const orc_mask* m, const orc_grid* g, uint8_t* out)
{
    const int64_t N = (int64_t)g->T * g->H * g->W;
    if (N > 65536) return -1;
    for (int64_t nq = 0; nq < N; ++nq)
        for (int64_t nk = 0; nk < N; ++nk)
            out[nq * N + nk] = (uint8_t)orc_keep(m, g, nq, nk);
    return 0;
}
