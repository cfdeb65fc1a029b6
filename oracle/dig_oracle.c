/*
 * dig_oracle.c -- plain, slow, fp64 CPU oracle for the DiG GLA hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke check and
 * the benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or helper with the CUDA path, and the CUDA path never calls it.
 *
 * What it computes, and where that is stated:
 *
 *  - Scan orders (DiG paper notes, "空间重定向与增强模块 (SREM)"): every block scans
 *    the 2D patch-token grid in one of four directions -- left-to-right,
 *    right-to-left, top-to-bottom, bottom-to-top -- obtained by transposing the
 *    2D token matrix and flipping the sequence.  Numbering follows the order in
 *    which the notes list them: 0 = L->R, 1 = R->L, 2 = T->B, 3 = B->T.
 *    Codes 4..11 are the eight zigzag orders (see zigzag_order).
 *    oracle_scan_order() materialises the order literally: it builds the grid of
 *    raster token ids, transposes it for 2/3, flattens row by row, and reverses
 *    the flattened sequence for 1/3.
 *
 *  - GLA recurrence (DiG: gated linear attention, S_t = Diag(alpha_t) S_{t-1} +
 *    k_t^T v_t, o_t = q_t S_t): per (batch, head) the state S (dk x dv) starts at
 *    zero (diffusers draft GatedLinearAttnProcessor2_0, "gated_linear_attention":
 *    the state is initialised to zeros); each step first decays row i of S by
 *    alpha_{t,i} = exp(log_alpha_{t,i}) -- the gate is per key channel and is
 *    broadcast over the value axis -- then adds k_t^T v_t, and only then reads
 *    o_t = q_t S_t (update before read, as in the same draft).  Steps run over
 *    scan positions p = 0..T-1 visiting token order[p]; the output for a token is
 *    written at that token's own (canonical) index.  Everything is fp64.  No
 *    feature map, normaliser or internal 1/sqrt(dk): callers pre-scale q, k, v.
 *
 *  - SREM depthwise 3x3 conv (DiG notes, SREM and DiG Block step (4)): after the
 *    token sequence is reshaped to the 2D grid, each channel is cross-correlated
 *    with its own 3x3 kernel, zero padding of one pixel ("same" output size), no
 *    bias.  Identity initialisation (centre 1, rest 0) makes it the identity map.
 *
 *  - SREM reorientation (DiG notes, SREM: transpose + flip are O(T) operations):
 *    gather of whole token rows by the scan-order table, y[b][p] = x[b][order[p]],
 *    or its inverse scatter y[b][order[p]] = x[b][p].  Rows are copied byte for
 *    byte, so the result is exact for any element type.
 *
 * Threads: independent (batch, head) pairs or conv image rows are spread over
 * POSIX threads; this changes no arithmetic, only which core runs it.
 *
 *  - GLA backward (DiG notes, "损失函数 / 训练策略": the model is trained like DiT,
 *    so gradients flow back through every GLA layer; "硬件友好的效率设计": the
 *    chunk-wise form is the training path).  The pages give no formula for it: it
 *    is the exact gradient of the recurrence above, written as reverse-mode
 *    differentiation of its steps, one step at a time in reverse scan order.  With
 *    dO the gradient of the loss with respect to out, and G the gradient with
 *    respect to the state S_p after step p (G = 0 past the last step):
 *        G    += q_p^T dO_p                        (o_p = q_p S_p reads S_p)
 *        dq_p  = dO_p S_p^T
 *        dk_p  = G v_p^T,   dv_p = k_p G           (S_p contains k_p^T v_p)
 *        dlog_alpha_p[i] = alpha_p[i] * sum_j G[i][j] S_{p-1}[i][j]
 *        G     = Diag(alpha_p) G                   (S_p = Diag(alpha_p) S_{p-1} + ...)
 *    The forward states S_p of the head are kept (T * dk * dv values) so that the
 *    reverse sweep reads them exactly.
 *
 *  - Normalised variant (the diffusers draft, page 4, `gated_linear_attention`): the
 *    features are elu(x) + 1 of q and k, the per-key-channel forget gate is
 *    sigmoid(q * k) of the raw q and k, and a gated denominator runs beside the
 *    state.  Per (batch, head), from S = 0 and z = 0, at every scan position:
 *        S <- Diag(g_t) S + phi(k_t)^T v_t,   z <- g_t * z + phi(k_t)
 *        o_t = (phi(q_t) S) / max(phi(q_t) . z, eps)
 *    all in fp64 (the draft computes in fp32 or wider).  Same scan orders and
 *    canonical output positions as the forward above.
 *
 * Planted mistakes: oracle_gla_fwd_planted() runs the same recurrence with one
 * deliberate error selected by `planted` (1..7), and oracle_gla_bwd_planted()
 * the backward sweep with one of 1..6, oracle_gla_norm_fwd_planted() the
 * normalised variant with one of 1..5.  Tests use them to show that the oracle's
 * pins catch each kind of mistake; the method itself is planted == 0.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG -1
#define ORACLE_NOMEM -6

/* ------------------------------------------------------------------------- */
/* Scan order: the raster token id visited at each scan position.             */
/* ------------------------------------------------------------------------- */
/*
 * Zigzag orders (ZigMa notes, "Zigzag 扫描方案": within every line the scan turns
 * back, a snake path, so that tokens adjacent in the sequence are adjacent in the
 * grid; eight schemes S_0..S_7 that differ in horizontal / vertical orientation,
 * start and direction).  Scheme j: lines are the grid's rows for j < 4 and its
 * columns (the transposed grid's rows) for j >= 4; the lines are visited first to
 * last when bit 1 of j is clear and last to first when it is set; the first visited
 * line is walked from its first entry when bit 0 of j is clear and from its last
 * entry when it is set, and every following line in the opposite direction of the
 * one before.  scan order code dir = 4 + j.
 */
static int zigzag_order(int j, int Hgrid, int Wgrid, int64_t *order)
{
    const int64_t T = (int64_t)Hgrid * Wgrid;
    int64_t *grid = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!grid) return ORACLE_NOMEM;
    int nl, len; /* lines and their length, in `grid` laid out line by line */
    if (j < 4) {
        nl = Hgrid;
        len = Wgrid;
        for (int y = 0; y < Hgrid; ++y)
            for (int x = 0; x < Wgrid; ++x) grid[(int64_t)y * Wgrid + x] = (int64_t)y * Wgrid + x;
    } else {
        nl = Wgrid;
        len = Hgrid;
        for (int y = 0; y < Hgrid; ++y)
            for (int x = 0; x < Wgrid; ++x) grid[(int64_t)x * Hgrid + y] = (int64_t)y * Wgrid + x;
    }
    const int lines_backwards = (j >> 1) & 1;
    int from_end = j & 1; /* direction of the line being walked */
    int64_t n = 0;
    for (int s = 0; s < nl; ++s) {
        const int line = lines_backwards ? nl - 1 - s : s;
        for (int e = 0; e < len; ++e) {
            const int at = from_end ? len - 1 - e : e;
            order[n++] = grid[(int64_t)line * len + at];
        }
        from_end = !from_end; /* the snake turns back */
    }
    free(grid);
    return ORACLE_OK;
}

int oracle_scan_order(int dir, int Hgrid, int Wgrid, int64_t *order)
{
    if (dir < 0 || dir > 11 || Hgrid <= 0 || Wgrid <= 0 || !order) return ORACLE_BAD_ARG;
    if (dir >= 4) return zigzag_order(dir - 4, Hgrid, Wgrid, order);
    const int64_t T = (int64_t)Hgrid * Wgrid;

    /* grid[y][x] holds the raster token id y*Wgrid + x */
    int64_t *grid = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!grid) return ORACLE_NOMEM;
    for (int y = 0; y < Hgrid; ++y)
        for (int x = 0; x < Wgrid; ++x) grid[(int64_t)y * Wgrid + x] = (int64_t)y * Wgrid + x;

    int64_t n = 0;
    if (dir == 0 || dir == 1) {
        /* flatten the grid row by row */
        for (int y = 0; y < Hgrid; ++y)
            for (int x = 0; x < Wgrid; ++x) order[n++] = grid[(int64_t)y * Wgrid + x];
    } else {
        /* transpose the grid (Wgrid rows of Hgrid entries), then flatten row by row */
        int64_t *tr = (int64_t *)malloc(sizeof(int64_t) * T);
        if (!tr) { free(grid); return ORACLE_NOMEM; }
        for (int y = 0; y < Hgrid; ++y)
            for (int x = 0; x < Wgrid; ++x) tr[(int64_t)x * Hgrid + y] = grid[(int64_t)y * Wgrid + x];
        for (int r = 0; r < Wgrid; ++r)
            for (int c = 0; c < Hgrid; ++c) order[n++] = tr[(int64_t)r * Hgrid + c];
        free(tr);
    }
    free(grid);

    if (dir == 1 || dir == 3) {
        /* flip the flattened sequence */
        for (int64_t a = 0, b = T - 1; a < b; ++a, --b) {
            int64_t t = order[a];
            order[a] = order[b];
            order[b] = t;
        }
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Thread pool helper: run fn(ctx, i) for i in [0, n) over POSIX threads.     */
/* ------------------------------------------------------------------------- */
typedef void (*work_fn)(void *ctx, int64_t i);

typedef struct {
    work_fn fn;
    void *ctx;
    int64_t n;
    int64_t next;
    pthread_mutex_t mu;
} pool_t;

static void *pool_worker(void *arg)
{
    pool_t *p = (pool_t *)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int64_t i = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (i >= p->n) break;
        p->fn(p->ctx, i);
    }
    return NULL;
}

static int resolve_threads(int nthreads)
{
    if (nthreads > 0) return nthreads;
    long c = sysconf(_SC_NPROCESSORS_ONLN);
    return c > 0 ? (int)c : 1;
}

/* Returns the number of threads actually used. */
static int run_pool(work_fn fn, void *ctx, int64_t n, int nthreads)
{
    nthreads = resolve_threads(nthreads);
    if (n < 1) return 0;
    if (nthreads > n) nthreads = (int)n;
    pool_t p;
    p.fn = fn;
    p.ctx = ctx;
    p.n = n;
    p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    int used = 1;
    if (nthreads <= 1) {
        pool_worker(&p);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
        int started = 0;
        if (th)
            for (int i = 0; i < nthreads; ++i)
                if (pthread_create(&th[i], NULL, pool_worker, &p) == 0) ++started;
        if (started == 0) pool_worker(&p);
        for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
        free(th);
        used = started > 0 ? started : 1;
    }
    pthread_mutex_destroy(&p.mu);
    return used;
}

int oracle_hardware_threads(void) { return resolve_threads(0); }

/* ------------------------------------------------------------------------- */
/* GLA forward recurrence (fp64).                                             */
/* ------------------------------------------------------------------------- */
typedef struct {
    const double *q, *k, *v, *la;
    double *out;
    const int64_t *order;
    int64_t T;
    int64_t bh_base;
    int B, H, dk, dv;
    int planted; /* 0 = the method; 1..7 = a planted mistake (tests only) */
    int status;
} gla_ctx;

/* Element offset of (b, t, h, 0) in the token-major [B][T][H][d] layout. */
static inline int64_t tok_off(int64_t b, int64_t t, int64_t h, int64_t T, int64_t H, int64_t d)
{
    return ((b * T + t) * H + h) * d;
}

static void gla_head(void *vctx, int64_t i_local)
{
    gla_ctx *c = (gla_ctx *)vctx;
    const int64_t bh = c->bh_base + i_local;
    const int64_t b = bh / c->H, h = bh % c->H;
    const int dk = c->dk, dv = c->dv;
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *Sprev = (double *)calloc((size_t)dk * dv, sizeof(double));
    if (!S || !Sprev) {
        free(S);
        free(Sprev);
        c->status = ORACLE_NOMEM;
        return;
    }

    for (int64_t p = 0; p < c->T; ++p) {
        const int64_t t = c->order[p];
        const double *qt = c->q + tok_off(b, t, h, c->T, c->H, dk);
        const double *kt = c->k + tok_off(b, t, h, c->T, c->H, dk);
        const double *vt = c->v + tok_off(b, t, h, c->T, c->H, dv);
        const double *lt = c->la + tok_off(b, t, h, c->T, c->H, dk);
        double *ot = c->out + tok_off(b, t, h, c->T, c->H, dv);

        if (c->planted == 1) memcpy(Sprev, S, sizeof(double) * (size_t)dk * dv);

        /* S <- Diag(alpha_t) S + k_t^T v_t */
        for (int i = 0; i < dk; ++i) {
            double alpha = exp(lt[i]);
            if (c->planted == 4) alpha = 1.0;          /* planted: gate dropped */
            if (c->planted == 6) alpha = exp(-lt[i]);  /* planted: sign of the log-gate */
            for (int j = 0; j < dv; ++j) {
                double a = alpha;
                if (c->planted == 2) a = exp(lt[j < dk ? j : dk - 1]); /* planted: gate on the value axis */
                if (c->planted == 3)
                    S[(int64_t)i * dv + j] = a * (S[(int64_t)i * dv + j] + kt[i] * vt[j]); /* planted: decay after write */
                else
                    S[(int64_t)i * dv + j] = a * S[(int64_t)i * dv + j] + kt[i] * vt[j];
            }
        }
        /* o_t = q_t S_t  (read after the update) */
        const double *Sread = (c->planted == 1) ? Sprev : S; /* planted: read before the update */
        const double *qread = (c->planted == 7) ? kt : qt;   /* planted: k read in place of q */
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += qread[i] * Sread[(int64_t)i * dv + j];
            ot[j] = acc;
        }
    }
    free(S);
    free(Sprev);
}

static int gla_common(const double *q, const double *k, const double *v, const double *log_alpha,
                      int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir, double *out,
                      int nthreads, int planted, int64_t bh_begin, int64_t bh_end)
{
    if (!q || !k || !v || !log_alpha || !out) return ORACLE_BAD_ARG;
    if (B <= 0 || H <= 0 || Hgrid <= 0 || Wgrid <= 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (dir < 0 || dir > 11) return ORACLE_BAD_ARG;
    const int64_t T = (int64_t)Hgrid * Wgrid;
    const int64_t BH = (int64_t)B * H;
    if (bh_begin < 0) bh_begin = 0;
    if (bh_end < 0 || bh_end > BH) bh_end = BH;
    if (bh_begin > bh_end) return ORACLE_BAD_ARG;

    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!order) return ORACLE_NOMEM;
    int rc;
    if (planted == 5 && dir >= 2)
        rc = oracle_scan_order(dir, Wgrid, Hgrid, order); /* planted: grid sides swapped */
    else
        rc = oracle_scan_order(dir, Hgrid, Wgrid, order);
    if (rc != ORACLE_OK) {
        free(order);
        return rc;
    }

    gla_ctx c;
    c.q = q;
    c.k = k;
    c.v = v;
    c.la = log_alpha;
    c.out = out;
    c.order = order;
    c.T = T;
    c.bh_base = bh_begin;
    c.B = B;
    c.H = H;
    c.dk = dk;
    c.dv = dv;
    c.planted = planted;
    c.status = ORACLE_OK;
    int used = run_pool(gla_head, &c, bh_end - bh_begin, nthreads);
    free(order);
    if (c.status != ORACLE_OK) return c.status;
    return used; /* >= 0: threads used */
}

/*
 * GLA forward over all (batch, head) pairs.  q, k, log_alpha: [B][T][H][dk];
 * v, out: [B][T][H][dv]; T = Hgrid*Wgrid, token t = y*Wgrid + x.  Returns the
 * number of threads used (>= 0) or a negative error code.
 */
int oracle_gla_fwd(const double *q, const double *k, const double *v, const double *log_alpha,
                   int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir, double *out,
                   int nthreads)
{
    return gla_common(q, k, v, log_alpha, B, H, Hgrid, Wgrid, dk, dv, dir, out, nthreads, 0, 0, -1);
}

/* The same, restricted to flattened heads bh = b*H + h in [bh_begin, bh_end). */
int oracle_gla_fwd_heads(const double *q, const double *k, const double *v, const double *log_alpha,
                         int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir, double *out,
                         int nthreads, int64_t bh_begin, int64_t bh_end)
{
    return gla_common(q, k, v, log_alpha, B, H, Hgrid, Wgrid, dk, dv, dir, out, nthreads, 0, bh_begin,
                      bh_end);
}

/*
 * The forward with the gate given as logits g (same layout as q): log_alpha =
 * logsigmoid(g) / gate_norm, the gate definition of the GLA configurations
 * (logsigmoid(g) = min(g, 0) - log(1 + e^{-|g|}), in fp64), then the recurrence.
 */
int oracle_gla_fwd_glogit(const double *q, const double *k, const double *v, const double *g, int B, int H,
                          int Hgrid, int Wgrid, int dk, int dv, int dir, double gate_norm, double *out, int nthreads)
{
    if (!g || !(gate_norm > 0.0) || B <= 0 || H <= 0 || Hgrid <= 0 || Wgrid <= 0 || dk <= 0) return ORACLE_BAD_ARG;
    const int64_t n = (int64_t)B * Hgrid * Wgrid * H * dk;
    double *la = (double *)malloc(sizeof(double) * (size_t)n);
    if (!la) return ORACLE_NOMEM;
    for (int64_t e = 0; e < n; ++e) {
        const double x = g[e];
        la[e] = ((x < 0.0 ? x : 0.0) - log1p(exp(-fabs(x)))) / gate_norm;
    }
    int rc = gla_common(q, k, v, la, B, H, Hgrid, Wgrid, dk, dv, dir, out, nthreads, 0, 0, -1);
    free(la);
    return rc;
}

/* The recurrence with one deliberate mistake (tests of the pins only). */
int oracle_gla_fwd_planted(const double *q, const double *k, const double *v, const double *log_alpha,
                           int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir, double *out,
                           int planted)
{
    if (planted < 0 || planted > 7) return ORACLE_BAD_ARG;
    return gla_common(q, k, v, log_alpha, B, H, Hgrid, Wgrid, dk, dv, dir, out, 1, planted, 0, -1);
}

/* ------------------------------------------------------------------------- */
/* GLA backward: reverse sweep of the recurrence (fp64).                      */
/* ------------------------------------------------------------------------- */
typedef struct {
    const double *q, *k, *v, *la, *dout;
    double *dq, *dk, *dv, *dla;
    const int64_t *order;
    int64_t T;
    int64_t bh_base;
    int H, dk_, dv_;
    int planted; /* 0 = the method; 1..6 = a planted mistake (tests only) */
    int status;
} gla_bwd_ctx;

static void gla_bwd_head(void *vctx, int64_t i_local)
{
    gla_bwd_ctx *c = (gla_bwd_ctx *)vctx;
    const int64_t bh = c->bh_base + i_local;
    const int64_t b = bh / c->H, h = bh % c->H;
    const int dk = c->dk_, dv = c->dv_;
    const int64_t T = c->T, H = c->H;
    const size_t sz = (size_t)dk * dv;
    /* states[p] = S after step p; states[-1] (the zero initial state) is `zero` */
    double *states = (double *)malloc(sizeof(double) * sz * (size_t)T);
    double *zero = (double *)calloc(sz, sizeof(double));
    double *G = (double *)calloc(sz, sizeof(double));
    if (!states || !zero || !G) {
        free(states);
        free(zero);
        free(G);
        c->status = ORACLE_NOMEM;
        return;
    }

    /* forward sweep: the states the reverse sweep reads */
    for (int64_t p = 0; p < T; ++p) {
        const int64_t t = c->order[p];
        const double *kt = c->k + tok_off(b, t, h, T, H, dk);
        const double *vt = c->v + tok_off(b, t, h, T, H, dv);
        const double *lt = c->la + tok_off(b, t, h, T, H, dk);
        const double *Sp = p ? states + (size_t)(p - 1) * sz : zero;
        double *Sn = states + (size_t)p * sz;
        for (int i = 0; i < dk; ++i) {
            const double alpha = exp(lt[i]);
            for (int j = 0; j < dv; ++j) Sn[(int64_t)i * dv + j] = alpha * Sp[(int64_t)i * dv + j] + kt[i] * vt[j];
        }
    }

    /* reverse sweep */
    for (int64_t p = T - 1; p >= 0; --p) {
        const int64_t t = c->order[p];
        const double *qt = c->q + tok_off(b, t, h, T, H, dk);
        const double *kt = c->k + tok_off(b, t, h, T, H, dk);
        const double *vt = c->v + tok_off(b, t, h, T, H, dv);
        const double *lt = c->la + tok_off(b, t, h, T, H, dk);
        const double *go = c->dout + tok_off(b, t, h, T, H, dv);
        double *gq = c->dq + tok_off(b, t, h, T, H, dk);
        double *gk = c->dk + tok_off(b, t, h, T, H, dk);
        double *gv = c->dv + tok_off(b, t, h, T, H, dv);
        double *gl = c->dla + tok_off(b, t, h, T, H, dk);
        const double *Sp = states + (size_t)p * sz;                     /* S_p     */
        const double *Sm = p ? states + (size_t)(p - 1) * sz : zero;     /* S_{p-1} */

        /* o_p = q_p S_p: S_p receives q_p^T dO_p (planted 1: it is forgotten) */
        if (c->planted != 1)
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) G[(int64_t)i * dv + j] += qt[i] * go[j];
        /* dq_p = dO_p S_p^T (planted 2: the state before the update is read) */
        const double *Sq = (c->planted == 2) ? Sm : Sp;
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += go[j] * Sq[(int64_t)i * dv + j];
            gq[i] = acc;
        }
        /* dk_p = G v_p^T, dv_p = k_p G (planted 3: q_p read in place of k_p) */
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += G[(int64_t)i * dv + j] * vt[j];
            gk[i] = acc;
        }
        const double *kv = (c->planted == 3) ? qt : kt;
        for (int j = 0; j < dv; ++j) {
            double acc = 0.0;
            for (int i = 0; i < dk; ++i) acc += kv[i] * G[(int64_t)i * dv + j];
            gv[j] = acc;
        }
        /* dlog_alpha_p[i] = alpha_p[i] sum_j G[i][j] S_{p-1}[i][j]
           (planted 4: S_p in place of S_{p-1}; planted 5: the factor alpha dropped) */
        const double *Sa = (c->planted == 4) ? Sp : Sm;
        for (int i = 0; i < dk; ++i) {
            double acc = 0.0;
            for (int j = 0; j < dv; ++j) acc += G[(int64_t)i * dv + j] * Sa[(int64_t)i * dv + j];
            gl[i] = (c->planted == 5) ? acc : exp(lt[i]) * acc;
        }
        /* gradient to S_{p-1}: G = Diag(alpha_p) G (planted 6: decay skipped) */
        if (c->planted != 6)
            for (int i = 0; i < dk; ++i) {
                const double alpha = exp(lt[i]);
                for (int j = 0; j < dv; ++j) G[(int64_t)i * dv + j] *= alpha;
            }
    }
    free(states);
    free(zero);
    free(G);
}

static int gla_bwd_common(const double *q, const double *k, const double *v, const double *log_alpha,
                          const double *dout, int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir,
                          double *dq, double *dk_out, double *dv_out, double *dla, int nthreads, int planted,
                          int64_t bh_begin, int64_t bh_end)
{
    if (!q || !k || !v || !log_alpha || !dout || !dq || !dk_out || !dv_out || !dla) return ORACLE_BAD_ARG;
    if (B <= 0 || H <= 0 || Hgrid <= 0 || Wgrid <= 0 || dk <= 0 || dv <= 0) return ORACLE_BAD_ARG;
    if (dir < 0 || dir > 11) return ORACLE_BAD_ARG;
    const int64_t T = (int64_t)Hgrid * Wgrid;
    const int64_t BH = (int64_t)B * H;
    if (bh_begin < 0) bh_begin = 0;
    if (bh_end < 0 || bh_end > BH) bh_end = BH;
    if (bh_begin > bh_end) return ORACLE_BAD_ARG;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!order) return ORACLE_NOMEM;
    int rc = oracle_scan_order(dir, Hgrid, Wgrid, order);
    if (rc != ORACLE_OK) {
        free(order);
        return rc;
    }
    gla_bwd_ctx c;
    c.q = q;
    c.k = k;
    c.v = v;
    c.la = log_alpha;
    c.dout = dout;
    c.dq = dq;
    c.dk = dk_out;
    c.dv = dv_out;
    c.dla = dla;
    c.order = order;
    c.T = T;
    c.bh_base = bh_begin;
    c.H = H;
    c.dk_ = dk;
    c.dv_ = dv;
    c.planted = planted;
    c.status = ORACLE_OK;
    int used = run_pool(gla_bwd_head, &c, bh_end - bh_begin, nthreads);
    free(order);
    if (c.status != ORACLE_OK) return c.status;
    return used;
}

/*
 * GLA backward over flattened heads bh = b*H + h in [bh_begin, bh_end) (bh_end < 0:
 * all).  Inputs as oracle_gla_fwd plus dout [B][T][H][dv]; outputs dq, dk,
 * dlog_alpha [B][T][H][dk] and dv [B][T][H][dv] (heads outside the range are not
 * written).  Each worker holds one head's T forward states.  Returns the number
 * of threads used or a negative error code.
 */
int oracle_gla_bwd(const double *q, const double *k, const double *v, const double *log_alpha,
                   const double *dout, int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir, double *dq,
                   double *dk_out, double *dv_out, double *dla, int nthreads, int64_t bh_begin, int64_t bh_end)
{
    return gla_bwd_common(q, k, v, log_alpha, dout, B, H, Hgrid, Wgrid, dk, dv, dir, dq, dk_out, dv_out, dla,
                          nthreads, 0, bh_begin, bh_end);
}

/* The backward sweep with one deliberate mistake (tests of the pins only). */
int oracle_gla_bwd_planted(const double *q, const double *k, const double *v, const double *log_alpha,
                           const double *dout, int B, int H, int Hgrid, int Wgrid, int dk, int dv, int dir,
                           double *dq, double *dk_out, double *dv_out, double *dla, int planted)
{
    if (planted < 0 || planted > 6) return ORACLE_BAD_ARG;
    return gla_bwd_common(q, k, v, log_alpha, dout, B, H, Hgrid, Wgrid, dk, dv, dir, dq, dk_out, dv_out, dla, 1,
                          planted, 0, -1);
}

/* ------------------------------------------------------------------------- */
/* Normalised variant (elu+1 features, sigmoid(q*k) gate, gated denominator). */
/* ------------------------------------------------------------------------- */
typedef struct {
    const double *q, *k, *v;
    double *out;
    const int64_t *order;
    int64_t T;
    int H, dk, dv;
    double eps;
    int planted; /* 0 = the method; 1..5 = a planted mistake (tests only) */
    int status;
} norm_ctx;

static double feature(double x, int planted)
{
    if (planted == 1) return x > 0.0 ? x : 0.0; /* planted: relu in place of elu + 1 */
    return x > 0.0 ? x + 1.0 : exp(x);         /* elu(x) + 1 = e^x for x <= 0 */
}

static void norm_head(void *vctx, int64_t bh)
{
    norm_ctx *c = (norm_ctx *)vctx;
    const int64_t b = bh / c->H, h = bh % c->H;
    const int dk = c->dk, dv = c->dv;
    double *S = (double *)calloc((size_t)dk * dv, sizeof(double));
    double *z = (double *)calloc((size_t)dk, sizeof(double));
    double *fq = (double *)malloc(sizeof(double) * dk);
    double *fk = (double *)malloc(sizeof(double) * dk);
    if (!S || !z || !fq || !fk) {
        free(S);
        free(z);
        free(fq);
        free(fk);
        c->status = ORACLE_NOMEM;
        return;
    }
    for (int64_t p = 0; p < c->T; ++p) {
        const int64_t t = c->order[p];
        const double *qt = c->q + tok_off(b, t, h, c->T, c->H, dk);
        const double *kt = c->k + tok_off(b, t, h, c->T, c->H, dk);
        const double *vt = c->v + tok_off(b, t, h, c->T, c->H, dv);
        double *ot = c->out + tok_off(b, t, h, c->T, c->H, dv);
        for (int i = 0; i < dk; ++i) {
            fq[i] = feature(qt[i], c->planted);
            fk[i] = feature(kt[i], c->planted);
        }
        for (int i = 0; i < dk; ++i) {
            /* the gate: sigmoid of the raw q * k (planted 2: of the features' product) */
            const double x = (c->planted == 2) ? fq[i] * fk[i] : qt[i] * kt[i];
            const double g = 1.0 / (1.0 + exp(-x));
            for (int j = 0; j < dv; ++j) S[(int64_t)i * dv + j] = g * S[(int64_t)i * dv + j] + fk[i] * vt[j];
            /* planted 3: the denominator is not gated */
            z[i] = (c->planted == 3 ? 1.0 : g) * z[i] + fk[i];
        }
        double den = 0.0;
        for (int i = 0; i < dk; ++i) den += fq[i] * z[i];
        if (c->planted != 4 && den < c->eps) den = c->eps; /* planted 4: no clamp */
        for (int j = 0; j < dv; ++j) {
            double num = 0.0;
            for (int i = 0; i < dk; ++i) num += fq[i] * S[(int64_t)i * dv + j];
            ot[j] = (c->planted == 5) ? num : num / den; /* planted 5: not normalised */
        }
    }
    free(S);
    free(z);
    free(fq);
    free(fk);
}

static int norm_common(const double *q, const double *k, const double *v, int B, int H, int Hgrid, int Wgrid,
                       int dk, int dv, int dir, double eps, double *out, int nthreads, int planted)
{
    if (!q || !k || !v || !out || B <= 0 || H <= 0 || Hgrid <= 0 || Wgrid <= 0 || dk <= 0 || dv <= 0)
        return ORACLE_BAD_ARG;
    if (dir < 0 || dir > 11 || !(eps > 0.0)) return ORACLE_BAD_ARG;
    const int64_t T = (int64_t)Hgrid * Wgrid;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!order) return ORACLE_NOMEM;
    int rc = oracle_scan_order(dir, Hgrid, Wgrid, order);
    if (rc != ORACLE_OK) {
        free(order);
        return rc;
    }
    norm_ctx c = {q, k, v, out, order, T, H, dk, dv, eps, planted, ORACLE_OK};
    int used = run_pool(norm_head, &c, (int64_t)B * H, nthreads);
    free(order);
    if (c.status != ORACLE_OK) return c.status;
    return used;
}

/* q, k: [B][T][H][dk]; v, out: [B][T][H][dv].  Returns the threads used or an error. */
int oracle_gla_norm_fwd(const double *q, const double *k, const double *v, int B, int H, int Hgrid, int Wgrid,
                        int dk, int dv, int dir, double eps, double *out, int nthreads)
{
    return norm_common(q, k, v, B, H, Hgrid, Wgrid, dk, dv, dir, eps, out, nthreads, 0);
}

/* The normalised variant with one deliberate mistake (tests of the pins only). */
int oracle_gla_norm_fwd_planted(const double *q, const double *k, const double *v, int B, int H, int Hgrid,
                                int Wgrid, int dk, int dv, int dir, double eps, double *out, int planted)
{
    if (planted < 0 || planted > 5) return ORACLE_BAD_ARG;
    return norm_common(q, k, v, B, H, Hgrid, Wgrid, dk, dv, dir, eps, out, 1, planted);
}

/* ------------------------------------------------------------------------- */
/* Depthwise 3x3 conv, zero padding 1, cross-correlation (fp64).              */
/* ------------------------------------------------------------------------- */
typedef struct {
    const double *x, *w;
    double *y;
    int B, Hgrid, Wgrid, C;
} conv_ctx;

static void conv_row(void *vctx, int64_t row)
{
    const conv_ctx *c = (const conv_ctx *)vctx;
    const int64_t b = row / c->Hgrid;
    const int yy = (int)(row % c->Hgrid);
    for (int xx = 0; xx < c->Wgrid; ++xx) {
        for (int ch = 0; ch < c->C; ++ch) {
            double acc = 0.0;
            for (int di = -1; di <= 1; ++di) {
                for (int dj = -1; dj <= 1; ++dj) {
                    const int ys = yy + di, xs = xx + dj;
                    if (ys < 0 || ys >= c->Hgrid || xs < 0 || xs >= c->Wgrid) continue; /* zero pad */
                    const double xv = c->x[((b * c->Hgrid + ys) * (int64_t)c->Wgrid + xs) * c->C + ch];
                    acc += c->w[(int64_t)ch * 9 + (di + 1) * 3 + (dj + 1)] * xv;
                }
            }
            c->y[((b * c->Hgrid + yy) * (int64_t)c->Wgrid + xx) * c->C + ch] = acc;
        }
    }
}

/* x, y: [B][Hgrid][Wgrid][C] channels-last; w: [C][3][3].  Returns threads used. */
int oracle_dwconv3x3(const double *x, const double *w, int B, int Hgrid, int Wgrid, int C, double *y,
                     int nthreads)
{
    if (!x || !w || !y || B <= 0 || Hgrid <= 0 || Wgrid <= 0 || C <= 0) return ORACLE_BAD_ARG;
    conv_ctx c = {x, w, y, B, Hgrid, Wgrid, C};
    return run_pool(conv_row, &c, (int64_t)B * Hgrid, nthreads);
}

/* ------------------------------------------------------------------------- */
/* Reorientation: byte-exact row gather / scatter by the scan-order table.    */
/* ------------------------------------------------------------------------- */
int oracle_reorient(const void *x, int dir, int inverse, int B, int Hgrid, int Wgrid, int64_t row_bytes,
                    void *y)
{
    if (!x || !y || B <= 0 || Hgrid <= 0 || Wgrid <= 0 || row_bytes <= 0) return ORACLE_BAD_ARG;
    if (dir < 0 || dir > 11 || (inverse != 0 && inverse != 1)) return ORACLE_BAD_ARG;
    const int64_t T = (int64_t)Hgrid * Wgrid;
    int64_t *order = (int64_t *)malloc(sizeof(int64_t) * T);
    if (!order) return ORACLE_NOMEM;
    int rc = oracle_scan_order(dir, Hgrid, Wgrid, order);
    if (rc != ORACLE_OK) {
        free(order);
        return rc;
    }
    const unsigned char *xs = (const unsigned char *)x;
    unsigned char *ys = (unsigned char *)y;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t p = 0; p < T; ++p) {
            const int64_t src = inverse ? p : order[p];
            const int64_t dst = inverse ? order[p] : p;
            memcpy(ys + (b * T + dst) * row_bytes, xs + (b * T + src) * row_bytes, (size_t)row_bytes);
        }
    }
    free(order);
    return ORACLE_OK;
}
