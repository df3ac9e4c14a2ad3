/*
 * oracle/ref_swattn.c -- fp64 CPU oracle for shifted local-window self-attention.
 *
 * TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, the smoke check
 * and the CPU-baseline leg of the benchmark load this library.  It shares no
 * source, header, table or helper with the CUDA path; the two meet only in
 * the seeded input generators, which hold none of the method's arithmetic.
 *
 * What it computes (paper: "Backend-Agnostic Sparse Attention for Fast
 * High-Resolution Visual Generation", BASA):
 *
 *   §3.1 "Shifted Window Sparse Attention": at each sparse-attention layer the
 *   token grid is cyclically shifted by -Delta, partitioned into
 *   non-overlapping windows, standard scaled dot-product softmax attention is
 *   applied inside each window with the unchanged Q/K/V, and the outputs are
 *   merged and shifted back by +Delta to their original positions.
 *
 *   Appendix A.1 "Regular execution with standard attention backends": the
 *   shift is a cyclic roll, the windows are formed by reshape/permute and
 *   folded into the batch dimension, each folded window is one dense
 *   attention problem.
 *
 * The four stages are carried out one after the other, each materialising its
 * result, with no fusion:
 *
 *   1. roll      R[t',h',w'] = X[(t'+Dt) mod T, (h'+Dh) mod H, (w'+Dw) mod W]
 *                (a roll by -Delta, the numpy/torch "roll(x, -Delta)" rule)
 *   2. partition windows are the boxes [m_a*w_a, min((m_a+1)*w_a, n_a)) of the
 *                rolled grid along each axis a, numbered in raster order over
 *                (m_t, m_h, m_w); slots inside a window are numbered in raster
 *                order over (s_t, s_h, s_w).
 *   3. attend    per (batch item, window, head): S = scale * Q_w K_w^T,
 *                P = softmax(S) row-wise (max-subtracted), O_w = P V_w, fp64.
 *   4. merge     window outputs are written back to their rolled positions,
 *      + unroll  and the grid is rolled by +Delta: Y[p] = R_O[(p - Delta) mod n].
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - the same cyclic rule applies on the temporal axis when w_t < T;
 *   - a grid that the window does not divide gets a truncated last window
 *     along that axis (no padded tokens take part in any softmax);
 *   - every head and every batch item uses the same partition;
 *   - the inputs are bf16 bit patterns, widened exactly to fp64.
 *
 *   §3.2 "K/V-Pooled Global Memory": K_bar, V_bar are means of K, V over
 *   spatial patches of the grid; each window's keys and values become
 *   [K_W; K_bar] and [V_W; V_bar] (oref_kv_pool builds the means,
 *   oref_swattn_fwd_mem attends over a window plus any extra segment).
 *
 *   §3.3 "Content-Adaptive True-Window Routing": window descriptors are the
 *   means of Q and K over each window, s_ij = q_i k_j^T / sqrt(d) over a
 *   candidate neighbourhood, the top-1 window is routed (oref_route), and each
 *   window attends to S_i = W_i u R_i u G (oref_swattn_fwd_route).
 *
 * Data layout: Q, K, V are bf16 [B, T*H*W, heads, d] (raster token order t,h,w),
 * passed as uint16 bit patterns; the output is fp64 [B, T*H*W, heads, d].
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OREF_OK 0
#define OREF_ERR_ARG (-1)
#define OREF_ERR_NOMEM (-2)

/* ------------------------------------------------------------------ */
/* scalar helpers                                                      */
/* ------------------------------------------------------------------ */

/* bf16 bit pattern -> fp64, exact (bf16 is the top half of an fp32). */
static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* mathematical modulus: result in [0, n) for any integer a and n > 0 */
static long pmod(long a, long n)
{
    long r = a % n;
    return r < 0 ? r + n : r;
}

/* ------------------------------------------------------------------ */
/* geometry                                                            */
/* ------------------------------------------------------------------ */

typedef struct {
    int n[3];      /* grid extent (T, H, W)                    */
    int w[3];      /* window extent (w_t, w_h, w_w)            */
    int delta[3];  /* shift Delta reduced into [0, n_a)        */
    int nwin[3];   /* windows per axis, ceil(n_a / w_a)        */
    long N;        /* tokens in the grid                       */
    long n_windows;/* windows in the grid                      */
    int nw_max;    /* tokens in a full window                  */
} geom_t;

static int geom_init(geom_t *g, int T, int H, int W, const int win[3], const int shift[3])
{
    int a;
    if (T < 1 || H < 1 || W < 1 || !win || !shift) return OREF_ERR_ARG;
    g->n[0] = T; g->n[1] = H; g->n[2] = W;
    g->N = (long)T * H * W;
    g->n_windows = 1;
    g->nw_max = 1;
    for (a = 0; a < 3; ++a) {
        if (win[a] < 1 || win[a] > g->n[a]) return OREF_ERR_ARG;
        g->w[a] = win[a];
        g->delta[a] = (int)pmod(shift[a], g->n[a]);
        g->nwin[a] = (g->n[a] + win[a] - 1) / win[a];
        g->n_windows *= g->nwin[a];
        g->nw_max *= win[a];
    }
    return OREF_OK;
}

/* extent of window index m_a along axis a: full, or truncated at the grid edge */
static int window_extent(const geom_t *g, int a, int m_a)
{
    int start = m_a * g->w[a];
    int left = g->n[a] - start;
    return left < g->w[a] ? left : g->w[a];
}

/* ------------------------------------------------------------------ */
/* stage 1 and stage 4b: cyclic roll of a (T, H, W, C) grid            */
/* ------------------------------------------------------------------ */

/*
 * sign = -1: roll by -Delta, out[i] = in[(i + Delta) mod n]   (stage 1)
 * sign = +1: roll by +Delta, out[i] = in[(i - Delta) mod n]   (stage 4)
 */
static void roll_grid(const double *in, double *out, const geom_t *g, long C, int sign)
{
    int t, h, w;
    for (t = 0; t < g->n[0]; ++t) {
        long ts = pmod((long)t - (long)sign * g->delta[0], g->n[0]);
        for (h = 0; h < g->n[1]; ++h) {
            long hs = pmod((long)h - (long)sign * g->delta[1], g->n[1]);
            for (w = 0; w < g->n[2]; ++w) {
                long wsrc = pmod((long)w - (long)sign * g->delta[2], g->n[2]);
                long dst = ((long)t * g->n[1] + h) * g->n[2] + w;
                long src = (ts * g->n[1] + hs) * g->n[2] + wsrc;
                memcpy(out + dst * C, in + src * C, (size_t)C * sizeof(double));
            }
        }
    }
}

/* ------------------------------------------------------------------ */
/* stage 2 and stage 4a: partition into windows, and its inverse       */
/* ------------------------------------------------------------------ */

/*
 * Window m (raster over m_t, m_h, m_w) of the rolled grid is copied into
 * wbuf[m][slot][C] with slots in raster order; count[m] receives its size.
 * to_windows = 0 performs the inverse copy (merge).
 */
static void partition_grid(double *grid, double *wbuf, int *count, const geom_t *g, long C,
                           int to_windows)
{
    long m = 0;
    int mt, mh, mw, st, sh, sw;
    for (mt = 0; mt < g->nwin[0]; ++mt)
        for (mh = 0; mh < g->nwin[1]; ++mh)
            for (mw = 0; mw < g->nwin[2]; ++mw, ++m) {
                int et = window_extent(g, 0, mt);
                int eh = window_extent(g, 1, mh);
                int ew = window_extent(g, 2, mw);
                long slot = 0;
                for (st = 0; st < et; ++st)
                    for (sh = 0; sh < eh; ++sh)
                        for (sw = 0; sw < ew; ++sw, ++slot) {
                            long t = (long)mt * g->w[0] + st;
                            long h = (long)mh * g->w[1] + sh;
                            long w = (long)mw * g->w[2] + sw;
                            double *gp = grid + ((t * g->n[1] + h) * g->n[2] + w) * C;
                            double *wp = wbuf + (m * g->nw_max + slot) * C;
                            if (to_windows)
                                memcpy(wp, gp, (size_t)C * sizeof(double));
                            else
                                memcpy(gp, wp, (size_t)C * sizeof(double));
                        }
                if (count) count[m] = (int)slot;
            }
}

/* ------------------------------------------------------------------ */
/* stage 3: dense softmax attention inside one window                  */
/* ------------------------------------------------------------------ */

/*
 * q, k, v, o: [n][d] row-major fp64.  S = scale * q k^T; each row of S goes
 * through a max-subtracted softmax; o = P v.  work holds n doubles.
 */
static void window_attention(const double *q, const double *k, const double *v, double *o,
                             int n, int d, double scale, double *work)
{
    int i, j, c;
    for (i = 0; i < n; ++i) {
        double mx = -INFINITY, sum = 0.0;
        for (j = 0; j < n; ++j) {
            double s = 0.0;
            for (c = 0; c < d; ++c) s += q[(long)i * d + c] * k[(long)j * d + c];
            work[j] = scale * s;
            if (work[j] > mx) mx = work[j];
        }
        for (j = 0; j < n; ++j) {
            work[j] = exp(work[j] - mx);
            sum += work[j];
        }
        for (c = 0; c < d; ++c) o[(long)i * d + c] = 0.0;
        for (j = 0; j < n; ++j) {
            double p = work[j] / sum;
            for (c = 0; c < d; ++c) o[(long)i * d + c] += p * v[(long)j * d + c];
        }
    }
}

/*
 * The same with an extra segment appended to the window's keys and values
 * (§3.2 "K/V-Pooled Global Memory": K^mem = [K_W; K_bar], V^mem = [V_W; V_bar]):
 * keys j < n are the window's, keys n <= j < n + E are kx/vx ([E][d]).
 * work holds n + E doubles.
 */
static void window_attention_mem(const double *q, const double *k, const double *v,
                                 const double *kx, const double *vx, double *o,
                                 int n, int E, int d, double scale, double *work)
{
    int i, j, c;
    for (i = 0; i < n; ++i) {
        double mx = -INFINITY, sum = 0.0;
        for (j = 0; j < n + E; ++j) {
            const double *kr = j < n ? k + (long)j * d : kx + (long)(j - n) * d;
            double s = 0.0;
            for (c = 0; c < d; ++c) s += q[(long)i * d + c] * kr[c];
            work[j] = scale * s;
            if (work[j] > mx) mx = work[j];
        }
        for (j = 0; j < n + E; ++j) {
            work[j] = exp(work[j] - mx);
            sum += work[j];
        }
        for (c = 0; c < d; ++c) o[(long)i * d + c] = 0.0;
        for (j = 0; j < n + E; ++j) {
            const double *vr = j < n ? v + (long)j * d : vx + (long)(j - n) * d;
            double pj = work[j] / sum;
            for (c = 0; c < d; ++c) o[(long)i * d + c] += pj * vr[c];
        }
    }
}

/* ------------------------------------------------------------------ */
/* index map: which original token sits in (window, slot)              */
/* ------------------------------------------------------------------ */

/*
 * token_of_slot: [n_windows][nw_max] int32, -1 where a truncated window has
 * no token in that slot.  count_of_window: [n_windows] int32 (may be NULL).
 * Computed by pushing the raster ids of the tokens through stages 1 and 2.
 */
int oref_index_map(int T, int H, int W, const int win[3], const int shift[3],
                   int32_t *token_of_slot, int32_t *count_of_window)
{
    geom_t g;
    double *ids, *rolled, *wbuf;
    int *count;
    long i;
    int rc = geom_init(&g, T, H, W, win, shift);
    if (rc) return rc;
    if (!token_of_slot) return OREF_ERR_ARG;
    ids = (double *)malloc(sizeof(double) * (size_t)g.N);
    rolled = (double *)malloc(sizeof(double) * (size_t)g.N);
    wbuf = (double *)malloc(sizeof(double) * (size_t)(g.n_windows * g.nw_max));
    count = (int *)malloc(sizeof(int) * (size_t)g.n_windows);
    if (!ids || !rolled || !wbuf || !count) {
        free(ids); free(rolled); free(wbuf); free(count);
        return OREF_ERR_NOMEM;
    }
    for (i = 0; i < g.N; ++i) ids[i] = (double)i;
    for (i = 0; i < g.n_windows * g.nw_max; ++i) wbuf[i] = -1.0;
    roll_grid(ids, rolled, &g, 1, -1);
    partition_grid(rolled, wbuf, count, &g, 1, 1);
    for (i = 0; i < g.n_windows * g.nw_max; ++i) token_of_slot[i] = (int32_t)wbuf[i];
    if (count_of_window)
        for (i = 0; i < g.n_windows; ++i) count_of_window[i] = count[i];
    free(ids); free(rolled); free(wbuf); free(count);
    return OREF_OK;
}

/* ------------------------------------------------------------------ */
/* the full forward                                                    */
/* ------------------------------------------------------------------ */

typedef struct {
    const geom_t *g;
    const double *qw, *kw, *vw; /* [n_windows][nw_max][d] for one (b, head) */
    double *ow;
    const int *count;
    int d;
    double scale;
    const double *kx, *vx;      /* extra key/value segment [E][d], or NULL */
    int E;
    long next;                  /* shared window counter */
    int failed;
} attn_job_t;

static void *attn_worker(void *arg)
{
    attn_job_t *job = (attn_job_t *)arg;
    double *work = (double *)malloc(sizeof(double) * (size_t)(job->g->nw_max + job->E));
    if (!work) {
        __atomic_store_n(&job->failed, 1, __ATOMIC_SEQ_CST);
        return NULL;
    }
    for (;;) {
        long m = __atomic_fetch_add(&job->next, 1, __ATOMIC_SEQ_CST);
        long off;
        if (m >= job->g->n_windows) break;
        off = m * job->g->nw_max * job->d;
        if (job->E > 0)
            window_attention_mem(job->qw + off, job->kw + off, job->vw + off, job->kx, job->vx,
                                 job->ow + off, job->count[m], job->E, job->d, job->scale, work);
        else
            window_attention(job->qw + off, job->kw + off, job->vw + off, job->ow + off,
                             job->count[m], job->d, job->scale, work);
    }
    free(work);
    return NULL;
}

/*
 * The forward, with an optional extra key/value segment (kxb, vxb: bf16
 * [B, E, heads, d]; E = 0 for none) appended to every window of its (b, head).
 * out[b, token, head, :] for head in [head_begin, head_end); other heads of
 * out are left untouched.  nthreads <= 0 means one thread.
 */
static int swattn_fwd_impl(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const uint16_t *kxb, const uint16_t *vxb, int E, double *out,
                           int B, int heads, int T, int H, int W, int d,
                           const int win[3], const int shift[3], double scale,
                           int head_begin, int head_end, int nthreads)
{
    geom_t g;
    long N, wsz, tok, c;
    int b, hd, i, rc;
    double *xq, *xk, *xv, *rq, *rk, *rv, *wq, *wk, *wv, *wo, *ro, *y;
    double *xkx = NULL, *xvx = NULL;
    int *count;
    rc = geom_init(&g, T, H, W, win, shift);
    if (rc) return rc;
    if (!q || !k || !v || !out || B < 1 || heads < 1 || d < 1) return OREF_ERR_ARG;
    if (head_begin < 0 || head_end > heads || head_begin >= head_end) return OREF_ERR_ARG;
    if (nthreads < 1) nthreads = 1;
    N = g.N;
    wsz = g.n_windows * g.nw_max * d;
    xq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    xk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    xv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    ro = (double *)malloc(sizeof(double) * (size_t)(N * d));
    y = (double *)malloc(sizeof(double) * (size_t)(N * d));
    wq = (double *)calloc((size_t)wsz, sizeof(double));
    wk = (double *)calloc((size_t)wsz, sizeof(double));
    wv = (double *)calloc((size_t)wsz, sizeof(double));
    wo = (double *)calloc((size_t)wsz, sizeof(double));
    count = (int *)malloc(sizeof(int) * (size_t)g.n_windows);
    if (E > 0) {
        xkx = (double *)malloc(sizeof(double) * (size_t)E * (size_t)d);
        xvx = (double *)malloc(sizeof(double) * (size_t)E * (size_t)d);
    }
    rc = OREF_OK;
    if (!xq || !xk || !xv || !rq || !rk || !rv || !ro || !y || !wq || !wk || !wv || !wo || !count ||
        (E > 0 && (!xkx || !xvx))) {
        rc = OREF_ERR_NOMEM;
        goto done;
    }
    for (b = 0; b < B; ++b) {
        for (hd = head_begin; hd < head_end; ++hd) {
            pthread_t *tids;
            attn_job_t job;
            /* this head's grid, widened to fp64 */
            for (tok = 0; tok < N; ++tok) {
                long src = (((long)b * N + tok) * heads + hd) * d;
                for (c = 0; c < d; ++c) {
                    xq[tok * d + c] = bf16_to_f64(q[src + c]);
                    xk[tok * d + c] = bf16_to_f64(k[src + c]);
                    xv[tok * d + c] = bf16_to_f64(v[src + c]);
                }
            }
            /* the extra segment of this (b, head), widened to fp64 */
            for (tok = 0; tok < E; ++tok) {
                long src = (((long)b * E + tok) * heads + hd) * d;
                for (c = 0; c < d; ++c) {
                    xkx[tok * d + c] = bf16_to_f64(kxb[src + c]);
                    xvx[tok * d + c] = bf16_to_f64(vxb[src + c]);
                }
            }
            /* stage 1: roll by -Delta */
            roll_grid(xq, rq, &g, d, -1);
            roll_grid(xk, rk, &g, d, -1);
            roll_grid(xv, rv, &g, d, -1);
            /* stage 2: partition */
            partition_grid(rq, wq, count, &g, d, 1);
            partition_grid(rk, wk, NULL, &g, d, 1);
            partition_grid(rv, wv, NULL, &g, d, 1);
            /* stage 3: attention in every window */
            job.g = &g; job.qw = wq; job.kw = wk; job.vw = wv; job.ow = wo;
            job.count = count; job.d = d; job.scale = scale; job.next = 0; job.failed = 0;
            job.kx = xkx; job.vx = xvx; job.E = E;
            tids = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
            if (!tids) { rc = OREF_ERR_NOMEM; goto done; }
            for (i = 0; i < nthreads; ++i)
                if (pthread_create(&tids[i], NULL, attn_worker, &job) != 0) break;
            {
                int started = i, j;
                if (started == 0) attn_worker(&job);
                for (j = 0; j < started; ++j) pthread_join(tids[j], NULL);
            }
            free(tids);
            if (job.failed) { rc = OREF_ERR_NOMEM; goto done; }
            /* stage 4: merge, then roll back by +Delta */
            partition_grid(ro, wo, NULL, &g, d, 0);
            roll_grid(ro, y, &g, d, +1);
            for (tok = 0; tok < N; ++tok) {
                long dst = (((long)b * N + tok) * heads + hd) * d;
                memcpy(out + dst, y + tok * d, sizeof(double) * (size_t)d);
            }
        }
    }
done:
    free(xq); free(xk); free(xv); free(rq); free(rk); free(rv); free(ro); free(y);
    free(wq); free(wk); free(wv); free(wo); free(count); free(xkx); free(xvx);
    return rc;
}

int oref_swattn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *out,
                    int B, int heads, int T, int H, int W, int d,
                    const int win[3], const int shift[3], double scale,
                    int head_begin, int head_end, int nthreads)
{
    return swattn_fwd_impl(q, k, v, NULL, NULL, 0, out, B, heads, T, H, W, d, win, shift, scale,
                           head_begin, head_end, nthreads);
}

/*
 * The forward with an extra key/value segment appended to every window
 * (§3.2): kx, vx are bf16 [B, E, heads, d]; every query of window m attends
 * to the window's tokens and to the E extra tokens of its own (b, head).
 */
int oref_swattn_fwd_mem(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                        const uint16_t *kx, const uint16_t *vx, int E, double *out,
                        int B, int heads, int T, int H, int W, int d,
                        const int win[3], const int shift[3], double scale,
                        int head_begin, int head_end, int nthreads)
{
    if (E < 0 || (E > 0 && (!kx || !vx))) return OREF_ERR_ARG;
    return swattn_fwd_impl(q, k, v, kx, vx, E, out, B, heads, T, H, W, d, win, shift, scale,
                           head_begin, head_end, nthreads);
}

/* ------------------------------------------------------------------ */
/* single output rows, for sampling large grids                        */
/* ------------------------------------------------------------------ */

/*
 * For each requested (b, token, head) triple, the same four stages restricted
 * to one query: the query's rolled position (stage 1), the window that holds
 * it and that window's tokens in slot order (stage 2), one softmax row over
 * the window (stage 3), and the result returned for the token it came from
 * (stage 4).  out_rows: [nrows][d].  Arithmetic order per row equals
 * oref_swattn_fwd's, so the two agree bit for bit.
 */
int oref_swattn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                     int B, int heads, int T, int H, int W, int d,
                     const int win[3], const int shift[3], double scale,
                     const int64_t *triples, long nrows, double *out_rows)
{
    geom_t g;
    long r;
    int rc = geom_init(&g, T, H, W, win, shift);
    double *kw, *vw, *qrow, *work;
    if (rc) return rc;
    if (!q || !k || !v || !triples || !out_rows || B < 1 || heads < 1 || d < 1) return OREF_ERR_ARG;
    kw = (double *)malloc(sizeof(double) * (size_t)g.nw_max * d);
    vw = (double *)malloc(sizeof(double) * (size_t)g.nw_max * d);
    qrow = (double *)malloc(sizeof(double) * (size_t)d);
    work = (double *)malloc(sizeof(double) * (size_t)g.nw_max);
    if (!kw || !vw || !qrow || !work) {
        free(kw); free(vw); free(qrow); free(work);
        return OREF_ERR_NOMEM;
    }
    for (r = 0; r < nrows; ++r) {
        long b = triples[3 * r], tok = triples[3 * r + 1], hd = triples[3 * r + 2];
        long p[3], rp[3], m[3], e[3], c, j, n;
        double mx = -INFINITY, sum = 0.0;
        if (b < 0 || b >= B || tok < 0 || tok >= g.N || hd < 0 || hd >= heads) {
            rc = OREF_ERR_ARG;
            break;
        }
        p[0] = tok / ((long)g.n[1] * g.n[2]);
        p[1] = (tok / g.n[2]) % g.n[1];
        p[2] = tok % g.n[2];
        /* stage 1: after the roll by -Delta the token sits at (p - Delta) mod n */
        for (c = 0; c < 3; ++c) {
            rp[c] = pmod(p[c] - g.delta[c], g.n[c]);
            m[c] = rp[c] / g.w[c];                   /* stage 2: its window */
            e[c] = window_extent(&g, (int)c, (int)m[c]);
        }
        /* stage 2: the window's tokens in slot order (rolled coordinate + Delta) */
        n = 0;
        {
            long st, sh, sw;
            for (st = 0; st < e[0]; ++st)
                for (sh = 0; sh < e[1]; ++sh)
                    for (sw = 0; sw < e[2]; ++sw, ++n) {
                        long ot = pmod(m[0] * g.w[0] + st + g.delta[0], g.n[0]);
                        long oh = pmod(m[1] * g.w[1] + sh + g.delta[1], g.n[1]);
                        long ow = pmod(m[2] * g.w[2] + sw + g.delta[2], g.n[2]);
                        long otok = (ot * g.n[1] + oh) * g.n[2] + ow;
                        long src = ((b * g.N + otok) * heads + hd) * d;
                        for (c = 0; c < d; ++c) {
                            kw[n * d + c] = bf16_to_f64(k[src + c]);
                            vw[n * d + c] = bf16_to_f64(v[src + c]);
                        }
                    }
        }
        {
            long src = ((b * g.N + tok) * heads + hd) * d;
            for (c = 0; c < d; ++c) qrow[c] = bf16_to_f64(q[src + c]);
        }
        /* stage 3: one softmax row, same operation order as window_attention */
        for (j = 0; j < n; ++j) {
            double s = 0.0;
            for (c = 0; c < d; ++c) s += qrow[c] * kw[j * d + c];
            work[j] = scale * s;
            if (work[j] > mx) mx = work[j];
        }
        for (j = 0; j < n; ++j) {
            work[j] = exp(work[j] - mx);
            sum += work[j];
        }
        for (c = 0; c < d; ++c) out_rows[r * d + c] = 0.0;
        for (j = 0; j < n; ++j) {
            double pj = work[j] / sum;
            for (c = 0; c < d; ++c) out_rows[r * d + c] += pj * vw[j * d + c];
        }
        /* stage 4: the row belongs to the token it was gathered from */
    }
    free(kw); free(vw); free(qrow); free(work);
    return rc;
}

/*
 * Algorithmic FLOPs of the windowed forward: every window contributes
 * 4 * n_m^2 * d per head and batch item (2 n_m^2 d for Q K^T, 2 n_m^2 d for P V),
 * following the O(N n_w d) cost in §3.1 "Attention complexity".
 */
double oref_flops(int B, int heads, int T, int H, int W, int d, const int win[3])
{
    geom_t g;
    int zero[3] = {0, 0, 0};
    int mt, mh, mw;
    double total = 0.0;
    if (geom_init(&g, T, H, W, win, zero)) return -1.0;
    for (mt = 0; mt < g.nwin[0]; ++mt)
        for (mh = 0; mh < g.nwin[1]; ++mh)
            for (mw = 0; mw < g.nwin[2]; ++mw) {
                double n = (double)window_extent(&g, 0, mt) * window_extent(&g, 1, mh) *
                           window_extent(&g, 2, mw);
                total += 4.0 * n * n * d;
            }
    return total * B * heads;
}

/* ------------------------------------------------------------------ */
/* K/V pooling (§3.2 "K/V-Pooled Global Memory")                       */
/* ------------------------------------------------------------------ */

/*
 * xbar[b, g, head, :] = the mean of x[b, token, head, :] over the tokens of
 * patch g, where the original (unshifted) grid is cut into patches of
 * p_t x p_h x p_w tokens, [g_a p_a, min((g_a + 1) p_a, n_a)) along each axis a
 * (a truncated last patch averages over the tokens it has), and patches are
 * numbered in raster order over (g_t, g_h, g_w).  x is bf16 [B, N, heads, d];
 * xbar is fp64 [B, G, heads, d] with G = prod ceil(n_a / p_a).
 */
int oref_kv_pool(const uint16_t *x, double *xbar, int B, int heads, int T, int H, int W, int d,
                 const int pool[3])
{
    const int n[3] = {T, H, W};
    int G[3], a;
    long g, Gt, N;
    int b, hd, c;
    if (!x || !xbar || !pool || B < 1 || heads < 1 || d < 1 || T < 1 || H < 1 || W < 1)
        return OREF_ERR_ARG;
    for (a = 0; a < 3; ++a) {
        if (pool[a] < 1) return OREF_ERR_ARG;
        G[a] = (n[a] + pool[a] - 1) / pool[a];
    }
    Gt = (long)G[0] * G[1] * G[2];
    N = (long)T * H * W;
    for (b = 0; b < B; ++b)
        for (g = 0; g < Gt; ++g) {
            const int gw = (int)(g % G[2]);
            const int gh = (int)((g / G[2]) % G[1]);
            const int gt = (int)(g / ((long)G[1] * G[2]));
            const int t0 = gt * pool[0], h0 = gh * pool[1], w0 = gw * pool[2];
            const int t1 = t0 + pool[0] < T ? t0 + pool[0] : T;
            const int h1 = h0 + pool[1] < H ? h0 + pool[1] : H;
            const int w1 = w0 + pool[2] < W ? w0 + pool[2] : W;
            const double cnt = (double)(t1 - t0) * (h1 - h0) * (w1 - w0);
            for (hd = 0; hd < heads; ++hd)
                for (c = 0; c < d; ++c) {
                    double acc = 0.0;
                    int t, h, w;
                    for (t = t0; t < t1; ++t)
                        for (h = h0; h < h1; ++h)
                            for (w = w0; w < w1; ++w) {
                                const long tok = ((long)t * H + h) * W + w;
                                acc += bf16_to_f64(x[(((long)b * N + tok) * heads + hd) * d + c]);
                            }
                    xbar[(((long)b * Gt + g) * heads + hd) * d + c] = acc / cnt;
                }
        }
    return OREF_OK;
}

/* ------------------------------------------------------------------ */
/* true-window routing (§3.3 "Content-Adaptive True-Window Routing")   */
/* ------------------------------------------------------------------ */

/*
 * routed[b, head, i] for every window i of the layer's (shifted) partition:
 * q_i = mean of Q over window i's tokens, k_j = mean of K over window j's
 * tokens, s_ij = q_i . k_j / sqrt(d), separately for every head and batch
 * item.  Routing is spatial: the candidates of i are the other windows with
 * the same temporal window index m_t whose spatial window coordinates
 * (m_h, m_w) are within Chebyshev distance `radius` of i's (no wrap-around:
 * the window grid has edges).  routed is the candidate with the largest s_ij
 * (the lowest window index on a tie), or -1 when there is none (K = 1).
 * Computed stage by stage: roll, partition, window means, scores.
 * q, k: bf16 [B, N, heads, d]; routed: int32 [B, heads, nW]; scores (may be
 * NULL): fp64 [B, heads, nW, nW], s_ij for the candidates, -inf elsewhere.
 */
int oref_route(const uint16_t *q, const uint16_t *k, int B, int heads, int T, int H, int W, int d,
               const int win[3], const int shift[3], int radius, int32_t *routed, double *scores)
{
    geom_t g;
    long N, tok, c, wsz;
    int b, hd, rc, m, j;
    double *xq = NULL, *xk = NULL, *rq = NULL, *rk = NULL, *wq = NULL, *wk = NULL;
    double *mq = NULL, *mk = NULL;
    int *count = NULL;
    rc = geom_init(&g, T, H, W, win, shift);
    if (rc) return rc;
    if (!q || !k || !routed || B < 1 || heads < 1 || d < 1 || radius < 0) return OREF_ERR_ARG;
    N = g.N;
    wsz = g.n_windows * g.nw_max * d;
    xq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    xk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    wq = (double *)calloc((size_t)wsz, sizeof(double));
    wk = (double *)calloc((size_t)wsz, sizeof(double));
    mq = (double *)malloc(sizeof(double) * (size_t)(g.n_windows * d));
    mk = (double *)malloc(sizeof(double) * (size_t)(g.n_windows * d));
    count = (int *)malloc(sizeof(int) * (size_t)g.n_windows);
    rc = OREF_OK;
    if (!xq || !xk || !rq || !rk || !wq || !wk || !mq || !mk || !count) { rc = OREF_ERR_NOMEM; goto done; }
    for (b = 0; b < B; ++b) {
        for (hd = 0; hd < heads; ++hd) {
            for (tok = 0; tok < N; ++tok) {
                long src = (((long)b * N + tok) * heads + hd) * d;
                for (c = 0; c < d; ++c) {
                    xq[tok * d + c] = bf16_to_f64(q[src + c]);
                    xk[tok * d + c] = bf16_to_f64(k[src + c]);
                }
            }
            roll_grid(xq, rq, &g, d, -1);
            roll_grid(xk, rk, &g, d, -1);
            partition_grid(rq, wq, count, &g, d, 1);
            partition_grid(rk, wk, NULL, &g, d, 1);
            /* window means */
            for (m = 0; m < g.n_windows; ++m) {
                int s;
                for (c = 0; c < d; ++c) {
                    double aq = 0.0, ak = 0.0;
                    for (s = 0; s < count[m]; ++s) {
                        aq += wq[((long)m * g.nw_max + s) * d + c];
                        ak += wk[((long)m * g.nw_max + s) * d + c];
                    }
                    mq[(long)m * d + c] = aq / count[m];
                    mk[(long)m * d + c] = ak / count[m];
                }
            }
            /* scores over the radius neighbourhood, top-1 */
            for (m = 0; m < g.n_windows; ++m) {
                const int mw = m % g.nwin[2], mh = (m / g.nwin[2]) % g.nwin[1], mt = m / (g.nwin[2] * g.nwin[1]);
                int best = -1;
                double best_s = -INFINITY;
                double *srow = scores ? scores + (((long)b * heads + hd) * g.n_windows + m) * g.n_windows : NULL;
                for (j = 0; j < g.n_windows; ++j) {
                    const int jw = j % g.nwin[2], jh = (j / g.nwin[2]) % g.nwin[1], jt = j / (g.nwin[2] * g.nwin[1]);
                    double s = 0.0;
                    if (srow) srow[j] = -INFINITY;
                    if (j == m || jt != mt || abs(jh - mh) > radius || abs(jw - mw) > radius)
                        continue;
                    for (c = 0; c < d; ++c) s += mq[(long)m * d + c] * mk[(long)j * d + c];
                    s /= sqrt((double)d);
                    if (srow) srow[j] = s;
                    if (s > best_s) { best_s = s; best = j; }
                }
                routed[((long)b * heads + hd) * g.n_windows + m] = best;
            }
        }
    }
done:
    free(xq); free(xk); free(rq); free(rk); free(wq); free(wk); free(mq); free(mk); free(count);
    return rc;
}

/*
 * The forward where window i's queries attend to the tokens of window i, of
 * window routed[b, head, i] (when >= 0; the routed window's own tokens, in its
 * own raster order) and of the extra segment kx, vx ([B, E, heads, d], E >= 0):
 * the key/value source S_i = W_i u R_i u G of §3.3.  Stage by stage as the
 * plain forward; out is fp64 [B, N, heads, d].
 */
int oref_swattn_fwd_route(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const int32_t *routed, const uint16_t *kx, const uint16_t *vx, int E,
                          double *out, int B, int heads, int T, int H, int W, int d,
                          const int win[3], const int shift[3], double scale)
{
    geom_t g;
    long N, tok, c, wsz;
    int b, hd, rc, m;
    double *xq = NULL, *xk = NULL, *xv = NULL, *rq = NULL, *rk = NULL, *rv = NULL;
    double *wq = NULL, *wk = NULL, *wv = NULL, *wo = NULL, *ro = NULL, *y = NULL;
    double *kk = NULL, *vv = NULL, *work = NULL;
    int *count = NULL;
    rc = geom_init(&g, T, H, W, win, shift);
    if (rc) return rc;
    if (!q || !k || !v || !routed || !out || B < 1 || heads < 1 || d < 1 || E < 0 ||
        (E > 0 && (!kx || !vx)))
        return OREF_ERR_ARG;
    N = g.N;
    wsz = g.n_windows * g.nw_max * d;
    xq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    xk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    xv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rq = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rk = (double *)malloc(sizeof(double) * (size_t)(N * d));
    rv = (double *)malloc(sizeof(double) * (size_t)(N * d));
    ro = (double *)malloc(sizeof(double) * (size_t)(N * d));
    y = (double *)malloc(sizeof(double) * (size_t)(N * d));
    wq = (double *)calloc((size_t)wsz, sizeof(double));
    wk = (double *)calloc((size_t)wsz, sizeof(double));
    wv = (double *)calloc((size_t)wsz, sizeof(double));
    wo = (double *)calloc((size_t)wsz, sizeof(double));
    kk = (double *)malloc(sizeof(double) * (size_t)((2 * g.nw_max + E) * d));
    vv = (double *)malloc(sizeof(double) * (size_t)((2 * g.nw_max + E) * d));
    work = (double *)malloc(sizeof(double) * (size_t)(2 * g.nw_max + E));
    count = (int *)malloc(sizeof(int) * (size_t)g.n_windows);
    rc = OREF_OK;
    if (!xq || !xk || !xv || !rq || !rk || !rv || !ro || !y || !wq || !wk || !wv || !wo || !kk || !vv ||
        !work || !count) { rc = OREF_ERR_NOMEM; goto done; }
    for (b = 0; b < B; ++b) {
        for (hd = 0; hd < heads; ++hd) {
            for (tok = 0; tok < N; ++tok) {
                long src = (((long)b * N + tok) * heads + hd) * d;
                for (c = 0; c < d; ++c) {
                    xq[tok * d + c] = bf16_to_f64(q[src + c]);
                    xk[tok * d + c] = bf16_to_f64(k[src + c]);
                    xv[tok * d + c] = bf16_to_f64(v[src + c]);
                }
            }
            roll_grid(xq, rq, &g, d, -1);
            roll_grid(xk, rk, &g, d, -1);
            roll_grid(xv, rv, &g, d, -1);
            partition_grid(rq, wq, count, &g, d, 1);
            partition_grid(rk, wk, NULL, &g, d, 1);
            partition_grid(rv, wv, NULL, &g, d, 1);
            for (m = 0; m < g.n_windows; ++m) {
                const int r = routed[((long)b * heads + hd) * g.n_windows + m];
                int n = 0, s, e;
                /* key/value source: window m, then window r, then the extra segment */
                for (s = 0; s < count[m]; ++s, ++n) {
                    memcpy(kk + (long)n * d, wk + ((long)m * g.nw_max + s) * d, sizeof(double) * (size_t)d);
                    memcpy(vv + (long)n * d, wv + ((long)m * g.nw_max + s) * d, sizeof(double) * (size_t)d);
                }
                if (r >= 0) {
                    if (r >= g.n_windows) { rc = OREF_ERR_ARG; goto done; }
                    for (s = 0; s < count[r]; ++s, ++n) {
                        memcpy(kk + (long)n * d, wk + ((long)r * g.nw_max + s) * d, sizeof(double) * (size_t)d);
                        memcpy(vv + (long)n * d, wv + ((long)r * g.nw_max + s) * d, sizeof(double) * (size_t)d);
                    }
                }
                for (e = 0; e < E; ++e, ++n) {
                    long src = (((long)b * E + e) * heads + hd) * d;
                    for (c = 0; c < d; ++c) {
                        kk[(long)n * d + c] = bf16_to_f64(kx[src + c]);
                        vv[(long)n * d + c] = bf16_to_f64(vx[src + c]);
                    }
                }
                /* dense softmax attention of window m's queries over the n keys */
                {
                    int i, jj;
                    for (i = 0; i < count[m]; ++i) {
                        const double *qi = wq + ((long)m * g.nw_max + i) * d;
                        double *oi = wo + ((long)m * g.nw_max + i) * d;
                        double mx = -INFINITY, sum = 0.0;
                        for (jj = 0; jj < n; ++jj) {
                            double sc = 0.0;
                            for (c = 0; c < d; ++c) sc += qi[c] * kk[(long)jj * d + c];
                            work[jj] = scale * sc;
                            if (work[jj] > mx) mx = work[jj];
                        }
                        for (jj = 0; jj < n; ++jj) { work[jj] = exp(work[jj] - mx); sum += work[jj]; }
                        for (c = 0; c < d; ++c) oi[c] = 0.0;
                        for (jj = 0; jj < n; ++jj) {
                            const double pj = work[jj] / sum;
                            for (c = 0; c < d; ++c) oi[c] += pj * vv[(long)jj * d + c];
                        }
                    }
                }
            }
            partition_grid(ro, wo, NULL, &g, d, 0);
            roll_grid(ro, y, &g, d, +1);
            for (tok = 0; tok < N; ++tok) {
                long dst = (((long)b * N + tok) * heads + hd) * d;
                memcpy(out + dst, y + tok * d, sizeof(double) * (size_t)d);
            }
        }
    }
done:
    free(xq); free(xk); free(xv); free(rq); free(rk); free(rv); free(ro); free(y);
    free(wq); free(wk); free(wv); free(wo); free(kk); free(vv); free(work); free(count);
    return rc;
}

/*
 * Output rows of oref_swattn_fwd_route for (b, token, head) triples only:
 * the token's window (found by the roll by -Delta, as in oref_swattn_rows),
 * then the tokens of its routed window routed[b, head, window] (when >= 0),
 * then the E extra tokens, one softmax row over them, in the same operation
 * order as oref_swattn_fwd_route.  out_rows: fp64 [nrows][d].
 */
int oref_swattn_rows_route(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const int32_t *routed, const uint16_t *kx, const uint16_t *vx, int E,
                           int B, int heads, int T, int H, int W, int d,
                           const int win[3], const int shift[3], double scale,
                           const int64_t *triples, long nrows, double *out_rows)
{
    geom_t g;
    long r, cap;
    int rc = geom_init(&g, T, H, W, win, shift);
    double *kk, *vv, *qrow, *work;
    if (rc) return rc;
    if (!q || !k || !v || !routed || !triples || !out_rows || B < 1 || heads < 1 || d < 1 || E < 0 ||
        (E > 0 && (!kx || !vx)))
        return OREF_ERR_ARG;
    cap = 2L * g.nw_max + E;
    kk = (double *)malloc(sizeof(double) * (size_t)cap * d);
    vv = (double *)malloc(sizeof(double) * (size_t)cap * d);
    qrow = (double *)malloc(sizeof(double) * (size_t)d);
    work = (double *)malloc(sizeof(double) * (size_t)cap);
    if (!kk || !vv || !qrow || !work) {
        free(kk); free(vv); free(qrow); free(work);
        return OREF_ERR_NOMEM;
    }
    for (r = 0; r < nrows; ++r) {
        long b = triples[3 * r], tok = triples[3 * r + 1], hd = triples[3 * r + 2];
        long p[3], rp[3], m[3], c, j, n, seg, wid, rt;
        double mx = -INFINITY, sum = 0.0;
        if (b < 0 || b >= B || tok < 0 || tok >= g.N || hd < 0 || hd >= heads) {
            rc = OREF_ERR_ARG;
            break;
        }
        p[0] = tok / ((long)g.n[1] * g.n[2]);
        p[1] = (tok / g.n[2]) % g.n[1];
        p[2] = tok % g.n[2];
        for (c = 0; c < 3; ++c) {
            rp[c] = pmod(p[c] - g.delta[c], g.n[c]);
            m[c] = rp[c] / g.w[c];
        }
        wid = (m[0] * g.nwin[1] + m[1]) * g.nwin[2] + m[2];
        rt = routed[(b * heads + hd) * g.n_windows + wid];
        if (rt >= g.n_windows) {
            rc = OREF_ERR_ARG;
            break;
        }
        /* keys: the token's window, then the routed window, each in slot order */
        n = 0;
        for (seg = 0; seg < 2; ++seg) {
            long mm[3], e[3], st, sh, sw, id = seg == 0 ? wid : rt;
            if (id < 0) continue;
            mm[2] = id % g.nwin[2];
            mm[1] = (id / g.nwin[2]) % g.nwin[1];
            mm[0] = id / ((long)g.nwin[2] * g.nwin[1]);
            for (c = 0; c < 3; ++c) e[c] = window_extent(&g, (int)c, (int)mm[c]);
            for (st = 0; st < e[0]; ++st)
                for (sh = 0; sh < e[1]; ++sh)
                    for (sw = 0; sw < e[2]; ++sw, ++n) {
                        long ot = pmod(mm[0] * g.w[0] + st + g.delta[0], g.n[0]);
                        long oh = pmod(mm[1] * g.w[1] + sh + g.delta[1], g.n[1]);
                        long ow = pmod(mm[2] * g.w[2] + sw + g.delta[2], g.n[2]);
                        long src = ((b * g.N + (ot * g.n[1] + oh) * g.n[2] + ow) * heads + hd) * d;
                        for (c = 0; c < d; ++c) {
                            kk[n * d + c] = bf16_to_f64(k[src + c]);
                            vv[n * d + c] = bf16_to_f64(v[src + c]);
                        }
                    }
        }
        /* then the extra segment */
        for (j = 0; j < E; ++j, ++n) {
            long src = ((b * E + j) * heads + hd) * d;
            for (c = 0; c < d; ++c) {
                kk[n * d + c] = bf16_to_f64(kx[src + c]);
                vv[n * d + c] = bf16_to_f64(vx[src + c]);
            }
        }
        {
            long src = ((b * g.N + tok) * heads + hd) * d;
            for (c = 0; c < d; ++c) qrow[c] = bf16_to_f64(q[src + c]);
        }
        for (j = 0; j < n; ++j) {
            double s = 0.0;
            for (c = 0; c < d; ++c) s += qrow[c] * kk[j * d + c];
            work[j] = scale * s;
            if (work[j] > mx) mx = work[j];
        }
        for (j = 0; j < n; ++j) {
            work[j] = exp(work[j] - mx);
            sum += work[j];
        }
        for (c = 0; c < d; ++c) out_rows[r * d + c] = 0.0;
        for (j = 0; j < n; ++j) {
            const double pj = work[j] / sum;
            for (c = 0; c < d; ++c) out_rows[r * d + c] += pj * vv[j * d + c];
        }
    }
    free(kk); free(vv); free(qrow); free(work);
    return rc;
}
