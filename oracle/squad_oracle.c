/*
 * squad_oracle.c - plain fp64 CPU oracle for SQuad-Attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call this file:
 * only the tests, the smoke check and the CPU-baseline leg of the benchmark
 * load it. It shares no code, header or table with the CUDA library.
 *
 * What it computes follows "SQuad: Sub-Quadratic Attention Distillation for
 * Efficient Video Generation", gist.science technical summary, Methodology
 * section 1 ("SQuad-Attention Operator"):
 *   - local pass: tokens mix inside fixed windows (full softmax per window);
 *   - global pass: tokens at the same relative position inside their window
 *     mix across all windows (full softmax per group);
 *   - composition: the local output is the value stream of the global pass.
 * Concrete reading used here (the pages leave these open):
 *   - tokens of a T x H x W latent grid are flattened as p = (t*H + y)*W + x;
 *   - a window is an aligned, non-overlapping tT x tH x tW box of the grid;
 *   - "same relative position" is the same (t mod tT, y mod tH, x mod tW);
 *   - both passes use the input Q and K and the scale 1/sqrt(d) (or the
 *     caller's scale); no mask, bias or residual; the output is the global
 *     pass output.
 * The backward is the textbook gradient of softmax attention applied to each
 * pass in turn (the pages only imply it, through fine-tuning through the
 * operator: gist.science technical summary, Methodology section 2).
 *
 * Everything is fp64 with libm exp/log. No blocking, fusion or reordering:
 * each query row is computed on its own, exactly as the definition reads.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int B, heads, d;
    int T, H, W;
    int tT, tH, tW;
    double scale; /* <= 0 means 1/sqrt(d) */
} oracle_desc;

enum { ORACLE_OK = 0, ORACLE_BAD_SHAPE = 1, ORACLE_NO_MEMORY = 2 };

/* ---- geometry: which window and which in-window position a token has ---- */

static long window_of(const oracle_desc* s, long p) {
    long x = p % s->W, y = (p / s->W) % s->H, t = p / ((long)s->W * s->H);
    long nW = s->W / s->tW, nH = s->H / s->tH;
    return ((t / s->tT) * nH + y / s->tH) * nW + x / s->tW;
}

static long offset_of(const oracle_desc* s, long p) {
    long x = p % s->W, y = (p / s->W) % s->H, t = p / ((long)s->W * s->H);
    return ((t % s->tT) * s->tH + y % s->tH) * s->tW + x % s->tW;
}

static int check_desc(const oracle_desc* s) {
    if (s->B <= 0 || s->heads <= 0 || s->d <= 0) return ORACLE_BAD_SHAPE;
    if (s->T <= 0 || s->H <= 0 || s->W <= 0) return ORACLE_BAD_SHAPE;
    if (s->tT <= 0 || s->tH <= 0 || s->tW <= 0) return ORACLE_BAD_SHAPE;
    if (s->T % s->tT || s->H % s->tH || s->W % s->tW) return ORACLE_BAD_SHAPE;
    return ORACLE_OK;
}

/* Bucket the n tokens by a key function: members[key*L + j] is the j-th token
 * (in increasing token order) whose key is `key`. Every bucket has L members. */
static long* bucket(const oracle_desc* s, long n, long nkeys, long L,
                    long (*key)(const oracle_desc*, long)) {
    long* members = (long*)malloc(sizeof(long) * n);
    long* fill = (long*)calloc((size_t)nkeys, sizeof(long));
    if (!members || !fill) { free(members); free(fill); return NULL; }
    for (long p = 0; p < n; p++) {
        long kk = key(s, p);
        members[kk * L + fill[kk]++] = p;
    }
    free(fill);
    return members;
}

/* ---- one softmax-attention problem over a token set ---- */

/* out[i] = sum_j softmax_j(scale * <q_i, k_j>) * val[j] for i, j in rows[0..L);
 * lse[i] = max_j z_ij + log sum_j exp(z_ij - max). */
static void attend_fwd(long L, const long* rows, int d, double scale,
                       const double* q, const double* k, const double* val,
                       double* out, double* lse, double* z, unsigned long long* macs) {
    for (long a = 0; a < L; a++) {
        const double* qi = q + rows[a] * d;
        double mu = -INFINITY;
        for (long b = 0; b < L; b++) {
            const double* kj = k + rows[b] * d;
            double dot = 0.0;
            for (int c = 0; c < d; c++) dot += qi[c] * kj[c];
            z[b] = scale * dot;
            if (z[b] > mu) mu = z[b];
        }
        double l = 0.0;
        for (long b = 0; b < L; b++) {
            z[b] = exp(z[b] - mu);
            l += z[b];
        }
        double* oi = out + rows[a] * d;
        for (int c = 0; c < d; c++) oi[c] = 0.0;
        for (long b = 0; b < L; b++) {
            const double* vj = val + rows[b] * d;
            for (int c = 0; c < d; c++) oi[c] += z[b] * vj[c];
        }
        for (int c = 0; c < d; c++) oi[c] /= l;
        lse[rows[a]] = mu + log(l);
        *macs += (unsigned long long)(2 * L * d);
    }
}

/* Gradient of attend_fwd. With P_ij = exp(z_ij - lse_i) and dP_ij = <dout_i, val_j>:
 *   dS_ij = P_ij * (dP_ij - sum_k P_ik dP_ik)
 *   dq_i += scale * sum_j dS_ij k_j,  dk_j += scale * sum_i dS_ij q_i,
 *   dval_j += sum_i P_ij dout_i. */
static void attend_bwd(long L, const long* rows, int d, double scale,
                       const double* q, const double* k, const double* val,
                       const double* dout, const double* lse,
                       double* dq, double* dk, double* dval, double* P, double* dP) {
    for (long a = 0; a < L; a++) {
        long i = rows[a];
        const double* qi = q + i * d;
        const double* gi = dout + i * d;
        double Di = 0.0;
        for (long b = 0; b < L; b++) {
            const double* kj = k + rows[b] * d;
            const double* vj = val + rows[b] * d;
            double dot = 0.0, gdot = 0.0;
            for (int c = 0; c < d; c++) { dot += qi[c] * kj[c]; gdot += gi[c] * vj[c]; }
            P[b] = exp(scale * dot - lse[i]);
            dP[b] = gdot;
            Di += P[b] * dP[b];
        }
        for (long b = 0; b < L; b++) {
            long j = rows[b];
            double dS = P[b] * (dP[b] - Di);
            for (int c = 0; c < d; c++) {
                dq[i * d + c] += scale * dS * k[j * d + c];
                dk[j * d + c] += scale * dS * qi[c];
                dval[j * d + c] += P[b] * gi[c];
            }
        }
    }
}

/* ---- thread pool over (b,h, problem) work items ---- */

typedef struct {
    const oracle_desc* s;
    long n, L, nprob;     /* tokens per (b,h), rows per problem, problems per (b,h) */
    const long* members;  /* nprob * L token ids */
    int bwd;
    const double *q, *k, *val, *dout, *lse_in;
    double *out, *lse_out, *dq, *dk, *dval;
    int tid, nth;
    unsigned long long macs;
    int failed;
} job_t;

static void* run_job(void* arg) {
    job_t* j = (job_t*)arg;
    const oracle_desc* s = j->s;
    int d = s->d;
    double scale = s->scale > 0 ? s->scale : 1.0 / sqrt((double)d);
    double* z = (double*)malloc(sizeof(double) * 2 * (size_t)j->L);
    if (!z) { j->failed = 1; return NULL; }
    long nbh = (long)s->B * s->heads;
    for (long item = j->tid; item < nbh * j->nprob; item += j->nth) {
        long bh = item / j->nprob, pr = item % j->nprob;
        long off = bh * j->n;                    /* first token of this (b,h) */
        const long* rows = j->members + pr * j->L;
        if (!j->bwd) {
            attend_fwd(j->L, rows, d, scale, j->q + off * d, j->k + off * d, j->val + off * d,
                       j->out + off * d, j->lse_out + off, z, &j->macs);
        } else {
            attend_bwd(j->L, rows, d, scale, j->q + off * d, j->k + off * d, j->val + off * d,
                       j->dout + off * d, j->lse_in + off, j->dq + off * d, j->dk + off * d,
                       j->dval + off * d, z, z + j->L);
        }
    }
    free(z);
    return NULL;
}

static int run_pass(const job_t* proto, int nthreads, unsigned long long* macs) {
    if (nthreads < 1) nthreads = 1;
    job_t* jobs = (job_t*)malloc(sizeof(job_t) * nthreads);
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * nthreads);
    if (!jobs || !th) { free(jobs); free(th); return ORACLE_NO_MEMORY; }
    int started = 0, failed = 0;
    for (int t = 0; t < nthreads; t++) {
        jobs[t] = *proto;
        jobs[t].tid = t;
        jobs[t].nth = nthreads;
        jobs[t].macs = 0;
        jobs[t].failed = 0;
    }
    for (int t = 1; t < nthreads; t++) {
        if (pthread_create(&th[t], NULL, run_job, &jobs[t]) != 0) break;
        started = t;
    }
    /* items of threads that could not be started run here, in thread 0 */
    for (int t = started + 1; t < nthreads; t++) run_job(&jobs[t]);
    run_job(&jobs[0]);
    for (int t = 1; t <= started; t++) pthread_join(th[t], NULL);
    for (int t = 0; t < nthreads; t++) {
        if (macs) *macs += jobs[t].macs;
        failed |= jobs[t].failed;
    }
    free(jobs);
    free(th);
    return failed ? ORACLE_NO_MEMORY : ORACLE_OK;
}

/* ---- public entry points (called through ctypes by the test harness) ---- */

/* Forward. q, k, v: [B, heads, n, d] row-major fp64. Writes o (global-pass
 * output) and, when non-NULL, o1 (local-pass output, token order), lse1, lse2
 * ([B, heads, n], natural log). *macs (optional) receives the number of
 * multiply-adds performed in scores and value sums. */
int oracle_fwd(const oracle_desc* s, const double* q, const double* k, const double* v,
               double* o, double* o1, double* lse1, double* lse2, int nthreads,
               unsigned long long* macs) {
    int rc = check_desc(s);
    if (rc) return rc;
    long n = (long)s->T * s->H * s->W;
    long w = (long)s->tT * s->tH * s->tW, m = n / w;
    long nbh = (long)s->B * s->heads;
    double* o1b = o1 ? o1 : (double*)malloc(sizeof(double) * nbh * n * s->d);
    double* l1b = lse1 ? lse1 : (double*)malloc(sizeof(double) * nbh * n);
    double* l2b = lse2 ? lse2 : (double*)malloc(sizeof(double) * nbh * n);
    long* win = bucket(s, n, m, w, window_of);   /* m windows of w tokens */
    long* grp = bucket(s, n, w, m, offset_of);   /* w groups of m tokens */
    if (macs) *macs = 0;
    if (!o1b || !l1b || !l2b || !win || !grp) { rc = ORACLE_NO_MEMORY; goto done; }

    job_t j;
    memset(&j, 0, sizeof j);
    j.s = s; j.n = n; j.bwd = 0;
    /* local pass: values V, output O1 */
    j.L = w; j.nprob = m; j.members = win;
    j.q = q; j.k = k; j.val = v; j.out = o1b; j.lse_out = l1b;
    rc = run_pass(&j, nthreads, macs);
    if (rc) goto done;
    /* global pass: same Q and K, values O1, output O */
    j.L = m; j.nprob = w; j.members = grp;
    j.val = o1b; j.out = o; j.lse_out = l2b;
    rc = run_pass(&j, nthreads, macs);
done:
    if (!o1) free(o1b);
    if (!lse1) free(l1b);
    if (!lse2) free(l2b);
    free(win);
    free(grp);
    return rc;
}

/* Backward of oracle_fwd for the loss sum(O * dout): writes dq, dk, dv
 * ([B, heads, n, d] fp64). The forward is recomputed here. */
int oracle_bwd(const oracle_desc* s, const double* q, const double* k, const double* v,
               const double* dout, double* dq, double* dk, double* dv, int nthreads) {
    int rc = check_desc(s);
    if (rc) return rc;
    long n = (long)s->T * s->H * s->W;
    long w = (long)s->tT * s->tH * s->tW, m = n / w;
    long nbh = (long)s->B * s->heads;
    size_t big = sizeof(double) * nbh * n * s->d, small = sizeof(double) * nbh * n;
    double* o = (double*)malloc(big);
    double* o1 = (double*)malloc(big);
    double* do1 = (double*)calloc(1, big);
    double* l1 = (double*)malloc(small);
    double* l2 = (double*)malloc(small);
    long* win = bucket(s, n, m, w, window_of);
    long* grp = bucket(s, n, w, m, offset_of);
    if (!o || !o1 || !do1 || !l1 || !l2 || !win || !grp) { rc = ORACLE_NO_MEMORY; goto done; }
    rc = oracle_fwd(s, q, k, v, o, o1, l1, l2, nthreads, NULL);
    if (rc) goto done;
    memset(dq, 0, big);
    memset(dk, 0, big);
    memset(dv, 0, big);

    job_t j;
    memset(&j, 0, sizeof j);
    j.s = s; j.n = n; j.bwd = 1;
    j.q = q; j.k = k;
    /* global pass backward: values O1, upstream dout -> dO1 (and dq, dk parts) */
    j.L = m; j.nprob = w; j.members = grp;
    j.val = o1; j.dout = dout; j.lse_in = l2;
    j.dq = dq; j.dk = dk; j.dval = do1;
    rc = run_pass(&j, nthreads, NULL);
    if (rc) goto done;
    /* local pass backward: values V, upstream dO1 -> dv (and the other dq, dk parts) */
    j.L = w; j.nprob = m; j.members = win;
    j.val = v; j.dout = do1; j.lse_in = l1;
    j.dval = dv;
    rc = run_pass(&j, nthreads, NULL);
done:
    free(o); free(o1); free(do1); free(l1); free(l2); free(win); free(grp);
    return rc;
}

/* ---- more than two passes ----
 *
 * The pages leave "composing more than two passes" as an outlook (gist.science
 * technical summary, Significance and Claims). Reading used here: nested tiles
 * t_1 | t_2 | ... | t_{k-1} | grid (each divides the next along every axis), with
 * t_0 = 1x1x1 and t_k = the grid. Pass j (1..k) attends among the tokens that lie
 * in the same t_j-window AND at the same position inside their t_{j-1}-window; the
 * values of pass j are the output of pass j-1 (V for j = 1), Q and K are the
 * inputs throughout, and the output is that of pass k. With k = 2 this is the
 * local pass followed by the global pass above. */

typedef struct {
    long T, H, W;
    long in[3], out[3]; /* (t, y, x) extents of the inner and the outer tile */
} pass_geom;

/* Group key: (outer window, position inside the inner window). */
static long pass_key(const pass_geom* g, long p) {
    long x = p % g->W, y = (p / g->W) % g->H, t = p / (g->W * g->H);
    long win = ((t / g->out[0]) * (g->H / g->out[1]) + y / g->out[1]) * (g->W / g->out[2]) + x / g->out[2];
    long pos = ((t % g->in[0]) * g->in[1] + y % g->in[1]) * g->in[2] + x % g->in[2];
    return win * (g->in[0] * g->in[1] * g->in[2]) + pos;
}

static long* bucket_pass(const pass_geom* g, long n, long nkeys, long L) {
    long* members = (long*)malloc(sizeof(long) * n);
    long* fill = (long*)calloc((size_t)nkeys, sizeof(long));
    if (!members || !fill) { free(members); free(fill); return NULL; }
    for (long p = 0; p < n; p++) {
        long kk = pass_key(g, p);
        members[kk * L + fill[kk]++] = p;
    }
    free(fill);
    return members;
}

/* Geometry of pass j (1-based) of the k = ntiles + 1 passes; 0 if the tiles do not nest. */
static int pass_of(const oracle_desc* s, int ntiles, const int* tiles, int j, pass_geom* g) {
    g->T = s->T; g->H = s->H; g->W = s->W;
    for (int a = 0; a < 3; a++) {
        g->in[a] = j == 1 ? 1 : tiles[3 * (j - 2) + a];
        g->out[a] = j == ntiles + 1 ? (a == 0 ? s->T : a == 1 ? s->H : s->W) : tiles[3 * (j - 1) + a];
        if (g->in[a] <= 0 || g->out[a] <= 0 || g->out[a] % g->in[a]) return 0;
    }
    return s->T % g->out[0] == 0 && s->H % g->out[1] == 0 && s->W % g->out[2] == 0;
}

static int check_multi(const oracle_desc* s, int ntiles, const int* tiles) {
    if (s->B <= 0 || s->heads <= 0 || s->d <= 0 || s->T <= 0 || s->H <= 0 || s->W <= 0) return ORACLE_BAD_SHAPE;
    if (ntiles < 1 || tiles == NULL) return ORACLE_BAD_SHAPE;
    pass_geom g;
    for (int j = 1; j <= ntiles + 1; j++)
        if (!pass_of(s, ntiles, tiles, j, &g)) return ORACLE_BAD_SHAPE;
    return ORACLE_OK;
}

/* Forward of the k = ntiles + 1 passes. tiles: 3*ntiles ints (tT, tH, tW), innermost
 * first. Writes o and, when non-NULL, inter (ntiles consecutive [B, heads, n, d]
 * tensors: the outputs of passes 1..k-1) and lse (k consecutive [B, heads, n]).
 * *macs (optional) counts the multiply-adds of scores and value sums. */
int oracle_fwd_multi(const oracle_desc* s, int ntiles, const int* tiles, const double* q, const double* k,
                     const double* v, double* o, double* inter, double* lse, int nthreads,
                     unsigned long long* macs) {
    int rc = check_multi(s, ntiles, tiles);
    if (rc) return rc;
    long n = (long)s->T * s->H * s->W;
    long nbh = (long)s->B * s->heads;
    size_t big = (size_t)nbh * n * s->d, small = (size_t)nbh * n;
    double* ib = inter ? inter : (double*)malloc(sizeof(double) * big * ntiles);
    double* lb = lse ? lse : (double*)malloc(sizeof(double) * small * (ntiles + 1));
    if (macs) *macs = 0;
    if (!ib || !lb) { rc = ORACLE_NO_MEMORY; goto done; }
    const double* val = v;
    for (int j = 1; j <= ntiles + 1 && rc == ORACLE_OK; j++) {
        pass_geom g;
        pass_of(s, ntiles, tiles, j, &g);
        long L = (g.out[0] / g.in[0]) * (g.out[1] / g.in[1]) * (g.out[2] / g.in[2]);
        long* members = bucket_pass(&g, n, n / L, L);
        if (!members) { rc = ORACLE_NO_MEMORY; break; }
        job_t jb;
        memset(&jb, 0, sizeof jb);
        jb.s = s; jb.n = n; jb.bwd = 0;
        jb.L = L; jb.nprob = n / L; jb.members = members;
        jb.q = q; jb.k = k; jb.val = val;
        jb.out = j == ntiles + 1 ? o : ib + big * (j - 1);
        jb.lse_out = lb + small * (j - 1);
        rc = run_pass(&jb, nthreads, macs);
        free(members);
        val = jb.out;
    }
done:
    if (!inter) free(ib);
    if (!lse) free(lb);
    return rc;
}

/* Backward of oracle_fwd_multi for the loss sum(O * dout): writes dq, dk, dv. The
 * forward is recomputed; the passes are differentiated from the last to the first,
 * each one's value gradient being the upstream gradient of the pass before. */
int oracle_bwd_multi(const oracle_desc* s, int ntiles, const int* tiles, const double* q, const double* k,
                     const double* v, const double* dout, double* dq, double* dk, double* dv, int nthreads) {
    int rc = check_multi(s, ntiles, tiles);
    if (rc) return rc;
    long n = (long)s->T * s->H * s->W;
    long nbh = (long)s->B * s->heads;
    size_t big = (size_t)nbh * n * s->d, small = (size_t)nbh * n;
    double* o = (double*)malloc(sizeof(double) * big);
    double* inter = (double*)malloc(sizeof(double) * big * ntiles);
    double* lse = (double*)malloc(sizeof(double) * small * (ntiles + 1));
    double* g_up = (double*)malloc(sizeof(double) * big);   /* upstream gradient of the current pass */
    double* g_val = (double*)malloc(sizeof(double) * big);  /* gradient of its values */
    if (!o || !inter || !lse || !g_up || !g_val) { rc = ORACLE_NO_MEMORY; goto done; }
    rc = oracle_fwd_multi(s, ntiles, tiles, q, k, v, o, inter, lse, nthreads, NULL);
    if (rc) goto done;
    memset(dq, 0, sizeof(double) * big);
    memset(dk, 0, sizeof(double) * big);
    memcpy(g_up, dout, sizeof(double) * big);
    for (int j = ntiles + 1; j >= 1 && rc == ORACLE_OK; j--) {
        pass_geom g;
        pass_of(s, ntiles, tiles, j, &g);
        long L = (g.out[0] / g.in[0]) * (g.out[1] / g.in[1]) * (g.out[2] / g.in[2]);
        long* members = bucket_pass(&g, n, n / L, L);
        if (!members) { rc = ORACLE_NO_MEMORY; break; }
        double* dval = j == 1 ? dv : g_val;
        memset(dval, 0, sizeof(double) * big);
        job_t jb;
        memset(&jb, 0, sizeof jb);
        jb.s = s; jb.n = n; jb.bwd = 1;
        jb.L = L; jb.nprob = n / L; jb.members = members;
        jb.q = q; jb.k = k;
        jb.val = j == 1 ? v : inter + big * (j - 2);
        jb.dout = g_up; jb.lse_in = lse + small * (j - 1);
        jb.dq = dq; jb.dk = dk; jb.dval = dval;
        rc = run_pass(&jb, nthreads, NULL);
        free(members);
        if (j > 1) { double* tmp = g_up; g_up = g_val; g_val = tmp; }
    }
done:
    free(o); free(inter); free(lse); free(g_up); free(g_val);
    return rc;
}
