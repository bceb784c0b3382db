/*
 * fp64 CPU oracle for the variable-length (packed, ragged) attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes is the packed attention forward defined by the boostr
 * 0.2.0 source page src/ops/cpu/attention/varlen_attention.rs
 * (VarLenAttentionOps::varlen_attention_fwd), written here from that
 * definition in double precision rather than in the shape of the page's
 * loop.  For sequence b, query head h and sequence-local query qi:
 *
 *   kv_h = h / (H / Hkv)                                  (GQA head map)
 *   V(qi) = { ki in [0, Lk_b) : not (causal and qi < ki) }  (visible keys)
 *   s_ki  = scale * <Q[cu_q[b]+qi, h, :], K[cu_k[b]+ki, kv_h, :]>  for ki in V(qi)
 *   LSE   = log-sum-exp of { s_ki : ki in V(qi) }          (natural log)
 *   O[cu_q[b]+qi, h, :] = sum over ki in V(qi) of exp(s_ki - LSE) * V[cu_k[b]+ki, kv_h, :]
 *
 * The visible keys are gathered first, the LSE comes from a separate
 * max-shifted log-sum-exp reduction, and the weights exp(s - LSE) are the
 * softmax over V(qi).  A row with an empty V(qi) gets O = 0 and LSE = -inf
 * (the page's result for a sequence without keys).
 *
 * Layouts are the page's packed ones: Q/O [Tq, H, D], K/V [Tk, Hkv, D],
 * LSE [Tq, H], all row-major.  The scale is an explicit argument; a value
 * <= 0 or NaN selects the page's default 1/sqrt(D).
 *
 * Extension (the `_ext` entry points): the sliding window and used-key count
 * that PyTorch pull request #176015 lists in the varlen forward schema
 * (window_size_left, window_size_right, seqused_k), read with the page's
 * sequence-local indices: key ki also leaves V(qi) when ki >= seqused_k[b]
 * (clipped to [0, Lk_b]), when left >= 0 and ki < qi - left, or when
 * right >= 0 and ki > qi + right.
 *
 * Attention sinks (the `sinks` argument of the `_ext` entry points; the
 * FLOAT32 per-head "sinks" input of the Ascend sparse shared-KV attention
 * page, which gives no formula): sinks[h] is one more logit, already in score
 * units (not multiplied by the scale), with no value row.  It is one more
 * term of the log-sum-exp, LSE = ln(sum_ki exp(s_ki) + exp(sinks[h])), and
 * the value sum keeps the weights exp(s_ki - LSE); a row with an empty V(qi)
 * then gets O = 0 and LSE = sinks[h].
 *
 * Backward (oracle_varlen_attn_bwd): the gradient of the forward as the
 * same page's VarLenAttentionOps::varlen_attention_bwd defines it, in double
 * precision, given dO, Q, K, V, the forward output O and LSE.  Per query row
 * (b, h, qi), over its visible keys ki:
 *
 *   P_ki  = exp(s_ki - LSE[qi, h])          (the softmax weights)
 *   dP_ki = <dO[qi, h], V[ki, kv_h]>
 *   delta = <dO[qi, h], O[qi, h]>
 *   dS_ki = P_ki (dP_ki - delta)
 *   dQ[qi, h]    = scale * sum_ki dS_ki K[ki, kv_h]
 *   dK[ki, kv_h] += scale * dS_ki Q[qi, h]      (summed over the group's heads)
 *   dV[ki, kv_h] += P_ki dO[qi, h]
 *
 * The row's vectors P, dP and dS are formed first; the three gradient sums
 * follow.  dO is 16-bit like Q/K/V; O and LSE are given in double (the caller
 * widens the stored bf16/fp16 O and float32 LSE exactly, or passes exact
 * values).  Work items are (b, kv_h): each owns the dK/dV rows of that
 * key/value head of sequence b and the dQ rows of its query heads, and runs
 * its rows in a fixed order, so the result does not depend on the thread
 * count.
 *
 * Inputs are bf16 or fp16 bit patterns; they are widened exactly to double
 * before any arithmetic (a format conversion, once per (b, kv_h) item for
 * K and V).  Forward work items (b, h), or single requested rows, are spread
 * over POSIX threads; each output row is computed by one thread, so the
 * result does not depend on the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_BF16 = 0, ORACLE_FP16 = 1 };

/* bf16 is the top half of an IEEE binary32 value: the widening is exact. */
static double oracle_bf16_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* IEEE binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double oracle_fp16_to_double(uint16_t bits) {
    int sign = (bits >> 15) & 1;
    int expo = (bits >> 10) & 0x1f;
    int frac = bits & 0x3ff;
    double mag;
    if (expo == 0) {
        mag = ldexp((double)frac, -24);                 /* subnormal or zero */
    } else if (expo == 31) {
        mag = frac ? NAN : INFINITY;
    } else {
        mag = ldexp((double)(1024 + frac), expo - 25);  /* (1 + f/1024) 2^(e-15) */
    }
    return sign ? -mag : mag;
}

double oracle_decode16(uint16_t bits, int dtype) {
    return dtype == ORACLE_FP16 ? oracle_fp16_to_double(bits) : oracle_bf16_to_double(bits);
}

typedef struct {
    const uint16_t *q, *k, *v;
    int dtype;
    const int32_t *cu_q, *cu_k;
    const int32_t *seqused_k; /* NULL: every key of the sequence */
    int B, H, Hkv, D, causal;
    int win_left, win_right;  /* < 0: unbounded */
    const double *sinks;      /* NULL, or one extra logit per query head */
    double scale;
    /* full mode */
    double *out, *lse;
    /* rows mode */
    const int64_t *row_tok;
    const int32_t *row_head;
    int64_t nrows;
    double *out_rows, *lse_rows;
    /* work distribution */
    int64_t next_item;
    int64_t n_items;
    int status;
} OracleCtx;

static double effective_scale(double scale, int D) {
    if (!(scale > 0.0)) return 1.0 / sqrt((double)D); /* <= 0 or NaN */
    return scale;
}

/* Keys of sequence b that exist for attention: Lk_b, or seqused_k[b] when
 * given (clipped to [0, Lk_b]). */
static int used_keys(const OracleCtx *c, int b) {
    int Lk = c->cu_k[b + 1] - c->cu_k[b];
    if (c->seqused_k) {
        int u = c->seqused_k[b];
        if (u < 0) u = 0;
        if (u < Lk) Lk = u;
    }
    return Lk;
}

static double head_sink(const OracleCtx *c, int h) {
    return c->sinks ? c->sinks[h] : -INFINITY;
}

static int key_hidden(const OracleCtx *c, int qi, int ki) {
    if (c->causal && qi < ki) return 1;
    if (c->win_left >= 0 && ki < qi - c->win_left) return 1;
    if (c->win_right >= 0 && ki > qi + c->win_right) return 1;
    return 0;
}

/* Indices of the keys of V(qi) among the first Lk keys of the sequence, in
 * increasing order, into idx; returns how many there are. */
static int visible_keys(const OracleCtx *c, int qi, int Lk, int *idx) {
    int n = 0;
    for (int ki = 0; ki < Lk; ++ki)
        if (!key_hidden(c, qi, ki)) idx[n++] = ki;
    return n;
}

static double dot_d(const double *a, const double *b, int D) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += a[d] * b[d];
    return acc;
}

/* ln(exp(extra) + sum_i exp(x[i])), shifted by the largest term; -inf for
 * an empty sum (n = 0 and extra = -inf). */
static double log_sum_exp(const double *x, int n, double extra) {
    double m = extra;
    for (int i = 0; i < n; ++i)
        if (x[i] > m) m = x[i];
    if (m == -INFINITY) return -INFINITY;
    double acc = exp(extra - m);
    for (int i = 0; i < n; ++i) acc += exp(x[i] - m);
    return m + log(acc);
}

/* One output row from the definition: the scores of the visible keys, their
 * log-sum-exp (with the head's sink logit as one more term), and the value
 * rows weighted by exp(s - LSE).  kd/vd hold the widened keys/values of head
 * kv_h of sequence b, [Lk][D]; idx and s are scratch of Lk entries. */
static void oracle_row(const OracleCtx *c, const double *qrow, int qi, int Lk, const double *kd,
                       const double *vd, int *idx, double *s, double sink, double *out_row,
                       double *lse_out) {
    const int D = c->D;
    const int n = visible_keys(c, qi, Lk, idx);
    for (int i = 0; i < n; ++i) s[i] = c->scale * dot_d(qrow, kd + (size_t)idx[i] * D, D);
    const double lse = log_sum_exp(s, n, sink);
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    *lse_out = lse;
    if (lse == -INFINITY) return;
    for (int i = 0; i < n; ++i) {
        const double w = exp(s[i] - lse);
        const double *vrow = vd + (size_t)idx[i] * D;
        for (int d = 0; d < D; ++d) out_row[d] += w * vrow[d];
    }
}

static void widen_kv(const OracleCtx *c, int b, int kv_h, double *kd, double *vd) {
    const int D = c->D, Hkv = c->Hkv;
    int k0 = c->cu_k[b], Lk = c->cu_k[b + 1] - c->cu_k[b];
    for (int ki = 0; ki < Lk; ++ki) {
        size_t off = ((size_t)(k0 + ki) * Hkv + kv_h) * D;
        for (int d = 0; d < D; ++d) {
            kd[(size_t)ki * D + d] = oracle_decode16(c->k[off + d], c->dtype);
            vd[(size_t)ki * D + d] = oracle_decode16(c->v[off + d], c->dtype);
        }
    }
}

static void widen_q(const OracleCtx *c, int64_t tok, int h, double *qd) {
    size_t off = ((size_t)tok * c->H + h) * c->D;
    for (int d = 0; d < c->D; ++d) qd[d] = oracle_decode16(c->q[off + d], c->dtype);
}

static int max_k_len(const OracleCtx *c) {
    int m = 0;
    for (int b = 0; b < c->B; ++b) {
        int L = c->cu_k[b + 1] - c->cu_k[b];
        if (L > m) m = L;
    }
    return m;
}

/* Full mode: work item = (b, h). */
static void *full_worker(void *arg) {
    OracleCtx *c = (OracleCtx *)arg;
    const int D = c->D, H = c->H, G = c->H / c->Hkv;
    int mk = max_k_len(c);
    size_t kvn = (size_t)(mk > 0 ? mk : 1) * D;
    double *kd = (double *)malloc(kvn * sizeof(double));
    double *vd = (double *)malloc(kvn * sizeof(double));
    double *scores = (double *)malloc((size_t)(mk > 0 ? mk : 1) * sizeof(double));
    int *idx = (int *)malloc((size_t)(mk > 0 ? mk : 1) * sizeof(int));
    double *qd = (double *)malloc((size_t)D * sizeof(double));
    if (!kd || !vd || !scores || !idx || !qd) {
        __atomic_store_n(&c->status, -1, __ATOMIC_RELAXED);
        free(kd); free(vd); free(scores); free(idx); free(qd);
        return NULL;
    }
    for (;;) {
        int64_t item = __atomic_fetch_add(&c->next_item, 1, __ATOMIC_RELAXED);
        if (item >= c->n_items) break;
        int b = (int)(item / H), h = (int)(item % H);
        int kv_h = h / G;
        int q0 = c->cu_q[b], Lq = c->cu_q[b + 1] - c->cu_q[b];
        int Lk = used_keys(c, b);
        if (Lq <= 0) continue;
        widen_kv(c, b, kv_h, kd, vd);
        for (int qi = 0; qi < Lq; ++qi) {
            int64_t tok = (int64_t)q0 + qi;
            widen_q(c, tok, h, qd);
            oracle_row(c, qd, qi, Lk, kd, vd, idx, scores, head_sink(c, h),
                       c->out + ((size_t)tok * H + h) * D, c->lse + (size_t)tok * H + h);
        }
    }
    free(kd); free(vd); free(scores); free(idx); free(qd);
    return NULL;
}

/* Sequence containing packed query token tok: largest b with cu_q[b] <= tok,
 * among sequences with Lq_b > 0. */
static int find_seq(const OracleCtx *c, int64_t tok) {
    int lo = 0, hi = c->B - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (c->cu_q[mid] <= tok) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* Rows mode: work item = one requested (token, head) row. */
static void *rows_worker(void *arg) {
    OracleCtx *c = (OracleCtx *)arg;
    const int D = c->D, G = c->H / c->Hkv;
    int mk = max_k_len(c);
    size_t kvn = (size_t)(mk > 0 ? mk : 1) * D;
    double *kd = (double *)malloc(kvn * sizeof(double));
    double *vd = (double *)malloc(kvn * sizeof(double));
    double *scores = (double *)malloc((size_t)(mk > 0 ? mk : 1) * sizeof(double));
    int *idx = (int *)malloc((size_t)(mk > 0 ? mk : 1) * sizeof(int));
    double *qd = (double *)malloc((size_t)D * sizeof(double));
    int cached_b = -1, cached_kvh = -1;
    if (!kd || !vd || !scores || !idx || !qd) {
        __atomic_store_n(&c->status, -1, __ATOMIC_RELAXED);
        free(kd); free(vd); free(scores); free(idx); free(qd);
        return NULL;
    }
    for (;;) {
        int64_t i = __atomic_fetch_add(&c->next_item, 1, __ATOMIC_RELAXED);
        if (i >= c->nrows) break;
        int64_t tok = c->row_tok[i];
        int h = c->row_head[i];
        int b = find_seq(c, tok);
        int kv_h = h / G;
        int qi = (int)(tok - c->cu_q[b]);
        int Lk = used_keys(c, b);
        if (b != cached_b || kv_h != cached_kvh) {
            widen_kv(c, b, kv_h, kd, vd);
            cached_b = b;
            cached_kvh = kv_h;
        }
        widen_q(c, tok, h, qd);
        oracle_row(c, qd, qi, Lk, kd, vd, idx, scores, head_sink(c, h),
                   c->out_rows + (size_t)i * D, c->lse_rows + i);
    }
    free(kd); free(vd); free(scores); free(idx); free(qd);
    return NULL;
}

static int run_threads(OracleCtx *c, void *(*fn)(void *), int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t tids[512];
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, fn, c) != 0) break;
        ++started;
    }
    if (started == 0) fn(c);
    for (int t = 0; t < started; ++t) pthread_join(tids[t], NULL);
    return c->status;
}

static int check_args(int B, int H, int Hkv, int D, int dtype) {
    if (B < 0 || H <= 0 || Hkv <= 0 || D <= 0) return -2;
    if (H % Hkv != 0) return -2;
    if (dtype != ORACLE_BF16 && dtype != ORACLE_FP16) return -3;
    return 0;
}

/* Full forward: writes out[Tq*H*D] and lse[Tq*H] (Tq = cu_q[B]).
 * Returns 0, or a negative code on bad arguments / allocation failure. */
int oracle_varlen_attn_fwd_ext(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                               int dtype, const int32_t *cu_q, const int32_t *cu_k,
                               const int32_t *seqused_k, int B, int H, int Hkv, int D, int causal,
                               int win_left, int win_right, const double *sinks, double scale,
                               double *out, double *lse, int nthreads) {
    int rc = check_args(B, H, Hkv, D, dtype);
    if (rc) return rc;
    OracleCtx c;
    memset(&c, 0, sizeof c);
    c.q = q; c.k = k; c.v = v; c.dtype = dtype; c.cu_q = cu_q; c.cu_k = cu_k;
    c.seqused_k = seqused_k;
    c.B = B; c.H = H; c.Hkv = Hkv; c.D = D; c.causal = causal != 0;
    c.win_left = win_left; c.win_right = win_right; c.sinks = sinks;
    c.scale = effective_scale(scale, D);
    c.out = out; c.lse = lse;
    c.n_items = (int64_t)B * H;
    return run_threads(&c, full_worker, nthreads);
}

int oracle_varlen_attn_fwd(const uint16_t *q, const uint16_t *k, const uint16_t *v, int dtype,
                           const int32_t *cu_q, const int32_t *cu_k, int B, int H, int Hkv,
                           int D, int causal, double scale, double *out, double *lse,
                           int nthreads) {
    return oracle_varlen_attn_fwd_ext(q, k, v, dtype, cu_q, cu_k, NULL, B, H, Hkv, D, causal,
                                      -1, -1, NULL, scale, out, lse, nthreads);
}

/* Selected rows: for i in [0, nrows) computes the output row of packed query
 * token row_tok[i], head row_head[i] into out_rows[i*D..] and lse_rows[i]. */
int oracle_varlen_attn_rows_ext(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                int dtype, const int32_t *cu_q, const int32_t *cu_k,
                                const int32_t *seqused_k, int B, int H, int Hkv, int D,
                                int causal, int win_left, int win_right, const double *sinks,
                                double scale, const int64_t *row_tok, const int32_t *row_head,
                                int64_t nrows, double *out_rows, double *lse_rows, int nthreads) {
    int rc = check_args(B, H, Hkv, D, dtype);
    if (rc) return rc;
    if (B < 1) return -2;
    OracleCtx c;
    memset(&c, 0, sizeof c);
    c.q = q; c.k = k; c.v = v; c.dtype = dtype; c.cu_q = cu_q; c.cu_k = cu_k;
    c.seqused_k = seqused_k;
    c.B = B; c.H = H; c.Hkv = Hkv; c.D = D; c.causal = causal != 0;
    c.win_left = win_left; c.win_right = win_right; c.sinks = sinks;
    c.scale = effective_scale(scale, D);
    c.row_tok = row_tok; c.row_head = row_head; c.nrows = nrows;
    c.out_rows = out_rows; c.lse_rows = lse_rows;
    return run_threads(&c, rows_worker, nthreads);
}

int oracle_varlen_attn_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, int dtype,
                            const int32_t *cu_q, const int32_t *cu_k, int B, int H, int Hkv,
                            int D, int causal, double scale, const int64_t *row_tok,
                            const int32_t *row_head, int64_t nrows, double *out_rows,
                            double *lse_rows, int nthreads) {
    return oracle_varlen_attn_rows_ext(q, k, v, dtype, cu_q, cu_k, NULL, B, H, Hkv, D, causal,
                                       -1, -1, NULL, scale, row_tok, row_head, nrows, out_rows,
                                       lse_rows, nthreads);
}


/* ------------------------------------------------------------------ backward */

typedef struct {
    const uint16_t *dout, *q, *k, *v;
    const double *o, *lse;
    int dtype;
    const int32_t *cu_q, *cu_k;
    int B, H, Hkv, D, causal;
    double scale;
    double *dq, *dk, *dv;
    int64_t next_item, n_items;
    int status;
} OracleBwdCtx;

/* Keys of the sequence visible to query qi (the causal rule only), in
 * increasing order, into idx; returns how many there are. */
static int bwd_visible_keys(const OracleBwdCtx *c, int qi, int Lk, int *idx) {
    int n = 0;
    for (int ki = 0; ki < Lk; ++ki) {
        if (c->causal && qi < ki) continue;
        idx[n++] = ki;
    }
    return n;
}

static void bwd_widen(const OracleBwdCtx *c, const uint16_t *t, size_t off, int D, double *dst) {
    for (int d = 0; d < D; ++d) dst[d] = oracle_decode16(t[off + d], c->dtype);
}

static void *bwd_worker(void *arg) {
    OracleBwdCtx *c = (OracleBwdCtx *)arg;
    const int D = c->D, H = c->H, Hkv = c->Hkv, G = c->H / c->Hkv;
    int mk = 0;
    for (int b = 0; b < c->B; ++b)
        if (c->cu_k[b + 1] - c->cu_k[b] > mk) mk = c->cu_k[b + 1] - c->cu_k[b];
    const size_t nk = (size_t)(mk > 0 ? mk : 1);
    double *kd = (double *)malloc(nk * D * sizeof(double));
    double *vd = (double *)malloc(nk * D * sizeof(double));
    double *p = (double *)malloc(nk * sizeof(double));
    double *dp = (double *)malloc(nk * sizeof(double));
    double *ds = (double *)malloc(nk * sizeof(double));
    int *idx = (int *)malloc(nk * sizeof(int));
    double *qd = (double *)malloc((size_t)D * sizeof(double));
    double *dod = (double *)malloc((size_t)D * sizeof(double));
    if (!kd || !vd || !p || !dp || !ds || !idx || !qd || !dod) {
        __atomic_store_n(&c->status, -1, __ATOMIC_RELAXED);
        free(kd); free(vd); free(p); free(dp); free(ds); free(idx); free(qd); free(dod);
        return NULL;
    }
    for (;;) {
        int64_t item = __atomic_fetch_add(&c->next_item, 1, __ATOMIC_RELAXED);
        if (item >= c->n_items) break;
        int b = (int)(item / Hkv), kv_h = (int)(item % Hkv);
        int q0 = c->cu_q[b], Lq = c->cu_q[b + 1] - c->cu_q[b];
        int k0 = c->cu_k[b], Lk = c->cu_k[b + 1] - c->cu_k[b];
        for (int ki = 0; ki < Lk; ++ki) {
            size_t koff = ((size_t)(k0 + ki) * Hkv + kv_h) * D;
            bwd_widen(c, c->k, koff, D, kd + (size_t)ki * D);
            bwd_widen(c, c->v, koff, D, vd + (size_t)ki * D);
        }
        for (int h = kv_h * G; h < (kv_h + 1) * G; ++h) {
            for (int qi = 0; qi < Lq; ++qi) {
                const size_t qoff = ((size_t)(q0 + qi) * H + h) * D;
                const double lse = c->lse[(size_t)(q0 + qi) * H + h];
                bwd_widen(c, c->q, qoff, D, qd);
                bwd_widen(c, c->dout, qoff, D, dod);
                const double delta = dot_d(dod, c->o + qoff, D);
                const int n = bwd_visible_keys(c, qi, Lk, idx);
                /* the row's softmax weights, dP and dS over its visible keys */
                for (int i = 0; i < n; ++i) {
                    const double *krow = kd + (size_t)idx[i] * D;
                    const double *vrow = vd + (size_t)idx[i] * D;
                    p[i] = exp(c->scale * dot_d(qd, krow, D) - lse);
                    dp[i] = dot_d(dod, vrow, D);
                }
                for (int i = 0; i < n; ++i) ds[i] = p[i] * (dp[i] - delta);
                /* dQ of the row: one weighted sum of key rows */
                for (int d = 0; d < D; ++d) {
                    double acc = 0.0;
                    for (int i = 0; i < n; ++i) acc += ds[i] * kd[(size_t)idx[i] * D + d];
                    c->dq[qoff + d] = c->scale * acc;
                }
                /* the row's contributions to dK and dV of its visible keys */
                for (int i = 0; i < n; ++i) {
                    double *dk_row = c->dk + ((size_t)(k0 + idx[i]) * Hkv + kv_h) * D;
                    double *dv_row = c->dv + ((size_t)(k0 + idx[i]) * Hkv + kv_h) * D;
                    for (int d = 0; d < D; ++d) {
                        dk_row[d] += c->scale * ds[i] * qd[d];
                        dv_row[d] += p[i] * dod[d];
                    }
                }
            }
        }
    }
    free(kd); free(vd); free(p); free(dp); free(ds); free(idx); free(qd); free(dod);
    return NULL;
}

/* Full backward: writes dq[Tq*H*D], dk[Tk*Hkv*D], dv[Tk*Hkv*D] (zeroed first
 * over the packed extents cu_q[B] / cu_k[B]).  Returns 0 or a negative code. */
int oracle_varlen_attn_bwd(const uint16_t *dout, const uint16_t *q, const uint16_t *k,
                           const uint16_t *v, const double *o, const double *lse, int dtype,
                           const int32_t *cu_q, const int32_t *cu_k, int B, int H, int Hkv,
                           int D, int causal, double scale, double *dq, double *dk, double *dv,
                           int nthreads) {
    int rc = check_args(B, H, Hkv, D, dtype);
    if (rc) return rc;
    OracleBwdCtx c;
    memset(&c, 0, sizeof c);
    c.dout = dout; c.q = q; c.k = k; c.v = v; c.o = o; c.lse = lse; c.dtype = dtype;
    c.cu_q = cu_q; c.cu_k = cu_k;
    c.B = B; c.H = H; c.Hkv = Hkv; c.D = D; c.causal = causal != 0;
    c.scale = effective_scale(scale, D);
    c.dq = dq; c.dk = dk; c.dv = dv;
    if (B > 0) {
        memset(dq, 0, (size_t)cu_q[B] * H * D * sizeof(double));
        memset(dk, 0, (size_t)cu_k[B] * Hkv * D * sizeof(double));
        memset(dv, 0, (size_t)cu_k[B] * Hkv * D * sizeof(double));
    }
    c.n_items = (int64_t)B * Hkv;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t tids[512];
    int started = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&tids[t], NULL, bwd_worker, &c) != 0) break;
        ++started;
    }
    if (started == 0) bwd_worker(&c);
    for (int t = 0; t < started; ++t) pthread_join(tids[t], NULL);
    return c.status;
}
