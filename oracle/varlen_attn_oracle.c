/*
 * fp64 CPU oracle for the variable-length (packed, ragged) attention forward.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the package's smoke check and the bench's
 * CPU-baseline leg use it.  It shares no code with the CUDA library.
 *
 * What it computes follows the CPU forward loop of boostr 0.2.0,
 * src/ops/cpu/attention/varlen_attention.rs (VarLenAttentionOps::
 * varlen_attention_fwd), step for step, with every f32 replaced by double:
 *
 *   for each sequence b, query head h, query qi in [0, Lq_b):
 *     kv_h = h / (H / Hkv)                           (GQA head map)
 *     for each key ki in [0, Lk_b):
 *       masked when causal and qi < ki                (sequence-local indices)
 *       s_ki = (sum_d Q[cu_q[b]+qi, h, d] * K[cu_k[b]+ki, kv_h, d]) * scale
 *     m = max of the unmasked s_ki
 *     e_ki = exp(s_ki - m)        (masked keys give exp(-inf) = 0)
 *     l = sum of e_ki
 *     O[cu_q[b]+qi, h, :] = sum_ki (e_ki / l) * V[cu_k[b]+ki, kv_h, :]
 *     LSE[cu_q[b]+qi, h]  = m + ln(l)
 *
 * Layouts are the page's packed ones: Q/O [Tq, H, D], K/V [Tk, Hkv, D],
 * LSE [Tq, H], all row-major.  The scale is an explicit argument; a value
 * <= 0 or NaN selects the page's default 1/sqrt(D).
 *
 * Extension (the `_ext` entry points): the sliding window and used-key count
 * that PyTorch pull request #176015 lists in the varlen forward schema
 * (window_size_left, window_size_right, seqused_k), read with the page's
 * sequence-local indices: key ki is also hidden when ki >= seqused_k[b]
 * (clipped to [0, Lk_b]), when left >= 0 and ki < qi - left, or when
 * right >= 0 and ki > qi + right.  A row with no visible key gets O = 0 and
 * LSE = -inf, what the page's loop gives for a sequence without keys.
 *
 * Attention sinks (the `sinks` argument of the `_ext` entry points; the
 * FLOAT32 per-head "sinks" input of the Ascend sparse shared-KV attention
 * page, which gives no formula): sinks[h] is one more logit, already in score
 * units (not multiplied by the scale), that joins the softmax of every row of
 * query head h but has no value row.  So m = max(max_ki s_ki, sinks[h]),
 * l = sum_ki exp(s_ki - m) + exp(sinks[h] - m), O = sum_ki exp(s_ki - m) / l
 * * V_ki, LSE = m + ln(l); a row without visible keys then gets O = 0 and
 * LSE = sinks[h].
 *
 * Backward (oracle_varlen_attn_bwd): the CPU backward loop of the same page
 * (VarLenAttentionOps::varlen_attention_bwd), step for step in double
 * precision.  Given dO, Q, K, V, the forward output O and LSE:
 *
 *   for each sequence b, query head h (kv_h = h / (H / Hkv)), query qi:
 *     delta = sum_d dO[qi, h, d] * O[qi, h, d]
 *     for each visible key ki (causal: skip qi < ki):
 *       s  = scale * <Q[qi, h], K[ki, kv_h]>
 *       p  = exp(s - LSE[qi, h])                 (the softmax weight)
 *       dp = <V[ki, kv_h], dO[qi, h]>
 *       ds = p * (dp - delta)
 *       dQ[qi, h]     += scale * ds * K[ki, kv_h]
 *       dK[ki, kv_h]  += scale * ds * Q[qi, h]
 *       dV[ki, kv_h]  += p * dO[qi, h]
 *
 * dK and dV sum over the H / Hkv query heads of their key/value head.  The
 * scale is the page's 1/sqrt(D) unless given (as in the forward).  dO is
 * 16-bit like Q/K/V; O and LSE are given in double (the caller widens the
 * stored bf16/fp16 O and float32 LSE exactly, or passes exact values).  Work items are (b, kv_h): each owns the dK/dV rows
 * of that key/value head of sequence b and the dQ rows of its query heads,
 * and runs the loop above serially, so the result does not depend on the
 * thread count.
 *
 * Inputs are bf16 or fp16 bit patterns; they are widened exactly to double
 * before any arithmetic.  The widening of a key/value head of one sequence
 * is done once per (b, h) work item; that is a format conversion, not a
 * change to the order of the attention arithmetic.
 *
 * Work items (b, h) are spread over POSIX threads; each output row is
 * computed by one thread with the serial loop above, so the result does not
 * depend on the thread count.
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

/* One query row: the page's two-pass softmax, in double precision.
 * kd/vd hold the widened keys/values of head kv_h of sequence b, [Lk][D]. */
static void oracle_attend_row(const OracleCtx *c, const double *qrow, int qi, int Lk,
                              const double *kd, const double *vd, double *scores, double sink,
                              double *out_row, double *lse_out) {
    const int D = c->D;
    double max_score = -INFINITY;
    for (int ki = 0; ki < Lk; ++ki) {
        if (key_hidden(c, qi, ki)) {
            scores[ki] = -INFINITY;
            continue;
        }
        double dot = 0.0;
        const double *krow = kd + (size_t)ki * D;
        for (int d = 0; d < D; ++d) dot += qrow[d] * krow[d];
        double s = dot * c->scale;
        if (s > max_score) max_score = s;
        scores[ki] = s;
    }
    if (sink > max_score) max_score = sink; /* the sink logit takes part in the max */
    if (max_score == -INFINITY) { /* no visible key and no sink */
        for (int d = 0; d < D; ++d) out_row[d] = 0.0;
        *lse_out = -INFINITY;
        return;
    }
    double sum_exp = 0.0;
    for (int ki = 0; ki < Lk; ++ki) {
        double e = exp(scores[ki] - max_score);
        sum_exp += e;
        scores[ki] = e;
    }
    sum_exp += exp(sink - max_score); /* ... and in the normalisation (0 without a sink) */
    for (int d = 0; d < D; ++d) out_row[d] = 0.0;
    for (int ki = 0; ki < Lk; ++ki) {
        double weight = scores[ki] / sum_exp;
        const double *vrow = vd + (size_t)ki * D;
        for (int d = 0; d < D; ++d) out_row[d] += weight * vrow[d];
    }
    *lse_out = max_score + log(sum_exp);
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
    double *qd = (double *)malloc((size_t)D * sizeof(double));
    if (!kd || !vd || !scores || !qd) {
        __atomic_store_n(&c->status, -1, __ATOMIC_RELAXED);
        free(kd); free(vd); free(scores); free(qd);
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
            oracle_attend_row(c, qd, qi, Lk, kd, vd, scores, head_sink(c, h),
                              c->out + ((size_t)tok * H + h) * D,
                              c->lse + (size_t)tok * H + h);
        }
    }
    free(kd); free(vd); free(scores); free(qd);
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
    double *qd = (double *)malloc((size_t)D * sizeof(double));
    int cached_b = -1, cached_kvh = -1;
    if (!kd || !vd || !scores || !qd) {
        __atomic_store_n(&c->status, -1, __ATOMIC_RELAXED);
        free(kd); free(vd); free(scores); free(qd);
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
        oracle_attend_row(c, qd, qi, Lk, kd, vd, scores, head_sink(c, h),
                          c->out_rows + (size_t)i * D, c->lse_rows + i);
    }
    free(kd); free(vd); free(scores); free(qd);
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

static double bwd_elem(const OracleBwdCtx *c, const uint16_t *t, size_t off) {
    return oracle_decode16(t[off], c->dtype);
}

static void *bwd_worker(void *arg) {
    OracleBwdCtx *c = (OracleBwdCtx *)arg;
    const int D = c->D, H = c->H, Hkv = c->Hkv, G = c->H / c->Hkv;
    for (;;) {
        int64_t item = __atomic_fetch_add(&c->next_item, 1, __ATOMIC_RELAXED);
        if (item >= c->n_items) break;
        int b = (int)(item / Hkv), kv_h = (int)(item % Hkv);
        int q0 = c->cu_q[b], Lq = c->cu_q[b + 1] - c->cu_q[b];
        int k0 = c->cu_k[b], Lk = c->cu_k[b + 1] - c->cu_k[b];
        for (int h = kv_h * G; h < (kv_h + 1) * G; ++h) {
            for (int qi = 0; qi < Lq; ++qi) {
                size_t qoff = ((size_t)(q0 + qi) * H + h) * D;
                double lse = c->lse[(size_t)(q0 + qi) * H + h];
                double delta = 0.0;
                for (int d = 0; d < D; ++d)
                    delta += bwd_elem(c, c->dout, qoff + d) * c->o[qoff + d];
                for (int ki = 0; ki < Lk; ++ki) {
                    if (c->causal && qi < ki) continue;
                    size_t koff = ((size_t)(k0 + ki) * Hkv + kv_h) * D;
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += bwd_elem(c, c->q, qoff + d) * bwd_elem(c, c->k, koff + d);
                    double prob = exp(dot * c->scale - lse);
                    double dp = 0.0;
                    for (int d = 0; d < D; ++d)
                        dp += bwd_elem(c, c->v, koff + d) * bwd_elem(c, c->dout, qoff + d);
                    double ds = prob * (dp - delta);
                    for (int d = 0; d < D; ++d) {
                        c->dq[qoff + d] += c->scale * ds * bwd_elem(c, c->k, koff + d);
                        c->dk[koff + d] += c->scale * ds * bwd_elem(c, c->q, qoff + d);
                        c->dv[koff + d] += prob * bwd_elem(c, c->dout, qoff + d);
                    }
                }
            }
        }
    }
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
