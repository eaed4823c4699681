/*
 * kda_oracle.c -- fp64 token-by-token oracle for Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE ONLY. This file is the plain, slow, obviously correct
 * CPU definition that the CUDA path is checked against. Only the test suite,
 * the smoke check and the CPU-baseline leg of the benchmark may load it. It
 * shares no code, header, table or helper with the CUDA library, and the CUDA
 * library never calls it.
 *
 * What it computes, per (sequence, head), token by token, in double precision:
 *
 *   g'   = max(g_t, lb)                       per key channel i
 *   S    = Diag(exp g') S                     row i of S decays by exp(g'_i)
 *   w    = S^T k_t                            what the decayed state recalls for k_t
 *   S    = S + beta_t * k_t (v_t - w)^T       delta-rule erase-then-write
 *   o_t  = scale * S^T q_t                    read-out from the UPDATED state
 *
 * i.e. S_t = (I - beta_t k_t k_t^T) Diag(exp g'_t) S_{t-1} + beta_t k_t v_t^T.
 * S is d_k x d_v (rows indexed by key channels).
 *
 * Optionally (kda_oracle_recurrent_ex) the inputs are raw: q_t, k_t are first divided by
 * their L2 norms, and/or g_t holds gate pre-activations a with g = lb * sigmoid(a); and
 * the state after every P tokens of a sequence can be recorded (prefix-cache snapshots).
 *
 * Sources (web pages about the Kimi K3 report):
 *  - "Kimi K3 深度拆解" (chenxutan.com), section 4.2 "线性注意力与 Delta Rule":
 *    the delta-rule update S_t = S_{t-1}(I - b k k^T) + b k v^T, the fixed-size
 *    [d, d_v] state, the per-token write strength beta in (0,1), and the toy
 *    single-head loop (erase, then write, then read from the new state).
 *    The printed formula only type-checks with S as d_v x d_k; with S stored
 *    d_k x d_v (as the toy does) the same map is the left-multiplied form above.
 *  - "Kimi K3 技術報告：三個架構改動" (akiraxclaw.com), section "長度":
 *    KDA extends Gated DeltaNet with channel-wise gating (each key channel
 *    forgets at its own rate), so the decay is Diag(exp g_t) with g_t in R^{d_k}.
 *  - "3 分钟看懂 Kimi K3" (landx.limxdynamics.com), "第一条主线" and Figure 3:
 *    the log decay is bounded below; here that is the clamp g' = max(g, lb).
 *  Reading taken where the pages are silent: the decay acts on the state before
 *  the erase/write (gated delta rule), and o_t uses 1/sqrt(d_k) by default
 *  (the caller passes `scale`).
 *
 * Inputs are read as float32 or as bfloat16 bit patterns and widened exactly
 * to double per token, so a 1M-token run never materialises fp64 copies.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KDA_ORACLE_F32 0
#define KDA_ORACLE_BF16 1

/* Optional input prologue (bit flags). */
#define KDA_ORACLE_QK_L2NORM 1   /* q_t, k_t <- x / max(||x||_2, 1e-12) per (token, head) */
#define KDA_ORACLE_GATE_SIGMOID 2 /* g holds pre-activations a: log decay = lb * sigmoid(a) */

/* Exact widening of one input element to double. */
static double load_elem(const void *base, int dtype, int64_t idx)
{
    if (dtype == KDA_ORACLE_F32) {
        return (double)((const float *)base)[idx];
    }
    /* bfloat16: the upper 16 bits of an IEEE float32. */
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[idx]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

typedef struct {
    int64_t T;
    int H, dk, dv, n_seqs;
    const int64_t *cu_seqlens;
    int dtype;
    const void *q, *k, *v, *g, *beta;
    const double *initial_state;
    double lb, scale;
    double *out;
    const int64_t *out_rows;
    int64_t n_out_rows;
    double *final_state;
    int64_t snap_tokens;       /* snapshot interval in tokens (0 = none) */
    const int64_t *snap_first; /* [n_seqs] index of each sequence's first snapshot */
    double *snaps;             /* [n_snaps, H, dk, dv] */
    int prologue;              /* KDA_ORACLE_* prologue flags */
    int64_t next_item; /* shared work counter over (seq, head) */
    pthread_mutex_t lock;
} job_t;

/* First index in the sorted list `rows` whose value is >= t. */
static int64_t lower_bound_rows(const int64_t *rows, int64_t n, int64_t t)
{
    int64_t lo = 0, hi = n;
    while (lo < hi) {
        int64_t mid = lo + (hi - lo) / 2;
        if (rows[mid] < t) lo = mid + 1; else hi = mid;
    }
    return lo;
}

/* One (sequence, head) pair, token by token. */
static void run_one(const job_t *J, int seq, int h, double *S, double *kt,
                    double *qt, double *vt, double *decay, double *w)
{
    const int dk = J->dk, dv = J->dv, H = J->H;
    const int64_t t0 = J->cu_seqlens[seq], t1 = J->cu_seqlens[seq + 1];
    const int64_t state_off = ((int64_t)seq * H + h) * dk * dv;

    if (J->initial_state) {
        memcpy(S, J->initial_state + state_off, sizeof(double) * dk * dv);
    } else {
        memset(S, 0, sizeof(double) * dk * dv);
    }

    int64_t next_out = J->out_rows ? lower_bound_rows(J->out_rows, J->n_out_rows, t0) : 0;

    for (int64_t t = t0; t < t1; ++t) {
        const int64_t tok_k = (t * H + h) * dk;
        const int64_t tok_v = (t * H + h) * dv;
        for (int i = 0; i < dk; ++i) {
            kt[i] = load_elem(J->k, J->dtype, tok_k + i);
            qt[i] = load_elem(J->q, J->dtype, tok_k + i);
            double gi = load_elem(J->g, J->dtype, tok_k + i);
            if (J->prologue & KDA_ORACLE_GATE_SIGMOID)
                gi = J->lb / (1.0 + exp(-gi));       /* lb * sigmoid(a), inside (lb, 0) */
            if (gi < J->lb) gi = J->lb;              /* lower bound on the log decay */
            decay[i] = exp(gi);
        }
        if (J->prologue & KDA_ORACLE_QK_L2NORM) {
            /* unit-length q and k (the delta rule assumes them normalised) */
            double nk = 0.0, nq = 0.0;
            for (int i = 0; i < dk; ++i) {
                nk += kt[i] * kt[i];
                nq += qt[i] * qt[i];
            }
            nk = sqrt(nk);
            nq = sqrt(nq);
            if (nk < 1e-12) nk = 1e-12;
            if (nq < 1e-12) nq = 1e-12;
            for (int i = 0; i < dk; ++i) {
                kt[i] /= nk;
                qt[i] /= nq;
            }
        }
        for (int j = 0; j < dv; ++j) vt[j] = load_elem(J->v, J->dtype, tok_v + j);
        const double b = load_elem(J->beta, J->dtype, t * H + h);

        /* S <- Diag(exp g') S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] *= decay[i];

        /* w = S^T k */
        for (int j = 0; j < dv; ++j) w[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) w[j] += kt[i] * S[i * dv + j];

        /* S <- S + beta k (v - w)^T */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] += b * kt[i] * (vt[j] - w[j]);

        /* o = scale * S^T q, written only where an output row is wanted */
        int64_t out_row = -1;
        if (J->out) {
            if (!J->out_rows) {
                out_row = t;
            } else if (next_out < J->n_out_rows && J->out_rows[next_out] == t) {
                out_row = next_out++;
            }
        }
        if (out_row >= 0) {
            double *o = J->out + (out_row * H + h) * dv;
            for (int j = 0; j < dv; ++j) o[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) o[j] += qt[i] * S[i * dv + j];
            for (int j = 0; j < dv; ++j) o[j] *= J->scale;
        }

        /* the state after the first m * snap_tokens tokens of the sequence */
        if (J->snaps && (t - t0 + 1) % J->snap_tokens == 0) {
            const int64_t idx = J->snap_first[seq] + (t - t0 + 1) / J->snap_tokens - 1;
            memcpy(J->snaps + (idx * H + h) * dk * dv, S, sizeof(double) * dk * dv);
        }
    }

    if (J->final_state) memcpy(J->final_state + state_off, S, sizeof(double) * dk * dv);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    const int dk = J->dk, dv = J->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *buf = (double *)malloc(sizeof(double) * (size_t)(3 * dk + 2 * dv));
    if (!S || !buf) {
        free(S);
        free(buf);
        return (void *)1;
    }
    double *kt = buf, *qt = buf + dk, *decay = buf + 2 * dk, *vt = buf + 3 * dk, *w = vt + dv;
    const int64_t n_items = (int64_t)J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t item = J->next_item++;
        pthread_mutex_unlock(&J->lock);
        if (item >= n_items) break;
        run_one(J, (int)(item / J->H), (int)(item % J->H), S, kt, qt, vt, decay, w);
    }
    free(S);
    free(buf);
    return NULL;
}

/*
 * Token-by-token fp64 recurrence over packed sequences.
 *
 *  q, k, g : [T, H, dk]   v : [T, H, dv]   beta : [T, H]   (dtype f32 or bf16 bits)
 *  cu_seqlens : [n_seqs + 1], cu_seqlens[0] = 0, non-decreasing, last = T
 *  initial_state / final_state : [n_seqs, H, dk, dv] fp64 (initial NULL = zeros)
 *  out : [T, H, dv] fp64, or [n_out_rows, H, dv] when out_rows (sorted token
 *        indices) is given; NULL skips the read-out.
 *  Returns 0 on success, -1 on a bad argument, -2 when a thread failed.
 */
static int run_all(int64_t T, int H, int dk, int dv, int n_seqs,
                   const int64_t *cu_seqlens, int dtype,
                   const void *q, const void *k, const void *v,
                   const void *g, const void *beta,
                   const double *initial_state, double lb, double scale,
                   double *out, const int64_t *out_rows, int64_t n_out_rows,
                   double *final_state, int64_t snap_tokens, const int64_t *snap_first,
                   double *snaps, int prologue, int n_threads)
{
    if (T < 0 || H <= 0 || dk <= 0 || dv <= 0 || n_seqs <= 0 || !cu_seqlens) return -1;
    if (dtype != KDA_ORACLE_F32 && dtype != KDA_ORACLE_BF16) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return -1;
    for (int s = 0; s < n_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    if (T > 0 && (!q || !k || !v || !g || !beta)) return -1;
    if (prologue & ~(KDA_ORACLE_QK_L2NORM | KDA_ORACLE_GATE_SIGMOID)) return -1;
    if (snap_tokens < 0 || (snap_tokens > 0 && (!snap_first || !snaps))) return -1;
    if (snap_tokens == 0) snaps = NULL;

    job_t J;
    memset(&J, 0, sizeof J);
    J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.n_seqs = n_seqs;
    J.cu_seqlens = cu_seqlens; J.dtype = dtype;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta;
    J.initial_state = initial_state; J.lb = lb; J.scale = scale;
    J.out = out; J.out_rows = out_rows; J.n_out_rows = n_out_rows;
    J.final_state = final_state;
    J.snap_tokens = snap_tokens; J.snap_first = snap_first; J.snaps = snaps;
    J.prologue = prologue;
    pthread_mutex_init(&J.lock, NULL);

    const int64_t n_items = (int64_t)n_seqs * H;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_items) n_threads = (int)n_items;

    int rc = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) {
        pthread_mutex_destroy(&J.lock);
        return -2;
    }
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) rc = -2;
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret != NULL) rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}

int kda_oracle_recurrent(int64_t T, int H, int dk, int dv, int n_seqs,
                         const int64_t *cu_seqlens, int dtype,
                         const void *q, const void *k, const void *v,
                         const void *g, const void *beta,
                         const double *initial_state, double lb, double scale,
                         double *out, const int64_t *out_rows, int64_t n_out_rows,
                         double *final_state, int n_threads)
{
    return run_all(T, H, dk, dv, n_seqs, cu_seqlens, dtype, q, k, v, g, beta, initial_state,
                   lb, scale, out, out_rows, n_out_rows, final_state, 0, NULL, NULL, 0,
                   n_threads);
}

/*
 * The general form: kda_oracle_recurrent with optional snapshots and an optional input
 * prologue.
 *  Snapshots (snap_tokens > 0; 0 = none): for every m >= 1 with m * snap_tokens <=
 *  len(seq), the state after the sequence's first m * snap_tokens tokens (seeded by its
 *  initial state) is copied to snaps[snap_first[seq] + m - 1] ([.., H, dk, dv] fp64).
 *  The caller sizes snaps and chooses snap_first so that the sequences' ranges do not
 *  overlap. A prefix cache keeps exactly these states ("3 分钟看懂 Kimi K3", 第一条主线:
 *  KDA state and prefix-cache scheduling for long requests).
 *  Prologue flags:
 *  KDA_ORACLE_QK_L2NORM    q_t and k_t are divided by max(||.||_2, 1e-12) per (token,
 *                          head) before use ("Kimi K3 深度拆解", section 4.2: the delta
 *                          rule takes L2-normalised q and k);
 *  KDA_ORACLE_GATE_SIGMOID g holds gate pre-activations a and the log decay is
 *                          lb * sigmoid(a), which lies inside (lb, 0) ("3 分钟看懂 Kimi K3",
 *                          第一条主线 / Figure 3: the log decay is bounded below).
 */
int kda_oracle_recurrent_ex(int64_t T, int H, int dk, int dv, int n_seqs,
                            const int64_t *cu_seqlens, int dtype,
                            const void *q, const void *k, const void *v,
                            const void *g, const void *beta,
                            const double *initial_state, double lb, double scale,
                            double *out, const int64_t *out_rows, int64_t n_out_rows,
                            double *final_state, int64_t snap_tokens,
                            const int64_t *snap_first, double *snaps, int prologue,
                            int n_threads)
{
    return run_all(T, H, dk, dv, n_seqs, cu_seqlens, dtype, q, k, v, g, beta, initial_state,
                   lb, scale, out, out_rows, n_out_rows, final_state, snap_tokens, snap_first,
                   snaps, prologue, n_threads);
}

/* ======================================================================== backward
 * Reverse-mode gradient of the token recurrence above (no prologue), in fp64.
 * Given upstream gradients dO = dL/do_t [T, H, dv] and dS_T = dL/dS_final [n, H, dk, dv]
 * (NULL = 0) of some scalar L, returns dL/dq, dL/dk, dL/dg, dL/dbeta, dL/dv and
 * dL/dS0. It differentiates, step by step in reverse, exactly the forward loop:
 *
 *   Sb = Diag(exp g') S_prev     w = Sb^T k     u = beta (v - w)
 *   S  = Sb + k u^T              o = scale S^T q
 *
 * so, with dS the gradient of S_t accumulated from later tokens:
 *   dS += scale q do^T;  dq = scale S do;  dk = dS u;  du = dS^T k;
 *   dbeta = du . (v - w);  dv = beta du;  dw = -beta du;
 *   dSb = dS + k dw^T;  dk += Sb dw;  dg'_i = sum_j Sb_ij dSb_ij;
 *   dg_i = dg'_i where g_i >= lb (the clamp passes the gradient), else 0;
 *   dS_prev = Diag(exp g') dSb.
 * The states S_{t-1} are recomputed per block of 64 tokens from checkpoints taken in
 * a forward sweep. Training needs this gradient ("Kimi K3 深度拆解", section 4.2
 * describes the chunk-parallel kernels the model is trained with).
 */
typedef struct {
    int64_t T;
    int H, dk, dv, n_seqs;
    const int64_t *cu_seqlens;
    int dtype;
    const void *q, *k, *v, *g, *beta;
    const double *initial_state, *d_out, *d_final;
    double lb, scale;
    double *dq, *dkk, *dvv, *dg, *dbeta, *ds0;
    int prologue;      /* KDA_ORACLE_* prologue flags: raw inputs, chain rule through them */
    int64_t next_item;
    pthread_mutex_t lock;
} bjob_t;

#define KDA_ORACLE_BWD_BLOCK 64

/* Inputs of token t (head h) as the recurrence uses them: k, q (unit length with the
 * L2 prologue; their norms in *nk, *nq), v, beta, the log decay before the clamp (the gate's
 * output with the gate prologue; sig = sigmoid(a) then) and the clamped decay. */
static void load_token(const bjob_t *J, int64_t t, int h, double *kt, double *qt, double *vt,
                       double *decay, double *graw, double *b, double *nk, double *nq,
                       double *sig)
{
    const int dk = J->dk, dv = J->dv, H = J->H;
    const int64_t tok_k = (t * H + h) * dk, tok_v = (t * H + h) * dv;
    for (int i = 0; i < dk; ++i) {
        kt[i] = load_elem(J->k, J->dtype, tok_k + i);
        qt[i] = load_elem(J->q, J->dtype, tok_k + i);
        graw[i] = load_elem(J->g, J->dtype, tok_k + i);
        if (J->prologue & KDA_ORACLE_GATE_SIGMOID) {
            sig[i] = 1.0 / (1.0 + exp(-graw[i]));
            graw[i] = J->lb * sig[i];
        }
        decay[i] = exp(graw[i] < J->lb ? J->lb : graw[i]);
    }
    *nk = *nq = 1.0;
    if (J->prologue & KDA_ORACLE_QK_L2NORM) {
        double a = 0.0, c = 0.0;
        for (int i = 0; i < dk; ++i) {
            a += kt[i] * kt[i];
            c += qt[i] * qt[i];
        }
        *nk = sqrt(a) < 1e-12 ? 1e-12 : sqrt(a);
        *nq = sqrt(c) < 1e-12 ? 1e-12 : sqrt(c);
        for (int i = 0; i < dk; ++i) {
            kt[i] /= *nk;
            qt[i] /= *nq;
        }
    }
    for (int j = 0; j < dv; ++j) vt[j] = load_elem(J->v, J->dtype, tok_v + j);
    *b = load_elem(J->beta, J->dtype, t * H + h);
}

/* One forward token step in place: S <- (I - b k k^T) Diag(decay) S + b k v^T. */
static void step_state(double *S, int dk, int dv, const double *kt, const double *vt,
                       const double *decay, double b, double *w)
{
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] *= decay[i];
    for (int j = 0; j < dv; ++j) w[j] = 0.0;
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) w[j] += kt[i] * S[i * dv + j];
    for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) S[i * dv + j] += b * kt[i] * (vt[j] - w[j]);
}

static int bwd_one(const bjob_t *J, int seq, int h)
{
    const int dk = J->dk, dv = J->dv, H = J->H, B = KDA_ORACLE_BWD_BLOCK;
    const int64_t t0 = J->cu_seqlens[seq], t1 = J->cu_seqlens[seq + 1];
    const int64_t nb = (t1 - t0 + B - 1) / B;
    const size_t st = (size_t)dk * dv;
    const int64_t state_off = ((int64_t)seq * H + h) * dk * dv;
    double *ckpt = (double *)malloc(sizeof(double) * st * (size_t)(nb > 0 ? nb : 1));
    double *pre = (double *)malloc(sizeof(double) * st * (size_t)B); /* S_{t-1} per token */
    double *S = (double *)malloc(sizeof(double) * st);
    double *Sb = (double *)malloc(sizeof(double) * st);
    double *dS = (double *)malloc(sizeof(double) * st);
    double *buf = (double *)malloc(sizeof(double) * (size_t)(6 * dk + 6 * dv));
    if (!ckpt || !pre || !S || !Sb || !dS || !buf) {
        free(ckpt); free(pre); free(S); free(Sb); free(dS); free(buf);
        return 1;
    }
    double *kt = buf, *qt = kt + dk, *decay = qt + dk, *graw = decay + dk, *dgp = graw + dk;
    double *sig = dgp + dk;
    double *vt = sig + dk, *w = vt + dv, *u = w + dv, *du = u + dv, *dw = du + dv, *dov = dw + dv;
    double b, nk, nq;

    /* forward sweep: the state at the start of every block */
    if (J->initial_state) memcpy(S, J->initial_state + state_off, sizeof(double) * st);
    else memset(S, 0, sizeof(double) * st);
    for (int64_t blk = 0; blk < nb; ++blk) {
        memcpy(ckpt + (size_t)blk * st, S, sizeof(double) * st);
        const int64_t e = t0 + (blk + 1) * B < t1 ? t0 + (blk + 1) * B : t1;
        for (int64_t t = t0 + blk * B; t < e; ++t) {
            load_token(J, t, h, kt, qt, vt, decay, graw, &b, &nk, &nq, sig);
            step_state(S, dk, dv, kt, vt, decay, b, w);
        }
    }

    if (J->d_final) memcpy(dS, J->d_final + state_off, sizeof(double) * st);
    else memset(dS, 0, sizeof(double) * st);
    for (int64_t blk = nb - 1; blk >= 0; --blk) {
        const int64_t s = t0 + blk * B, e = s + B < t1 ? s + B : t1;
        memcpy(S, ckpt + (size_t)blk * st, sizeof(double) * st);
        for (int64_t t = s; t < e; ++t) {
            memcpy(pre + (size_t)(t - s) * st, S, sizeof(double) * st);
            load_token(J, t, h, kt, qt, vt, decay, graw, &b, &nk, &nq, sig);
            step_state(S, dk, dv, kt, vt, decay, b, w);
        }
        for (int64_t t = e - 1; t >= s; --t) {
            load_token(J, t, h, kt, qt, vt, decay, graw, &b, &nk, &nq, sig);
            const double *Sp = pre + (size_t)(t - s) * st;
            /* recompute the step: Sb, w, u and S_t (in S) */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) Sb[i * dv + j] = decay[i] * Sp[i * dv + j];
            for (int j = 0; j < dv; ++j) w[j] = 0.0;
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) w[j] += kt[i] * Sb[i * dv + j];
            for (int j = 0; j < dv; ++j) u[j] = b * (vt[j] - w[j]);
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) S[i * dv + j] = Sb[i * dv + j] + kt[i] * u[j];

            const int64_t tk = (t * H + h) * dk, tv = (t * H + h) * dv;
            for (int j = 0; j < dv; ++j) dov[j] = J->d_out ? J->d_out[tv + j] : 0.0;
            /* o = scale S^T q */
            for (int i = 0; i < dk; ++i)
                for (int j = 0; j < dv; ++j) dS[i * dv + j] += J->scale * qt[i] * dov[j];
            for (int i = 0; i < dk; ++i) {
                double a = 0.0;
                for (int j = 0; j < dv; ++j) a += S[i * dv + j] * dov[j];
                J->dq[tk + i] = J->scale * a;
            }
            /* S = Sb + k u^T */
            for (int j = 0; j < dv; ++j) du[j] = 0.0;
            for (int i = 0; i < dk; ++i) {
                double a = 0.0;
                for (int j = 0; j < dv; ++j) {
                    a += dS[i * dv + j] * u[j];
                    du[j] += dS[i * dv + j] * kt[i];
                }
                J->dkk[tk + i] = a;
            }
            /* u = beta (v - w) */
            double db = 0.0;
            for (int j = 0; j < dv; ++j) {
                db += du[j] * (vt[j] - w[j]);
                J->dvv[tv + j] = b * du[j];
                dw[j] = -b * du[j];
            }
            J->dbeta[t * H + h] = db;
            /* w = Sb^T k: dSb = dS + k dw^T, dk += Sb dw */
            for (int i = 0; i < dk; ++i) {
                double a = 0.0;
                for (int j = 0; j < dv; ++j) {
                    dS[i * dv + j] += kt[i] * dw[j];
                    a += Sb[i * dv + j] * dw[j];
                }
                J->dkk[tk + i] += a;
            }
            /* Sb = Diag(exp g') S_prev */
            for (int i = 0; i < dk; ++i) {
                double a = 0.0;
                for (int j = 0; j < dv; ++j) a += Sb[i * dv + j] * dS[i * dv + j];
                dgp[i] = a;
                J->dg[tk + i] = graw[i] >= J->lb ? dgp[i] : 0.0;
                for (int j = 0; j < dv; ++j) dS[i * dv + j] *= decay[i];
            }
            /* through the prologue, to the raw inputs */
            if (J->prologue & KDA_ORACLE_GATE_SIGMOID)
                for (int i = 0; i < dk; ++i) J->dg[tk + i] *= J->lb * sig[i] * (1.0 - sig[i]);
            if (J->prologue & KDA_ORACLE_QK_L2NORM) {
                /* x = r / max(|r|, eps): dr = (dx - x (x . dx)) / |r| above eps, dx / eps below */
                double pk = 0.0, pq = 0.0;
                for (int i = 0; i < dk; ++i) {
                    pk += kt[i] * J->dkk[tk + i];
                    pq += qt[i] * J->dq[tk + i];
                }
                if (nk <= 1e-12) pk = 0.0;
                if (nq <= 1e-12) pq = 0.0;
                for (int i = 0; i < dk; ++i) {
                    J->dkk[tk + i] = (J->dkk[tk + i] - kt[i] * pk) / nk;
                    J->dq[tk + i] = (J->dq[tk + i] - qt[i] * pq) / nq;
                }
            }
        }
    }
    if (J->ds0) memcpy(J->ds0 + state_off, dS, sizeof(double) * st);
    free(ckpt); free(pre); free(S); free(Sb); free(dS); free(buf);
    return 0;
}

static void *bwd_worker(void *arg)
{
    bjob_t *J = (bjob_t *)arg;
    const int64_t n_items = (int64_t)J->n_seqs * J->H;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int64_t item = J->next_item++;
        pthread_mutex_unlock(&J->lock);
        if (item >= n_items) break;
        if (bwd_one(J, (int)(item / J->H), (int)(item % J->H)) != 0) return (void *)1;
    }
    return NULL;
}

/*
 * Gradients of the recurrence (see the block comment above). Layouts as in the forward;
 * d_out [T, H, dv] fp64 (NULL = 0), d_final [n_seqs, H, dk, dv] fp64 (NULL = 0); outputs
 * dq, dk, dg [T, H, dk], dv [T, H, dv], dbeta [T, H], ds0 [n_seqs, H, dk, dv] (NULL to
 * skip), all fp64. With prologue flags the inputs are raw (as in kda_oracle_recurrent_ex)
 * and the gradients are those of the raw q, k and gate pre-activations.
 * Returns 0, -1 on a bad argument, -2 when a thread failed.
 */
int kda_oracle_backward(int64_t T, int H, int dk, int dv, int n_seqs,
                        const int64_t *cu_seqlens, int dtype,
                        const void *q, const void *k, const void *v,
                        const void *g, const void *beta,
                        const double *initial_state, double lb, double scale,
                        const double *d_out, const double *d_final,
                        double *dq, double *dkk, double *dvv, double *dg, double *dbeta,
                        double *ds0, int prologue, int n_threads)
{
    if (T < 0 || H <= 0 || dk <= 0 || dv <= 0 || n_seqs <= 0 || !cu_seqlens) return -1;
    if (dtype != KDA_ORACLE_F32 && dtype != KDA_ORACLE_BF16) return -1;
    if (cu_seqlens[0] != 0 || cu_seqlens[n_seqs] != T) return -1;
    for (int s = 0; s < n_seqs; ++s)
        if (cu_seqlens[s + 1] < cu_seqlens[s]) return -1;
    if (T > 0 && (!q || !k || !v || !g || !beta || !dq || !dkk || !dvv || !dg || !dbeta))
        return -1;
    if (prologue & ~(KDA_ORACLE_QK_L2NORM | KDA_ORACLE_GATE_SIGMOID)) return -1;

    bjob_t J;
    memset(&J, 0, sizeof J);
    J.T = T; J.H = H; J.dk = dk; J.dv = dv; J.n_seqs = n_seqs;
    J.cu_seqlens = cu_seqlens; J.dtype = dtype;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta;
    J.initial_state = initial_state; J.d_out = d_out; J.d_final = d_final;
    J.lb = lb; J.scale = scale;
    J.dq = dq; J.dkk = dkk; J.dvv = dvv; J.dg = dg; J.dbeta = dbeta; J.ds0 = ds0;
    J.prologue = prologue;
    pthread_mutex_init(&J.lock, NULL);

    const int64_t n_items = (int64_t)n_seqs * H;
    if (n_threads < 1) n_threads = 1;
    if (n_threads > n_items) n_threads = (int)n_items;
    int rc = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    if (!th) {
        pthread_mutex_destroy(&J.lock);
        return -2;
    }
    int started = 0;
    for (int i = 0; i < n_threads; ++i) {
        if (pthread_create(&th[i], NULL, bwd_worker, &J) != 0) break;
        ++started;
    }
    if (started == 0) rc = -2;
    for (int i = 0; i < started; ++i) {
        void *ret = NULL;
        pthread_join(th[i], &ret);
        if (ret != NULL) rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&J.lock);
    return rc;
}
