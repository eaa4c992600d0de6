/*
 * ua_oracle.c -- plain, slow, fp64 CPU oracle for Universal Attention (UA).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline leg do.
 * It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (the pages describe the structure; they print no equations):
 *   [S1] "A Self-Pruning Transformer: Extreme KV-Cache Compression with Universal
 *        Attention", paperlayer.ai source-linked summary: §3 (causal softmax attention,
 *        FoX additive forget gate), §4 and §4.1 (three decay mechanisms combined by a
 *        geometric mean), §4.2 (threshold-p eviction with a monotone per-pair bias),
 *        App. C (decay applied inside the online softmax).
 *   [S3] "Universal Attention composes decay gates for over 10x KV-cache compression
 *        and beats unpruned Llama3 on RULER", ai4snews synopsis: Fig. 1 caption
 *        (L2-normalised keys, low-rank sigmoid output gate, geometric mean ->
 *        log space -> causal accumulation into Lambda), the veto property, and the
 *        eviction paragraph (scalar bias per key/value pair, evicted entries never return).
 *
 * Parameterisation adopted by this library (the pages fix structure only):
 *   khat_j   = k_j / max(||k_j||, 1e-12)
 *   r_q(l)   = softplus(a_q[l]),  r_k(j) = softplus(a_k[j])
 *   r_sim(l,j) = softplus(alpha * <khat_l, khat_j> + beta)          (pre-RoPE keys)
 *   D[l,j]   = cbrt(r_q(l) * r_k(j) * r_sim(l,j))                   (geometric mean)
 *   Lambda_ij = -sum_{l=j+1..i} D[l,j]   (i >= j; Lambda_ii = 0)
 *   O_i = softmax_j<=i( scale * RoPE(q_i).RoPE(khat_j) + Lambda_ij ) V  (.) sigmoid(g_i)
 *   RoPE: rotate-half pairs (m, m+d/2), frequency theta^(-2m/d), position = token index.
 * Everything is computed in fp64 from the (already rounded) inputs, directly from
 * these definitions, with no blocking, fusion or reordering.
 *
 * Layouts (row-major, innermost last):
 *   q, g, o, do : [B, T, H, d]      k, v : [B, T, Hkv, d]
 *   a_q, a_k    : [B, T, Hkv]       alpha, beta : [Hkv]
 *   lse         : [B, H, T]         b_final : [B, Hkv, T]     lambda : [B, Hkv, T, T]
 * Query head h reads KV head h / (H / Hkv); decay parameters belong to the KV head.
 *
 * Variants (the ablations of [S1] §5.4 with Table 3 and App. E with Table 6; [S3]
 * interpretation paragraph), selected by a `variant` bit field, 0 = the method above:
 *   bit 0 / 1 / 2 set: the query / key / similarity mechanism is switched off, and D is
 *     the geometric mean of the rates left on: (prod of the n active rates)^(1/n).
 *     All three off is rejected.
 *   bit 3 set: queries are RMS-normalised per head before RoPE (Qwen3-style query norm,
 *     unit gain): q' = q / sqrt(mean(q^2) + 1e-6).  Keys keep their L2 normalisation.
 *
 * Chunked pruned prefill ([S1] §5: prefill pruning proceeds in chunks of 128 tokens), when
 * prune_logp > -inf: before the chunk that starts at row c (c a multiple of 128, c > 0), every
 * pair j < c whose bias Lambda_{c-1,j} is below log p is evicted for good (Lambda only
 * decreases down a column, so it would never come back).  A row of that chunk attends over
 * the surviving pairs and every pair of its own chunk, with the same biases as before.
 * Lambda and b_final do not change; with prune_logp = -inf (p = 0) nothing is evicted.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ scalar pieces */

/* softplus(x) = log(1 + e^x), written in the overflow-free form. */
static double softplus(double x) { return fmax(x, 0.0) + log1p(exp(-fabs(x))); }

static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* d softplus / dx divided by softplus, i.e. sigmoid(x)/softplus(x).  When softplus
 * underflows to zero the decay that multiplies this factor is zero too, so 0 is returned
 * for the product's sake (the limit of the ratio is 1 but it is always multiplied by D). */
static double sig_over_softplus(double x) {
    double sp = softplus(x);
    if (sp == 0.0) return 0.0;
    return sigmoid(x) / sp;
}

static double dot(const double* a, const double* b, int n) {
    double s = 0.0;
    for (int c = 0; c < n; ++c) s += a[c] * b[c];
    return s;
}

/* Key L2 normalisation ([S3] Fig. 1 caption: keys are L2-normalised). */
static double l2_normalise(const double* x, int d, double* out) {
    double n = sqrt(dot(x, x, d));
    double den = n > 1e-12 ? n : 1e-12;
    for (int c = 0; c < d; ++c) out[c] = x[c] / den;
    return n;
}

/* RoPE with rotate-half pairing: (x_m, x_{m+d/2}) rotated by pos * theta^(-2m/d).
 * sign = +1 applies the rotation, -1 applies its inverse (= transpose). */
static void rope(const double* x, int d, double pos, double theta, double sign, double* out) {
    int half = d / 2;
    for (int m = 0; m < half; ++m) {
        double freq = pow(theta, -2.0 * (double)m / (double)d);
        double ang = sign * pos * freq;
        double c = cos(ang), s = sin(ang);
        double x0 = x[m], x1 = x[m + half];
        out[m] = x0 * c - x1 * s;
        out[m + half] = x1 * c + x0 * s;
    }
}

/* Combined decay: geometric mean of the three rates ([S1] §4; [S3] Fig. 1 right and the
 * veto property: a zero rate in any factor gives exactly zero). */
static double decay_rate(double rq, double rk, double rsim) { return cbrt(rq * rk * rsim); }

/* Variant bits (see the header). */
enum { VAR_NO_Q = 1, VAR_NO_K = 2, VAR_NO_SIM = 4, VAR_QNORM = 8, VAR_ALL = 15 };

static int n_active(int variant) {
    return !(variant & VAR_NO_Q) + !(variant & VAR_NO_K) + !(variant & VAR_NO_SIM);
}

/* Geometric mean of the rates whose mechanisms are on ([S1] §5.4, App. E: the ablations
 * drop mechanisms from the combination).  With all three on this is decay_rate. */
static double decay_active(double rq, double rk, double rsim, int variant) {
    if (!(variant & (VAR_NO_Q | VAR_NO_K | VAR_NO_SIM))) return decay_rate(rq, rk, rsim);
    double prod = 1.0;
    if (!(variant & VAR_NO_Q)) prod *= rq;
    if (!(variant & VAR_NO_K)) prod *= rk;
    if (!(variant & VAR_NO_SIM)) prod *= rsim;
    return n_active(variant) == 2 ? sqrt(prod) : prod;
}

/* Qwen3-style query normalisation ([S1] App. E): RMS norm over the head dimension with
 * unit gain and eps 1e-6.  Returns the factor 1/sqrt(mean(x^2) + eps). */
static double rms_normalise(const double* x, int d, double* out) {
    double r = 1.0 / sqrt(dot(x, x, d) / (double)d + 1e-6);
    for (int c = 0; c < d; ++c) out[c] = x[c] * r;
    return r;
}

/* RoPE of a query, RMS-normalised first when the variant asks for it. */
static void rope_query(const double* q, int d, double pos, double theta, int variant,
                       double* tmp, double* out) {
    if (variant & VAR_QNORM) {
        rms_normalise(q, d, tmp);
        q = tmp;
    }
    rope(q, d, pos, theta, 1.0, out);
}

/* ------------------------------------------------------------------ tiny thread pool */

typedef void (*unit_fn)(void* ctx, int unit);
typedef struct { unit_fn fn; void* ctx; int n_units; int next; pthread_mutex_t mu; } pool_t;

static void* pool_worker(void* arg) {
    pool_t* p = (pool_t*)arg;
    for (;;) {
        pthread_mutex_lock(&p->mu);
        int u = p->next++;
        pthread_mutex_unlock(&p->mu);
        if (u >= p->n_units) break;
        p->fn(p->ctx, u);
    }
    return NULL;
}

static void run_units(unit_fn fn, void* ctx, int n_units, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > n_units) nthreads = n_units;
    pool_t p;
    p.fn = fn; p.ctx = ctx; p.n_units = n_units; p.next = 0;
    pthread_mutex_init(&p.mu, NULL);
    if (nthreads <= 1) {
        pool_worker(&p);
    } else {
        pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
        for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, pool_worker, &p);
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
        free(th);
    }
    pthread_mutex_destroy(&p.mu);
}

/* ------------------------------------------------------------------ prefill forward */

/* Nearest bf16 value (8 significant bits) of x, ties to even, by way of the nearest float.
 * Used only by the tolerance models (bf16 operands of the forward, saved outputs of the
 * backward). */
static double round_bf16(double x) {
    float f = (float)x;
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) != 0x7f800000u) {
        u += 0x7fffu + ((u >> 16) & 1u);
        u &= 0xffff0000u;
        memcpy(&f, &u, sizeof f);
    }
    return (double)f;
}

/* Forward.  Operand model (optional, for deriving tolerances only; bf16_operands set): the
 * unit keys, the rotated keys and the rotated queries are rounded to bf16 where they enter the
 * similarity and the logits, as in an implementation whose products take bf16 operands; the
 * logit error that leaves grows with scale*||q||. */
typedef struct {
    int B, T, H, Hkv, d;
    double scale, theta;
    const double *q, *k, *v, *g, *aq, *ak, *alpha, *beta;
    const uint8_t* unit_mask; /* [B*Hkv] or NULL = all units */
    const uint8_t* row_mask;  /* [T] or NULL = all rows get attention outputs */
    double *o, *lse, *bfinal, *lambda;
    int variant;
    double prune_logp;        /* log p of the chunked prefill pruning, -inf = dense */
    int bf16_operands;        /* operand model (see above) */
} fwd_ctx;

static void fwd_unit(void* vctx, int unit) {
    fwd_ctx* c = (fwd_ctx*)vctx;
    if (c->unit_mask && !c->unit_mask[unit]) return;
    const int B = c->B, T = c->T, H = c->H, Hkv = c->Hkv, d = c->d, G = H / Hkv;
    (void)B;
    const int b = unit / Hkv, kvh = unit % Hkv;
    const double alpha = c->alpha[kvh], beta = c->beta[kvh];

    double* khat = (double*)malloc(sizeof(double) * (size_t)T * d);
    double* krot = (double*)malloc(sizeof(double) * (size_t)T * d);
    double* rk = (double*)malloc(sizeof(double) * (size_t)T);
    double* lam = (double*)malloc(sizeof(double) * (size_t)T);   /* row i of Lambda */
    double* srow = (double*)malloc(sizeof(double) * (size_t)T);
    double* qrot = (double*)malloc(sizeof(double) * (size_t)d);
    double* qtmp = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    double* lamb = (double*)malloc(sizeof(double) * (size_t)T);  /* Lambda at the last chunk boundary */
    int cs = 0;                                                  /* first row of the current chunk */

    for (int t = 0; t < T; ++t) {
        const double* kt = c->k + (((size_t)b * T + t) * Hkv + kvh) * d;
        l2_normalise(kt, d, khat + (size_t)t * d);
        rope(khat + (size_t)t * d, d, (double)t, c->theta, 1.0, krot + (size_t)t * d);
        rk[t] = softplus(c->ak[((size_t)b * T + t) * Hkv + kvh]);
        if (c->bf16_operands)
            for (int x = 0; x < d; ++x) {
                khat[(size_t)t * d + x] = round_bf16(khat[(size_t)t * d + x]);
                krot[(size_t)t * d + x] = round_bf16(krot[(size_t)t * d + x]);
            }
    }

    for (int i = 0; i < T; ++i) {
        if (i > 0 && i % 128 == 0) {
            /* chunk boundary: lam still holds row i-1, the biases the eviction decides on */
            cs = i;
            for (int j = 0; j < i; ++j) lamb[j] = lam[j];
        }
        /* Causal accumulation, column prefix form: Lambda_ij = Lambda_{i-1,j} - D[i,j]. */
        double rq_i = softplus(c->aq[((size_t)b * T + i) * Hkv + kvh]);
        for (int j = 0; j < i; ++j) {
            double sim = dot(khat + (size_t)i * d, khat + (size_t)j * d, d);
            double rsim = softplus(alpha * sim + beta);
            lam[j] -= decay_active(rq_i, rk[j], rsim, c->variant);
        }
        lam[i] = 0.0;
        if (c->lambda) {
            double* row = c->lambda + (((size_t)b * Hkv + kvh) * T + i) * (size_t)T;
            for (int j = 0; j < T; ++j) row[j] = (j <= i) ? lam[j] : 0.0;
        }
        if (c->row_mask && !c->row_mask[i]) continue;
        for (int hh = 0; hh < G; ++hh) {
            int h = kvh * G + hh;
            const double* qi = c->q + (((size_t)b * T + i) * H + h) * d;
            rope_query(qi, d, (double)i, c->theta, c->variant, qtmp, qrot);
            if (c->bf16_operands)
                for (int x = 0; x < d; ++x) qrot[x] = round_bf16(qrot[x]);
            double m = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                /* evicted at the chunk boundary: no longer in the cache */
                if (j < cs && !(lamb[j] >= c->prune_logp)) {
                    srow[j] = -INFINITY;
                    continue;
                }
                srow[j] = c->scale * dot(qrot, krot + (size_t)j * d, d) + lam[j];
                if (srow[j] > m) m = srow[j];
            }
            double l = 0.0;
            for (int x = 0; x < d; ++x) acc[x] = 0.0;
            for (int j = 0; j <= i; ++j) {
                if (srow[j] == -INFINITY) continue;
                double p = exp(srow[j] - m);
                l += p;
                const double* vj = c->v + (((size_t)b * T + j) * Hkv + kvh) * d;
                for (int x = 0; x < d; ++x) acc[x] += p * vj[x];
            }
            const double* gi = c->g + (((size_t)b * T + i) * H + h) * d;
            double* oi = c->o + (((size_t)b * T + i) * H + h) * d;
            for (int x = 0; x < d; ++x) oi[x] = acc[x] / l * sigmoid(gi[x]);
            if (c->lse) c->lse[((size_t)b * H + h) * T + i] = m + log(l);
        }
    }
    if (c->bfinal) {
        double* bf = c->bfinal + ((size_t)b * Hkv + kvh) * T;
        for (int j = 0; j < T; ++j) bf[j] = lam[j];
    }
    free(khat); free(krot); free(rk); free(lam); free(srow); free(qrot); free(qtmp); free(acc);
    free(lamb);
}

/* Prefill forward.  Outputs that are NULL are skipped.  Only units with unit_mask set
 * (all if NULL) and rows with row_mask set (all if NULL) are written. */
int ora_prefill_fwd(int B, int T, int H, int Hkv, int d, double scale, double theta,
                    const double* q, const double* k, const double* v, const double* g,
                    const double* aq, const double* ak, const double* alpha, const double* beta,
                    const uint8_t* unit_mask, const uint8_t* row_mask,
                    double* o, double* lse, double* bfinal, double* lambda, int variant,
                    double prune_logp, int bf16_operands, int nthreads) {
    if (B < 1 || T < 1 || H < 1 || Hkv < 1 || d < 2 || (d & 1) || H % Hkv) return 1;
    if ((variant & ~VAR_ALL) || n_active(variant) == 0) return 1;
    if (isnan(prune_logp) || prune_logp > 0.0) return 1;
    fwd_ctx c = {B, T, H, Hkv, d, scale, theta, q, k, v, g, aq, ak, alpha, beta,
                 unit_mask, row_mask, o, lse, bfinal, lambda, variant, prune_logp, bf16_operands != 0};
    run_units(fwd_unit, &c, B * Hkv, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ brute-force Lambda */

typedef struct {
    int B, T, Hkv, d;
    const double *k, *aq, *ak, *alpha, *beta;
    double* lambda;
    int variant;
} brute_ctx;

static void brute_unit(void* vctx, int unit) {
    brute_ctx* c = (brute_ctx*)vctx;
    const int T = c->T, Hkv = c->Hkv, d = c->d;
    const int b = unit / Hkv, kvh = unit % Hkv;
    double* kl = (double*)malloc(sizeof(double) * (size_t)d);
    double* kj = (double*)malloc(sizeof(double) * (size_t)d);
    for (int i = 0; i < T; ++i) {
        for (int j = 0; j < T; ++j) {
            double s = 0.0;
            if (j <= i) {
                /* Direct per-(i,j) sum over l = j+1 .. i, every factor recomputed. */
                for (int l = j + 1; l <= i; ++l) {
                    l2_normalise(c->k + (((size_t)b * T + l) * Hkv + kvh) * d, d, kl);
                    l2_normalise(c->k + (((size_t)b * T + j) * Hkv + kvh) * d, d, kj);
                    double rq = softplus(c->aq[((size_t)b * T + l) * Hkv + kvh]);
                    double rk = softplus(c->ak[((size_t)b * T + j) * Hkv + kvh]);
                    double rsim = softplus(c->alpha[kvh] * dot(kl, kj, d) + c->beta[kvh]);
                    s -= decay_active(rq, rk, rsim, c->variant);
                }
            }
            c->lambda[(((size_t)b * Hkv + kvh) * T + i) * (size_t)T + j] = s;
        }
    }
    free(kl); free(kj);
}

/* O(T^3 d) Lambda straight from its definition (tiny T only). */
int ora_lambda_bruteforce(int B, int T, int Hkv, int d, const double* k, const double* aq,
                          const double* ak, const double* alpha, const double* beta,
                          double* lambda, int variant, int nthreads) {
    if ((variant & ~VAR_ALL) || n_active(variant) == 0) return 1;
    brute_ctx c = {B, T, Hkv, d, k, aq, ak, alpha, beta, lambda, variant};
    run_units(brute_unit, &c, B * Hkv, nthreads);
    return 0;
}

/* ------------------------------------------------------------------ decode step */
/*
 * One decode step for every (b, KV head) cache ([S1] §4.2, [S3] eviction paragraph):
 *   1. every cached pair j takes the new row's decay: b_j -= D[t, j];
 *   2. it is evicted when exp(b_j) < p, i.e. b_j < log p (kept when b_j >= log p);
 *   3. the new token's query heads attend over the surviving pairs plus the new token,
 *      whose own bias is Lambda_tt = 0;
 *   4. the survivors are compacted stably (ascending old slot) and the new token is
 *      appended with b = 0.
 * The cache holds the raw key (k), value, a_k logit, token position and the bias.
 * Keys are normalised and rotated from scratch at every use.
 *
 * adopt_keep (optional, [B,Hkv,cap]): for pairs whose new bias lies strictly within
 * `band` of log p the oracle takes this decision instead of its own, so that two
 * implementations whose roundings differ near the threshold stay in lockstep.
 * in_band (optional out) flags those pairs.
 *
 * defer != 0 (deferred compaction): step 4 moves nothing.  Every pair keeps its slot and its
 * updated bias, evicted ones included (their bias stays below log p: it only decreases), and the
 * new token goes to slot n.  kept_order then holds s at slot s.  Step 3 attends over the same
 * pairs either way, since an evicted pair's bias never rises back above log p.
 */
typedef struct {
    int B, H, Hkv, d, cap;
    double scale, theta, logp, band, pos_t;
    int* n_kept;
    double *kc, *vc, *akc, *posc, *bc;
    const double *q, *k, *v, *g, *aq, *ak, *alpha, *beta;
    const uint8_t* adopt_keep;
    double* o;
    uint8_t *evict, *in_band;
    int64_t* kept_order;
    int variant;
    int defer;
} dec_ctx;

static void dec_unit(void* vctx, int unit) {
    dec_ctx* c = (dec_ctx*)vctx;
    const int H = c->H, Hkv = c->Hkv, d = c->d, cap = c->cap, G = H / Hkv;
    const int b = unit / Hkv, kvh = unit % Hkv;
    const size_t base = (size_t)unit * cap;
    int n = c->n_kept[unit];
    double* kt_hat = (double*)malloc(sizeof(double) * (size_t)d);
    double* kt_rot = (double*)malloc(sizeof(double) * (size_t)d);
    double* kj_hat = (double*)malloc(sizeof(double) * (size_t)d);
    double* kj_rot = (double*)malloc(sizeof(double) * (size_t)d);
    double* qrot = (double*)malloc(sizeof(double) * (size_t)d);
    double* qtmp = (double*)malloc(sizeof(double) * (size_t)d);
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    double* logits = (double*)malloc(sizeof(double) * (size_t)(n + 1));
    uint8_t* keep = (uint8_t*)malloc((size_t)(n + 1));

    const double* kt = c->k + ((size_t)b * Hkv + kvh) * d;
    const double* vt = c->v + ((size_t)b * Hkv + kvh) * d;
    l2_normalise(kt, d, kt_hat);
    rope(kt_hat, d, c->pos_t, c->theta, 1.0, kt_rot);
    double rq_t = softplus(c->aq[(size_t)b * Hkv + kvh]);
    const double alpha = c->alpha[kvh], beta = c->beta[kvh];

    /* 1-2: bias update and eviction decision (a pair left in place by a deferred compaction
     * already has b < log p and stays evicted) */
    for (int j = 0; j < n; ++j) {
        l2_normalise(c->kc + (base + j) * d, d, kj_hat);
        double rsim = softplus(alpha * dot(kt_hat, kj_hat, d) + beta);
        double rk = softplus(c->akc[base + j]);
        c->bc[base + j] -= decay_active(rq_t, rk, rsim, c->variant);
        double bj = c->bc[base + j];
        keep[j] = bj >= c->logp;
        int inb = fabs(bj - c->logp) < c->band;
        if (c->in_band) c->in_band[base + j] = (uint8_t)inb;
        if (inb && c->adopt_keep) keep[j] = c->adopt_keep[base + j] ? 1 : 0;
        if (c->evict) c->evict[base + j] = (uint8_t)!keep[j];
    }
    /* 3: attention of the G query heads over survivors + the new token */
    for (int hh = 0; hh < G; ++hh) {
        int h = kvh * G + hh;
        rope_query(c->q + ((size_t)b * H + h) * d, d, c->pos_t, c->theta, c->variant, qtmp, qrot);
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
            if (!keep[j]) continue;
            l2_normalise(c->kc + (base + j) * d, d, kj_hat);
            rope(kj_hat, d, c->posc[base + j], c->theta, 1.0, kj_rot);
            logits[j] = c->scale * dot(qrot, kj_rot, d) + c->bc[base + j];
            if (logits[j] > m) m = logits[j];
        }
        logits[n] = c->scale * dot(qrot, kt_rot, d) + 0.0;
        if (logits[n] > m) m = logits[n];
        double l = 0.0;
        for (int x = 0; x < d; ++x) acc[x] = 0.0;
        for (int j = 0; j <= n; ++j) {
            if (j < n && !keep[j]) continue;
            double p = exp(logits[j] - m);
            l += p;
            const double* vj = (j < n) ? c->vc + (base + j) * d : vt;
            for (int x = 0; x < d; ++x) acc[x] += p * vj[x];
        }
        const double* gh = c->g + ((size_t)b * H + h) * d;
        double* oh = c->o + ((size_t)b * H + h) * d;
        for (int x = 0; x < d; ++x) oh[x] = acc[x] / l * sigmoid(gh[x]);
    }
    /* 4: stable compaction (or none, deferred), then append */
    int w = 0;
    if (c->defer) {
        for (int j = 0; j < n; ++j)
            if (c->kept_order) c->kept_order[base + j] = j;
        w = n;
    }
    for (int j = 0; j < n && !c->defer; ++j) {
        if (!keep[j]) continue;
        if (c->kept_order) c->kept_order[base + w] = j;
        if (w != j) {
            memmove(c->kc + (base + w) * d, c->kc + (base + j) * d, sizeof(double) * d);
            memmove(c->vc + (base + w) * d, c->vc + (base + j) * d, sizeof(double) * d);
            c->akc[base + w] = c->akc[base + j];
            c->posc[base + w] = c->posc[base + j];
            c->bc[base + w] = c->bc[base + j];
        }
        ++w;
    }
    if (w < cap) {
        memcpy(c->kc + (base + w) * d, kt, sizeof(double) * d);
        memcpy(c->vc + (base + w) * d, vt, sizeof(double) * d);
        c->akc[base + w] = c->ak[(size_t)b * Hkv + kvh];
        c->posc[base + w] = c->pos_t;
        c->bc[base + w] = 0.0;
        c->n_kept[unit] = w + 1;
    } else {
        c->n_kept[unit] = -1; /* capacity exceeded */
    }
    free(kt_hat); free(kt_rot); free(kj_hat); free(kj_rot); free(qrot); free(qtmp); free(acc);
    free(logits); free(keep);
}

int ora_decode_step(int B, int H, int Hkv, int d, int cap, double scale, double theta,
                    int* n_kept, double* kc, double* vc, double* akc, double* posc, double* bc,
                    const double* q, const double* k, const double* v, const double* g,
                    const double* aq, const double* ak, const double* alpha, const double* beta,
                    double pos_t, double logp, double band, const uint8_t* adopt_keep,
                    double* o, uint8_t* evict, uint8_t* in_band, int64_t* kept_order,
                    int variant, int defer, int nthreads) {
    if (H % Hkv) return 1;
    if ((variant & ~VAR_ALL) || n_active(variant) == 0) return 1;
    dec_ctx c = {B, H, Hkv, d, cap, scale, theta, logp, band, pos_t, n_kept, kc, vc, akc,
                 posc, bc, q, k, v, g, aq, ak, alpha, beta, adopt_keep, o, evict, in_band,
                 kept_order, variant, defer};
    run_units(dec_unit, &c, B * Hkv, nthreads);
    for (int u = 0; u < B * Hkv; ++u)
        if (n_kept[u] < 0) return 2;
    return 0;
}

/* Stable compaction of one slot list by a keep mask: the kept slot indices in ascending
 * order (the order std::stable_partition leaves them in).  Returns the kept count. */
int ora_compact_order(int n, const uint8_t* keep, int64_t* order) {
    int w = 0;
    for (int j = 0; j < n; ++j)
        if (keep[j]) order[w++] = j;
    return w;
}

/* ------------------------------------------------------------------ prefill backward */
/*
 * Analytic fp64 gradient of L = sum(dO * O) through the definitions above:
 *   A_i = sum_j P_ij v_j,  O_i = A_i * sigmoid(g_i),  P_ij = softmax_j(S_ij)
 *   dA = dO*sigmoid(g);   dg = dO*A*sigmoid(g)*(1-sigmoid(g))
 *   dP_ij = dA_i.v_j;     dS_ij = P_ij (dP_ij - sum_j' P_ij' dP_ij')
 *   dv_j += P_ij dA_i;    dqrot_i += s dS_ij krot_j;   dkrot_j += s dS_ij qrot_i
 *   dLambda_ij = sum over the group's heads of dS_ij
 *   dD[l,j] = -sum_{i>=l} dLambda_ij                                   (l > j)
 *   w = dD * D / 3  (D = cbrt of the product, so dD/dr = D/(3r))
 *   d a_q[l] += w sigmoid(a_q)/softplus(a_q);  d a_k[j] += w sigmoid(a_k)/softplus(a_k)
 *   dX = w sigmoid(X)/softplus(X), X = alpha c + beta, c = <khat_l, khat_j>
 *   d alpha += dX c;  d beta += dX;  dkhat_l += alpha dX khat_j;  dkhat_j += alpha dX khat_l
 *   then dq = RoPE^T dqrot, dkhat += RoPE^T dkrot, dk = (dkhat - khat <khat,dkhat>)/||k||.
 * Variants: with n mechanisms on, D = (product of the active rates)^(1/n), so
 *   w = dD * D / n, and the a_q / a_k / (alpha, beta, khat-similarity) terms appear only
 *   for the mechanisms that are on.  With the query norm q' = r q, r = 1/sqrt(mean(q^2)+eps):
 *   dq = r (dq' - q' <q', dq'> / d), dq' = RoPE^T dqrot.
 * Lambda and dLambda are held as packed lower-triangular T x T matrices per unit.
 * dalpha / dbeta are summed over the batch: [Hkv].
 *
 * Saved-output model (optional, for deriving tolerances only; model_c > 0): the backward is
 * fed what a bf16 forward saves.  That forward rounds each unnormalised probability
 * e_ij = c exp(s_ij - m_i) to bf16 before its PV and row-sum products (c <= 1: its softmax
 * shift need not be the row maximum; c picks which values round up), so its normaliser is
 * l_i = sum_j bf16(c e_ij) / c and its output o = sigmoid(g) (.) sum_j bf16(c e_ij) v_j / (c l_i),
 * stored in bf16.  The backward recomputes P_ij = e_ij / l_i from the saved lse (rows then sum to
 * 1 + eta_i, not 1) and forms delta_i = sum_x dO_ix o_ix from the saved output.  In exact
 * arithmetic all of this is the method; each row's error eps_i in (dP - delta) terms moves
 * every gradient by about -sum_i eps_i * grad(lse_i) (an extra -eps_i P_ij in dS_ij is the
 * derivative of -eps_i lse_i), which the per-head sums dalpha, dbeta feel most.
 */
typedef struct {
    int B, T, H, Hkv, d;
    double scale, theta;
    const double *q, *k, *v, *g, *aq, *ak, *alpha, *beta, *dout;
    const uint8_t* unit_mask;
    double *dq, *dk, *dv, *dg, *daq, *dak;
    double *dalpha_u, *dbeta_u; /* per unit partials [B*Hkv] */
    int variant;
    double model_c;             /* saved-output model (see above); 0 = off */
} bwd_ctx;



static size_t tri(int i, int j) { return (size_t)i * (size_t)(i + 1) / 2 + (size_t)j; }

static void bwd_unit(void* vctx, int unit) {
    bwd_ctx* c = (bwd_ctx*)vctx;
    if (c->unit_mask && !c->unit_mask[unit]) return;
    const int T = c->T, H = c->H, Hkv = c->Hkv, d = c->d, G = H / Hkv;
    const int b = unit / Hkv, kvh = unit % Hkv;
    const double alpha = c->alpha[kvh], beta = c->beta[kvh], s = c->scale;
    const size_t TT = (size_t)T * (size_t)(T + 1) / 2;

    double* khat = (double*)calloc((size_t)T * d, sizeof(double));
    double* knorm = (double*)calloc((size_t)T, sizeof(double));
    double* krot = (double*)calloc((size_t)T * d, sizeof(double));
    double* rq = (double*)calloc((size_t)T, sizeof(double));
    double* rk = (double*)calloc((size_t)T, sizeof(double));
    double* lam = (double*)calloc(TT, sizeof(double));
    double* dlam = (double*)calloc(TT, sizeof(double));
    double* dkhat = (double*)calloc((size_t)T * d, sizeof(double));
    double* dkrot = (double*)calloc((size_t)T * d, sizeof(double));
    double* dvl = (double*)calloc((size_t)T * d, sizeof(double));
    double* daq = (double*)calloc((size_t)T, sizeof(double));
    double* dak = (double*)calloc((size_t)T, sizeof(double));
    double* qrot = (double*)calloc((size_t)d, sizeof(double));
    double* dqrot = (double*)calloc((size_t)d, sizeof(double));
    double* tmp = (double*)calloc((size_t)d, sizeof(double));
    double* qn = (double*)calloc((size_t)d, sizeof(double));
    double* A = (double*)calloc((size_t)d, sizeof(double));
    double* dA = (double*)calloc((size_t)d, sizeof(double));
    double* P = (double*)calloc((size_t)T, sizeof(double));
    double* dP = (double*)calloc((size_t)T, sizeof(double));

    for (int t = 0; t < T; ++t) {
        knorm[t] = l2_normalise(c->k + (((size_t)b * T + t) * Hkv + kvh) * d, d, khat + (size_t)t * d);
        rope(khat + (size_t)t * d, d, (double)t, c->theta, 1.0, krot + (size_t)t * d);
        rq[t] = softplus(c->aq[((size_t)b * T + t) * Hkv + kvh]);
        rk[t] = softplus(c->ak[((size_t)b * T + t) * Hkv + kvh]);
    }
    /* Lambda by column prefix */
    for (int i = 0; i < T; ++i) {
        lam[tri(i, i)] = 0.0;
        for (int j = 0; j < i; ++j) {
            double rsim = softplus(alpha * dot(khat + (size_t)i * d, khat + (size_t)j * d, d) + beta);
            double prev = (i - 1 >= j) ? lam[tri(i - 1, j)] : 0.0;
            lam[tri(i, j)] = prev - decay_active(rq[i], rk[j], rsim, c->variant);
        }
    }
    /* attention part, head by head, row by row */
    for (int hh = 0; hh < G; ++hh) {
        int h = kvh * G + hh;
        for (int i = 0; i < T; ++i) {
            const double* qi = c->q + (((size_t)b * T + i) * H + h) * d;
            const double* gi = c->g + (((size_t)b * T + i) * H + h) * d;
            const double* doi = c->dout + (((size_t)b * T + i) * H + h) * d;
            rope_query(qi, d, (double)i, c->theta, c->variant, qn, qrot);
            double m = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                P[j] = s * dot(qrot, krot + (size_t)j * d, d) + lam[tri(i, j)];
                if (P[j] > m) m = P[j];
            }
            const double mc = c->model_c;
            double l = 0.0;
            for (int j = 0; j <= i; ++j) {
                P[j] = exp(P[j] - m);
                l += mc > 0.0 ? round_bf16(mc * P[j]) / mc : P[j];
            }
            for (int x = 0; x < d; ++x) A[x] = 0.0;
            for (int j = 0; j <= i; ++j) {
                const double* vj = c->v + (((size_t)b * T + j) * Hkv + kvh) * d;
                const double pj = (mc > 0.0 ? round_bf16(mc * P[j]) / mc : P[j]) / l;
                for (int x = 0; x < d; ++x) A[x] += pj * vj[x];
            }
            for (int j = 0; j <= i; ++j) P[j] /= l;
            double* dgi = c->dg + (((size_t)b * T + i) * H + h) * d;
            for (int x = 0; x < d; ++x) {
                double sg = sigmoid(gi[x]);
                dA[x] = doi[x] * sg;
                dgi[x] = doi[x] * A[x] * sg * (1.0 - sg);
            }
            double delta = 0.0;
            for (int j = 0; j <= i; ++j) {
                const double* vj = c->v + (((size_t)b * T + j) * Hkv + kvh) * d;
                dP[j] = dot(dA, vj, d);
                delta += P[j] * dP[j];
            }
            if (mc > 0.0) {
                delta = 0.0;
                for (int x = 0; x < d; ++x) delta += doi[x] * round_bf16(sigmoid(gi[x]) * A[x]);
            }
            for (int x = 0; x < d; ++x) dqrot[x] = 0.0;
            for (int j = 0; j <= i; ++j) {
                double dS = P[j] * (dP[j] - delta);
                dlam[tri(i, j)] += dS;
                for (int x = 0; x < d; ++x) {
                    dqrot[x] += s * dS * krot[(size_t)j * d + x];
                    dkrot[(size_t)j * d + x] += s * dS * qrot[x];
                    dvl[(size_t)j * d + x] += P[j] * dA[x];
                }
            }
            double* dqi = c->dq + (((size_t)b * T + i) * H + h) * d;
            rope(dqrot, d, (double)i, c->theta, -1.0, dqi);
            if (c->variant & VAR_QNORM) {
                /* back through q' = r q: qn holds q' from rope_query */
                double r = rms_normalise(qi, d, qn);
                double pr = dot(qn, dqi, d);
                for (int x = 0; x < d; ++x) dqi[x] = r * (dqi[x] - qn[x] * pr / (double)d);
            }
        }
    }
    /* dD[l,j] = -sum_{i>=l} dLambda_ij, then through the geometric mean and softplus */
    double dal = 0.0, dbe = 0.0;
    for (int j = 0; j < T; ++j) {
        double suffix = 0.0;
        for (int l = T - 1; l > j; --l) {
            suffix += dlam[tri(l, j)];
            double dD = -suffix;
            double cs = dot(khat + (size_t)l * d, khat + (size_t)j * d, d);
            double X = alpha * cs + beta;
            double D = decay_active(rq[l], rk[j], softplus(X), c->variant);
            if (D == 0.0) continue;
            double w = dD * D / (double)n_active(c->variant);
            if (!(c->variant & VAR_NO_Q))
                daq[l] += w * sig_over_softplus(c->aq[((size_t)b * T + l) * Hkv + kvh]);
            if (!(c->variant & VAR_NO_K))
                dak[j] += w * sig_over_softplus(c->ak[((size_t)b * T + j) * Hkv + kvh]);
            double dX = (c->variant & VAR_NO_SIM) ? 0.0 : w * sig_over_softplus(X);
            dal += dX * cs;
            dbe += dX;
            for (int x = 0; x < d; ++x) {
                dkhat[(size_t)l * d + x] += alpha * dX * khat[(size_t)j * d + x];
                dkhat[(size_t)j * d + x] += alpha * dX * khat[(size_t)l * d + x];
            }
        }
    }
    for (int t = 0; t < T; ++t) {
        rope(dkrot + (size_t)t * d, d, (double)t, c->theta, -1.0, tmp);
        double* dkh = dkhat + (size_t)t * d;
        for (int x = 0; x < d; ++x) dkh[x] += tmp[x];
        const double* kh = khat + (size_t)t * d;
        double* dkt = c->dk + (((size_t)b * T + t) * Hkv + kvh) * d;
        if (knorm[t] > 1e-12) {
            double proj = dot(kh, dkh, d);
            for (int x = 0; x < d; ++x) dkt[x] = (dkh[x] - kh[x] * proj) / knorm[t];
        } else {
            for (int x = 0; x < d; ++x) dkt[x] = dkh[x] / 1e-12;
        }
        double* dvt = c->dv + (((size_t)b * T + t) * Hkv + kvh) * d;
        for (int x = 0; x < d; ++x) dvt[x] = dvl[(size_t)t * d + x];
        c->daq[((size_t)b * T + t) * Hkv + kvh] = daq[t];
        c->dak[((size_t)b * T + t) * Hkv + kvh] = dak[t];
    }
    c->dalpha_u[unit] = dal;
    c->dbeta_u[unit] = dbe;

    free(khat); free(knorm); free(krot); free(rq); free(rk); free(lam); free(dlam);
    free(dkhat); free(dkrot); free(dvl); free(daq); free(dak); free(qrot); free(dqrot);
    free(tmp); free(qn); free(A); free(dA); free(P); free(dP);
}

int ora_prefill_bwd(int B, int T, int H, int Hkv, int d, double scale, double theta,
                    const double* q, const double* k, const double* v, const double* g,
                    const double* aq, const double* ak, const double* alpha, const double* beta,
                    const double* dout, const uint8_t* unit_mask,
                    double* dq, double* dk, double* dv, double* dg, double* daq, double* dak,
                    double* dalpha, double* dbeta, int variant, double model_c, int nthreads) {
    if (B < 1 || T < 1 || H < 1 || Hkv < 1 || d < 2 || (d & 1) || H % Hkv) return 1;
    if ((variant & ~VAR_ALL) || n_active(variant) == 0) return 1;
    double* dal_u = (double*)calloc((size_t)B * Hkv, sizeof(double));
    double* dbe_u = (double*)calloc((size_t)B * Hkv, sizeof(double));
    bwd_ctx c = {B, T, H, Hkv, d, scale, theta, q, k, v, g, aq, ak, alpha, beta, dout,
                 unit_mask, dq, dk, dv, dg, daq, dak, dal_u, dbe_u, variant, model_c > 0.0 ? model_c : 0.0};
    run_units(bwd_unit, &c, B * Hkv, nthreads);
    for (int h = 0; h < Hkv; ++h) {
        dalpha[h] = 0.0;
        dbeta[h] = 0.0;
        for (int b = 0; b < B; ++b) {
            dalpha[h] += dal_u[b * Hkv + h];
            dbeta[h] += dbe_u[b * Hkv + h];
        }
    }
    free(dal_u); free(dbe_u);
    return 0;
}
