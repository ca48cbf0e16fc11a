/*
 * lbca_oracle.c -- plain fp64 CPU oracle for block-compressed attention
 * (the LBCA retrofit and the HCA form).
 *
 * TEST INFRASTRUCTURE ONLY.  The tests, the smoke check and the benchmark's
 * CPU-baseline leg load this library; the product path never does.  It shares
 * no code, header, table or helper with the CUDA library.
 *
 * What it computes, and where the pages define it:
 *   - Block pooling: each complete, non-overlapping block of m raw tokens
 *     becomes one entry by a per-channel softmax over the block's positions of
 *     content logits Z plus a learnable positional bias B_pos, weighting the
 *     raw values.  ("mSeek" README, section "How LBCA works", steps 2-3; HCA
 *     page, section "What is implemented": single-series pooling, Eqs 20-23.)
 *     K and V are pooled as separate series, each with its own Z and B_pos
 *     (GQA retrofit); in the HCA form one series C serves as key and value.
 *   - Entry finalisation: RMSNorm (HCA form) and RoPE at the block-start
 *     position (CSA page, section "Deviations from paper": compressed entries
 *     take RoPE at their block-start index).
 *   - Attention: one softmax over every causally visible pooled entry plus an
 *     exact raw recent window, plus an optional sink logit that enters only the
 *     denominator; in the shared-KV form the output's RoPE dims are rotated by
 *     the negative query position.  ("mSeek" README, "How LBCA works", steps
 *     4-5; HCA page, "What is implemented"; CSA page, "What is implemented":
 *     core attention Eqs 18-19, sink Eq 27, partial RoPE with the -i output
 *     rotation.)
 *
 * Readings taken where the pages are silent (the design notes list them all):
 *   - Visibility is a block-aligned partition: a query at 0-based position t
 *     (L = t + 1 tokens) sees pooled entries j < P(L) = max(0, floor((L-w)/m))
 *     and raw tokens s in [P*m, t].  This is the reading under which the
 *     README's cache figures (section "Results": 7.116 GiB at 128K, 304,343
 *     tokens in the 154,624-token budget) come out exactly.
 *   - RoPE rotates consecutive pairs (2k, 2k+1) of the last rho dims by
 *     pos * theta^(-2k/rho).  RMSNorm is x / sqrt(mean(x^2) + eps) * gamma,
 *     applied to queries and to key entries (pooled and raw) before RoPE; in
 *     the GQA form values are never normalised or rotated.
 *   - Softmax scale defaults to 1/sqrt(D); kv head of query head h is h / r.
 *
 * Layouts (row-major): raw x, z, k, v [B, T, G, D]; B_pos [m, G*D];
 * queries [B, nq, Hq, D]; pooled entries [B, NB, G, D]; outputs [B, nq, Hq, D].
 */
#include <math.h>
#include <stddef.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int n_q_heads;        /* Hq */
    int n_kv_heads;       /* G */
    int head_dim;         /* D */
    int shared_kv;        /* 1: one entry serves as key and value */
    int block_m;          /* m */
    int n_win;            /* w */
    int rope_dims;        /* rho, 0 = no RoPE */
    int rmsnorm;          /* 1: RMSNorm on queries and key entries */
    double rope_theta;
    double rms_eps;
    double softmax_scale; /* <= 0 selects 1/sqrt(D) */
} orc_config;

enum { ORC_KEY = 0, ORC_VALUE = 1 };

static int cfg_ok(const orc_config* c)
{
    if (!c) return 0;
    if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 1) return 0;
    if (c->n_q_heads % c->n_kv_heads) return 0;
    if (c->block_m < 1 || c->n_win < 0) return 0;
    if (c->rope_dims < 0 || c->rope_dims > c->head_dim || (c->rope_dims & 1)) return 0;
    return 1;
}

/* Number of pooled entries a query with L visible tokens sees. */
long orc_visible_blocks(long L, int m, int w)
{
    long p = L - (long)w;
    if (p <= 0) return 0;
    return p / m;
}

/* x <- x / sqrt(mean(x^2) + eps) * gamma */
static void rmsnorm(double* x, int D, const double* gamma, double eps)
{
    double ss = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    double inv = 1.0 / sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) x[d] = x[d] * inv * (gamma ? gamma[d] : 1.0);
}

/* Rotate consecutive pairs of the last rho dims by pos * theta^(-2k/rho). */
static void rope(double* x, int D, int rho, double theta, double pos)
{
    int base = D - rho;
    for (int k = 0; k < rho / 2; ++k) {
        double inv_freq = pow(theta, -2.0 * k / rho);
        double ang = pos * inv_freq;
        double cs = cos(ang), sn = sin(ang);
        double a = x[base + 2 * k], b = x[base + 2 * k + 1];
        x[base + 2 * k] = a * cs - b * sn;
        x[base + 2 * k + 1] = a * sn + b * cs;
    }
}

/* Key-side finalisation of one entry (pooled or raw) at absolute position pos. */
static void finalise_key(const orc_config* c, double* e, const double* gamma, double pos)
{
    if (c->rmsnorm) rmsnorm(e, c->head_dim, gamma, c->rms_eps);
    if (c->rope_dims) rope(e, c->head_dim, c->rope_dims, c->rope_theta, pos);
}

/*
 * Pool one complete block for kv head g: per channel, softmax over the m
 * positions of z + b_pos, then the weighted sum of x.
 * xb, zb point at the block's first token ([m, G, D] slice).
 */
static void pool_block(const orc_config* c, const double* xb, const double* zb,
                       const double* bpos, int g, double* out)
{
    const int m = c->block_m, G = c->n_kv_heads, D = c->head_dim;
    const long ts = (long)G * D;
    for (int ch = 0; ch < D; ++ch) {
        double amax = -INFINITY;
        for (int i = 0; i < m; ++i) {
            double a = zb[i * ts + (long)g * D + ch] + bpos[i * ts + (long)g * D + ch];
            if (a > amax) amax = a;
        }
        double den = 0.0, num = 0.0;
        for (int i = 0; i < m; ++i) {
            double a = zb[i * ts + (long)g * D + ch] + bpos[i * ts + (long)g * D + ch];
            double e = exp(a - amax);
            den += e;
            num += e * xb[i * ts + (long)g * D + ch];
        }
        out[ch] = num / den;
    }
}

/*
 * Pool the floor(T/m) complete blocks of one series and finalise them.
 * series ORC_KEY: RMSNorm (if enabled) and RoPE at pos0 + j*m;
 * series ORC_VALUE: the pooled value as is.
 * x, z: [B, T, G, D]; bpos: [m, G*D]; gamma: [D] or NULL; out: [B, T/m, G, D].
 */
int orc_pool(const orc_config* c, int series, int B, long T, long pos0,
             const double* x, const double* z, const double* bpos,
             const double* gamma, double* out)
{
    if (!cfg_ok(c) || B < 0 || T < 0 || !x || !z || !bpos || !out) return -1;
    const int m = c->block_m, G = c->n_kv_heads, D = c->head_dim;
    const long NB = T / m;
    const long ts = (long)G * D;
    long total = (long)B * NB * G;
#pragma omp parallel for schedule(static)
    for (long idx = 0; idx < total; ++idx) {
        int g = (int)(idx % G);
        long j = (idx / G) % NB;
        long b = idx / ((long)G * NB);
        const double* xb = x + (b * T + j * m) * ts;
        const double* zb = z + (b * T + j * m) * ts;
        double* e = out + ((b * NB + j) * G + g) * (long)D;
        pool_block(c, xb, zb, bpos, g, e);
        if (series == ORC_KEY) finalise_key(c, e, gamma, (double)(pos0 + j * m));
    }
    return 0;
}

/*
 * Attention for selected query rows.
 *   q     [B, nq, Hq, D] raw queries; qpos [B, nq] their 0-based positions.
 *   ek    [B, NB, G, D] finalised pooled key entries (shared form: the entries);
 *   ev    [B, NB, G, D] pooled values (GQA) or NULL (shared form).
 *   k, v  [B, T_hist, G, D] raw history (v NULL in the shared form).
 *   lens  [B] tokens of history available; a query needs qpos < lens.
 *   sink  [Hq] logits or NULL; gq, gkv RMSNorm gains [D] or NULL.
 *   out   [B, nq, Hq, D].
 * Returns 0, or -1 on a bad argument (a query outside its history, or a
 * visible pooled entry beyond NB).
 */
int orc_attend(const orc_config* c, int B, int nq, const long* qpos,
               const double* q, const double* ek, const double* ev, long NB,
               const double* k, const double* v, long T_hist, const long* lens,
               const double* sink, const double* gq, const double* gkv,
               double* out)
{
    if (!cfg_ok(c) || B < 0 || nq < 0 || !qpos || !q || !k || !lens || !out) return -1;
    if (!c->shared_kv && !v) return -1;
    const int Hq = c->n_q_heads, G = c->n_kv_heads, D = c->head_dim;
    const int m = c->block_m, w = c->n_win, r = Hq / G;
    const double scale = c->softmax_scale > 0 ? c->softmax_scale : 1.0 / sqrt((double)D);
    const long ts = (long)G * D;

    for (int b = 0; b < B; ++b) {
        if (lens[b] > T_hist) return -1;
        for (int i = 0; i < nq; ++i) {
            long t = qpos[(long)b * nq + i];
            if (t < 0 || t >= lens[b]) return -1;
            long P = orc_visible_blocks(t + 1, m, w);
            if (P > NB || (P > 0 && !ek)) return -1;
            if (!c->shared_kv && P > 0 && !ev) return -1;
        }
    }

    int err = 0;
    long total = (long)B * nq * Hq;
#pragma omp parallel for schedule(dynamic, 4)
    for (long idx = 0; idx < total; ++idx) {
        const int h = (int)(idx % Hq);
        const long i = (idx / Hq) % nq;
        const long b = idx / ((long)Hq * nq);
        const int g = h / r;
        const long t = qpos[b * nq + i];
        const long L = t + 1;
        const long P = orc_visible_blocks(L, m, w);
        const long s0 = P * m;
        const long n_raw = t - s0 + 1;
        const long n = P + n_raw;

        double* qt = malloc(sizeof(double) * D);
        double* kt = malloc(sizeof(double) * D);
        double* sc = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        double* o = out + ((b * nq + i) * Hq + h) * (long)D;
        if (!qt || !kt || !sc) {
            free(qt); free(kt); free(sc);
#pragma omp atomic write
            err = 1;
            continue;
        }
        memcpy(qt, q + ((b * nq + i) * Hq + h) * (long)D, sizeof(double) * D);
        if (c->rmsnorm) rmsnorm(qt, D, gq, c->rms_eps);
        if (c->rope_dims) rope(qt, D, c->rope_dims, c->rope_theta, (double)t);

        /* scores: pooled entries j < P, then raw tokens s in [P*m, t] */
        double smax = sink ? sink[h] : -INFINITY;
        for (long j = 0; j < P; ++j) {
            const double* e = ek + ((b * NB + j) * G + g) * (long)D;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += qt[d] * e[d];
            sc[j] = acc * scale;
            if (sc[j] > smax) smax = sc[j];
        }
        for (long s = s0; s <= t; ++s) {
            memcpy(kt, k + (b * T_hist + s) * ts + (long)g * D, sizeof(double) * D);
            finalise_key(c, kt, gkv, (double)s);
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += qt[d] * kt[d];
            sc[P + (s - s0)] = acc * scale;
            if (sc[P + (s - s0)] > smax) smax = sc[P + (s - s0)];
        }

        /* one softmax over all scores plus the sink (denominator only) */
        double den = sink ? exp(sink[h] - smax) : 0.0;
        for (long e = 0; e < n; ++e) {
            sc[e] = exp(sc[e] - smax);
            den += sc[e];
        }
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (long j = 0; j < P; ++j) {
            const double* val = c->shared_kv ? ek + ((b * NB + j) * G + g) * (long)D
                                             : ev + ((b * NB + j) * G + g) * (long)D;
            for (int d = 0; d < D; ++d) o[d] += sc[j] * val[d];
        }
        for (long s = s0; s <= t; ++s) {
            const double p = sc[P + (s - s0)];
            if (c->shared_kv) {
                memcpy(kt, k + (b * T_hist + s) * ts + (long)g * D, sizeof(double) * D);
                finalise_key(c, kt, gkv, (double)s);
                for (int d = 0; d < D; ++d) o[d] += p * kt[d];
            } else {
                const double* val = v + (b * T_hist + s) * ts + (long)g * D;
                for (int d = 0; d < D; ++d) o[d] += p * val[d];
            }
        }
        for (int d = 0; d < D; ++d) o[d] /= den;

        /* shared form: undo the query-position rotation on the RoPE dims */
        if (c->shared_kv && c->rope_dims) rope(o, D, c->rope_dims, c->rope_theta, -(double)t);
        free(qt); free(kt); free(sc);
    }
    return err ? -1 : 0;
}

/* ===================================================================== *
 * CSA form: dual overlapped pooling, lightning-indexer relevance, sparse *
 * attention over the selected entries and an overlapping raw window.    *
 * (CSA page, section "What is implemented": dual overlapped compression *
 * Eqs 9-12, lightning indexer Eqs 13-17, shared-KV MQA core attention   *
 * Eqs 18-19 with the sliding-window branch, sink Eq 27.)                *
 * ===================================================================== */

/*
 * Dual overlapped pooling of the floor(T/m) complete blocks.  Two series,
 * a and b, each with raw values x and content logits z ([B, T, G, D]) and a
 * positional bias ([m, G*D], by in-block offset).  Entry i pools, per
 * channel, its own block i from the a-series and the preceding block i-1 from
 * the b-series under ONE softmax over the 2m logits (block 0 has no preceding
 * block: its softmax runs over its m a-series logits alone):
 *     w = softmax( [z_a[i m + r] + B_a[r]]_r , [z_b[(i-1) m + r] + B_b[r]]_r )
 *     entry_i = sum_r w_a[r] x_a[i m + r] + sum_r w_b[r] x_b[(i-1) m + r]
 * series ORC_KEY then finalises (RMSNorm when on, RoPE at the entry's own
 * block start i*m); ORC_VALUE keeps the pooled value.  out [B, T/m, G, D].
 */
int orc_pool_dual(const orc_config* c, int series, int B, long T,
                  const double* xa, const double* za, const double* xb, const double* zb,
                  const double* bpos_a, const double* bpos_b, const double* gamma, double* out)
{
    if (!cfg_ok(c) || B < 0 || T < 0 || !xa || !za || !xb || !zb || !bpos_a || !bpos_b || !out) return -1;
    const int m = c->block_m, G = c->n_kv_heads, D = c->head_dim;
    const long NB = T / m;
    const long ts = (long)G * D;
    long total = (long)B * NB * G;
#pragma omp parallel for schedule(static)
    for (long idx = 0; idx < total; ++idx) {
        const int g = (int)(idx % G);
        const long i = (idx / G) % NB;
        const long b = idx / ((long)G * NB);
        double* e = out + ((b * NB + i) * G + g) * (long)D;
        for (int ch = 0; ch < D; ++ch) {
            const long col = (long)g * D + ch;
            /* the joint list of logits: own block (a), then the preceding one (b) */
            double amax = -INFINITY;
            for (int r = 0; r < m; ++r) {
                double a = za[(b * T + i * m + r) * ts + col] + bpos_a[r * ts + col];
                if (a > amax) amax = a;
            }
            if (i > 0)
                for (int r = 0; r < m; ++r) {
                    double a = zb[(b * T + (i - 1) * m + r) * ts + col] + bpos_b[r * ts + col];
                    if (a > amax) amax = a;
                }
            double den = 0.0, num = 0.0;
            for (int r = 0; r < m; ++r) {
                double p = exp(za[(b * T + i * m + r) * ts + col] + bpos_a[r * ts + col] - amax);
                den += p;
                num += p * xa[(b * T + i * m + r) * ts + col];
            }
            if (i > 0)
                for (int r = 0; r < m; ++r) {
                    double p = exp(zb[(b * T + (i - 1) * m + r) * ts + col] + bpos_b[r * ts + col] - amax);
                    den += p;
                    num += p * xb[(b * T + (i - 1) * m + r) * ts + col];
                }
            e[ch] = num / den;
        }
        if (series == ORC_KEY) finalise_key(c, e, gamma, (double)(i * m));
    }
    return 0;
}

/*
 * Lightning-indexer relevance of every complete entry to one query per
 * sequence: I_j = sum_h w_h * ReLU(q_h . k_j) over the indexer heads h, for
 * the entries j < nvis[b] (the complete blocks the query can see); the rest
 * of the row is -infinity.
 *   q [B, HI, DI] indexer queries, w [B, HI] head weights,
 *   kx [B, NB, DI] compressed indexer keys, out [B, NB].
 */
int orc_indexer_scores(int B, long NB, int HI, int DI, const double* q, const double* w,
                       const double* kx, const long* nvis, double* out)
{
    if (B < 0 || NB < 0 || HI < 1 || DI < 1 || !q || !w || !kx || !nvis || !out) return -1;
    for (int b = 0; b < B; ++b)
        if (nvis[b] < 0 || nvis[b] > NB) return -1;
    long total = (long)B * NB;
#pragma omp parallel for schedule(static)
    for (long idx = 0; idx < total; ++idx) {
        const long j = idx % NB, b = idx / NB;
        if (j >= nvis[b]) {
            out[idx] = -INFINITY;
            continue;
        }
        double s = 0.0;
        for (int h = 0; h < HI; ++h) {
            double dot = 0.0;
            for (int d = 0; d < DI; ++d) dot += q[((long)b * HI + h) * DI + d] * kx[(b * NB + j) * DI + d];
            s += w[(long)b * HI + h] * (dot > 0.0 ? dot : 0.0);
        }
        out[idx] = s;
    }
    return 0;
}

/*
 * Sparse core attention of the shared-KV form for one query per sequence at
 * position t = lens[b] - 1: one softmax over the selected entries (finalised
 * compressed entries, sel[b, i] >= 0; -1 entries are unused) and the raw
 * window of the last n_win tokens s in [max(0, lens - n_win), t] (finalised
 * at s), plus the sink; the output's RoPE dims turn back by -t.
 *   q [B, Hq, D]; ek [B, NB, 1, D]; sel [B, K]; k [B, T_hist, 1, D] raw history;
 *   sink [Hq] or NULL; gq, gkv [D] or NULL; out [B, Hq, D].
 * The window may cover tokens that a selected entry also summarises (the
 * two branches overlap).
 */
int orc_attend_sparse(const orc_config* c, int B, const double* q, const double* ek, long NB,
                      const long* sel, int K, const double* k, long T_hist, const long* lens,
                      const double* sink, const double* gq, const double* gkv, double* out)
{
    if (!cfg_ok(c) || !c->shared_kv || c->n_kv_heads != 1 || B < 0 || K < 0 || !q || !k || !lens || !out)
        return -1;
    if (K > 0 && (!sel || !ek)) return -1;
    const int Hq = c->n_q_heads, D = c->head_dim, w = c->n_win;
    const double scale = c->softmax_scale > 0 ? c->softmax_scale : 1.0 / sqrt((double)D);
    for (int b = 0; b < B; ++b) {
        if (lens[b] < 1 || lens[b] > T_hist) return -1;
        for (int i = 0; i < K; ++i)
            if (sel[(long)b * K + i] >= NB) return -1;
    }
    int err = 0;
    long total = (long)B * Hq;
#pragma omp parallel for schedule(dynamic, 4)
    for (long idx = 0; idx < total; ++idx) {
        const int h = (int)(idx % Hq);
        const long b = idx / Hq;
        const long t = lens[b] - 1;
        const long s0 = lens[b] - w > 0 ? lens[b] - w : 0;
        const long n = K + (t - s0 + 1);
        double* qt = malloc(sizeof(double) * D);
        double* rows = malloc(sizeof(double) * D * (size_t)(n > 0 ? n : 1));
        double* sc = malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        char* use = malloc((size_t)(n > 0 ? n : 1));
        double* o = out + (b * Hq + h) * (long)D;
        if (!qt || !rows || !sc || !use) {
            free(qt); free(rows); free(sc); free(use);
#pragma omp atomic write
            err = 1;
            continue;
        }
        memcpy(qt, q + (b * Hq + h) * (long)D, sizeof(double) * D);
        if (c->rmsnorm) rmsnorm(qt, D, gq, c->rms_eps);
        if (c->rope_dims) rope(qt, D, c->rope_dims, c->rope_theta, (double)t);
        /* the visible rows: selected entries, then the window */
        for (int i = 0; i < K; ++i) {
            long j = sel[b * K + i];
            use[i] = j >= 0;
            if (j >= 0) memcpy(rows + (long)i * D, ek + (b * NB + j) * (long)D, sizeof(double) * D);
        }
        for (long s = s0; s <= t; ++s) {
            double* r = rows + (K + (s - s0)) * (long)D;
            memcpy(r, k + (b * T_hist + s) * (long)D, sizeof(double) * D);
            finalise_key(c, r, gkv, (double)s);
            use[K + (s - s0)] = 1;
        }
        double smax = sink ? sink[h] : -INFINITY;
        for (long e = 0; e < n; ++e) {
            if (!use[e]) continue;
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += qt[d] * rows[e * D + d];
            sc[e] = acc * scale;
            if (sc[e] > smax) smax = sc[e];
        }
        double den = sink ? exp(sink[h] - smax) : 0.0;
        for (int d = 0; d < D; ++d) o[d] = 0.0;
        for (long e = 0; e < n; ++e) {
            if (!use[e]) continue;
            double p = exp(sc[e] - smax);
            den += p;
            for (int d = 0; d < D; ++d) o[d] += p * rows[e * D + d];
        }
        for (int d = 0; d < D; ++d) o[d] /= den;
        if (c->rope_dims) rope(o, D, c->rope_dims, c->rope_theta, -(double)t);
        free(qt); free(rows); free(sc); free(use);
    }
    return err ? -1 : 0;
}

/* ===================================================================== *
 * Backward of the prefill (pooling + attention), for training.          *
 * ("mSeek" README, "Experiment at a glance": the LBCA layers are trained *
 * by continued pretraining, so gradients flow through the pooling       *
 * weights Z, the positional bias B_pos, the raw keys and values, and the *
 * queries.)  Plain reverse-mode differentiation of orc_pool + orc_attend *
 * as written above, in fp64.                                            *
 * ===================================================================== */

/* dx of y = x * r * gamma, r = 1/sqrt(mean(x^2) + eps), given dy (all [D]). */
static void rmsnorm_bwd(const double* x, const double* dy, int D, const double* gamma, double eps, double* dx)
{
    double ss = 0.0, dot = 0.0;
    for (int d = 0; d < D; ++d) ss += x[d] * x[d];
    const double r = 1.0 / sqrt(ss / D + eps);
    for (int d = 0; d < D; ++d) dot += (gamma ? gamma[d] : 1.0) * dy[d] * x[d];
    for (int d = 0; d < D; ++d) dx[d] = r * (gamma ? gamma[d] : 1.0) * dy[d] - x[d] * r * r * r * dot / D;
}

/* d(input of the key finalisation) from d(finalised), at position pos. */
static void finalise_key_bwd(const orc_config* c, const double* raw, const double* dfin, const double* gamma,
                             double pos, double* dx)
{
    const int D = c->head_dim;
    double* t = malloc(sizeof(double) * D);
    memcpy(t, dfin, sizeof(double) * D);
    if (c->rope_dims) rope(t, D, c->rope_dims, c->rope_theta, -pos);  /* rotations are orthogonal */
    if (c->rmsnorm) rmsnorm_bwd(raw, t, D, gamma, c->rms_eps, dx);
    else memcpy(dx, t, sizeof(double) * D);
    free(t);
}

/*
 * Gradients of sum(dout * out) for out = the prefill of every row (all T
 * queries of each sequence), with respect to every input.
 *   q [B, T, Hq, D]; k, v, zk, zv [B, T, G, D] (v, zv NULL in the shared form);
 *   bpk, bpv [m, G*D]; sink [Hq] or NULL; gq, gkv [D] or NULL; dout [B, T, Hq, D].
 * Outputs (zeroed here; any may be NULL except dq): dq, dk, dv, dzk, dzv like
 * their inputs, dbk, dbv [m, G*D], dsink [Hq].  Gains are not differentiated.
 */
int orc_prefill_backward(const orc_config* c, int B, long T, const double* q, const double* k, const double* v,
                         const double* zk, const double* zv, const double* bpk, const double* bpv,
                         const double* sink, const double* gq, const double* gkv, const double* dout,
                         double* dq, double* dk, double* dv, double* dzk, double* dzv, double* dbk,
                         double* dbv, double* dsink)
{
    if (!cfg_ok(c) || B < 0 || T < 0 || !q || !k || !zk || !bpk || !dout || !dq) return -1;
    if (!c->shared_kv && (!v || !zv || !bpv)) return -1;
    const int Hq = c->n_q_heads, G = c->n_kv_heads, D = c->head_dim, m = c->block_m, w = c->n_win;
    const int r = Hq / G, S = c->shared_kv ? 1 : 2;
    const long NB = T / m, ts = (long)G * D;
    const double scale = c->softmax_scale > 0 ? c->softmax_scale : 1.0 / sqrt((double)D);
    const long nx = (long)B * T * ts;
    memset(dq, 0, sizeof(double) * (size_t)B * T * Hq * D);
    double* dX[2] = {dk, dv};
    double* dZ[2] = {dzk, dzv};
    double* dBp[2] = {dbk, dbv};
    /* scratch: the pooled and finalised entries, their gradients, the raw
       finalised keys and their gradients, the pooling weights */
    double* P = calloc((size_t)S * B * NB * ts + 1, sizeof(double));    /* pooled, before finalisation */
    double* E = calloc((size_t)S * B * NB * ts + 1, sizeof(double));    /* keys finalised; values as pooled */
    double* dE = calloc((size_t)S * B * NB * ts + 1, sizeof(double));
    double* Kf = calloc((size_t)nx + 1, sizeof(double));                /* raw keys finalised */
    double* dKf = calloc((size_t)nx + 1, sizeof(double));
    double* dVr = calloc((size_t)nx + 1, sizeof(double));               /* raw values (GQA) */
    double* Wt = calloc((size_t)S * B * NB * m * ts + 1, sizeof(double)); /* pooling weights [S][B][NB][m][G][D] */
    double* gX = calloc((size_t)S * nx + 1, sizeof(double));            /* d raw x of each series */
    double* gZ = calloc((size_t)S * nx + 1, sizeof(double));
    double* gB = calloc((size_t)S * m * ts + 1, sizeof(double));
    double* ds = calloc((size_t)Hq + 1, sizeof(double));
    double* qt = malloc(sizeof(double) * D);
    double* dqt = malloc(sizeof(double) * D);
    double* dof = malloc(sizeof(double) * D);
    double* o = malloc(sizeof(double) * D);
    double* sc = malloc(sizeof(double) * (size_t)(NB + T + 1));
    double* tmp = malloc(sizeof(double) * D);
    if (!P || !E || !dE || !Kf || !dKf || !dVr || !Wt || !gX || !gZ || !gB || !ds || !qt || !dqt || !dof || !o ||
        !sc || !tmp) {
        free(P); free(E); free(dE); free(Kf); free(dKf); free(dVr); free(Wt); free(gX); free(gZ); free(gB);
        free(ds); free(qt); free(dqt); free(dof); free(o); free(sc); free(tmp);
        return -1;
    }
    /* ---- forward: pooling weights, pooled and finalised entries, finalised raw keys ---- */
    for (int sr = 0; sr < S; ++sr) {
        const double* x = sr ? v : k;
        const double* z = sr ? zv : zk;
        const double* bp = sr ? bpv : bpk;
        for (int b = 0; b < B; ++b)
            for (long j = 0; j < NB; ++j)
                for (int g = 0; g < G; ++g)
                    for (int ch = 0; ch < D; ++ch) {
                        const long col = (long)g * D + ch;
                        double amax = -INFINITY;
                        for (int i = 0; i < m; ++i) {
                            double a = z[(b * T + j * m + i) * ts + col] + bp[i * ts + col];
                            if (a > amax) amax = a;
                        }
                        double den = 0.0, num = 0.0;
                        for (int i = 0; i < m; ++i)
                            den += exp(z[(b * T + j * m + i) * ts + col] + bp[i * ts + col] - amax);
                        for (int i = 0; i < m; ++i) {
                            double wi = exp(z[(b * T + j * m + i) * ts + col] + bp[i * ts + col] - amax) / den;
                            Wt[((((long)sr * B + b) * NB + j) * m + i) * ts + col] = wi;
                            num += wi * x[(b * T + j * m + i) * ts + col];
                        }
                        P[(((long)sr * B + b) * NB + j) * ts + col] = num;
                    }
        for (int b = 0; b < B; ++b)
            for (long j = 0; j < NB; ++j)
                for (int g = 0; g < G; ++g) {
                    const long o_ = (((long)sr * B + b) * NB + j) * ts + (long)g * D;
                    memcpy(E + o_, P + o_, sizeof(double) * D);
                    if (sr == 0) finalise_key(c, E + o_, gkv, (double)(j * m));
                }
    }
    for (long idx = 0; idx < (long)B * T * G; ++idx) {
        memcpy(Kf + idx * D, k + idx * D, sizeof(double) * D);
        finalise_key(c, Kf + idx * D, gkv, (double)((idx / G) % T));
    }
    /* ---- attention backward, row by row ---- */
    for (int b = 0; b < B; ++b)
        for (long t = 0; t < T; ++t)
            for (int h = 0; h < Hq; ++h) {
                const int g = h / r;
                const long L = t + 1, Pv = orc_visible_blocks(L, m, w), s0 = Pv * m;
                const long n = Pv + (t - s0 + 1);
                memcpy(qt, q + ((b * T + t) * Hq + h) * (long)D, sizeof(double) * D);
                if (c->rmsnorm) rmsnorm(qt, D, gq, c->rms_eps);
                if (c->rope_dims) rope(qt, D, c->rope_dims, c->rope_theta, (double)t);
                /* keys and values of the visible list, entry e */
#define KEY(e) ((e) < Pv ? E + (((long)0 * B + b) * NB + (e)) * ts + (long)g * D \
                         : Kf + (b * T + s0 + ((e) - Pv)) * ts + (long)g * D)
#define VAL(e) (c->shared_kv ? KEY(e) : ((e) < Pv ? E + (((long)1 * B + b) * NB + (e)) * ts + (long)g * D \
                                                  : v + (b * T + s0 + ((e) - Pv)) * ts + (long)g * D))
                double smax = sink ? sink[h] : -INFINITY;
                for (long e = 0; e < n; ++e) {
                    const double* kk = KEY(e);
                    double acc = 0.0;
                    for (int d = 0; d < D; ++d) acc += qt[d] * kk[d];
                    sc[e] = acc * scale;
                    if (sc[e] > smax) smax = sc[e];
                }
                double den = sink ? exp(sink[h] - smax) : 0.0;
                for (long e = 0; e < n; ++e) {
                    sc[e] = exp(sc[e] - smax);
                    den += sc[e];
                }
                for (long e = 0; e < n; ++e) sc[e] /= den;                     /* p_e */
                const double psink = sink ? exp(sink[h] - smax) / den : 0.0;
                for (int d = 0; d < D; ++d) o[d] = 0.0;
                for (long e = 0; e < n; ++e) {
                    const double* vv = VAL(e);
                    for (int d = 0; d < D; ++d) o[d] += sc[e] * vv[d];
                }
                /* d of o: the output of the shared form was turned back by -t */
                memcpy(dof, dout + ((b * T + t) * Hq + h) * (long)D, sizeof(double) * D);
                if (c->shared_kv && c->rope_dims) rope(dof, D, c->rope_dims, c->rope_theta, (double)t);
                double Dsum = 0.0;
                for (int d = 0; d < D; ++d) Dsum += dof[d] * o[d];
                for (int d = 0; d < D; ++d) dqt[d] = 0.0;
                for (long e = 0; e < n; ++e) {
                    const double* kk = KEY(e);
                    const double* vv = VAL(e);
                    double dp = 0.0;
                    for (int d = 0; d < D; ++d) dp += dof[d] * vv[d];
                    const double dS = sc[e] * (dp - Dsum);
                    double* dkey = e < Pv ? dE + (((long)0 * B + b) * NB + e) * ts + (long)g * D
                                          : dKf + (b * T + s0 + (e - Pv)) * ts + (long)g * D;
                    double* dval = c->shared_kv ? dkey
                                                : (e < Pv ? dE + (((long)1 * B + b) * NB + e) * ts + (long)g * D
                                                          : dVr + (b * T + s0 + (e - Pv)) * ts + (long)g * D);
                    for (int d = 0; d < D; ++d) {
                        dqt[d] += scale * dS * kk[d];
                        dkey[d] += scale * dS * qt[d];
                        dval[d] += sc[e] * dof[d];
                    }
                }
#undef KEY
#undef VAL
                ds[h] += -psink * Dsum;
                /* back through the query's RoPE at t and RMSNorm */
                double* dqo = dq + ((b * T + t) * Hq + h) * (long)D;
                const double* qraw = q + ((b * T + t) * Hq + h) * (long)D;
                if (c->rope_dims) rope(dqt, D, c->rope_dims, c->rope_theta, -(double)t);
                if (c->rmsnorm) rmsnorm_bwd(qraw, dqt, D, gq, c->rms_eps, dqo);
                else memcpy(dqo, dqt, sizeof(double) * D);
            }
    /* ---- raw keys and values: their own gradient, through the key finalisation ---- */
    for (long idx = 0; idx < (long)B * T * G; ++idx) {
        finalise_key_bwd(c, k + idx * D, dKf + idx * D, gkv, (double)((idx / G) % T), tmp);
        for (int d = 0; d < D; ++d) gX[idx * D + d] = tmp[d];
        if (!c->shared_kv)
            for (int d = 0; d < D; ++d) gX[nx + idx * D + d] = dVr[idx * D + d];
    }
    /* ---- pooled entries: through the finalisation, then the pooling softmax ---- */
    for (int sr = 0; sr < S; ++sr) {
        const double* x = sr ? v : k;
        for (int b = 0; b < B; ++b)
            for (long j = 0; j < NB; ++j)
                for (int g = 0; g < G; ++g) {
                    const long o_ = (((long)sr * B + b) * NB + j) * ts + (long)g * D;
                    if (sr == 0) finalise_key_bwd(c, P + o_, dE + o_, gkv, (double)(j * m), tmp);
                    else memcpy(tmp, dE + o_, sizeof(double) * D);
                    for (int ch = 0; ch < D; ++ch) {
                        const long col = (long)g * D + ch;
                        const double dPc = tmp[ch], Pc = P[o_ + ch];
                        for (int i = 0; i < m; ++i) {
                            const long tok = (b * T + j * m + i) * ts + col;
                            const double wi = Wt[((((long)sr * B + b) * NB + j) * m + i) * ts + col];
                            const double da = wi * (x[tok] - Pc) * dPc;
                            gX[(long)sr * nx + tok] += wi * dPc;
                            gZ[(long)sr * nx + tok] += da;
                            gB[((long)sr * m + i) * ts + col] += da;
                        }
                    }
                }
    }
    for (int sr = 0; sr < S; ++sr) {
        if (dX[sr]) memcpy(dX[sr], gX + (long)sr * nx, sizeof(double) * (size_t)nx);
        if (dZ[sr]) memcpy(dZ[sr], gZ + (long)sr * nx, sizeof(double) * (size_t)nx);
        if (dBp[sr]) memcpy(dBp[sr], gB + (long)sr * m * ts, sizeof(double) * (size_t)m * ts);
    }
    if (dsink) memcpy(dsink, ds, sizeof(double) * Hq);
    free(P); free(E); free(dE); free(Kf); free(dKf); free(dVr); free(Wt); free(gX); free(gZ); free(gB);
    free(ds); free(qt); free(dqt); free(dof); free(o); free(sc); free(tmp);
    return 0;
}
