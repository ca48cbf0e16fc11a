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
