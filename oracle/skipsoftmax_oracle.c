/*
 * Plain fp64 CPU oracle for Skip Softmax attention (prefill and decode).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or
 * call this file; it exists so that tests, the smoke check and the bench's CPU
 * baseline can check the CUDA kernels against an obviously correct program.
 * It shares no code, header, table or constant with the CUDA path.
 *
 * What it computes (source: "Accelerating Long-Context Inference with Skip
 * Softmax in NVIDIA TensorRT-LLM", Key Points and Detailed Analysis):
 *   attention scores S = Q K^T / sqrt(d) are visited one key block (tile) at a
 *   time, in ascending key order.  For each visited tile j the local maximum
 *   of every query row, mt_r = max_{k in tile} s_rk, is compared with the
 *   running row maximum m_r minus the threshold tau.  If every row of the row
 *   block has mt_r < m_r - tau (strict), the whole tile is skipped: none of its
 *   exponentials is formed and none of its values is accumulated.  Otherwise
 *   the usual online-softmax update runs:
 *        m' = max(m, mt);   l = l e^{m-m'} + sum_k e^{s-m'};
 *        acc = acc e^{m-m'} + sum_k e^{s-m'} v_k;   m = m'.
 *   The output row is acc / l.  (The page's comparison value is garbled in
 *   the transcript; it is read as m_i - tau, the running maximum minus the
 *   threshold the page calls Tau.)
 *
 * Conventions fixed where the page is silent:
 *   - causal attention is top-left aligned: query i sees keys k <= i; tiles
 *     whose first key lies beyond the last row of the row block are not
 *     visited at all (mask value 2);
 *   - a row whose running max is still -inf cannot be skipped (tile 0 is
 *     therefore always kept); a row whose tile max is -inf (fully masked in
 *     this tile) does not prevent skipping;
 *   - tau >= 0, tau = +inf means exact attention;
 *   - decode: the rows of the test are the g query heads that share one KV
 *     head; the key range is cut into splits of Ls keys, each split runs the
 *     tile loop with its own running max starting at -inf, and the split
 *     results are merged exactly (log-sum-exp).
 *   - decode rule variants (bits of `rule`; 0 is the rule above):
 *       ORACLE_RULE_PER_HEAD: each query head takes the test on its own row
 *         (skips its own exponentials and value sums); the shared value tile
 *         is needed iff some head of the group keeps the tile.  Mask and
 *         margin are then per query head, [B, Hq, tiles].
 *       ORACLE_RULE_SINK_SEED: every split's running max starts at the row
 *         maximum over the first key tile of the sequence (keys [0, Bt)),
 *         where attention sinks sit, instead of -inf; a split's first tile
 *         can then be skipped.  With one split (Ls >= L) this changes
 *         nothing, as tile 0 is that split's first tile.
 *
 * Every floating-point quantity is fp64; inputs are bf16 bit patterns that are
 * widened exactly.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_NO_MEMORY 2
#define ORACLE_RULE_PER_HEAD 1
#define ORACLE_RULE_SINK_SEED 2

/* bf16 -> fp64: a bf16 value is the top half of an IEEE fp32 word. */
static double widen_bf16(uint16_t bits)
{
    uint32_t w = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static double dot_widened(const uint16_t *a, const uint16_t *b, int d)
{
    double s = 0.0;
    for (int t = 0; t < d; ++t)
        s += widen_bf16(a[t]) * widen_bf16(b[t]);
    return s;
}

/* Contribution of one row to the tile margin  max_r (mt_r - m_r + tau).
 * The tile is skipped iff the maximum over rows is < 0.                   */
static double row_margin(double mt, double m, double tau)
{
    if (m == -INFINITY) return INFINITY;     /* nothing seen yet: never skippable */
    if (mt == -INFINITY) return -INFINITY;   /* row fully masked in this tile      */
    return mt - m + tau;                     /* tau = +inf gives +inf               */
}

/* ------------------------------------------------------------------------- */
/* Prefill                                                                   */
/* ------------------------------------------------------------------------- */

typedef struct {
    const uint16_t *Q, *K, *V;
    int B, Hq, Hkv, N, d, causal, Br, Bc;
    double tau;
    double *O, *O_exact, *margin, *pskip;
    uint8_t *mask;
} prefill_args;

/* One row block: rows [r0, r1) of query head h in batch b. */
static int prefill_row_block(const prefill_args *a, int b, int h, int rb)
{
    const int N = a->N, d = a->d, Br = a->Br, Bc = a->Bc;
    const int g = a->Hq / a->Hkv;
    const int kvh = h / g;                       /* query head h reads KV head floor(h/g) */
    const int n_rb = (N + Br - 1) / Br;
    const int n_tiles = (N + Bc - 1) / Bc;
    const int r0 = rb * Br;
    const int r1 = (r0 + Br < N) ? r0 + Br : N;
    const int nr = r1 - r0;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);

    const uint16_t *q = a->Q + ((size_t)(b * a->Hq + h) * N) * d;
    const uint16_t *k = a->K + ((size_t)(b * a->Hkv + kvh) * N) * d;
    const uint16_t *v = a->V + ((size_t)(b * a->Hkv + kvh) * N) * d;

    double *m = malloc(sizeof(double) * nr);
    double *l = malloc(sizeof(double) * nr);
    double *acc = calloc((size_t)nr * d, sizeof(double));
    double *s = malloc(sizeof(double) * (size_t)nr * Bc);
    double *mt = malloc(sizeof(double) * nr);
    uint8_t *skipped = calloc(n_tiles, 1);
    if (!m || !l || !acc || !s || !mt || !skipped) {
        free(m); free(l); free(acc); free(s); free(mt); free(skipped);
        return ORACLE_NO_MEMORY;
    }
    for (int r = 0; r < nr; ++r) { m[r] = -INFINITY; l[r] = 0.0; }

    const size_t tile_base = (((size_t)b * a->Hq + h) * n_rb + rb) * n_tiles;

    for (int j = 0; j < n_tiles; ++j) {
        const int c0 = j * Bc;
        const int c1 = (c0 + Bc < N) ? c0 + Bc : N;
        if (a->causal && c0 > r1 - 1) {          /* tile lies wholly above the diagonal */
            if (a->mask) a->mask[tile_base + j] = 2;
            if (a->margin) a->margin[tile_base + j] = NAN;
            continue;
        }
        /* scores of this tile and the local (tile) maximum of every row */
        for (int r = 0; r < nr; ++r) {
            const int qi = r0 + r;
            mt[r] = -INFINITY;
            for (int c = c0; c < c1; ++c) {
                double x;
                if (a->causal && c > qi) x = -INFINITY;
                else x = dot_widened(q + (size_t)qi * d, k + (size_t)c * d, d) * inv_sqrt_d;
                s[(size_t)r * Bc + (c - c0)] = x;
                if (x > mt[r]) mt[r] = x;
            }
        }
        /* the block-skip test */
        double margin = -INFINITY;
        for (int r = 0; r < nr; ++r) {
            double x = row_margin(mt[r], m[r], a->tau);
            if (x > margin) margin = x;
        }
        const int skip = margin < 0.0;
        if (a->mask) a->mask[tile_base + j] = (uint8_t)skip;
        if (a->margin) a->margin[tile_base + j] = margin;
        if (skip) { skipped[j] = 1; continue; }

        /* online-softmax update with this tile */
        for (int r = 0; r < nr; ++r) {
            const double m_new = (mt[r] > m[r]) ? mt[r] : m[r];
            if (m_new == -INFINITY) continue;    /* row has seen no visible key yet */
            const double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - m_new);
            l[r] *= alpha;
            double *ar = acc + (size_t)r * d;
            for (int t = 0; t < d; ++t) ar[t] *= alpha;
            for (int c = c0; c < c1; ++c) {
                const double x = s[(size_t)r * Bc + (c - c0)];
                if (x == -INFINITY) continue;
                const double p = exp(x - m_new);
                l[r] += p;
                const uint16_t *vc = v + (size_t)c * d;
                for (int t = 0; t < d; ++t) ar[t] += p * widen_bf16(vc[t]);
            }
            m[r] = m_new;
        }
    }

    for (int r = 0; r < nr; ++r) {
        double *o = a->O + ((size_t)(b * a->Hq + h) * N + r0 + r) * d;
        for (int t = 0; t < d; ++t) o[t] = acc[(size_t)r * d + t] / l[r];
    }

    /* exact attention (every visible key) and the probability mass the skip
     * removed, both straight from the softmax definition                     */
    if (a->O_exact || a->pskip) {
        double *w = malloc(sizeof(double) * N);
        double *ex = malloc(sizeof(double) * d);
        if (!w || !ex) { free(w); free(ex); free(m); free(l); free(acc); free(s); free(mt); free(skipped); return ORACLE_NO_MEMORY; }
        for (int r = 0; r < nr; ++r) {
            const int qi = r0 + r;
            const int kend = a->causal ? qi + 1 : N;
            double M = -INFINITY;
            for (int c = 0; c < kend; ++c) {
                w[c] = dot_widened(q + (size_t)qi * d, k + (size_t)c * d, d) * inv_sqrt_d;
                if (w[c] > M) M = w[c];
            }
            double total = 0.0, lost = 0.0;
            for (int t = 0; t < d; ++t) ex[t] = 0.0;
            for (int c = 0; c < kend; ++c) {
                const double p = exp(w[c] - M);
                total += p;
                if (skipped[c / Bc]) lost += p;
                const uint16_t *vc = v + (size_t)c * d;
                for (int t = 0; t < d; ++t) ex[t] += p * widen_bf16(vc[t]);
            }
            const size_t row = (size_t)(b * a->Hq + h) * N + qi;
            if (a->O_exact)
                for (int t = 0; t < d; ++t) a->O_exact[row * d + t] = ex[t] / total;
            if (a->pskip) a->pskip[row] = lost / total;
        }
        free(w); free(ex);
    }

    free(m); free(l); free(acc); free(s); free(mt); free(skipped);
    return ORACLE_OK;
}

/*
 * Q [B,Hq,N,d], K/V [B,Hkv,N,d] bf16 bits, contiguous, d fastest.
 * units: NULL for every row block, else n_units triples (b, h, rb).
 * O [B,Hq,N,d] fp64 (required).  Optional (may be NULL):
 *   O_exact [B,Hq,N,d]      exact attention (no skipping)
 *   mask    [B,Hq,nRB,nT]   0 kept, 1 skipped, 2 not visited (causal)
 *   margin  [B,Hq,nRB,nT]   max_r (mt_r - m_r + tau), NaN if not visited
 *   pskip   [B,Hq,N]        softmax probability mass in skipped tiles
 * Only the entries belonging to the computed row blocks are written.
 */
int oracle_prefill(const uint16_t *Q, const uint16_t *K, const uint16_t *V,
                   int B, int Hq, int Hkv, int N, int d, int causal, double tau,
                   int Br, int Bc, const int32_t *units, int64_t n_units,
                   double *O, double *O_exact, uint8_t *mask, double *margin,
                   double *pskip, int nthreads)
{
    if (!Q || !K || !V || !O) return ORACLE_BAD_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || N <= 0 || d <= 0 || Br <= 0 || Bc <= 0) return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0) return ORACLE_BAD_ARG;
    if (isnan(tau) || tau < 0.0) return ORACLE_BAD_ARG;

    prefill_args a = {Q, K, V, B, Hq, Hkv, N, d, causal, Br, Bc, tau, O, O_exact, margin, pskip, mask};
    const int n_rb = (N + Br - 1) / Br;
    const int64_t total = units ? n_units : (int64_t)B * Hq * n_rb;
    int status = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t u = 0; u < total; ++u) {
        int b, h, rb;
        if (units) { b = units[3 * u]; h = units[3 * u + 1]; rb = units[3 * u + 2]; }
        else { rb = (int)(u % n_rb); h = (int)((u / n_rb) % Hq); b = (int)(u / ((int64_t)n_rb * Hq)); }
        int st;
        if (b < 0 || b >= B || h < 0 || h >= Hq || rb < 0 || rb >= n_rb) st = ORACLE_BAD_ARG;
        else st = prefill_row_block(&a, b, h, rb);
        if (st != ORACLE_OK) {
#pragma omp critical
            status = st;
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* Decode                                                                    */
/* ------------------------------------------------------------------------- */

/*
 * q [B,Hq,d]; K/V [B,Hkv,L,d]; one query token per (batch, query head) that
 * attends to all L cached keys.  Rows of the skip test: the g = Hq/Hkv query
 * heads of one KV head.  Splits of Ls keys, tiles of Bt keys inside a split.
 * o [B,Hq,d] fp64.  Optional: o_exact [B,Hq,d]; mask/margin [B,Hkv,ceil(L/Bt)]
 * (tiles are numbered globally: tile j covers keys [j*Bt, (j+1)*Bt) cut at the
 * split end, so Ls must be a multiple of Bt); pskip [B,Hq].  With
 * ORACLE_RULE_PER_HEAD in `rule`, mask and margin are [B,Hq,ceil(L/Bt)].
 */
int oracle_decode(const uint16_t *q, const uint16_t *K, const uint16_t *V,
                  int B, int Hq, int Hkv, int L, int d, double tau, int Ls, int Bt,
                  int rule, double *o, double *o_exact, uint8_t *mask, double *margin,
                  double *pskip, int nthreads)
{
    const int per_head = (rule & ORACLE_RULE_PER_HEAD) != 0;
    const int seeded = (rule & ORACLE_RULE_SINK_SEED) != 0;
    if (rule & ~(ORACLE_RULE_PER_HEAD | ORACLE_RULE_SINK_SEED)) return ORACLE_BAD_ARG;
    if (!q || !K || !V || !o) return ORACLE_BAD_ARG;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || L <= 0 || d <= 0 || Ls <= 0 || Bt <= 0) return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0 || Ls % Bt != 0) return ORACLE_BAD_ARG;
    if (isnan(tau) || tau < 0.0) return ORACLE_BAD_ARG;
    const int g = Hq / Hkv;
    const int n_tiles = (L + Bt - 1) / Bt;
    const int n_splits = (L + Ls - 1) / Ls;
    const double inv_sqrt_d = 1.0 / sqrt((double)d);
    int status = ORACLE_OK;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t grp = 0; grp < (int64_t)B * Hkv; ++grp) {
        const int b = (int)(grp / Hkv), kvh = (int)(grp % Hkv);
        const uint16_t *k = K + ((size_t)(b * Hkv + kvh) * L) * d;
        const uint16_t *v = V + ((size_t)(b * Hkv + kvh) * L) * d;
        double *s = malloc(sizeof(double) * (size_t)L * g);       /* all scores, [key][row] */
        double *m = malloc(sizeof(double) * g), *l = malloc(sizeof(double) * g);
        double *acc = malloc(sizeof(double) * (size_t)g * d);
        double *sm = malloc(sizeof(double) * (size_t)n_splits * g);   /* per-split max   */
        double *sl = malloc(sizeof(double) * (size_t)n_splits * g);   /* per-split sum   */
        double *sa = malloc(sizeof(double) * (size_t)n_splits * g * d);/* per-split acc  */
        double *mt = malloc(sizeof(double) * g);
        uint8_t *skipped = calloc((size_t)n_tiles * g, 1);  /* [row][tile] */
        double *seed = malloc(sizeof(double) * g);
        if (!s || !m || !l || !acc || !sm || !sl || !sa || !mt || !skipped || !seed) {
#pragma omp critical
            status = ORACLE_NO_MEMORY;
            free(s); free(m); free(l); free(acc); free(sm); free(sl); free(sa); free(mt); free(skipped);
            free(seed);
            continue;
        }
        for (int c = 0; c < L; ++c)
            for (int r = 0; r < g; ++r) {
                const uint16_t *qr = q + ((size_t)b * Hq + (size_t)kvh * g + r) * d;
                s[(size_t)c * g + r] = dot_widened(qr, k + (size_t)c * d, d) * inv_sqrt_d;
            }
        /* sink seed: row maximum over the first key tile of the sequence */
        for (int r = 0; r < g; ++r) {
            seed[r] = -INFINITY;
            for (int c = 0; c < Bt && c < L; ++c)
                if (s[(size_t)c * g + r] > seed[r]) seed[r] = s[(size_t)c * g + r];
        }
        for (int sp = 0; sp < n_splits; ++sp) {
            const int k0 = sp * Ls, k1 = (k0 + Ls < L) ? k0 + Ls : L;
            for (int r = 0; r < g; ++r) { m[r] = seeded ? seed[r] : -INFINITY; l[r] = 0.0; }
            for (size_t t = 0; t < (size_t)g * d; ++t) acc[t] = 0.0;
            for (int c0 = k0; c0 < k1; c0 += Bt) {
                const int c1 = (c0 + Bt < k1) ? c0 + Bt : k1;
                const int j = c0 / Bt;
                double margin_j = -INFINITY;
                for (int r = 0; r < g; ++r) {
                    mt[r] = -INFINITY;
                    for (int c = c0; c < c1; ++c)
                        if (s[(size_t)c * g + r] > mt[r]) mt[r] = s[(size_t)c * g + r];
                    double x = row_margin(mt[r], m[r], tau);
                    if (x > margin_j) margin_j = x;
                }
                if (per_head) {
                    /* each row decides for itself; margins per query head */
                    for (int r = 0; r < g; ++r) {
                        const double x = row_margin(mt[r], m[r], tau);
                        const size_t ti = ((size_t)b * Hq + (size_t)kvh * g + r) * n_tiles + j;
                        if (mask) mask[ti] = (uint8_t)(x < 0.0);
                        if (margin) margin[ti] = x;
                    }
                } else {
                    const int skip = margin_j < 0.0;
                    const size_t ti = (size_t)(b * Hkv + kvh) * n_tiles + j;
                    if (mask) mask[ti] = (uint8_t)skip;
                    if (margin) margin[ti] = margin_j;
                    if (skip) {
                        for (int r = 0; r < g; ++r) skipped[(size_t)r * n_tiles + j] = 1;
                        continue;
                    }
                }
                for (int r = 0; r < g; ++r) {
                    if (per_head && row_margin(mt[r], m[r], tau) < 0.0) {
                        skipped[(size_t)r * n_tiles + j] = 1;
                        continue;
                    }
                    const double m_new = (mt[r] > m[r]) ? mt[r] : m[r];
                    const double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - m_new);
                    l[r] *= alpha;
                    for (int t = 0; t < d; ++t) acc[(size_t)r * d + t] *= alpha;
                    for (int c = c0; c < c1; ++c) {
                        const double p = exp(s[(size_t)c * g + r] - m_new);
                        l[r] += p;
                        for (int t = 0; t < d; ++t) acc[(size_t)r * d + t] += p * widen_bf16(v[(size_t)c * d + t]);
                    }
                    m[r] = m_new;
                }
            }
            for (int r = 0; r < g; ++r) {
                sm[(size_t)sp * g + r] = m[r];
                sl[(size_t)sp * g + r] = l[r];
                for (int t = 0; t < d; ++t) sa[((size_t)sp * g + r) * d + t] = acc[(size_t)r * d + t];
            }
        }
        /* exact merge of the splits: rescale each to the common maximum */
        for (int r = 0; r < g; ++r) {
            double M = -INFINITY;
            for (int sp = 0; sp < n_splits; ++sp)
                if (sm[(size_t)sp * g + r] > M) M = sm[(size_t)sp * g + r];
            double den = 0.0;
            double *orow = o + ((size_t)b * Hq + (size_t)kvh * g + r) * d;
            for (int t = 0; t < d; ++t) orow[t] = 0.0;
            for (int sp = 0; sp < n_splits; ++sp) {
                if (sl[(size_t)sp * g + r] == 0.0) continue;  /* every tile of the split skipped */
                const double w = exp(sm[(size_t)sp * g + r] - M);
                den += w * sl[(size_t)sp * g + r];
                for (int t = 0; t < d; ++t) orow[t] += w * sa[((size_t)sp * g + r) * d + t];
            }
            for (int t = 0; t < d; ++t) orow[t] /= den;
        }
        /* exact attention and skipped probability mass, from the definition */
        if (o_exact || pskip) {
            for (int r = 0; r < g; ++r) {
                double M = -INFINITY;
                for (int c = 0; c < L; ++c) if (s[(size_t)c * g + r] > M) M = s[(size_t)c * g + r];
                double total = 0.0, lost = 0.0;
                for (int t = 0; t < d; ++t) acc[t] = 0.0;
                for (int c = 0; c < L; ++c) {
                    const double p = exp(s[(size_t)c * g + r] - M);
                    total += p;
                    if (skipped[(size_t)r * n_tiles + c / Bt]) lost += p;
                    for (int t = 0; t < d; ++t) acc[t] += p * widen_bf16(v[(size_t)c * d + t]);
                }
                const size_t row = (size_t)b * Hq + (size_t)kvh * g + r;
                if (o_exact) for (int t = 0; t < d; ++t) o_exact[row * d + t] = acc[t] / total;
                if (pskip) pskip[row] = lost / total;
            }
        }
        free(s); free(m); free(l); free(acc); free(sm); free(sl); free(sa); free(mt); free(skipped);
        free(seed);
    }
    return status;
}

/*
 * e4m3 quantisation for the FP8 Q K^T path (the page names FP8 attention as
 * the path the skip rule combines with; the scale rule is this library's
 * own, stated here in full).
 *
 * Format (OCP 8-bit floating point, E4M3): sign bit, 4 exponent bits with
 * bias 7, 3 mantissa bits; exponent field 0 holds the subnormals
 * m * 2^-9 (m = 0..7); field 15 with mantissa 7 is NaN; there are no
 * infinities, and the largest finite value is 1.75 * 2^8 = 448.
 *
 * Quantisation of one group x[0..n): s = 2^k with k the smallest integer
 * >= -126 such that max|x| <= 448 * 2^k (s = 1 for a group of zeros, NaN for
 * a group holding inf or NaN); code_i = the e4m3 value nearest to x_i / s,
 * ties to the code with an even mantissa.
 */
double oracle_e4m3_value(uint8_t code)
{
    const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

/* Nearest code to y (|y| <= 448), ties to even: the non-negative codes
 * 0..126 are in increasing order of value, so find (by bisection) the last
 * code whose value does not exceed |y| and compare it with the next one. */
static uint8_t e4m3_nearest(double y)
{
    const double a = fabs(y);
    int lo = 0, hi = 126;  /* value(lo) <= a always; the answer lies in [lo, hi] */
    while (lo < hi) {
        const int mid = (lo + hi + 1) / 2;
        if (oracle_e4m3_value((uint8_t)mid) <= a)
            lo = mid;
        else
            hi = mid - 1;
    }
    int c = lo;
    if (lo < 126) {
        const double dl = a - oracle_e4m3_value((uint8_t)lo);
        const double dh = oracle_e4m3_value((uint8_t)(lo + 1)) - a;
        if (dh < dl || (dh == dl && ((lo + 1) & 1) == 0))
            c = lo + 1;
    }
    return (uint8_t)(c | ((y < 0 || (y == 0 && signbit(y))) ? 0x80 : 0));
}

int oracle_quantize_e4m3(const uint16_t *x, int64_t groups, int64_t group_elems, uint8_t *q,
                         double *scales)
{
    if (!x || !q || !scales || groups <= 0 || group_elems <= 0)
        return ORACLE_BAD_ARG;
    for (int64_t g = 0; g < groups; ++g) {
        const uint16_t *xg = x + g * group_elems;
        double amax = 0.0;
        int finite = 1;
        for (int64_t i = 0; i < group_elems; ++i) {
            const double v = widen_bf16(xg[i]);
            if (!isfinite(v))
                finite = 0;
            else if (fabs(v) > amax)
                amax = fabs(v);
        }
        double s;
        if (!finite) {
            s = NAN;
        } else if (amax == 0.0) {
            s = 1.0;
        } else {
            int k = -126;
            while (amax > ldexp(448.0, k))
                ++k;
            s = ldexp(1.0, k);
        }
        scales[g] = s;
        for (int64_t i = 0; i < group_elems; ++i)
            q[g * group_elems + i] = finite ? e4m3_nearest(widen_bf16(xg[i]) / s) : 0x7f;
    }
    return ORACLE_OK;
}

/*
 * int8 quantisation for the integer Q K^T path ("TurboAttention", Technical
 * Deep Dive, quantises Q and K to integers inside the tile loop; the scale
 * rule is this library's own, stated here in full): s = 2^k with k the
 * smallest integer >= -126 such that max|x| <= 127 * 2^k (s = 1 for a group of
 * zeros, NaN for a group holding inf or NaN); code_i = the integer nearest
 * x_i / s, ties to the even integer, as a two's-complement byte (|code| <= 127).
 */
static int8_t nearest_int_even(double y)
{
    const double f = floor(y);
    const double r = y - f;  /* exact: y has few significant bits */
    double n;
    if (r < 0.5)
        n = f;
    else if (r > 0.5)
        n = f + 1.0;
    else
        n = (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
    return (int8_t)n;
}

int oracle_quantize_i8(const uint16_t *x, int64_t groups, int64_t group_elems, int8_t *q,
                       double *scales)
{
    if (!x || !q || !scales || groups <= 0 || group_elems <= 0)
        return ORACLE_BAD_ARG;
    for (int64_t g = 0; g < groups; ++g) {
        const uint16_t *xg = x + g * group_elems;
        double amax = 0.0;
        int finite = 1;
        for (int64_t i = 0; i < group_elems; ++i) {
            const double v = widen_bf16(xg[i]);
            if (!isfinite(v))
                finite = 0;
            else if (fabs(v) > amax)
                amax = fabs(v);
        }
        double s;
        if (!finite) {
            s = NAN;
        } else if (amax == 0.0) {
            s = 1.0;
        } else {
            int k = -126;
            while (amax > ldexp(127.0, k))
                ++k;
            s = ldexp(1.0, k);
        }
        scales[g] = s;
        for (int64_t i = 0; i < group_elems; ++i)
            q[g * group_elems + i] = finite ? nearest_int_even(widen_bf16(xg[i]) / s) : 0;
    }
    return ORACLE_OK;
}
