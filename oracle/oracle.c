/*
 * oracle.c -- plain, slow, double-precision CPU oracle for selector-driven
 * block-sparse attention.  TEST INFRASTRUCTURE ONLY: the test-suite, the
 * smoke check and the benchmark's CPU-baseline leg are the only callers.  It
 * shares no code, header, table or constant with the CUDA library.
 *
 * Pages followed (cited by title and section):
 *   [SAS]  "Учёные научили трансформеры отбирать контекст напрямую, а не через
 *          имитацию полного внимания" -- opening section (a light selector
 *          scores context units, hard top-K keeps the best; the gate enters the
 *          attention logits, inside the softmax, in log form, normalised
 *          against the always-kept current block), "Ключевые факты",
 *          "Как это применить".
 *   [HiLS] "HiLS-Attention: иерархическое разреженное внимание для
 *          сверхдлинного контекста в языковых моделях" -- opening section
 *          (each query reads every selected chunk on its own; the per-chunk
 *          results are combined with weights given by the chunks' retrieval
 *          scores), "Ключевые факты".
 *   [LSA]  the Latent Sparse Attention post (rit.work) -- section
 *          "Индекс перестаёт перебирать весь контекст" (adjacent keys are
 *          pooled before scoring; the start of the context and the recent
 *          window are always added).
 *
 * The pages print no formula.  The concrete forms used here are the plainest
 * ones consistent with them: landmark = mean of the block's keys; score =
 * scaled dot product of the pooled query with the landmark; gate =
 * log_sigmoid(s_b - s_local) on selected blocks; hierarchical weights =
 * softmax of the retrieval scores.  Every arithmetic step runs in double.
 *
 * Flag bits (the same numbers the C ABI publishes; defined here on their own):
 *   1 sink block 0 always kept, 2 local block always kept, 4 gate on,
 *   8 hierarchical mode, 16 causal mask inside the local block.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_SINK 1
#define ORC_LOCAL 2
#define ORC_GATE 4
#define ORC_HIER 8
#define ORC_CAUSAL 16

/* Round a double to the nearest bfloat16 value (ties to even), returned as a
 * double.  bfloat16 keeps 8 significant bits and fp32's exponent range. */
double orc_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                  /* x = m * 2^e, 0.5 <= |m| < 1 */
    int qexp = e - 8;              /* weight of the last kept bit */
    if (qexp < -133) qexp = -133;  /* bfloat16 subnormal quantum 2^-133 */
    double q = ldexp(1.0, qexp);
    double r = rint(x / q) * q;    /* rint: current mode, ties to even */
    if (fabs(r) > 3.3895313892515355e38) r = copysign(INFINITY, x);
    return r;
}

static double store_round(double x, int mode)
{
    if (mode == 1) return orc_round_bf16(x);
    if (mode == 2) return (double)(float)x;
    return x;
}

/* Landmarks of one (batch, kv-head): the mean of each block's keys.
 * [HiLS] names the per-chunk summary a landmark; [LSA] pools adjacent keys
 * before scoring.  A ragged last block averages only the keys that exist.
 *   k   [n][d] keys;  lmk [ceil(n/bs)][d] out;
 *   round_mode 0 keep double, 1 round to bfloat16, 2 round to fp32. */
void orc_landmarks(const double *k, long n, int d, int bs, int round_mode,
                   double *lmk)
{
    long nb = (n + bs - 1) / bs;
    for (long b = 0; b < nb; ++b) {
        long t0 = b * bs, t1 = t0 + bs < n ? t0 + bs : n;
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (long t = t0; t < t1; ++t) s += k[t * d + c];
            lmk[b * d + c] = store_round(s / (double)(t1 - t0), round_mode);
        }
    }
}

/* Pooled query of one selection unit: the mean over `nheads` query heads and
 * query rows [row0, row0 + nrows) (clipped to n).  q [nheads][n][d]. */
void orc_pool_queries(const double *q, int nheads, long n, int d, long row0,
                      int nrows, double *qbar)
{
    long r1 = row0 + nrows < n ? row0 + nrows : n;
    double cnt = (double)nheads * (double)(r1 - row0);
    for (int c = 0; c < d; ++c) {
        double s = 0.0;
        for (int h = 0; h < nheads; ++h)
            for (long r = row0; r < r1; ++r) s += q[((long)h * n + r) * d + c];
        qbar[c] = s / cnt;
    }
}

/* log(sigmoid(x)) without overflow. */
double orc_log_sigmoid(double x)
{
    return x >= 0.0 ? -log1p(exp(-x)) : x - log1p(exp(x));
}

typedef struct { float key; int idx; } cand_t;

static int cand_cmp(const void *pa, const void *pb)
{
    const cand_t *a = (const cand_t *)pa, *b = (const cand_t *)pb;
    if (a->key > b->key) return -1;     /* higher score first */
    if (a->key < b->key) return 1;
    return a->idx < b->idx ? -1 : (a->idx > b->idx); /* then lower index */
}

static int int_cmp(const void *pa, const void *pb)
{
    int a = *(const int *)pa, b = *(const int *)pb;
    return (a > b) - (a < b);
}

/* Selection for one unit whose own (current / local) block is `local`.
 *
 *   score s_b = scale * <qbar, lmk[b]> for b = 0..local            [SAS]
 *   candidates: blocks before `local`, block 0 excluded when the sink is
 *   forced; hard top-K of the candidates by (score desc, index asc), the
 *   comparison taken on scores rounded to fp32 (the precision in which the
 *   GPU decides); forced blocks: 0 with ORC_SINK [LSA], `local` with
 *   ORC_LOCAL [SAS].  The kept list is sorted ascending without duplicates.
 *   gate of a selected block = log_sigmoid(s_b - s_local) with ORC_GATE
 *   [SAS: inside the softmax, log form, normalised against the current
 *   block]; forced blocks carry gate 0.
 *
 * Outputs (capacity top_k + 2): idx, sc (= s_b of each kept block), gate.
 * *rel_gap = (s_(K) - s_(K+1)) / max(|s_(K)|, 1e-30) over the fp32 decision
 * keys when more than K candidates exist, else +inf.  s_all (capacity
 * local + 1, may be NULL) receives every score.  Returns the kept count. */
int orc_select(const double *qbar, const double *lmk, int d, int local,
               int top_k, int flags, double scale, int *idx, double *sc,
               double *gate, double *rel_gap, double *s_all)
{
    double *s = (double *)malloc(sizeof(double) * (size_t)(local + 1));
    for (int b = 0; b <= local; ++b) {
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qbar[c] * lmk[(long)b * d + c];
        s[b] = scale * acc;
        if (s_all) s_all[b] = s[b];
    }
    int first = (flags & ORC_SINK) ? 1 : 0;
    int ncand = local - first > 0 ? local - first : 0;
    cand_t *cand = (cand_t *)malloc(sizeof(cand_t) * (size_t)(ncand + 1));
    for (int i = 0; i < ncand; ++i) {
        cand[i].key = (float)s[first + i];
        cand[i].idx = first + i;
    }
    qsort(cand, (size_t)ncand, sizeof(cand_t), cand_cmp);
    int nsel = top_k < ncand ? top_k : ncand;
    if (nsel < 0) nsel = 0;
    *rel_gap = INFINITY;
    if (top_k > 0 && ncand > top_k) {
        double a = cand[top_k - 1].key, b = cand[top_k].key;
        double den = fabs(a) > 1e-30 ? fabs(a) : 1e-30;
        *rel_gap = (a - b) / den;
    }
    int *kept = (int *)malloc(sizeof(int) * (size_t)(nsel + 2));
    char *is_sel = (char *)calloc((size_t)(local + 1), 1);
    int cnt = 0;
    for (int i = 0; i < nsel; ++i) {
        kept[cnt++] = cand[i].idx;
        is_sel[cand[i].idx] = 1;
    }
    if (flags & ORC_SINK) kept[cnt++] = 0;
    if ((flags & ORC_LOCAL) && !((flags & ORC_SINK) && local == 0))
        kept[cnt++] = local;
    qsort(kept, (size_t)cnt, sizeof(int), int_cmp);
    for (int i = 0; i < cnt; ++i) {
        int b = kept[i];
        idx[i] = b;
        sc[i] = s[b];
        gate[i] = ((flags & ORC_GATE) && is_sel[b])
                      ? orc_log_sigmoid(s[b] - s[local]) : 0.0;
    }
    free(is_sel);
    free(kept);
    free(cand);
    free(s);
    return cnt;
}

/* Is key t of kept block b visible from query position i? */
static int visible(long t, long i, int b, int local, int flags)
{
    return !((flags & ORC_CAUSAL) && b == local && t > i);
}

/* Gated block-sparse attention for `nrows` query rows that share one kept
 * list.  For query position i and key t of kept block b (t < n, and t <= i
 * inside the local block when causal):
 *     z_t = scale * <q_i, k_t> + gate_b,     O_i = softmax(z) V,
 *     LSE_i = log sum_t exp(z_t)
 * -- the gate sits inside the softmax as an additive log-domain term [SAS].
 * An empty key set gives O = 0, LSE = -inf.
 *   q [nrows][d]; qpos [nrows]; k, v [n][d] of the row's kv-head;
 *   o [nrows][d]; lse [nrows]. */
void orc_attend_gated(const double *q, int nrows, const long *qpos,
                      const double *k, const double *v, long n, int d, int bs,
                      int local, const int *idx, const double *gate,
                      int count, int flags, double scale, double *o,
                      double *lse)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)count * bs + 1);
    long *tk = (long *)malloc(sizeof(long) * (size_t)count * bs + 1);
    for (int r = 0; r < nrows; ++r) {
        const double *qi = q + (long)r * d;
        long i = qpos[r];
        int m = 0;
        for (int c = 0; c < count; ++c) {
            int b = idx[c];
            long t1 = (long)(b + 1) * bs < n ? (long)(b + 1) * bs : n;
            for (long t = (long)b * bs; t < t1; ++t) {
                if (!visible(t, i, b, local, flags)) continue;
                double dot = 0.0;
                for (int e = 0; e < d; ++e) dot += qi[e] * k[t * d + e];
                z[m] = scale * dot + gate[c];
                tk[m] = t;
                ++m;
            }
        }
        double *oi = o + (long)r * d;
        for (int e = 0; e < d; ++e) oi[e] = 0.0;
        if (m == 0) { lse[r] = -INFINITY; continue; }
        double mx = z[0];
        for (int u = 1; u < m; ++u) mx = z[u] > mx ? z[u] : mx;
        double den = 0.0;
        for (int u = 0; u < m; ++u) {
            double p = exp(z[u] - mx);
            den += p;
            for (int e = 0; e < d; ++e) oi[e] += p * v[tk[u] * d + e];
        }
        for (int e = 0; e < d; ++e) oi[e] /= den;
        lse[r] = mx + log(den);
    }
    free(tk);
    free(z);
}

/* Hierarchical (HiLS-style) attention for `nrows` query rows that share one
 * kept list [HiLS]: every kept block b is read on its own,
 *     o_b = softmax_{t in b visible}(scale * <q_i, k_t>) V_b,
 * and the block outputs are combined with weights w = softmax_b(sc_b) of the
 * retrieval scores:  O_i = sum_b w_b o_b.  No gate is applied.  LSE_i is the
 * log-sum-exp of the retrieval scores of the blocks that contribute.  A block
 * with no visible key (not reachable with the candidate rules) contributes
 * nothing; no contributing block gives O = 0, LSE = -inf. */
void orc_attend_hier(const double *q, int nrows, const long *qpos,
                     const double *k, const double *v, long n, int d, int bs,
                     int local, const int *idx, const double *sc, int count,
                     int flags, double scale, double *o, double *lse)
{
    double *z = (double *)malloc(sizeof(double) * (size_t)bs);
    double *ob = (double *)malloc(sizeof(double) * (size_t)count * d + 1);
    char *has = (char *)malloc((size_t)count + 1);
    for (int r = 0; r < nrows; ++r) {
        const double *qi = q + (long)r * d;
        long i = qpos[r];
        for (int c = 0; c < count; ++c) {
            int b = idx[c];
            long t0 = (long)b * bs;
            long t1 = t0 + bs < n ? t0 + bs : n;
            int m = 0;
            double mx = -INFINITY;
            for (long t = t0; t < t1; ++t) {
                double dot = -INFINITY;
                if (visible(t, i, b, local, flags)) {
                    dot = 0.0;
                    for (int e = 0; e < d; ++e) dot += qi[e] * k[t * d + e];
                    dot *= scale;
                    ++m;
                    mx = dot > mx ? dot : mx;
                }
                z[t - t0] = dot;
            }
            has[c] = m > 0;
            double *o_b = ob + (long)c * d;
            for (int e = 0; e < d; ++e) o_b[e] = 0.0;
            if (!m) continue;
            double den = 0.0;
            for (long t = t0; t < t1; ++t) {
                if (z[t - t0] == -INFINITY) continue;
                double p = exp(z[t - t0] - mx);
                den += p;
                for (int e = 0; e < d; ++e) o_b[e] += p * v[t * d + e];
            }
            for (int e = 0; e < d; ++e) o_b[e] /= den;
        }
        double smx = -INFINITY;
        for (int c = 0; c < count; ++c)
            if (has[c] && sc[c] > smx) smx = sc[c];
        double *oi = o + (long)r * d;
        for (int e = 0; e < d; ++e) oi[e] = 0.0;
        if (smx == -INFINITY) { lse[r] = -INFINITY; continue; }
        double wden = 0.0;
        for (int c = 0; c < count; ++c)
            if (has[c]) wden += exp(sc[c] - smx);
        for (int c = 0; c < count; ++c) {
            if (!has[c]) continue;
            double w = exp(sc[c] - smx) / wden;
            for (int e = 0; e < d; ++e) oi[e] += w * ob[(long)c * d + e];
        }
        lse[r] = smx + log(wden);
    }
    free(has);
    free(ob);
    free(z);
}
