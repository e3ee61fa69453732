/*
 * PaTH attention oracle — plain, slow, fp64 CPU reference.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test-suite, the smoke check and the
 * benchmark's CPU-baseline leg load this library. The product path (the CUDA
 * library) shares no code with it and never calls it.
 *
 * What it computes (per head (b, h), heads independent; 0-based positions):
 *
 *   H_s   = I - beta_s w_s w_s^T
 *       "PaTH Attention" (gist.science summary), section 2 "Kernmechanisme",
 *       transition-matrix equation; Paper-Notes page, "关键设计" equation for H_t.
 *   z_ij  = scale * q_i^T (H_i H_{i-1} ... H_{j+1}) k_j + (c_i - c_j),  j <= i
 *         = -inf,                                                        j >  i
 *       logit equation A_ij ∝ exp(k_j^T (prod_{s=j+1}^{i} H_s) q_i): gist.science
 *       section 2, Paper-Notes "整体框架". The product order is fixed by the
 *       decode rule (each new H_t multiplies the cached keys from the left,
 *       Paper-Notes "训练策略", inference paragraph) and by H being symmetric.
 *   c_t   = sum_{s<=t} log f_s  (PaTH-FoX forget gate, Paper-Notes "PaTH-FoX 扩展"
 *       equation: the product of f_s over s = j+1..i multiplies exp(.)); 0 without FoX.
 *   lse_i = log sum_j exp(z_ij);   o_i = sum_j exp(z_ij - lse_i) v_j.
 *
 * Forward: the key-cache recurrence. Before position t attends, every cached
 * key is multiplied in place by H_t, then k_t is appended untransformed (the
 * in-place key update of the inference paragraph, Paper-Notes "训练策略";
 * gist.science section 3 "Inferentie").
 *
 * Backward (the pages state none; this is the chain rule on the definition).
 * For query i let p_i = q_i and p_{j-1} = H_j p_j, so z_ij = scale k_j.p_j +
 * c_i - c_j. With loss sum(o * dO): P_ij = exp(z_ij - lse_i), dv_j += P_ij dO_i,
 * dZ_ij = P_ij (dO_i.v_j - dO_i.o_i), ds_j = scale dZ_ij, dk_j += ds_j p_j.
 * The adjoint g_j = dloss/dp_j obeys g_0 = ds_0 k_0 and
 * g_{j+1} = ds_{j+1} k_{j+1} + H_{j+1} g_j (H symmetric); from
 * p_j = p_{j+1} - b u (u.p_{j+1}) with u = w_{j+1}, b = beta_{j+1}:
 * dbeta_{j+1} -= (g_j.u)(u.p_{j+1}) and dw_{j+1} -= b[(u.p_{j+1}) g_j +
 * (g_j.u) p_{j+1}]; dq_i = g_i. The gate enters as +dZ_ij on c_i and -dZ_ij
 * on c_j, and dlogf_s = sum_{t>=s} dc_t.
 *
 * Decode: one step of the in-place key update, append, then one-query
 * softmax attention over the n+1 keys; optionally rounding each updated key
 * to bfloat16 (round to nearest, ties to even) as a bf16 cache must hold it.
 * With the forget gate, each cached key also carries g_j = c_t - c_j, the
 * gate's logit bias for the current position t: a step adds log f_t to every
 * cached g_j and appends g_t = 0 (the PaTH-FoX logit term c_i - c_j, carried
 * in the same in-place manner as the keys).
 *
 * Prefill cache: the decode rule replayed over positions 0..L-1 without the
 * attention, i.e. the cache a decoder holds after position L-1: row j of the
 * key cache is H_{L-1} ... H_{j+1} k_j, row j of the value cache is v_j, and
 * g_j = c_{L-1} - c_j.
 *
 * All arrays are contiguous row-major fp64: q, k, v, w, out, grads
 * [B,H,L,d]; beta, log_f, lse, dbeta, dlog_f [B,H,L]. log_f may be NULL
 * (no forget gate); then dlog_f is ignored.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int n_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static double dot(const double *a, const double *b, int d)
{
    double s = 0.0;
    for (int e = 0; e < d; ++e) s += a[e] * b[e];
    return s;
}

/* x <- H_s x = x - beta_s w_s (w_s . x) */
static void apply_h(double *x, const double *w_s, double beta_s, int d)
{
    double a = beta_s * dot(w_s, x, d);
    for (int e = 0; e < d; ++e) x[e] -= a * w_s[e];
}

static void prefix_gate(const double *logf, int L, double *c)
{
    double acc = 0.0;
    for (int t = 0; t < L; ++t) {
        if (logf) acc += logf[t];
        c[t] = acc;
    }
}

/*
 * One head of the forward via the key-cache recurrence.
 * kc: scratch [L,d] holding the cache; row: scratch [L]; c: scratch [L].
 * If z_out is non-NULL it receives the full [L,L] logit matrix (-inf above
 * the diagonal); out/lse may be NULL when only logits are wanted.
 */
static void head_forward(const double *q, const double *k, const double *v,
                         const double *w, const double *beta,
                         const double *logf, double scale, int L, int d,
                         double *out, double *lse, double *z_out,
                         double *kc, double *row, double *c, int inner_par)
{
    prefix_gate(logf, L, c);
    for (int t = 0; t < L; ++t) {
        const double *w_t = w + (size_t)t * d;
        const double *q_t = q + (size_t)t * d;
        /* 1. every cached key j < t is multiplied by H_t */
#pragma omp parallel for schedule(static) if (inner_par && t > 256)
        for (int j = 0; j < t; ++j) apply_h(kc + (size_t)j * d, w_t, beta[t], d);
        /* 2. append k_t untransformed */
        memcpy(kc + (size_t)t * d, k + (size_t)t * d, sizeof(double) * d);
        /* 3. logits against the n = t+1 cached keys */
#pragma omp parallel for schedule(static) if (inner_par && t > 256)
        for (int j = 0; j <= t; ++j)
            row[j] = scale * dot(q_t, kc + (size_t)j * d, d) + (c[t] - c[j]);
        if (z_out) {
            for (int j = 0; j <= t; ++j) z_out[(size_t)t * L + j] = row[j];
            for (int j = t + 1; j < L; ++j) z_out[(size_t)t * L + j] = -INFINITY;
        }
        if (!out) continue;
        /* 4. two-pass stable softmax, output row and log-sum-exp */
        double m = row[0];
        for (int j = 1; j <= t; ++j) m = row[j] > m ? row[j] : m;
        double s = 0.0;
        for (int j = 0; j <= t; ++j) s += exp(row[j] - m);
        double l = m + log(s);
        lse[t] = l;
        double *o_t = out + (size_t)t * d;
        for (int e = 0; e < d; ++e) o_t[e] = 0.0;
        for (int j = 0; j <= t; ++j) {
            double p = exp(row[j] - l);
            const double *v_j = v + (size_t)j * d;
            for (int e = 0; e < d; ++e) o_t[e] += p * v_j[e];
        }
    }
}

int path_oracle_fwd(const double *q, const double *k, const double *v,
                    const double *w, const double *beta, const double *log_f,
                    double scale, int B, int H, int L, int d, double *out,
                    double *lse)
{
    if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return 1;
    const int nh = B * H;
    const size_t hd = (size_t)L * d;
    const int outer = nh >= n_threads();
#pragma omp parallel for schedule(dynamic, 1) if (outer)
    for (int h = 0; h < nh; ++h) {
        double *kc = malloc(sizeof(double) * hd);
        double *row = malloc(sizeof(double) * L);
        double *c = malloc(sizeof(double) * L);
        head_forward(q + h * hd, k + h * hd, v + h * hd, w + h * hd,
                     beta + (size_t)h * L, log_f ? log_f + (size_t)h * L : NULL,
                     scale, L, d, out + h * hd, lse + (size_t)h * L, NULL, kc,
                     row, c, !outer);
        free(kc);
        free(row);
        free(c);
    }
    return 0;
}

/* Full logit matrices z [B,H,L,L] (tiny sizes only; for the self-tests). */
int path_oracle_scores(const double *q, const double *k, const double *w,
                       const double *beta, const double *log_f, double scale,
                       int B, int H, int L, int d, double *z)
{
    if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return 1;
    const size_t hd = (size_t)L * d;
    for (int h = 0; h < B * H; ++h) {
        double *kc = malloc(sizeof(double) * hd);
        double *row = malloc(sizeof(double) * L);
        double *c = malloc(sizeof(double) * L);
        head_forward(q + h * hd, k + h * hd, NULL, w + h * hd,
                     beta + (size_t)h * L, log_f ? log_f + (size_t)h * L : NULL,
                     scale, L, d, NULL, NULL, z + (size_t)h * L * L, kc, row, c,
                     0);
        free(kc);
        free(row);
        free(c);
    }
    return 0;
}

/* Per-thread gradient accumulators of one head. */
typedef struct {
    double *dk, *dv, *dw, *dbeta, *dc;
} grad_acc;

static void acc_alloc(grad_acc *a, int L, int d)
{
    a->dk = calloc((size_t)L * d, sizeof(double));
    a->dv = calloc((size_t)L * d, sizeof(double));
    a->dw = calloc((size_t)L * d, sizeof(double));
    a->dbeta = calloc((size_t)L, sizeof(double));
    a->dc = calloc((size_t)L, sizeof(double));
}

static void acc_free(grad_acc *a)
{
    free(a->dk);
    free(a->dv);
    free(a->dw);
    free(a->dbeta);
    free(a->dc);
}

/*
 * Backward of one query row i (loss = sum_e o_i[e] dO_i[e]).
 * p: scratch [L,d] for the chain p_j; s: scratch [L].
 * Writes dq_i; adds into the per-thread accumulators.
 */
static void query_backward(int i, const double *q, const double *k,
                           const double *v, const double *w,
                           const double *beta, const double *c, double scale,
                           int d, const double *o, const double *lse,
                           const double *dout, double *dq, grad_acc *a,
                           double *p, double *s)
{
    const double *do_i = dout + (size_t)i * d;
    /* chain p_i = q_i, p_{j-1} = H_j p_j */
    memcpy(p + (size_t)i * d, q + (size_t)i * d, sizeof(double) * d);
    for (int j = i; j >= 1; --j) {
        double *dst = p + (size_t)(j - 1) * d;
        memcpy(dst, p + (size_t)j * d, sizeof(double) * d);
        apply_h(dst, w + (size_t)j * d, beta[j], d);
    }
    /* probabilities, dV, dZ, dK */
    const double delta = dot(do_i, o + (size_t)i * d, d);
    for (int j = 0; j <= i; ++j) {
        const double *p_j = p + (size_t)j * d;
        const double zij = scale * dot(k + (size_t)j * d, p_j, d) + (c[i] - c[j]);
        const double pij = exp(zij - lse[i]);
        const double dpij = dot(do_i, v + (size_t)j * d, d);
        const double dz = pij * (dpij - delta);
        double *dv_j = a->dv + (size_t)j * d;
        for (int e = 0; e < d; ++e) dv_j[e] += pij * do_i[e];
        s[j] = scale * dz; /* d loss / d (k_j . p_j) */
        double *dk_j = a->dk + (size_t)j * d;
        for (int e = 0; e < d; ++e) dk_j[e] += s[j] * p_j[e];
        a->dc[i] += dz;
        a->dc[j] -= dz;
    }
    /* adjoint carried back up the chain: g = d loss / d p_j */
    double *g = dq + (size_t)i * d;
    for (int e = 0; e < d; ++e) g[e] = 0.0;
    for (int j = 0; j <= i; ++j) {
        const double *k_j = k + (size_t)j * d;
        for (int e = 0; e < d; ++e) g[e] += s[j] * k_j[e];
        if (j == i) break;
        /* p_j = H_{j+1} p_{j+1} with H = I - b u u^T */
        const double *u = w + (size_t)(j + 1) * d;
        const double b = beta[j + 1];
        const double *x = p + (size_t)(j + 1) * d;
        const double gu = dot(g, u, d);
        const double ux = dot(u, x, d);
        a->dbeta[j + 1] -= gu * ux;
        double *dw_u = a->dw + (size_t)(j + 1) * d;
        for (int e = 0; e < d; ++e) dw_u[e] -= b * (ux * g[e] + gu * x[e]);
        for (int e = 0; e < d; ++e) g[e] -= b * gu * u[e]; /* g <- H^T g */
    }
}

int path_oracle_bwd(const double *q, const double *k, const double *v,
                    const double *w, const double *beta, const double *log_f,
                    double scale, int B, int H, int L, int d,
                    const double *dout, double *dq, double *dk, double *dv,
                    double *dw, double *dbeta, double *dlog_f)
{
    if (B <= 0 || H <= 0 || L <= 0 || d <= 0) return 1;
    const int nh = B * H;
    const size_t hd = (size_t)L * d;
    const int nt = n_threads();
    const int outer = nh >= nt;
#pragma omp parallel for schedule(dynamic, 1) if (outer)
    for (int h = 0; h < nh; ++h) {
        const double *qh = q + h * hd, *kh = k + h * hd, *vh = v + h * hd;
        const double *wh = w + h * hd, *bh = beta + (size_t)h * L;
        const double *fh = log_f ? log_f + (size_t)h * L : NULL;
        double *o = malloc(sizeof(double) * hd);
        double *lse = malloc(sizeof(double) * L);
        double *c = malloc(sizeof(double) * L);
        {
            double *kc = malloc(sizeof(double) * hd);
            double *row = malloc(sizeof(double) * L);
            head_forward(qh, kh, vh, wh, bh, fh, scale, L, d, o, lse, NULL, kc,
                         row, c, !outer);
            free(kc);
            free(row);
        }
        const int nacc = outer ? 1 : nt;
        grad_acc *acc = malloc(sizeof(grad_acc) * nacc);
        for (int a = 0; a < nacc; ++a) acc_alloc(&acc[a], L, d);
#pragma omp parallel if (!outer)
        {
            int tid = 0;
#ifdef _OPENMP
            if (!outer) tid = omp_get_thread_num();
#endif
            double *p = malloc(sizeof(double) * hd);
            double *s = malloc(sizeof(double) * L);
#pragma omp for schedule(dynamic, 8)
            for (int i = L - 1; i >= 0; --i)
                query_backward(i, qh, kh, vh, wh, bh, c, scale, d, o, lse,
                               dout + h * hd, dq + h * hd, &acc[tid], p, s);
            free(p);
            free(s);
        }
        /* reduce the per-thread accumulators */
        double *dkh = dk + h * hd, *dvh = dv + h * hd, *dwh = dw + h * hd;
        double *dbh = dbeta + (size_t)h * L;
        for (size_t e = 0; e < hd; ++e) {
            double sk = 0, sv = 0, sw = 0;
            for (int a = 0; a < nacc; ++a) {
                sk += acc[a].dk[e];
                sv += acc[a].dv[e];
                sw += acc[a].dw[e];
            }
            dkh[e] = sk;
            dvh[e] = sv;
            dwh[e] = sw;
        }
        for (int t = 0; t < L; ++t) {
            double sb = 0;
            for (int a = 0; a < nacc; ++a) sb += acc[a].dbeta[t];
            dbh[t] = sb;
        }
        if (fh && dlog_f) {
            /* c_t = sum_{s<=t} logf_s  =>  dlogf_s = sum_{t>=s} dc_t */
            double run = 0.0;
            for (int t = L - 1; t >= 0; --t) {
                for (int a = 0; a < nacc; ++a) run += acc[a].dc[t];
                dlog_f[(size_t)h * L + t] = run;
            }
        }
        for (int a = 0; a < nacc; ++a) acc_free(&acc[a]);
        free(acc);
        free(o);
        free(lse);
        free(c);
    }
    return 0;
}

/*
 * Round a double to the nearest bfloat16 value, ties to even: keep 8
 * significant bits (1 implicit + 7 stored) at the binade of x, with the
 * fixed spacing 2^-133 below the smallest normal 2^-126.
 */
double path_oracle_round_bf16(double x)
{
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e); /* |x| = m 2^e, m in [0.5, 1) */
    if (e < -125) e = -125;
    const double ulp = ldexp(1.0, e - 8);
    return nearbyint(x / ulp) * ulp; /* default rounding mode: ties to even */
}

/*
 * One decode step of one head (Paper-Notes "训练策略", inference paragraph;
 * gist.science section 3 "Inferentie"). K / V [capacity,d] hold n valid rows;
 * g (NULL without the gate) holds their gate biases c_t - c_j (Paper-Notes
 * "PaTH-FoX 扩展" logit term) and logf_t is log f_t.
 */
static void decode_head(const double *q_t, const double *k_new, const double *v_new,
                        const double *w_t, double beta_t, const double *logf_t, double scale,
                        int d, int n, int round_bf16, double *K, double *V, double *g,
                        double *o)
{
    for (int j = 0; j < n; ++j) {
        double *k_j = K + (size_t)j * d;
        apply_h(k_j, w_t, beta_t, d);
        if (round_bf16)
            for (int e = 0; e < d; ++e) k_j[e] = path_oracle_round_bf16(k_j[e]);
        if (g) g[j] += *logf_t;
    }
    memcpy(K + (size_t)n * d, k_new, sizeof(double) * d);
    memcpy(V + (size_t)n * d, v_new, sizeof(double) * d);
    if (g) g[n] = 0.0;
    double *z = malloc(sizeof(double) * (n + 1));
    double m = -INFINITY;
    for (int j = 0; j <= n; ++j) {
        z[j] = scale * dot(q_t, K + (size_t)j * d, d) + (g ? g[j] : 0.0);
        m = z[j] > m ? z[j] : m;
    }
    double ssum = 0.0;
    for (int j = 0; j <= n; ++j) ssum += exp(z[j] - m);
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int j = 0; j <= n; ++j) {
        const double pj = exp(z[j] - m) / ssum;
        const double *v_j = V + (size_t)j * d;
        for (int e = 0; e < d; ++e) o[e] += pj * v_j[e];
    }
    free(z);
}

/*
 * One decode step for every head. k_cache / v_cache [B,H,capacity,d] hold
 * n_cached valid rows. Rows 0..n-1 of k_cache are multiplied in place by
 * H_t = I - beta w w^T (rounded to bf16 when round_bf16 != 0), then row n of
 * k_cache / v_cache receives k_new / v_new, and out = softmax(scale q K^T) V
 * over the n+1 rows. q, k_new, v_new, w, out: [B,H,d]; beta: [B,H].
 */
int path_oracle_decode_step(const double *q, const double *k_new,
                            const double *v_new, const double *w,
                            const double *beta, double scale, int B, int H,
                            int d, int n_cached, int capacity, int round_bf16,
                            double *k_cache, double *v_cache, double *out)
{
    if (B <= 0 || H <= 0 || d <= 0 || n_cached < 0 || n_cached + 1 > capacity)
        return 1;
    const int nh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        decode_head(q + (size_t)h * d, k_new + (size_t)h * d, v_new + (size_t)h * d,
                    w + (size_t)h * d, beta[h], NULL, scale, d, n_cached, round_bf16,
                    k_cache + (size_t)h * capacity * d, v_cache + (size_t)h * capacity * d,
                    NULL, out + (size_t)h * d);
    return 0;
}

/*
 * The decode step with the forget gate: as path_oracle_decode_step, and
 * g_cache [B,H,capacity] holds the cached keys' gate biases: g_j += log_f
 * (log_f [B,H], log f_t of the new position) for j < n, g_n = 0, and the
 * logits are scale q.k_j + g_j.
 */
int path_oracle_decode_step_gated(const double *q, const double *k_new,
                                  const double *v_new, const double *w,
                                  const double *beta, const double *log_f,
                                  double scale, int B, int H, int d, int n_cached,
                                  int capacity, int round_bf16, double *k_cache,
                                  double *v_cache, double *g_cache, double *out)
{
    if (B <= 0 || H <= 0 || d <= 0 || n_cached < 0 || n_cached + 1 > capacity ||
        !log_f || !g_cache)
        return 1;
    const int nh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h)
        decode_head(q + (size_t)h * d, k_new + (size_t)h * d, v_new + (size_t)h * d,
                    w + (size_t)h * d, beta[h], log_f + h, scale, d, n_cached, round_bf16,
                    k_cache + (size_t)h * capacity * d, v_cache + (size_t)h * capacity * d,
                    g_cache + (size_t)h * capacity, out + (size_t)h * d);
    return 0;
}

/*
 * The cache after a prefill of positions 0..L-1, by replaying the in-place
 * update of the inference paragraph (Paper-Notes "训练策略") position by position: before position t is appended, each key
 * already held is multiplied by H_t and each gate bias grows by log f_t.
 * k, v, w [B,H,L,d]; beta, log_f [B,H,L] (log_f may be NULL; g_cache is then
 * untouched). Writes rows 0..L-1 of k_cache, v_cache [B,H,capacity,d] and
 * g_cache [B,H,capacity].
 */
int path_oracle_prefill_cache(const double *k, const double *v, const double *w,
                              const double *beta, const double *log_f, int B, int H,
                              int L, int d, int capacity, double *k_cache,
                              double *v_cache, double *g_cache)
{
    if (B <= 0 || H <= 0 || L <= 0 || d <= 0 || L > capacity || (log_f && !g_cache))
        return 1;
    const int nh = B * H;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < nh; ++h) {
        const size_t in0 = (size_t)h * L;
        double *K = k_cache + (size_t)h * capacity * d;
        double *V = v_cache + (size_t)h * capacity * d;
        double *g = log_f ? g_cache + (size_t)h * capacity : NULL;
        for (int t = 0; t < L; ++t) {
            const double *w_t = w + (in0 + t) * d;
            for (int j = t - 1; j >= 0; --j) {
                apply_h(K + (size_t)j * d, w_t, beta[in0 + t], d);
                if (g) g[j] += log_f[in0 + t];
            }
            memcpy(K + (size_t)t * d, k + (in0 + t) * d, sizeof(double) * d);
            memcpy(V + (size_t)t * d, v + (in0 + t) * d, sizeof(double) * d);
            if (g) g[t] = 0.0;
        }
    }
    return 0;
}
