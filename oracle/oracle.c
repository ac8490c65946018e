/*
 * Plain fp64 CPU oracle for causal multi-head scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes is the plain definition, written out row by row with no
 * tiling, no online rescaling and no reordering beyond what the definition
 * states:
 *
 *   Forward ("NanoGPT Speedrun baseline", section "El Mecanismo de Atencion",
 *   the Attn(Q,K,V) = softmax(QK^T / sqrt(d_k)) V equation and the mask rule
 *   Attn_ij = 0 for j > i; the boolean triu(diagonal=1) mask of "Un GPT desde
 *   cero + nanoGPT", Laboratorio L2.1, True = blocked):
 *     S_ij  = scale * sum_d Q_id K_jd            for visible (i, j)
 *     m_i   = max_j S_ij
 *     lse_i = m_i + ln sum_j exp(S_ij - m_i)     (natural log)
 *     P_ij  = exp(S_ij - lse_i)                  (0 where not visible)
 *     O_i   = sum_j P_ij V_j
 *   Key j is visible to query i iff j <= i and (window <= 0 or j > i - window);
 *   the window is the sliding-window variant named in the modded-nanogpt
 *   README's technique list (long/short sliding-window attention).  Masked
 *   entries are -inf before the softmax, so every row renormalises over its
 *   visible keys.  The masked entry points add, from the same list, a window
 *   per head (the long/short pattern) and document boundaries (batches
 *   aligned to document ends): key j must also not lie before the start of
 *   the document that holds token i.
 *
 *   Backward: the exact gradient of L = sum(O * dO) with respect to Q, K, V
 *   (the pages only call loss.backward(); the gradient of the definition
 *   above is the one reading):
 *     dV_j    = sum_i P_ij dO_i
 *     dP_ij   = dO_i . V_j
 *     Delta_i = sum_j P_ij dP_ij
 *     dS_ij   = P_ij (dP_ij - Delta_i)
 *     dQ_i    = scale * sum_j dS_ij K_j
 *     dK_j    = scale * sum_i dS_ij Q_i
 *
 * Layout: contiguous [NH, T, D] row-major doubles (NH = B*H heads as an extra
 * batch dimension, as in the GPT-2 lecture's attention module).  Each head is
 * independent; heads are spread over OpenMP threads.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Key j is visible to query i iff j <= i, (window <= 0 or j > i - window), and
 * j >= first, the position where the document holding token i starts (0 when
 * the sequence is one document).  The document rule is the reading taken of the
 * modded-nanogpt README's item on aligning batches to document ends: attention
 * stays inside a document. */
static int visible(long i, long j, long window, long first) {
    if (j > i) return 0;
    if (window > 0 && j <= i - window) return 0;
    if (j < first) return 0;
    return 1;
}

/* Row i of the softmax: fills p[0..i] (p[j] = 0 where not visible), returns lse. */
static double softmax_row(const double* q, const double* k, long T, long D,
                          double scale, long window, long first, long i, double* p) {
    (void)T;
    double m = -INFINITY;
    for (long j = 0; j <= i; ++j) {
        if (!visible(i, j, window, first)) { p[j] = -INFINITY; continue; }
        double s = 0.0;
        for (long d = 0; d < D; ++d) s += q[i * D + d] * k[j * D + d];
        s *= scale;
        p[j] = s;
        if (s > m) m = s;
    }
    double sum = 0.0;
    for (long j = 0; j <= i; ++j)
        if (visible(i, j, window, first)) sum += exp(p[j] - m);
    double lse = m + log(sum);
    for (long j = 0; j <= i; ++j)
        p[j] = visible(i, j, window, first) ? exp(p[j] - lse) : 0.0;
    return lse;
}

/* first: per query row, the start of its document (NULL: one document). */
static void fwd_head(const double* q, const double* k, const double* v,
                     long T, long D, double scale, long window, const long* first,
                     double* o, double* lse, double* p) {
    for (long i = 0; i < T; ++i) {
        lse[i] = softmax_row(q, k, T, D, scale, window, first ? first[i] : 0, i, p);
        for (long d = 0; d < D; ++d) {
            double acc = 0.0;
            for (long j = 0; j <= i; ++j) acc += p[j] * v[j * D + d];
            o[i * D + d] = acc;
        }
    }
}

static void bwd_head(const double* q, const double* k, const double* v,
                     const double* dO, long T, long D, double scale, long window,
                     const long* first, double* dq, double* dk, double* dv,
                     double* delta, double* p, double* dp) {
    memset(dk, 0, sizeof(double) * T * D);
    memset(dv, 0, sizeof(double) * T * D);
    for (long i = 0; i < T; ++i) {
        const long fi = first ? first[i] : 0;
        softmax_row(q, k, T, D, scale, window, fi, i, p);
        /* dV_j += P_ij dO_i ; dP_ij = dO_i . V_j */
        for (long j = 0; j <= i; ++j) {
            if (p[j] != 0.0)
                for (long d = 0; d < D; ++d) dv[j * D + d] += p[j] * dO[i * D + d];
            double s = 0.0;
            if (visible(i, j, window, fi))
                for (long d = 0; d < D; ++d) s += dO[i * D + d] * v[j * D + d];
            dp[j] = s;
        }
        double del = 0.0;
        for (long j = 0; j <= i; ++j) del += p[j] * dp[j];
        delta[i] = del;
        for (long d = 0; d < D; ++d) dq[i * D + d] = 0.0;
        for (long j = 0; j <= i; ++j) {
            double ds = p[j] * (dp[j] - del);
            if (ds == 0.0) continue;
            for (long d = 0; d < D; ++d) {
                dq[i * D + d] += scale * ds * k[j * D + d];
                dk[j * D + d] += scale * ds * q[i * D + d];
            }
        }
    }
}

static int bad_args(long NH, long T, long D) {
    return NH < 0 || T < 0 || D <= 0;
}

/* A document-start row must name, for every token, a position at or before it. */
static int bad_doc_start(const long* doc_start, long NB, long T) {
    if (!doc_start) return 0;
    for (long n = 0; n < NB * T; ++n)
        if (doc_start[n] < 0 || doc_start[n] > n % T) return 1;
    return 0;
}

/* Heads are numbered h = b * H + hh (b batch row, hh head within the row).
 * head_window: H windows, one per head position hh, or NULL for `window`
 * everywhere.  doc_start: [NB, T] document starts, or NULL for one document
 * per row.  Returns 0 on success, 1 on bad arguments, 2 on allocation failure. */
int oracle_attn_fwd_masked(const double* q, const double* k, const double* v,
                           long NB, long H, long T, long D, double scale,
                           const long* head_window, long window, const long* doc_start,
                           double* o, double* lse, int nthreads) {
    if (NB < 0 || H <= 0 || bad_args(NB * H, T, D) || bad_doc_start(doc_start, NB, T)) return 1;
    const long NH = NB * H;
    if (NH == 0 || T == 0) return 0;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : fail)
#endif
    {
        double* p = (double*)malloc(sizeof(double) * T);
        if (!p) fail = 1;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long h = 0; h < NH; ++h) {
            if (!p) continue;
            const long w = head_window ? head_window[h % H] : window;
            const long* first = doc_start ? doc_start + (h / H) * T : NULL;
            fwd_head(q + h * T * D, k + h * T * D, v + h * T * D, T, D, scale,
                     w, first, o + h * T * D, lse + h * T, p);
        }
        free(p);
    }
    (void)nthreads;
    return fail ? 2 : 0;
}

int oracle_attn_bwd_masked(const double* q, const double* k, const double* v,
                           const double* dO, long NB, long H, long T, long D, double scale,
                           const long* head_window, long window, const long* doc_start,
                           double* dq, double* dk, double* dv, double* delta, int nthreads) {
    if (NB < 0 || H <= 0 || bad_args(NB * H, T, D) || bad_doc_start(doc_start, NB, T)) return 1;
    const long NH = NB * H;
    if (NH == 0 || T == 0) return 0;
    int fail = 0;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel num_threads(nthreads) reduction(| : fail)
#endif
    {
        double* p = (double*)malloc(sizeof(double) * T);
        double* dp = (double*)malloc(sizeof(double) * T);
        if (!p || !dp) fail = 1;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (long h = 0; h < NH; ++h) {
            if (!p || !dp) continue;
            const long w = head_window ? head_window[h % H] : window;
            const long* first = doc_start ? doc_start + (h / H) * T : NULL;
            bwd_head(q + h * T * D, k + h * T * D, v + h * T * D, dO + h * T * D,
                     T, D, scale, w, first, dq + h * T * D, dk + h * T * D,
                     dv + h * T * D, delta + h * T, p, dp);
        }
        free(p);
        free(dp);
    }
    (void)nthreads;
    return fail ? 2 : 0;
}

/* Every head with the one window and no document boundaries. */
int oracle_attn_fwd(const double* q, const double* k, const double* v,
                    long NH, long T, long D, double scale, long window,
                    double* o, double* lse, int nthreads) {
    if (bad_args(NH, T, D)) return 1;
    return oracle_attn_fwd_masked(q, k, v, NH, 1, T, D, scale, NULL, window, NULL, o, lse, nthreads);
}

int oracle_attn_bwd(const double* q, const double* k, const double* v,
                    const double* dO, long NH, long T, long D, double scale,
                    long window, double* dq, double* dk, double* dv,
                    double* delta, int nthreads) {
    if (bad_args(NH, T, D)) return 1;
    return oracle_attn_bwd_masked(q, k, v, dO, NH, 1, T, D, scale, NULL, window, NULL, dq, dk, dv,
                                  delta, nthreads);
}

/* Decode: one new query per (b, h) against its cached keys and values, as the
 * generation loop of "Un GPT desde cero + nanoGPT" (Laboratorio L2.1, generate)
 * runs the model on the growing sequence and keeps only the last position.  The
 * query is the last token of a sequence of length L = lens[b] (clamped to
 * [0, T_max]); it sees keys j < L, and with a window W >= 1 only j >= L - W.
 *   q: [NB*H, D]; k, v: [NB*H, T_max, D]; o: [NB*H, D]; lse: [NB*H] (natural log;
 *   -inf and o = 0 when no key is visible).
 * Returns 0 on success, 1 on bad arguments. */
int oracle_attn_decode(const double* q, const double* k, const double* v, const long* lens,
                       long NB, long H, long T_max, long D, double scale, long window,
                       double* o, double* lse, int nthreads) {
    if (NB < 0 || H <= 0 || T_max < 0 || D <= 0 || !lens) return 1;
    const long NH = NB * H;
#ifdef _OPENMP
    if (nthreads <= 0) nthreads = omp_get_max_threads();
#pragma omp parallel for num_threads(nthreads) schedule(dynamic, 1)
#endif
    for (long h = 0; h < NH; ++h) {
        long L = lens[h / H];
        if (L < 0) L = 0;
        if (L > T_max) L = T_max;
        const long lo = (window > 0 && L - window > 0) ? L - window : 0;
        const double* qh = q + h * D;
        const double* kh = k + h * T_max * D;
        const double* vh = v + h * T_max * D;
        double m = -INFINITY;
        for (long j = lo; j < L; ++j) {
            double s = 0.0;
            for (long d = 0; d < D; ++d) s += qh[d] * kh[j * D + d];
            s *= scale;
            if (s > m) m = s;
        }
        for (long d = 0; d < D; ++d) o[h * D + d] = 0.0;
        if (L <= lo) { lse[h] = -INFINITY; continue; }
        double sum = 0.0;
        for (long j = lo; j < L; ++j) {
            double s = 0.0;
            for (long d = 0; d < D; ++d) s += qh[d] * kh[j * D + d];
            sum += exp(s * scale - m);
        }
        const double l = m + log(sum);
        lse[h] = l;
        for (long j = lo; j < L; ++j) {
            double s = 0.0;
            for (long d = 0; d < D; ++d) s += qh[d] * kh[j * D + d];
            const double p = exp(s * scale - l);
            for (long d = 0; d < D; ++d) o[h * D + d] += p * vh[j * D + d];
        }
    }
    (void)nthreads;
    return 0;
}

/* QK-Norm + rotary prologue, the step before attention in the modded-nanogpt README page's
 * "modernised architecture" item (rotary embeddings, QK-Norm) and the RoPE exercise of "Un GPT
 * desde cero + nanoGPT".  For each row x (D values) at token position t:
 *   n = x / max(|x|, 1e-12)                 (QK-Norm: unit L2 norm, no gain)
 *   y[i]       = n[i] cos a_i - n[i + D/2] sin a_i        i < D/2
 *   y[i + D/2] = n[i] sin a_i + n[i + D/2] cos a_i        a_i = t * base^(-2i/D)
 * (each half-split pair is rotated by a_i; norm = 0 skips the normalisation, base <= 0 skips the
 * rotation).  Rows are [NH, T, D]; head h's token t is row h * T + t. */
static void prologue_row(const double* x, long D, long t, int norm, double base, double* y, double* nrm) {
    double ss = 0.0;
    for (long d = 0; d < D; ++d) ss += x[d] * x[d];
    double r = sqrt(ss);
    double inv = 1.0;
    if (norm) inv = 1.0 / (r > 1e-12 ? r : 1e-12);
    if (nrm) *nrm = r;
    const long h = D / 2;
    for (long i = 0; i < h; ++i) {
        const double a = base > 0 ? (double)t * pow(base, -2.0 * (double)i / (double)D) : 0.0;
        const double c = cos(a), s = sin(a);
        const double x1 = x[i] * inv, x2 = x[i + h] * inv;
        y[i] = x1 * c - x2 * s;
        y[i + h] = x1 * s + x2 * c;
    }
}

int oracle_qk_prologue_fwd(const double* x, long NH, long T, long D, int norm, double base, double* y) {
    if (NH < 0 || T < 0 || D <= 0 || (D & 1)) return 1;
    for (long h = 0; h < NH; ++h)
        for (long t = 0; t < T; ++t) prologue_row(x + (h * T + t) * D, D, t, norm, base, y + (h * T + t) * D, NULL);
    return 0;
}

/* Exact gradient of the prologue: dn = R^T dy (rotate back by a_i), then through the
 * normalisation dx = (dn - n (n . dn)) / |x| when |x| > 1e-12, else dn / 1e-12. */
int oracle_qk_prologue_bwd(const double* x, const double* dy, long NH, long T, long D, int norm, double base,
                           double* dx) {
    if (NH < 0 || T < 0 || D <= 0 || (D & 1)) return 1;
    const long hD = D / 2;
    for (long h = 0; h < NH; ++h)
        for (long t = 0; t < T; ++t) {
            const double* xr = x + (h * T + t) * D;
            const double* g = dy + (h * T + t) * D;
            double* o = dx + (h * T + t) * D;
            for (long i = 0; i < hD; ++i) {
                const double a = base > 0 ? (double)t * pow(base, -2.0 * (double)i / (double)D) : 0.0;
                const double c = cos(a), s = sin(a);
                o[i] = g[i] * c + g[i + hD] * s;
                o[i + hD] = -g[i] * s + g[i + hD] * c;
            }
            if (!norm) continue;
            double ss = 0.0;
            for (long d = 0; d < D; ++d) ss += xr[d] * xr[d];
            const double r = sqrt(ss);
            if (r > 1e-12) {
                double nd = 0.0;
                for (long d = 0; d < D; ++d) nd += xr[d] / r * o[d];
                for (long d = 0; d < D; ++d) o[d] = (o[d] - xr[d] / r * nd) / r;
            } else {
                for (long d = 0; d < D; ++d) o[d] /= 1e-12;
            }
        }
    return 0;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
