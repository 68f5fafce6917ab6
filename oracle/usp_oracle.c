/*
 * usp_oracle.c -- plain, slow, fp64 CPU oracle for the USP attention hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this library. The product
 * path (libusp.so and its Python binding) never calls it, and the two share no
 * code, headers, tables or helpers.
 *
 * What it computes (sources: the pages on long_context_exact_tma; none of them
 * prints a formula, so the readings below are the plain standard definitions):
 *   - exact softmax attention: LongNet slides (page 4, "Abstract": dilated
 *     attention is a drop-in replacement for standard attention; "Results":
 *     built on FlashAttention, i.e. exact attention). Per batch b, query head h,
 *     key/value head g = h / (Hq/Hkv):
 *         s_ij   = scale * sum_d Q[b,i,h,d] K[b,j,g,d]
 *         V(i)   = { j : j <= i } if causal else all j   (original token order)
 *         LSE_i  = log sum_{j in V(i)} exp(s_ij)         (natural log)
 *         O_i    = sum_{j in V(i)} exp(s_ij - LSE_i) V[b,j,g,:]
 *   - backward of the same definition (pages silent; calculus of the above):
 *         Delta_i = sum_d dO_id O_id,  P_ij = exp(s_ij - LSE_i),
 *         dP_ij = dO_i . V_j,  dS_ij = P_ij (dP_ij - Delta_i),
 *         dQ_i = scale sum_j dS_ij K_j,  dK_j = scale sum_{i,h in group} dS_ij Q_i,
 *         dV_j = sum_{i,h in group} P_ij dO_i
 *   - log-sum-exp merge of ring-step partials (Boosting Spec Eagle, "Ring
 *     Attention": each device works on its slice and passes data on, so a
 *     query's result arrives as per-step partials):
 *         LSE = m + log sum_t exp(LSE_t - m),  m = max_t LSE_t
 *         O   = sum_t exp(LSE_t - LSE) O_t      (partials with LSE_t = -inf skipped)
 *   - zigzag sharding (Boosting Spec Eagle, "Implementation Details": load
 *     balancing across the ring; read as 2P chunks of c = S/(2P) tokens, rank r
 *     holding chunks r and 2P-1-r) and the Ulysses sequence->head all-to-all
 *     (DeepSpeed-Ulysses summary, "Wie DeepSpeed-Ulysses funktioniert": an
 *     all-to-all before attention gives each GPU the whole sequence for a subset
 *     of heads; results are regathered afterwards). The permutes here loop over
 *     SOURCE coordinates ("push"), the opposite direction of a gather kernel.
 *
 * Inputs are bf16 bit patterns (uint16), converted exactly to double, or plain
 * doubles (the f64 flag), which the finite-difference pins need.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double bf16_to_f64(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Element i of an input tensor: bf16 bit patterns, or doubles when f64 != 0. */
static double ld(const void *base, long i, int f64) {
    return f64 ? ((const double *)base)[i] : bf16_to_f64(((const uint16_t *)base)[i]);
}

static long idx4(long b, long s, long h, long d, long S, long H, long D) {
    return ((b * S + s) * H + h) * D + d;
}

static void set_threads(int n_threads) {
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#else
    (void)n_threads;
#endif
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Visible key interval list for query position i: [lo, hi) pieces of the key
 * ranges (all of [0,S) when ranges == NULL), cut at i+1 when causal. */
static long visible_pieces(long i, long S, int causal, long n_ranges, const long *ranges,
                           long *lo, long *hi, long cap) {
    long limit = causal ? i + 1 : S;
    long n = 0;
    if (ranges == NULL) {
        lo[0] = 0;
        hi[0] = limit;
        return limit > 0 ? 1 : 0;
    }
    for (long r = 0; r < n_ranges && n < cap; r++) {
        long a = ranges[2 * r], e = ranges[2 * r + 1];
        if (e > limit) e = limit;
        if (a < 0) a = 0;
        if (a < e) {
            lo[n] = a;
            hi[n] = e;
            n++;
        }
    }
    return n;
}

/* One query row of the forward definition. s_buf holds S doubles. */
static void fwd_row(const void *q, const void *k, const void *v, int f64, long S, long Hq,
                    long Hkv, long D, int causal, double scale, long b, long h, long i,
                    long n_ranges, const long *ranges, double *s_buf, long *lo, long *hi,
                    double *o, double *lse) {
    long g = h / (Hq / Hkv);
    long np = visible_pieces(i, S, causal, n_ranges, ranges, lo, hi, n_ranges > 0 ? n_ranges : 1);
    long qi = idx4(b, i, h, 0, S, Hq, D);
    double m = -INFINITY;
    for (long p = 0; p < np; p++) {
        for (long j = lo[p]; j < hi[p]; j++) {
            long kj = idx4(b, j, g, 0, S, Hkv, D);
            double acc = 0.0;
            for (long d = 0; d < D; d++) acc += ld(q, qi + d, f64) * ld(k, kj + d, f64);
            s_buf[j] = scale * acc;
            if (s_buf[j] > m) m = s_buf[j];
        }
    }
    for (long d = 0; d < D; d++) o[d] = 0.0;
    if (m == -INFINITY) { /* no visible key: an empty partial */
        *lse = -INFINITY;
        return;
    }
    double l = 0.0;
    for (long p = 0; p < np; p++)
        for (long j = lo[p]; j < hi[p]; j++) l += exp(s_buf[j] - m);
    double L = m + log(l);
    *lse = L;
    for (long p = 0; p < np; p++) {
        for (long j = lo[p]; j < hi[p]; j++) {
            double w = exp(s_buf[j] - L);
            long vj = idx4(b, j, g, 0, S, Hkv, D);
            for (long d = 0; d < D; d++) o[d] += w * ld(v, vj + d, f64);
        }
    }
}

static int rows_ok(long n_rows, const long *rows, long B, long H, long S) {
    for (long r = 0; r < n_rows; r++)
        if (rows[3 * r] < 0 || rows[3 * r] >= B || rows[3 * r + 1] < 0 || rows[3 * r + 1] >= H ||
            rows[3 * r + 2] < 0 || rows[3 * r + 2] >= S)
            return 0;
    return 1;
}

/*
 * Forward for a list of query rows. rows = [n_rows][3] (b, h, i) with i the
 * original token position. ranges = [n_ranges][2] key intervals [start, end)
 * restricting the key set (NULL = every key). o = [n_rows][D], lse = [n_rows].
 * Inputs are [B][S][H][D]; f64 selects double inputs instead of bf16 bits.
 */
int oracle_attn_fwd_rows(const void *q, const void *k, const void *v, int f64, long B, long S,
                         long Hq, long Hkv, long D, int causal, double scale, long n_rows,
                         const long *rows, long n_ranges, const long *ranges, double *o,
                         double *lse, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !rows_ok(n_rows, rows, B, Hq, S)) return -1;
    set_threads(n_threads);
    long cap = n_ranges > 0 ? n_ranges : 1;
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        long *lo = (long *)malloc(sizeof(long) * (size_t)cap);
        long *hi = (long *)malloc(sizeof(long) * (size_t)cap);
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; r++) {
            fwd_row(q, k, v, f64, S, Hq, Hkv, D, causal, scale, rows[3 * r], rows[3 * r + 1],
                    rows[3 * r + 2], n_ranges, ranges, s_buf, lo, hi, o + r * D, lse + r);
        }
        free(s_buf);
        free(lo);
        free(hi);
    }
    return 0;
}

/*
 * Backward of one query row, given its forward (s_buf filled by fwd_row, LSE L,
 * exact O row o). Writes dQ_i to dqi (when not NULL) and, when dk/dv are not
 * NULL, accumulates into the key rows of kv-head g of batch b.
 */
static double bwd_row(const void *q, const void *k, const void *v, const void *dO, int f64,
                      long S, long Hq, long Hkv, long D, int causal, double scale, long b, long h,
                      long i, const double *s_buf, double L, const double *o, double *dqi,
                      double *dk, double *dv) {
    long g = h / (Hq / Hkv);
    long qi = idx4(b, i, h, 0, S, Hq, D);
    double delta = 0.0;
    for (long d = 0; d < D; d++) delta += ld(dO, qi + d, f64) * o[d];
    if (dqi)
        for (long d = 0; d < D; d++) dqi[d] = 0.0;
    long jmax = causal ? i + 1 : S;
    for (long j = 0; j < jmax; j++) {
        double p = exp(s_buf[j] - L);
        long kj = idx4(b, j, g, 0, S, Hkv, D);
        double dp = 0.0;
        for (long d = 0; d < D; d++) dp += ld(dO, qi + d, f64) * ld(v, kj + d, f64);
        double ds = p * (dp - delta);
        for (long d = 0; d < D; d++) {
            if (dqi) dqi[d] += scale * ds * ld(k, kj + d, f64);
            if (dk) dk[kj + d] += scale * ds * ld(q, qi + d, f64);
            if (dv) dv[kj + d] += p * ld(dO, qi + d, f64);
        }
    }
    return delta;
}

/*
 * Full forward + backward on whole tensors (small shapes). Global layouts:
 * q, dO, o, dq: [B][S][Hq][D]; k, v, dk, dv: [B][S][Hkv][D]; lse: [B][S][Hq].
 * Work is split over (b, kv-head g) so that each task owns its dK/dV rows.
 */
int oracle_attn_full(const void *q, const void *k, const void *v, const void *dO, int f64, long B,
                     long S, long Hq, long Hkv, long D, int causal, double scale, double *o,
                     double *lse, double *dq, double *dk, double *dv, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0) return -1;
    long G = Hq / Hkv;
    set_threads(n_threads);
    memset(dk, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
    memset(dv, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        long lo[1], hi[1];
#pragma omp for schedule(dynamic, 1)
        for (long bg = 0; bg < B * Hkv; bg++) {
            long b = bg / Hkv, g = bg % Hkv;
            for (long hh = 0; hh < G; hh++) {
                long h = g * G + hh;
                for (long i = 0; i < S; i++) {
                    double *oi = o + idx4(b, i, h, 0, S, Hq, D);
                    double L;
                    fwd_row(q, k, v, f64, S, Hq, Hkv, D, causal, scale, b, h, i, 0, NULL, s_buf,
                            lo, hi, oi, &L);
                    lse[(b * S + i) * Hq + h] = L;
                    bwd_row(q, k, v, dO, f64, S, Hq, Hkv, D, causal, scale, b, h, i, s_buf, L, oi,
                            dq + idx4(b, i, h, 0, S, Hq, D), dk, dv);
                }
            }
        }
        free(s_buf);
    }
    return 0;
}

/*
 * dQ for a list of query rows (b, h, i): the forward row, Delta_i from the
 * exact O_i, then dQ_i = scale * sum_j P_ij (dP_ij - Delta_i) K_j.
 * Also returns lse and delta of those rows.
 */
int oracle_attn_dq_rows(const void *q, const void *k, const void *v, const void *dO, int f64,
                        long B, long S, long Hq, long Hkv, long D, int causal, double scale,
                        long n_rows, const long *rows, double *dq, double *lse, double *delta,
                        int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !rows_ok(n_rows, rows, B, Hq, S)) return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        double *o = (double *)malloc(sizeof(double) * (size_t)D);
        long lo[1], hi[1];
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; r++) {
            long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            double L;
            fwd_row(q, k, v, f64, S, Hq, Hkv, D, causal, scale, b, h, i, 0, NULL, s_buf, lo, hi,
                    o, &L);
            lse[r] = L;
            delta[r] = bwd_row(q, k, v, dO, f64, S, Hq, Hkv, D, causal, scale, b, h, i, s_buf, L,
                               o, dq + r * D, NULL, NULL);
        }
        free(s_buf);
        free(o);
    }
    return 0;
}

/*
 * dK, dV for a list of key columns (b, g, j). Needs LSE_i and Delta_i of every
 * query row that sees key j, in every q-head of group g, passed as tables
 * lse_tab / delta_tab of shape [B][S][Hq] (rows that are not needed may hold
 * anything; a needed row holding NaN makes the call return -2).
 */
int oracle_attn_dkdv_cols(const void *q, const void *k, const void *v, const void *dO, int f64,
                          long B, long S, long Hq, long Hkv, long D, int causal, double scale,
                          long n_cols, const long *cols, const double *lse_tab,
                          const double *delta_tab, double *dk, double *dv, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !rows_ok(n_cols, cols, B, Hkv, S)) return -1;
    long G = Hq / Hkv;
    int bad = 0;
    set_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (long c = 0; c < n_cols; c++) {
        long b = cols[3 * c], g = cols[3 * c + 1], j = cols[3 * c + 2];
        double *dkj = dk + c * D, *dvj = dv + c * D;
        for (long d = 0; d < D; d++) dkj[d] = dvj[d] = 0.0;
        long kj = idx4(b, j, g, 0, S, Hkv, D);
        for (long hh = 0; hh < G; hh++) {
            long h = g * G + hh;
            for (long i = causal ? j : 0; i < S; i++) {
                double L = lse_tab[(b * S + i) * Hq + h];
                double dl = delta_tab[(b * S + i) * Hq + h];
                if (isnan(L) || isnan(dl)) {
                    bad |= 1;
                    continue;
                }
                long qi = idx4(b, i, h, 0, S, Hq, D);
                double s = 0.0, dp = 0.0;
                for (long d = 0; d < D; d++) {
                    s += ld(q, qi + d, f64) * ld(k, kj + d, f64);
                    dp += ld(dO, qi + d, f64) * ld(v, kj + d, f64);
                }
                double p = exp(scale * s - L);
                double ds = p * (dp - dl);
                for (long d = 0; d < D; d++) {
                    dkj[d] += scale * ds * ld(q, qi + d, f64);
                    dvj[d] += p * ld(dO, qi + d, f64);
                }
            }
        }
    }
    return bad ? -2 : 0;
}

/* Log-sum-exp merge of n partials: o_parts [n][rows][D], lse_parts [n][rows]. */
int oracle_lse_merge(long n, long rows, long D, const double *o_parts, const double *lse_parts,
                     double *o, double *lse, int n_threads) {
    set_threads(n_threads);
#pragma omp parallel for schedule(static)
    for (long r = 0; r < rows; r++) {
        double m = -INFINITY;
        for (long t = 0; t < n; t++)
            if (lse_parts[t * rows + r] > m) m = lse_parts[t * rows + r];
        double *orow = o + r * D;
        for (long d = 0; d < D; d++) orow[d] = 0.0;
        if (m == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double acc = 0.0;
        for (long t = 0; t < n; t++) acc += exp(lse_parts[t * rows + r] - m);
        double L = m + log(acc);
        lse[r] = L;
        for (long t = 0; t < n; t++) {
            double lt = lse_parts[t * rows + r];
            if (lt == -INFINITY) continue;
            double w = exp(lt - L);
            const double *ot = o_parts + (t * rows + r) * D;
            for (long d = 0; d < D; d++) orow[d] += w * ot[d];
        }
    }
    return 0;
}

/* ---- layout transforms; every element is `esize` bytes, rows are H x D elements ---- */

/* global [B][S][H][D] -> rank-major [P][B][2c][H][D], pushing each global token. */
int oracle_zigzag_shard(const uint8_t *src, uint8_t *dst, long B, long S, long H, long D,
                        long esize, long P) {
    if (P <= 0 || S % (2 * P) != 0) return -1;
    long c = S / (2 * P), tok = H * D * esize;
    for (long b = 0; b < B; b++)
        for (long s = 0; s < S; s++) {
            long chunk = s / c;
            long r = chunk < P ? chunk : 2 * P - 1 - chunk;
            long t = (chunk < P ? 0 : c) + s % c;
            memcpy(dst + ((r * B + b) * 2 * c + t) * tok, src + (b * S + s) * tok, (size_t)tok);
        }
    return 0;
}

/* rank-major [P][B][2c][H][D] -> global [B][S][H][D], pushing each local token. */
int oracle_zigzag_unshard(const uint8_t *src, uint8_t *dst, long B, long S, long H, long D,
                          long esize, long P) {
    if (P <= 0 || S % (2 * P) != 0) return -1;
    long c = S / (2 * P), tok = H * D * esize;
    for (long r = 0; r < P; r++)
        for (long b = 0; b < B; b++)
            for (long t = 0; t < 2 * c; t++) {
                long s = t < c ? r * c + t : (2 * P - 1 - r) * c + (t - c);
                memcpy(dst + (b * S + s) * tok, src + ((r * B + b) * 2 * c + t) * tok, (size_t)tok);
            }
    return 0;
}

/* rank-major [P][B][2c][H][D] -> head-sharded [P_r][P_u][B][2c*P_u][H/P_u][D].
 * Source rank r = i*P_u + u' sends head group u to rank (i, u), where its tokens
 * land at local offset u'*2c. Pushes each source (rank, b, token, head). */
int oracle_seq2head(const uint8_t *src, uint8_t *dst, long B, long S, long H, long D, long esize,
                    long P_u, long P_r) {
    long P = P_u * P_r;
    if (P <= 0 || S % (2 * P) != 0 || H % P_u != 0) return -1;
    long c2 = S / P, Hl = H / P_u, L = c2 * P_u, row = D * esize;
    for (long r = 0; r < P; r++) {
        long i = r / P_u, up = r % P_u;
        for (long b = 0; b < B; b++)
            for (long t = 0; t < c2; t++)
                for (long h = 0; h < H; h++) {
                    long u = h / Hl, hl = h % Hl, tau = up * c2 + t;
                    long d_off = ((((i * P_u + u) * B + b) * L + tau) * Hl + hl) * row;
                    long s_off = (((r * B + b) * c2 + t) * H + h) * row;
                    memcpy(dst + d_off, src + s_off, (size_t)row);
                }
    }
    return 0;
}

/* head-sharded [P_r][P_u][B][2c*P_u][H/P_u][D] -> rank-major [P][B][2c][H][D],
 * pushing each head-sharded (i, u, b, local token, local head). */
int oracle_head2seq(const uint8_t *src, uint8_t *dst, long B, long S, long H, long D, long esize,
                    long P_u, long P_r) {
    long P = P_u * P_r;
    if (P <= 0 || S % (2 * P) != 0 || H % P_u != 0) return -1;
    long c2 = S / P, Hl = H / P_u, L = c2 * P_u, row = D * esize;
    for (long i = 0; i < P_r; i++)
        for (long u = 0; u < P_u; u++)
            for (long b = 0; b < B; b++)
                for (long tau = 0; tau < L; tau++)
                    for (long hl = 0; hl < Hl; hl++) {
                        long up = tau / c2, t = tau % c2, r = i * P_u + up, h = u * Hl + hl;
                        long s_off = ((((i * P_u + u) * B + b) * L + tau) * Hl + hl) * row;
                        long d_off = (((r * B + b) * c2 + t) * H + h) * row;
                        memcpy(dst + d_off, src + s_off, (size_t)row);
                    }
    return 0;
}

/*
 * LongNet dilated attention, forward, for a list of query rows.
 *
 * Source: the LongNet slides (page 4): "Abstract" (dilated attention is a
 * drop-in replacement for standard attention; attention allocation falls
 * exponentially with distance) and "Results" (segment lengths w = {2048, 4096,
 * 8192, 16384, 32768} with dilation ratios r = {1, 2, 4, 6, 12}). The page's
 * formula figures did not survive extraction; the steps below are the
 * published method those slides summarise, in its order:
 *   1. for each (w_k, r_k), split the sequence into segments of w_k tokens
 *      (the last one shorter when w_k does not divide S);
 *   2. in every segment keep every r_k-th row, starting at the offset
 *      o = h mod r_k of the query head h: positions s*w + o + m*r, m >= 0,
 *      inside the segment (key/value rows of kv head h / (Hq/Hkv) at the same
 *      positions);
 *   3. dense softmax attention among the kept rows of the segment (causal:
 *      key position <= query position), giving the output O_k and the softmax
 *      denominator Z_k = sum_j exp(s_ij) at every kept row; a row that is not
 *      kept, or sees no key, has an empty result (Z_k = 0);
 *   4. the k results are combined with weights proportional to their softmax
 *      denominators: O = sum_k Z_k O_k / sum_k Z_k. The row's LSE is
 *      log sum_k Z_k (-inf and O = 0 when every Z_k is 0).
 * Denominators are carried as logarithms (LSE_k = log Z_k) so that they do not
 * overflow; step 4 is then the log-sum-exp merge.
 * pairs = [n_pairs][2] (w, r), w >= 1, 1 <= r. Layouts and rows as in
 * oracle_attn_fwd_rows.
 */
int oracle_dilated_fwd_rows(const void *q, const void *k, const void *v, int f64, long B, long S,
                            long Hq, long Hkv, long D, int causal, double scale, long n_pairs,
                            const long *pairs, long n_rows, const long *rows, double *o,
                            double *lse, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !rows_ok(n_rows, rows, B, Hq, S) || n_pairs <= 0) return -1;
    for (long p = 0; p < n_pairs; p++)
        if (pairs[2 * p] < 1 || pairs[2 * p + 1] < 1) return -1;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        double *o_k = (double *)malloc(sizeof(double) * (size_t)(n_pairs * D));
        double *l_k = (double *)malloc(sizeof(double) * (size_t)n_pairs);
#pragma omp for schedule(dynamic, 1)
        for (long r_ = 0; r_ < n_rows; r_++) {
            long b = rows[3 * r_], h = rows[3 * r_ + 1], i = rows[3 * r_ + 2];
            long g = h / (Hq / Hkv);
            long qi = idx4(b, i, h, 0, S, Hq, D);
            /* steps 1-3 for every pair */
            for (long p = 0; p < n_pairs; p++) {
                long w = pairs[2 * p], r = pairs[2 * p + 1];
                long off = h % r;
                long seg0 = (i / w) * w;
                long seg1 = seg0 + w < S ? seg0 + w : S;
                double *op = o_k + p * D;
                for (long d = 0; d < D; d++) op[d] = 0.0;
                l_k[p] = -INFINITY;
                if (i - seg0 < off || (i - seg0 - off) % r != 0) continue; /* row not kept */
                long jend = causal ? i + 1 : seg1;
                double m = -INFINITY;
                for (long j = seg0 + off; j < jend; j += r) {
                    long kj = idx4(b, j, g, 0, S, Hkv, D);
                    double acc = 0.0;
                    for (long d = 0; d < D; d++) acc += ld(q, qi + d, f64) * ld(k, kj + d, f64);
                    s_buf[j] = scale * acc;
                    if (s_buf[j] > m) m = s_buf[j];
                }
                if (m == -INFINITY) continue;
                double z = 0.0;
                for (long j = seg0 + off; j < jend; j += r) z += exp(s_buf[j] - m);
                l_k[p] = m + log(z);
                for (long j = seg0 + off; j < jend; j += r) {
                    double wgt = exp(s_buf[j] - l_k[p]);
                    long vj = idx4(b, j, g, 0, S, Hkv, D);
                    for (long d = 0; d < D; d++) op[d] += wgt * ld(v, vj + d, f64);
                }
            }
            /* step 4: weights proportional to the denominators exp(LSE_k) */
            double *orow = o + r_ * D;
            for (long d = 0; d < D; d++) orow[d] = 0.0;
            double mx = -INFINITY;
            for (long p = 0; p < n_pairs; p++)
                if (l_k[p] > mx) mx = l_k[p];
            if (mx == -INFINITY) {
                lse[r_] = -INFINITY;
                continue;
            }
            double zsum = 0.0;
            for (long p = 0; p < n_pairs; p++) zsum += exp(l_k[p] - mx);
            double L = mx + log(zsum);
            lse[r_] = L;
            for (long p = 0; p < n_pairs; p++) {
                if (l_k[p] == -INFINITY) continue;
                double alpha = exp(l_k[p] - L);
                for (long d = 0; d < D; d++) orow[d] += alpha * o_k[p * D + d];
            }
        }
        free(s_buf);
        free(o_k);
        free(l_k);
    }
    return 0;
}

/*
 * Attention with a visibility mask: block-sparse and packed variable-length
 * (document) attention.
 *
 * Source: DeepSpeed-Ulysses summary (page 3), "Hauptmerkmale von
 * DeepSpeed-Ulysses", item 3: the Ulysses layout serves dense and sparse
 * attention alike (after the all-to-all every rank holds whole sequences for
 * its heads, so any attention pattern applies unchanged). The pages give no
 * pattern; the readings are the plain ones:
 *   - block-sparse: a 0/1 mask over (query block, key block) of bs x bs
 *     positions, per batch and query head: bm[b][h][i / bs][j / bs];
 *   - packed variable-length sequences: documents [cu[d], cu[d+1]) of the
 *     sequence (cu[0] = 0, cu[n_docs] = S, shared by the batch); a query sees
 *     only keys of its own document.
 * Key j is visible to query i iff (not causal or j <= i) and the block bit is
 * set (when bm != NULL) and doc(i) == doc(j) (when cu != NULL). Otherwise the
 * definition is that of oracle_attn_fwd_rows / oracle_attn_full over the
 * visible set V(i); a row with an empty V(i) has O = 0, LSE = -inf and
 * contributes no gradient.
 */
static long doc_of(const long *cu, long n_docs, long x) {
    long d = 0;
    while (d + 1 < n_docs && cu[d + 1] <= x) d++;
    return d;
}

static int masked_visible(long b, long h, long i, long j, long Hq, int causal, const uint8_t *bm,
                          long bs, long nb, const long *cu, long n_docs) {
    if (causal && j > i) return 0;
    if (bm && !bm[((b * Hq + h) * nb + i / bs) * nb + j / bs]) return 0;
    if (cu && doc_of(cu, n_docs, i) != doc_of(cu, n_docs, j)) return 0;
    return 1;
}

/* Forward of one query row over its visible set; s_buf holds S doubles and
 * vis S flags. Returns LSE (-inf for an empty visible set). */
static double masked_fwd_row(const void *q, const void *k, const void *v, int f64, long S, long Hq,
                             long Hkv, long D, double scale, long b, long h, long i,
                             const char *vis, double *s_buf, double *o) {
    long g = h / (Hq / Hkv);
    long qi = idx4(b, i, h, 0, S, Hq, D);
    double m = -INFINITY;
    for (long j = 0; j < S; j++) {
        if (!vis[j]) continue;
        long kj = idx4(b, j, g, 0, S, Hkv, D);
        double acc = 0.0;
        for (long d = 0; d < D; d++) acc += ld(q, qi + d, f64) * ld(k, kj + d, f64);
        s_buf[j] = scale * acc;
        if (s_buf[j] > m) m = s_buf[j];
    }
    for (long d = 0; d < D; d++) o[d] = 0.0;
    if (m == -INFINITY) return -INFINITY;
    double l = 0.0;
    for (long j = 0; j < S; j++)
        if (vis[j]) l += exp(s_buf[j] - m);
    double L = m + log(l);
    for (long j = 0; j < S; j++) {
        if (!vis[j]) continue;
        double w = exp(s_buf[j] - L);
        long vj = idx4(b, j, g, 0, S, Hkv, D);
        for (long d = 0; d < D; d++) o[d] += w * ld(v, vj + d, f64);
    }
    return L;
}

static int masked_args_ok(long S, const uint8_t *bm, long bs, const long *cu, long n_docs) {
    if (bm && bs <= 0) return 0;
    if (cu) {
        if (n_docs < 1 || cu[0] != 0 || cu[n_docs] != S) return 0;
        for (long d = 0; d < n_docs; d++)
            if (cu[d + 1] < cu[d]) return 0;
    }
    return 1;
}

/* Forward rows (b, h, i) of the masked attention: o [n_rows][D], lse [n_rows].
 * bm = [B][Hq][nb][nb] bytes with nb = ceil(S / bs), or NULL; cu = [n_docs + 1]
 * or NULL. */
int oracle_masked_fwd_rows(const void *q, const void *k, const void *v, int f64, long B, long S,
                           long Hq, long Hkv, long D, int causal, double scale, const uint8_t *bm,
                           long bs, const long *cu, long n_docs, long n_rows, const long *rows,
                           double *o, double *lse, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !rows_ok(n_rows, rows, B, Hq, S) ||
        !masked_args_ok(S, bm, bs, cu, n_docs))
        return -1;
    long nb = bm ? (S + bs - 1) / bs : 0;
    set_threads(n_threads);
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        char *vis = (char *)malloc((size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (long r = 0; r < n_rows; r++) {
            long b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
            for (long j = 0; j < S; j++)
                vis[j] = (char)masked_visible(b, h, i, j, Hq, causal, bm, bs, nb, cu, n_docs);
            lse[r] = masked_fwd_row(q, k, v, f64, S, Hq, Hkv, D, scale, b, h, i, vis, s_buf, o + r * D);
        }
        free(s_buf);
        free(vis);
    }
    return 0;
}

/* Whole-tensor forward and backward of the masked attention (layouts as in
 * oracle_attn_full). Backward over the visible set: Delta_i = dO_i . O_i,
 * P_ij = exp(s_ij - LSE_i), dS_ij = P_ij (dO_i . V_j - Delta_i),
 * dQ_i = scale sum_j dS_ij K_j, dK_j = scale sum dS_ij Q_i, dV_j = sum P_ij dO_i.
 * Work is split over (b, kv-head) so each task owns its dK/dV rows. */
int oracle_masked_attn_full(const void *q, const void *k, const void *v, const void *dO, int f64,
                            long B, long S, long Hq, long Hkv, long D, int causal, double scale,
                            const uint8_t *bm, long bs, const long *cu, long n_docs, double *o,
                            double *lse, double *dq, double *dk, double *dv, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || !masked_args_ok(S, bm, bs, cu, n_docs)) return -1;
    long G = Hq / Hkv;
    long nb = bm ? (S + bs - 1) / bs : 0;
    set_threads(n_threads);
    memset(dk, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
    memset(dv, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        char *vis = (char *)malloc((size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (long bg = 0; bg < B * Hkv; bg++) {
            long b = bg / Hkv, g = bg % Hkv;
            for (long hh = 0; hh < G; hh++) {
                long h = g * G + hh;
                for (long i = 0; i < S; i++) {
                    for (long j = 0; j < S; j++)
                        vis[j] = (char)masked_visible(b, h, i, j, Hq, causal, bm, bs, nb, cu, n_docs);
                    long qi = idx4(b, i, h, 0, S, Hq, D);
                    double *oi = o + qi;
                    double L = masked_fwd_row(q, k, v, f64, S, Hq, Hkv, D, scale, b, h, i, vis, s_buf, oi);
                    lse[(b * S + i) * Hq + h] = L;
                    double *dqi = dq + qi;
                    for (long d = 0; d < D; d++) dqi[d] = 0.0;
                    if (L == -INFINITY) continue;
                    double delta = 0.0;
                    for (long d = 0; d < D; d++) delta += ld(dO, qi + d, f64) * oi[d];
                    for (long j = 0; j < S; j++) {
                        if (!vis[j]) continue;
                        double p = exp(s_buf[j] - L);
                        long kj = idx4(b, j, g, 0, S, Hkv, D);
                        double dp = 0.0;
                        for (long d = 0; d < D; d++) dp += ld(dO, qi + d, f64) * ld(v, kj + d, f64);
                        double ds = p * (dp - delta);
                        for (long d = 0; d < D; d++) {
                            dqi[d] += scale * ds * ld(k, kj + d, f64);
                            dk[kj + d] += scale * ds * ld(q, qi + d, f64);
                            dv[kj + d] += p * ld(dO, qi + d, f64);
                        }
                    }
                }
            }
        }
        free(s_buf);
        free(vis);
    }
    return 0;
}

/*
 * LongNet dilated attention, whole-tensor forward AND backward (small shapes).
 * The forward is that of oracle_dilated_fwd_rows written over the multiset of
 * keys the pairs show a row: key j counts C_ij times, C_ij = the number of
 * pairs (w, r) that keep both i and j in one segment (with j <= i if causal);
 * then O_i = sum_j C_ij e^{s_ij} V_j / sum_j C_ij e^{s_ij} -- the same result as
 * combining the pairs by their softmax denominators. The backward is the
 * calculus of that expression: P_ij = C_ij exp(s_ij - LSE_i),
 * Delta_i = dO_i . O_i, dS_ij = P_ij (dO_i . V_j - Delta_i),
 * dQ_i = scale sum_j dS_ij K_j, dK_j = scale sum dS_ij Q_i, dV_j = sum P_ij dO_i.
 * Work is split over (b, kv-head) so that each task owns its dK/dV rows.
 */
static long dilated_count(long i, long j, long h, long S, int causal, long n_pairs, const long *pairs) {
    if (causal && j > i) return 0;
    long n = 0;
    for (long p = 0; p < n_pairs; p++) {
        long w = pairs[2 * p], r = pairs[2 * p + 1], off = h % r;
        long si = i / w, sj = j / w;
        if (si != sj) continue;
        long ri = i - si * w, rj = j - sj * w;
        if (ri >= off && (ri - off) % r == 0 && rj >= off && (rj - off) % r == 0) n++;
    }
    (void)S;
    return n;
}

int oracle_dilated_attn_full(const void *q, const void *k, const void *v, const void *dO, int f64,
                             long B, long S, long Hq, long Hkv, long D, int causal, double scale,
                             long n_pairs, const long *pairs, double *o, double *lse, double *dq,
                             double *dk, double *dv, int n_threads) {
    if (Hkv <= 0 || Hq % Hkv != 0 || n_pairs <= 0) return -1;
    for (long p = 0; p < n_pairs; p++)
        if (pairs[2 * p] < 1 || pairs[2 * p + 1] < 1) return -1;
    long G = Hq / Hkv;
    set_threads(n_threads);
    memset(dk, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
    memset(dv, 0, sizeof(double) * (size_t)(B * S * Hkv * D));
#pragma omp parallel
    {
        double *s_buf = (double *)malloc(sizeof(double) * (size_t)S);
        long *cnt = (long *)malloc(sizeof(long) * (size_t)S);
#pragma omp for schedule(dynamic, 1)
        for (long bg = 0; bg < B * Hkv; bg++) {
            long b = bg / Hkv, g = bg % Hkv;
            for (long hh = 0; hh < G; hh++) {
                long h = g * G + hh;
                for (long i = 0; i < S; i++) {
                    long qi = idx4(b, i, h, 0, S, Hq, D);
                    double *oi = o + qi, *dqi = dq + qi;
                    double m = -INFINITY;
                    for (long j = 0; j < S; j++) {
                        cnt[j] = dilated_count(i, j, h, S, causal, n_pairs, pairs);
                        if (!cnt[j]) continue;
                        long kj = idx4(b, j, g, 0, S, Hkv, D);
                        double acc = 0.0;
                        for (long d = 0; d < D; d++) acc += ld(q, qi + d, f64) * ld(k, kj + d, f64);
                        s_buf[j] = scale * acc;
                        if (s_buf[j] > m) m = s_buf[j];
                    }
                    for (long d = 0; d < D; d++) oi[d] = dqi[d] = 0.0;
                    if (m == -INFINITY) {
                        lse[(b * S + i) * Hq + h] = -INFINITY;
                        continue;
                    }
                    double l = 0.0;
                    for (long j = 0; j < S; j++)
                        if (cnt[j]) l += (double)cnt[j] * exp(s_buf[j] - m);
                    double L = m + log(l);
                    lse[(b * S + i) * Hq + h] = L;
                    for (long j = 0; j < S; j++) {
                        if (!cnt[j]) continue;
                        double p = (double)cnt[j] * exp(s_buf[j] - L);
                        long vj = idx4(b, j, g, 0, S, Hkv, D);
                        for (long d = 0; d < D; d++) oi[d] += p * ld(v, vj + d, f64);
                    }
                    double delta = 0.0;
                    for (long d = 0; d < D; d++) delta += ld(dO, qi + d, f64) * oi[d];
                    for (long j = 0; j < S; j++) {
                        if (!cnt[j]) continue;
                        double p = (double)cnt[j] * exp(s_buf[j] - L);
                        long kj = idx4(b, j, g, 0, S, Hkv, D);
                        double dp = 0.0;
                        for (long d = 0; d < D; d++) dp += ld(dO, qi + d, f64) * ld(v, kj + d, f64);
                        double ds = p * (dp - delta);
                        for (long d = 0; d < D; d++) {
                            dqi[d] += scale * ds * ld(k, kj + d, f64);
                            dk[kj + d] += scale * ds * ld(q, qi + d, f64);
                            dv[kj + d] += p * ld(dO, qi + d, f64);
                        }
                    }
                }
            }
        }
        free(s_buf);
        free(cnt);
    }
    return 0;
}
