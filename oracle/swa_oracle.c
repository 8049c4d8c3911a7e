/*
 * swa_oracle.c -- plain, slow, float64 CPU oracle for the fused
 * softmax-weighted average (causal attention and the Nadaraya-Watson
 * regrid).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it.  It shares no code, header or constant with the
 * CUDA library.
 *
 * Source of every formula: "Show HN: Automatic deduction of FlashAttention
 * kernel from ~25 lines of SQL" (page 2, the demo script
 * benchmarks/ml/01_attention.py):
 *   - view ATTENTION_WINDOW / ATTENTION_GROUP_BY: scores = SUM(q.x*k.x)/8
 *     over the join on d with the predicate q.t >= k.t; w = exp(s - row max);
 *     z = SUM(w) per row; out = SUM(w/z * v.x) per (i, d).
 *   - query GRADIENT: loss = SUM(x*x)/2 over the view, gradient with respect
 *     to every value of q, k and v (one backward pass).
 *   - query NADARAYA_WATSON: w = exp(-((tx-sx)^2 + (ty-sy)^2)/0.25),
 *     out = SUM(w*v)/SUM(w) per target.
 *   - check_masks_are_absent_rows: a masked pair is a row that does not
 *     exist, so it is never visited (no 0*inf).
 * The order max -> exp(x - max) -> sum -> divide also follows the softmax
 * of "Wiki notes" (page 5, the Python softmax and its worked example).
 *
 * Arithmetic is IEEE float64 with no fast-math and no FMA contraction
 * (build with -O2 -ffp-contract=off).  Non-finite values in V (and in the
 * backward's dout) propagate by IEEE rules over the existing pairs only.
 *
 * Layout: q, k, v, out, dout, dq, dk, dv are [B, H, N, D] row-major;
 * lse is [B, H, N]; NW targets/sources are [M, 2] / [S, 2] (x, y).
 *
 * Return codes: 0 ok; 1 invalid argument; 2 some existing pair had a weight
 * that underflowed to exactly 0 (the inf/NaN pattern would then depend on
 * 0*inf; the result is still written); 3 out of memory.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_OK 0
#define OR_EINVAL 1
#define OR_UNDERFLOW 2
#define OR_ENOMEM 3

static void set_threads(int nthreads) {
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Number of the key range of row i: J(i) = {0..i} if causal, else {0..N-1}. */
static int64_t row_len(int64_t i, int64_t N, int causal) {
    return causal ? i + 1 : N;
}

/*
 * Scores of one query row against its key range (the "scores" CTE):
 *   s[j] = (sum_d q[i,d] * k[j,d]) * scale,  j in J(i).
 * Returns the row max m (the window MAX(s) OVER (PARTITION BY i)).
 */
static double row_scores(const double* qi, const double* kbh, int64_t len,
                         int64_t D, double scale, double* s) {
    double m = -INFINITY;
    for (int64_t j = 0; j < len; ++j) {
        const double* kj = kbh + j * D;
        double acc = 0.0;
        for (int64_t d = 0; d < D; ++d) acc += qi[d] * kj[d];
        s[j] = acc * scale;
        if (s[j] > m) m = s[j];
    }
    return m;
}

/*
 * Row statistics of the forward for row i of head bh (steps 1-6 of the
 * forward): w[j] = exp(s_j - m), z = sum w, out_i[d] = sum_j (w_j/z) v[j,d]
 * with the division inside the sum as the SQL writes SUM(w.w / n.z * v.x),
 * lse = m + ln z.  w must hold N doubles.  Returns 1 if some w underflowed.
 */
static int row_forward(const double* qi, const double* kbh, const double* vbh,
                       int64_t i, int64_t N, int64_t D, int causal, double scale,
                       double* w, double* m_out, double* z_out, double* out_i,
                       double* lse_out) {
    int64_t len = row_len(i, N, causal);
    double m = row_scores(qi, kbh, len, D, scale, w);
    double z = 0.0;
    int under = 0;
    for (int64_t j = 0; j < len; ++j) {
        w[j] = exp(w[j] - m);
        if (w[j] == 0.0) under = 1;
        z += w[j];
    }
    if (out_i) {
        for (int64_t d = 0; d < D; ++d) out_i[d] = 0.0;
        for (int64_t j = 0; j < len; ++j) {
            double p = w[j] / z;
            const double* vj = vbh + j * D;
            for (int64_t d = 0; d < D; ++d) out_i[d] += p * vj[d];
        }
    }
    if (m_out) *m_out = m;
    if (z_out) *z_out = z;
    if (lse_out) *lse_out = m + log(z);
    return under;
}

/* Forward over every (b, h, i). */
int oracle_attn_fwd(const double* q, const double* k, const double* v,
                    double* out, double* lse, int64_t B, int64_t H, int64_t N,
                    int64_t D, int causal, double scale, int nthreads) {
    if (!q || !k || !v || !out || B < 0 || H < 0 || N < 0 || D <= 0) return OR_EINVAL;
    set_threads(nthreads);
    int64_t rows = B * H * N;
    int status = OR_OK;
    int nomem = 0;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)(N > 0 ? N : 1));
        if (!w) {
#pragma omp atomic write
            nomem = 1;
        }
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            if (!w) continue;
            int64_t bh = r / N, i = r % N;
            const double* base_q = q + bh * N * D;
            const double* base_k = k + bh * N * D;
            const double* base_v = v + bh * N * D;
            double l;
            int u = row_forward(base_q + i * D, base_k, base_v, i, N, D, causal,
                                scale, w, NULL, NULL, out + r * D, &l);
            if (lse) lse[r] = l;
            if (u) {
#pragma omp atomic write
                status = OR_UNDERFLOW;
            }
        }
        free(w);
    }
    if (nomem) return OR_ENOMEM;
    return status;
}

/*
 * Forward for a list of sampled rows: sample t is row rows[t] of head
 * heads[t] (heads index the flattened B*H).  out_s is [nsamp, D], lse_s
 * is [nsamp].
 */
int oracle_attn_fwd_rows(const double* q, const double* k, const double* v,
                         int64_t N, int64_t D, int causal, double scale,
                         const int64_t* heads, const int64_t* rows, int64_t nsamp,
                         double* out_s, double* lse_s, int nthreads) {
    if (!q || !k || !v || !heads || !rows || !out_s || N <= 0 || D <= 0) return OR_EINVAL;
    set_threads(nthreads);
    int status = OR_OK;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < nsamp; ++t) {
            if (!w) continue;
            int64_t bh = heads[t], i = rows[t];
            double l;
            int u = row_forward(q + (bh * N + i) * D, k + bh * N * D, v + bh * N * D,
                                i, N, D, causal, scale, w, NULL, NULL,
                                out_s + t * D, &l);
            if (lse_s) lse_s[t] = l;
            if (u) {
#pragma omp atomic write
                status = OR_UNDERFLOW;
            }
        }
        free(w);
    }
    return status;
}

/*
 * Backward of loss = 1/2 sum out^2 generalised to an arbitrary upstream
 * gradient dout (the GRADIENT query uses dout = out).  Hand-derived:
 *   P_ij  = w_ij / z_i
 *   dV_j  = sum_{i: j in J(i)} P_ij dO_i
 *   dP_ij = sum_d dO_id v_jd
 *   Delta_i = sum_d dO_id out_id
 *   dS_ij = P_ij (dP_ij - Delta_i)
 *   dQ_i  = scale * sum_{j in J(i)} dS_ij k_j
 *   dK_j  = scale * sum_{i: j in J(i)} dS_ij q_i
 * Phase 1 (per row i): m_i, z_i, out_i, Delta_i and dQ_i.
 * Phase 2 (per key j): dK_j and dV_j, summing over the rows i that see j.
 * Every sum runs over existing pairs only.  Delta is the streaming form
 * dout_i . out_i; a caller may pass the stored forward output (what a
 * backward pass is given) for it, otherwise the oracle's own float64 out_i
 * is used.  On exact inputs both equal sum_j P_ij dP_ij.
 */

/*
 * Phase-1 work for one row; stats = {m, z, Delta}.  Delta_i is evaluated on
 * the given output row when `given` is non-NULL (the stored forward output a
 * backward pass receives), else on this oracle's own float64 out_i.
 */
static int bwd_row(const double* qbh, const double* kbh, const double* vbh,
                   const double* dobh, const double* given_bh, int64_t i, int64_t N,
                   int64_t D, int causal, double scale, double* w, double* out_i,
                   double* stats, double* dq_i) {
    double m, z;
    int u = row_forward(qbh + i * D, kbh, vbh, i, N, D, causal, scale, w, &m, &z,
                        out_i, NULL);
    const double* doi = dobh + i * D;
    const double* oi = given_bh ? given_bh + i * D : out_i;
    double delta = 0.0;
    for (int64_t d = 0; d < D; ++d) delta += doi[d] * oi[d];
    stats[0] = m;
    stats[1] = z;
    stats[2] = delta;
    if (dq_i) {
        int64_t len = row_len(i, N, causal);
        for (int64_t d = 0; d < D; ++d) dq_i[d] = 0.0;
        for (int64_t j = 0; j < len; ++j) {
            const double* vj = vbh + j * D;
            const double* kj = kbh + j * D;
            double p = w[j] / z;
            double dp = 0.0;
            for (int64_t d = 0; d < D; ++d) dp += doi[d] * vj[d];
            double ds = p * (dp - delta);
            for (int64_t d = 0; d < D; ++d) dq_i[d] += ds * kj[d];
        }
        for (int64_t d = 0; d < D; ++d) dq_i[d] *= scale;
    }
    return u;
}

/*
 * Phase-2 work for one key j, given the per-row stats {m, z, Delta} of
 * every row that sees j (stats is [N, 3] for the head).
 */
static void bwd_key(const double* qbh, const double* kbh, const double* vbh,
                    const double* dobh, const double* stats, int64_t j,
                    int64_t N, int64_t D, int causal, double scale,
                    double* dk_j, double* dv_j) {
    const double* kj = kbh + j * D;
    const double* vj = vbh + j * D;
    for (int64_t d = 0; d < D; ++d) { dk_j[d] = 0.0; dv_j[d] = 0.0; }
    int64_t i0 = causal ? j : 0;
    for (int64_t i = i0; i < N; ++i) {
        const double* qi = qbh + i * D;
        const double* doi = dobh + i * D;
        double s = 0.0;
        for (int64_t d = 0; d < D; ++d) s += qi[d] * kj[d];
        s *= scale;
        double p = exp(s - stats[3 * i + 0]) / stats[3 * i + 1];
        double dp = 0.0;
        for (int64_t d = 0; d < D; ++d) dp += doi[d] * vj[d];
        double ds = p * (dp - stats[3 * i + 2]);
        for (int64_t d = 0; d < D; ++d) {
            dv_j[d] += p * doi[d];
            dk_j[d] += ds * qi[d];
        }
    }
    for (int64_t d = 0; d < D; ++d) dk_j[d] *= scale;
}

/* out_given: NULL, or the stored forward output [B,H,N,D] for Delta. */
int oracle_attn_bwd(const double* q, const double* k, const double* v,
                    const double* dout, const double* out_given, double* dq, double* dk,
                    double* dv, int64_t B, int64_t H, int64_t N, int64_t D, int causal,
                    double scale, int nthreads) {
    if (!q || !k || !v || !dout || !dq || !dk || !dv || B < 0 || H < 0 || N < 0 || D <= 0)
        return OR_EINVAL;
    set_threads(nthreads);
    int64_t BH = B * H;
    if (BH == 0 || N == 0) return OR_OK;
    double* stats = (double*)malloc(sizeof(double) * (size_t)(BH * N * 3));
    if (!stats) return OR_ENOMEM;
    int status = OR_OK;
    int64_t rows = BH * N;
#pragma omp parallel
    {
        double* w = (double*)malloc(sizeof(double) * (size_t)N);
        double* out_i = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            if (!w || !out_i) continue;
            int64_t bh = r / N, i = r % N;
            int u = bwd_row(q + bh * N * D, k + bh * N * D, v + bh * N * D,
                            dout + bh * N * D, out_given ? out_given + bh * N * D : NULL, i,
                            N, D, causal, scale, w, out_i, stats + r * 3, dq + r * D);
            if (u) {
#pragma omp atomic write
                status = OR_UNDERFLOW;
            }
        }
        free(w);
        free(out_i);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            int64_t bh = r / N, j = r % N;
            bwd_key(q + bh * N * D, k + bh * N * D, v + bh * N * D, dout + bh * N * D,
                    stats + bh * N * 3, j, N, D, causal, scale, dk + r * D, dv + r * D);
        }
    }
    free(stats);
    return status;
}

/*
 * Sampled backward.  dq rows: sample t is query row qrows[t] of head
 * qheads[t]; dk/dv rows: sample t is key row krows[t] of head kheads[t].
 * The key samples need the row stats of every row i >= j (causal) or all
 * rows (non-causal) of their head; those are computed for the rows needed
 * only.  dq_s is [nq, D]; dk_s, dv_s are [nk, D].
 */
int oracle_attn_bwd_rows(const double* q, const double* k, const double* v,
                         const double* dout, const double* out_given, int64_t N, int64_t D,
                         int causal,
                         double scale, const int64_t* qheads, const int64_t* qrows,
                         int64_t nq, double* dq_s, const int64_t* kheads,
                         const int64_t* krows, int64_t nk, double* dk_s,
                         double* dv_s, int nthreads) {
    if (!q || !k || !v || !dout || N <= 0 || D <= 0) return OR_EINVAL;
    set_threads(nthreads);
    int status = OR_OK;
    if (nq > 0) {
#pragma omp parallel
        {
            double* w = (double*)malloc(sizeof(double) * (size_t)N);
            double* out_i = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 1)
            for (int64_t t = 0; t < nq; ++t) {
                if (!w || !out_i) continue;
                int64_t bh = qheads[t];
                double st[3];
                int u = bwd_row(q + bh * N * D, k + bh * N * D, v + bh * N * D,
                                dout + bh * N * D, out_given ? out_given + bh * N * D : NULL,
                                qrows[t], N, D, causal, scale, w, out_i, st, dq_s + t * D);
                if (u) {
#pragma omp atomic write
                    status = OR_UNDERFLOW;
                }
            }
            free(w);
            free(out_i);
        }
    }
    for (int64_t t = 0; t < nk; ++t) {
        int64_t bh = kheads[t], j = krows[t];
        int64_t i0 = causal ? j : 0;
        double* stats = (double*)calloc((size_t)(N * 3), sizeof(double));
        if (!stats) return OR_ENOMEM;
#pragma omp parallel
        {
            double* w = (double*)malloc(sizeof(double) * (size_t)N);
            double* out_i = (double*)malloc(sizeof(double) * (size_t)D);
#pragma omp for schedule(dynamic, 4)
            for (int64_t i = i0; i < N; ++i) {
                if (!w || !out_i) continue;
                int u = bwd_row(q + bh * N * D, k + bh * N * D, v + bh * N * D,
                                dout + bh * N * D, out_given ? out_given + bh * N * D : NULL,
                                i, N, D, causal, scale, w, out_i, stats + i * 3, NULL);
                if (u) {
#pragma omp atomic write
                    status = OR_UNDERFLOW;
                }
            }
            free(w);
            free(out_i);
        }
        bwd_key(q + bh * N * D, k + bh * N * D, v + bh * N * D, dout + bh * N * D,
                stats, j, N, D, causal, scale, dk_s + t * D, dv_s + t * D);
        free(stats);
    }
    return status;
}

/*
 * Nadaraya-Watson regrid (query NADARAYA_WATSON):
 *   w_pq  = exp(-((tx_p - sx_q)^2 + (ty_p - sy_q)^2) / h^2)
 *   out_p = (sum_q w_pq v_q) / (sum_q w_pq)
 * The pages' divisor 0.25 with "bandwidth h = 0.5" is read as h^2.  No max
 * is subtracted: every weight is <= 1.  If every weight of a target
 * underflows, 0/0 gives NaN.
 */
int oracle_nw(const double* targets, int64_t M, const double* sources,
              const double* vals, int64_t S, double h, double* out, int nthreads) {
    if (!targets || !sources || !vals || !out || M < 0 || S < 0 || !(h > 0.0)) return OR_EINVAL;
    set_threads(nthreads);
    double h2 = h * h;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < M; ++p) {
        double tx = targets[2 * p], ty = targets[2 * p + 1];
        double sw = 0.0, swv = 0.0;
        for (int64_t s = 0; s < S; ++s) {
            double dx = tx - sources[2 * s];
            double dy = ty - sources[2 * s + 1];
            double w = exp(-(dx * dx + dy * dy) / h2);
            sw += w;
            swv += w * vals[s];
        }
        out[p] = swv / sw;
    }
    return OR_OK;
}

/*
 * Nadaraya-Watson regrid with points of `dims` coordinates (1, 2 or 3):
 * the NADARAYA_WATSON query's weight with the squared distance summed over
 * every coordinate (the pages' points are (x, y); a point table with more
 * coordinate columns gives the same view with more terms):
 *   w_pq  = exp(-sum_c (t_pc - s_qc)^2 / h^2)
 *   Z_p   = sum_q w_pq
 *   out_p = (sum_q w_pq v_q) / Z_p
 * targets [M, dims], sources [S, dims]; z_out (may be NULL) receives Z_p.
 */
static void nw_row(const double* tp, const double* sources, const double* vals, int64_t S,
                   int dims, double h2, double* z, double* o) {
    double sw = 0.0, swv = 0.0;
    for (int64_t q = 0; q < S; ++q) {
        double d2 = 0.0;
        for (int c = 0; c < dims; ++c) {
            double d = tp[c] - sources[q * dims + c];
            d2 += d * d;
        }
        double w = exp(-d2 / h2);
        sw += w;
        swv += w * vals[q];
    }
    *z = sw;
    *o = swv / sw;
}

int oracle_nw_nd(const double* targets, int64_t M, const double* sources, const double* vals,
                 int64_t S, int dims, double h, double* out, double* z_out, int nthreads) {
    if (!targets || !sources || !vals || !out || M < 0 || S < 0 || dims < 1 || dims > 3 ||
        !(h > 0.0))
        return OR_EINVAL;
    set_threads(nthreads);
    double h2 = h * h;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < M; ++p) {
        double z;
        nw_row(targets + p * dims, sources, vals, S, dims, h2, &z, out + p);
        if (z_out) z_out[p] = z;
    }
    return OR_OK;
}

/*
 * Backward of the regrid for an upstream gradient g_p = dL/dout_p,
 * hand-derived from the definition above (every sum over all pairs):
 *   P_pq  = w_pq / Z_p                       (so out_p = sum_q P_pq v_q)
 *   dv_q  = sum_p g_p P_pq
 *   dw_pq = g_p (v_q - out_p) / Z_p          (dL/dw_pq through Z_p and the sum)
 *   dw_pq/dt_p = w_pq (-2 / h^2) (t_p - s_q),  dw_pq/ds_q = -dw_pq/dt_p
 *   dt_p  = sum_q dw_pq w_pq (-2 / h^2) (t_p - s_q)
 *   ds_q  = sum_p dw_pq w_pq (+2 / h^2) (t_p - s_q)
 * Phase 1 (per target): Z_p, out_p and dt_p.  Phase 2 (per source): ds_q and
 * dv_q from every target's (Z_p, out_p).  dtargets [M, dims], dsources
 * [S, dims], dvals [S].
 */
int oracle_nw_bwd(const double* targets, int64_t M, const double* sources, const double* vals,
                  int64_t S, int dims, double h, const double* gout, double* dtargets,
                  double* dsources, double* dvals, int nthreads) {
    if (!targets || !sources || !vals || !gout || !dtargets || !dsources || !dvals || M < 0 ||
        S < 0 || dims < 1 || dims > 3 || !(h > 0.0))
        return OR_EINVAL;
    set_threads(nthreads);
    double h2 = h * h;
    double* zo = (double*)malloc(sizeof(double) * (size_t)(2 * (M > 0 ? M : 1)));
    if (!zo) return OR_ENOMEM;
#pragma omp parallel for schedule(static)
    for (int64_t p = 0; p < M; ++p) {
        const double* tp = targets + p * dims;
        double z, o;
        nw_row(tp, sources, vals, S, dims, h2, &z, &o);
        zo[2 * p] = z;
        zo[2 * p + 1] = o;
        double acc[3] = {0.0, 0.0, 0.0};
        for (int64_t q = 0; q < S; ++q) {
            double d2 = 0.0, diff[3];
            for (int c = 0; c < dims; ++c) {
                diff[c] = tp[c] - sources[q * dims + c];
                d2 += diff[c] * diff[c];
            }
            double w = exp(-d2 / h2);
            double dw = gout[p] * (vals[q] - o) / z;
            for (int c = 0; c < dims; ++c) acc[c] += dw * w * (-2.0 / h2) * diff[c];
        }
        for (int c = 0; c < dims; ++c) dtargets[p * dims + c] = acc[c];
    }
#pragma omp parallel for schedule(static)
    for (int64_t q = 0; q < S; ++q) {
        const double* sq = sources + q * dims;
        double acc[3] = {0.0, 0.0, 0.0}, dv = 0.0;
        for (int64_t p = 0; p < M; ++p) {
            double d2 = 0.0, diff[3];
            for (int c = 0; c < dims; ++c) {
                diff[c] = targets[p * dims + c] - sq[c];
                d2 += diff[c] * diff[c];
            }
            double w = exp(-d2 / h2);
            double z = zo[2 * p], o = zo[2 * p + 1];
            dv += gout[p] * w / z;
            double dw = gout[p] * (vals[q] - o) / z;
            for (int c = 0; c < dims; ++c) acc[c] += dw * w * (2.0 / h2) * diff[c];
        }
        for (int c = 0; c < dims; ++c) dsources[q * dims + c] = acc[c];
        dvals[q] = dv;
    }
    free(zo);
    return OR_OK;
}

int oracle_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
