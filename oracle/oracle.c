/*
 * Plain, slow CPU oracle for the KV-streams hot path (fp64).
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the library's product path may call,
 * link or load this file; it shares no code, header, table or helper with the
 * CUDA kernels. Only the tests, the package's smoke check and the CPU-baseline
 * leg of the benchmark use it.
 *
 * What it follows (the pages; citations are page title + section):
 *  - "KV-streams: speeding up agentic RL by operating on the KV cache directly"
 *    (thread): cached keys keep the rotary rotation of their original logical
 *    position while moving to other physical slots; new queries/keys continue
 *    the original position count; the cache is paged in fixed 16-token blocks
 *    found through a block table, and compaction removes whole blocks and joins
 *    the remaining references with no holes; the SGLang setup uses 1-token
 *    blocks; every compaction event is recorded during generation and the
 *    trainer replays the continuous trace, masking from each query the spans
 *    that an eviction at or before its position had removed.
 *  - "KV-streams for Efficient Compaction in Agentic Reinforcement Learning"
 *    (paper listing), Fig. 2(A): re-prefill recomputes the retained tokens,
 *    KV-streams trains on one continuous trace with an attention mask that
 *    reproduces eviction.
 *
 * Readings where the pages are silent:
 *  - an event (seq, tau, start, end) removes logical positions [start, end)
 *    before the token at logical position tau is generated; so key j is
 *    visible to query t iff j <= t < kappa_j, kappa_j = min tau over the
 *    events covering j (INT32_MAX if none);
 *  - rotary embedding is rotate-half: pairs (i, i + d/2), angle p*theta^(-2i/d);
 *  - attention scale is 1/sqrt(d); GQA maps query head h to kv head h / G;
 *  - a 128x128 tile is EMPTY when none of its 16384 (query, key) pairs is
 *    visible, FULL when all are (pairs outside [0, N) count as not visible),
 *    PARTIAL otherwise.
 *
 * Every function is a direct transcription of the definition: loops over
 * elements in ascending index order, fp64 accumulation, no blocking. OpenMP is
 * only used to run independent rows/tiles in parallel.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_INF_TAU 2147483647

enum { ORC_EMPTY = 0, ORC_FULL = 1, ORC_PARTIAL = 2 };
enum { ORC_OK = 0, ORC_ERR_UNALIGNED = 2, ORC_ERR_CAPACITY = 4 };

/* ------------------------------------------------------------------------- */
/* Event log -> kill time kappa                                              */
/* ------------------------------------------------------------------------- */

/* kappa[b][j] = smallest tau of an event of sequence b whose range covers j. */
void orc_kappa(const int32_t *ev, int64_t n_ev, int32_t B, int32_t N, int32_t *kappa) {
    for (int64_t i = 0; i < (int64_t)B * N; ++i) kappa[i] = ORC_INF_TAU;
    for (int64_t e = 0; e < n_ev; ++e) {
        int32_t b = ev[4 * e], tau = ev[4 * e + 1], s = ev[4 * e + 2], t = ev[4 * e + 3];
        if (b < 0 || b >= B) continue;
        for (int32_t j = s; j < t; ++j) {
            if (j < 0 || j >= N) continue;
            int32_t *k = &kappa[(int64_t)b * N + j];
            if (tau < *k) *k = tau;
        }
    }
}

static inline int orc_visible(const int32_t *kap, int32_t N, int64_t t, int64_t j) {
    if (t < 0 || j < 0 || t >= N || j >= N) return 0;
    return j <= t && t < (int64_t)kap[j];
}

/* Count of visible pairs sum_j (min(kappa_j, N) - j): the unmasked work. */
int64_t orc_visible_pairs(const int32_t *kappa, int32_t B, int32_t N) {
    int64_t tot = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t j = 0; j < N; ++j) {
            int64_t hi = kappa[b * N + j] < N ? kappa[b * N + j] : N;
            if (hi > j) tot += hi - j;
        }
    return tot;
}

/* ------------------------------------------------------------------------- */
/* Tile mask by brute force over every element of every 128x128 tile         */
/* ------------------------------------------------------------------------- */

/* Class of every tile; cls is [B][T][T] with T = ceil(N/128). */
void orc_tile_classes(const int32_t *kappa, int32_t B, int32_t N, uint8_t *cls) {
    const int32_t T = (N + 127) / 128;
#pragma omp parallel for collapse(2) schedule(dynamic, 4)
    for (int32_t b = 0; b < B; ++b)
        for (int32_t qi = 0; qi < T; ++qi) {
            const int32_t *kap = kappa + (int64_t)b * N;
            for (int32_t kj = 0; kj < T; ++kj) {
                int64_t cnt = 0;
                for (int r = 0; r < 128; ++r)
                    for (int c = 0; c < 128; ++c)
                        cnt += orc_visible(kap, N, (int64_t)qi * 128 + r, (int64_t)kj * 128 + c);
                cls[((int64_t)b * T + qi) * T + kj] =
                    cnt == 0 ? ORC_EMPTY : (cnt == 128 * 128 ? ORC_FULL : ORC_PARTIAL);
            }
        }
}

/* Bits of one tile: bit (c % 32) of word (c / 32) of row r = visible(q0 + r, k0 + c). */
void orc_tile_bits(const int32_t *kappa, int32_t N, int32_t b, int32_t qi, int32_t kj,
                   uint32_t *bits /* [128][4] */) {
    const int32_t *kap = kappa + (int64_t)b * N;
    for (int r = 0; r < 128; ++r)
        for (int w = 0; w < 4; ++w) {
            uint32_t word = 0;
            for (int c = 32 * w; c < 32 * w + 32; ++c)
                if (orc_visible(kap, N, (int64_t)qi * 128 + r, (int64_t)kj * 128 + c))
                    word |= 1u << (c % 32);
            bits[r * 4 + w] = word;
        }
}

/*
 * Sparse tile lists from the classes:
 *  row-CSR over (b, qi): non-empty kj ascending, pidx = partial index or -1;
 *  partial indices are numbered in row-CSR order;
 *  col-CSR over (b, kj): non-empty qi ascending, with the same pidx.
 * Sizes always written; lists written when caps suffice (else ORC_ERR_CAPACITY).
 */
int orc_tile_lists(const int32_t *kappa, const uint8_t *cls, int32_t B, int32_t N,
                   int32_t *row_ptr, int32_t *row_col, int32_t *row_pidx,
                   int32_t *col_ptr, int32_t *col_row, int32_t *col_pidx,
                   uint32_t *bits, int64_t cap_nnz, int64_t cap_part,
                   int64_t *nnz_out, int64_t *npart_out) {
    const int32_t T = (N + 127) / 128;
    int64_t nnz = 0, np = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t qi = 0; qi < T; ++qi)
            for (int64_t kj = 0; kj < T; ++kj) {
                uint8_t c = cls[(b * T + qi) * T + kj];
                if (c != ORC_EMPTY) ++nnz;
                if (c == ORC_PARTIAL) ++np;
            }
    *nnz_out = nnz;
    *npart_out = np;
    if (!row_col) return ORC_OK;
    if (nnz > cap_nnz || np > cap_part) return ORC_ERR_CAPACITY;
    /* per-tile partial index, in row-major (b, qi, kj) order */
    int32_t *pid = (int32_t *)malloc(sizeof(int32_t) * (size_t)B * T * T);
    int64_t e = 0, p = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t qi = 0; qi < T; ++qi) {
            row_ptr[b * T + qi] = (int32_t)e;
            for (int64_t kj = 0; kj < T; ++kj) {
                int64_t id = (b * T + qi) * T + kj;
                uint8_t c = cls[id];
                pid[id] = -1;
                if (c == ORC_EMPTY) continue;
                if (c == ORC_PARTIAL) {
                    pid[id] = (int32_t)p;
                    orc_tile_bits(kappa, N, (int32_t)b, (int32_t)qi, (int32_t)kj, bits + p * 512);
                    ++p;
                }
                row_col[e] = (int32_t)kj;
                row_pidx[e] = pid[id];
                ++e;
            }
        }
    row_ptr[(int64_t)B * T] = (int32_t)e;
    e = 0;
    for (int64_t b = 0; b < B; ++b)
        for (int64_t kj = 0; kj < T; ++kj) {
            col_ptr[b * T + kj] = (int32_t)e;
            for (int64_t qi = 0; qi < T; ++qi) {
                int64_t id = (b * T + qi) * T + kj;
                if (cls[id] == ORC_EMPTY) continue;
                col_row[e] = (int32_t)qi;
                col_pidx[e] = pid[id];
                ++e;
            }
        }
    col_ptr[(int64_t)B * T] = (int32_t)e;
    free(pid);
    return ORC_OK;
}

/* ------------------------------------------------------------------------- */
/* Rotary embedding at logical positions                                     */
/* ------------------------------------------------------------------------- */

/* y[n][h][:] = R(+-lpos[n]) x[n][h][:], rotate-half pairs (i, i + d/2). */
/* One head row of d values rotated by the angle of position p (rotate-half). */
static void rope_row(const double *xr, double *yr, int32_t d, double p, double theta) {
    const int32_t half = d / 2;
    for (int32_t i = 0; i < half; ++i) {
        double ang = p * pow(theta, -2.0 * (double)i / (double)d);
        double c = cos(ang), s = sin(ang);
        double a = xr[i], b = xr[i + half];
        yr[i] = a * c - b * s;
        yr[i + half] = a * s + b * c;
    }
}

void orc_rope(const double *x, double *y, const int32_t *lpos, int64_t n_tok, int32_t H,
              int32_t d, double theta, int32_t inverse) {
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < n_tok; ++n) {
        double p = (double)lpos[n];
        if (inverse) p = -p;
        for (int32_t h = 0; h < H; ++h) rope_row(x + (n * H + h) * d, y + (n * H + h) * d, d, p, theta);
    }
}

/* ------------------------------------------------------------------------- */
/* Attention of one query over an ordered list of keys                       */
/* ------------------------------------------------------------------------- */

/*
 * o = sum_e softmax_e(scale * <q, key_e>) val_e over the n entries in the given
 * order; *lse = natural log of sum_e exp(scale * <q, key_e>). Accumulation in
 * list order. Used by the generation simulator (list = physical cache in
 * block-table order) and by the replay (list = visible keys, ascending j).
 */
static void orc_attend(const double *q, const double *const *keys, const double *const *vals,
                       int64_t n, int32_t d, double scale, double *o, double *lse, double *sbuf) {
    double m = -INFINITY;
    for (int64_t e = 0; e < n; ++e) {
        double s = 0.0;
        for (int32_t i = 0; i < d; ++i) s += q[i] * keys[e][i];
        s *= scale;
        sbuf[e] = s;
        if (s > m) m = s;
    }
    double l = 0.0;
    for (int32_t i = 0; i < d; ++i) o[i] = 0.0;
    for (int64_t e = 0; e < n; ++e) {
        double p = exp(sbuf[e] - m);
        sbuf[e] = p;
        l += p;
    }
    for (int64_t e = 0; e < n; ++e) {
        double w = sbuf[e] / l;
        for (int32_t i = 0; i < d; ++i) o[i] += w * vals[e][i];
    }
    if (lse) *lse = m + log(l);
}

/*
 * Replay forward for one (sequence, kv head): for each requested query row
 * (vector qrow[r], logical position trow[r]) attend over the keys with
 * j <= t < kappa_j, ascending j. k, v are [N][d] (already rotated).
 */
void orc_attn_rows(const double *qrow, const int32_t *trow, int64_t nrow, const double *k,
                   const double *v, const int32_t *kappa, int32_t N, int32_t d, double scale,
                   double *o, double *lse) {
#pragma omp parallel
    {
        const double **kp = (const double **)malloc(sizeof(double *) * (size_t)N);
        const double **vp = (const double **)malloc(sizeof(double *) * (size_t)N);
        double *sb = (double *)malloc(sizeof(double) * (size_t)N);
#pragma omp for schedule(dynamic, 8)
        for (int64_t r = 0; r < nrow; ++r) {
            int64_t t = trow[r], n = 0;
            for (int64_t j = 0; j <= t && j < N; ++j)
                if (orc_visible(kappa, N, t, j)) {
                    kp[n] = k + j * d;
                    vp[n] = v + j * d;
                    ++n;
                }
            orc_attend(qrow + r * d, kp, vp, n, d, scale, o + r * d, lse ? lse + r : NULL, sb);
        }
        free(kp);
        free(vp);
        free(sb);
    }
}

/* ------------------------------------------------------------------------- */
/* Backward (textbook formulas), one (sequence, kv head) group               */
/* ------------------------------------------------------------------------- */

/*
 * Full backward for a group of G query heads sharing one kv head.
 * q, dout, o_out: [G][N][d]; k, v, dk, dv: [N][d]; lse: [G][N].
 *   O, LSE   : forward (computed here, returned in o_out / lse)
 *   D_t      = sum_i dO_t,i O_t,i
 *   P_tj     = exp(scale <q_t,k_j> - LSE_t)      (visible pairs only)
 *   dV_j     = sum_{g,t} P_tj dO_t
 *   dP_tj    = <dO_t, v_j>
 *   dS_tj    = P_tj (dP_tj - D_t)
 *   dQ_t     = scale sum_j dS_tj k_j
 *   dK_j     = scale sum_{g,t} dS_tj q_t
 */
void orc_attn_bwd_group(const double *q, const double *k, const double *v, const double *dout,
                        const int32_t *kappa, int32_t N, int32_t G, int32_t d, double scale,
                        double *o_out, double *lse, double *dq, double *dk, double *dv) {
    int32_t *trow = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    for (int32_t t = 0; t < N; ++t) trow[t] = t;
    for (int32_t g = 0; g < G; ++g)
        orc_attn_rows(q + (int64_t)g * N * d, trow, N, k, v, kappa, N, d, scale,
                      o_out + (int64_t)g * N * d, lse + (int64_t)g * N);
    free(trow);
    memset(dk, 0, sizeof(double) * (size_t)N * d);
    memset(dv, 0, sizeof(double) * (size_t)N * d);
    for (int32_t g = 0; g < G; ++g) {
        const double *qg = q + (int64_t)g * N * d, *dog = dout + (int64_t)g * N * d;
        const double *og = o_out + (int64_t)g * N * d;
        for (int64_t t = 0; t < N; ++t) {
            const double *qt = qg + t * d, *dot = dog + t * d;
            double D = 0.0;
            for (int32_t i = 0; i < d; ++i) D += dot[i] * og[t * d + i];
            double *dqt = dq + ((int64_t)g * N + t) * d;
            for (int32_t i = 0; i < d; ++i) dqt[i] = 0.0;
            for (int64_t j = 0; j <= t; ++j) {
                if (!orc_visible(kappa, N, t, j)) continue;
                double s = 0.0, dp = 0.0;
                for (int32_t i = 0; i < d; ++i) s += qt[i] * k[j * d + i];
                for (int32_t i = 0; i < d; ++i) dp += dot[i] * v[j * d + i];
                double P = exp(scale * s - lse[(int64_t)g * N + t]);
                double dS = P * (dp - D);
                for (int32_t i = 0; i < d; ++i) {
                    dv[j * d + i] += P * dot[i];
                    dk[j * d + i] += scale * dS * qt[i];
                    dqt[i] += scale * dS * k[j * d + i];
                }
            }
        }
    }
}

/* dQ rows only: rows (g, t) of a group; needs only row-local quantities. */
void orc_attn_dq_rows(const double *q, const double *k, const double *v, const double *dout,
                      const int32_t *kappa, int32_t N, int32_t d, double scale,
                      const int32_t *grow, const int32_t *trow, int64_t nrow, double *dq) {
#pragma omp parallel
    {
        const double **kp = (const double **)malloc(sizeof(double *) * (size_t)N);
        const double **vp = (const double **)malloc(sizeof(double *) * (size_t)N);
        double *sb = (double *)malloc(sizeof(double) * (size_t)N);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < nrow; ++r) {
            int64_t t = trow[r], n = 0;
            const double *qt = q + ((int64_t)grow[r] * N + t) * d;
            const double *dot = dout + ((int64_t)grow[r] * N + t) * d;
            for (int64_t j = 0; j <= t; ++j)
                if (orc_visible(kappa, N, t, j)) {
                    kp[n] = k + j * d;
                    vp[n] = v + j * d;
                    ++n;
                }
            double lse;
            orc_attend(qt, kp, vp, n, d, scale, o, &lse, sb);
            double D = 0.0;
            for (int32_t i = 0; i < d; ++i) D += dot[i] * o[i];
            double *dqt = dq + r * d;
            for (int32_t i = 0; i < d; ++i) dqt[i] = 0.0;
            for (int64_t e = 0; e < n; ++e) {
                double s = 0.0, dp = 0.0;
                for (int32_t i = 0; i < d; ++i) s += qt[i] * kp[e][i];
                for (int32_t i = 0; i < d; ++i) dp += dot[i] * vp[e][i];
                double P = exp(scale * s - lse);
                double dS = P * (dp - D);
                for (int32_t i = 0; i < d; ++i) dqt[i] += scale * dS * kp[e][i];
            }
        }
        free(kp);
        free(vp);
        free(sb);
        free(o);
    }
}

/*
 * dK, dV for selected key positions cols[r] of a group of G query heads; every
 * query row that sees the key has its own softmax recomputed from scratch.
 */
void orc_attn_dkdv_cols(const double *q, const double *k, const double *v, const double *dout,
                        const int32_t *kappa, int32_t N, int32_t G, int32_t d, double scale,
                        const int32_t *cols, int64_t ncol, double *dk, double *dv) {
#pragma omp parallel
    {
        const double **kp = (const double **)malloc(sizeof(double *) * (size_t)N);
        const double **vp = (const double **)malloc(sizeof(double *) * (size_t)N);
        double *sb = (double *)malloc(sizeof(double) * (size_t)N);
        double *o = (double *)malloc(sizeof(double) * (size_t)d);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < ncol; ++r) {
            int64_t j = cols[r];
            double *dkj = dk + r * d, *dvj = dv + r * d;
            for (int32_t i = 0; i < d; ++i) dkj[i] = dvj[i] = 0.0;
            for (int32_t g = 0; g < G; ++g) {
                for (int64_t t = j; t < N; ++t) {
                    if (!orc_visible(kappa, N, t, j)) continue;
                    const double *qt = q + ((int64_t)g * N + t) * d;
                    const double *dot = dout + ((int64_t)g * N + t) * d;
                    int64_t n = 0;
                    for (int64_t jj = 0; jj <= t; ++jj)
                        if (orc_visible(kappa, N, t, jj)) {
                            kp[n] = k + jj * d;
                            vp[n] = v + jj * d;
                            ++n;
                        }
                    double lse;
                    orc_attend(qt, kp, vp, n, d, scale, o, &lse, sb);
                    double D = 0.0, s = 0.0, dp = 0.0;
                    for (int32_t i = 0; i < d; ++i) D += dot[i] * o[i];
                    for (int32_t i = 0; i < d; ++i) s += qt[i] * k[j * d + i];
                    for (int32_t i = 0; i < d; ++i) dp += dot[i] * v[j * d + i];
                    double P = exp(scale * s - lse);
                    double dS = P * (dp - D);
                    for (int32_t i = 0; i < d; ++i) {
                        dvj[i] += P * dot[i];
                        dkj[i] += scale * dS * qt[i];
                    }
                }
            }
        }
        free(kp);
        free(vp);
        free(sb);
        free(o);
    }
}

/*
 * dK, dV for key positions cols[r] of a group of G query heads, given each
 * query row's forward output o[g][t] and log-sum-exp lse[g][t] (as returned by
 * orc_attn_rows): the textbook formulas summed over the rows that see j,
 *   P_tj = exp(scale <q_t,k_j> - LSE_t),  D_t = <dO_t, O_t>,
 *   dV_j = sum_{g,t} P_tj dO_t,  dK_j = scale sum_{g,t} P_tj (<dO_t,v_j> - D_t) q_t.
 * A row whose dO is zero contributes nothing; callers may pass o = 0 and
 * lse = +inf for such rows (then P_tj = 0).
 */
void orc_attn_dkdv_cols_fwd(const double *q, const double *k, const double *v,
                            const double *dout, const double *o, const double *lse,
                            const int32_t *kappa, int32_t N, int32_t G, int32_t d, double scale,
                            const int32_t *cols, int64_t ncol, double *dk, double *dv) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < ncol; ++r) {
        int64_t j = cols[r];
        double *dkj = dk + r * d, *dvj = dv + r * d;
        for (int32_t i = 0; i < d; ++i) dkj[i] = dvj[i] = 0.0;
        for (int32_t g = 0; g < G; ++g) {
            for (int64_t t = j; t < N; ++t) {
                if (!orc_visible(kappa, N, t, j)) continue;
                const double *qt = q + ((int64_t)g * N + t) * d;
                const double *dot = dout + ((int64_t)g * N + t) * d;
                const double *ot = o + ((int64_t)g * N + t) * d;
                double D = 0.0, s = 0.0, dp = 0.0;
                for (int32_t i = 0; i < d; ++i) D += dot[i] * ot[i];
                for (int32_t i = 0; i < d; ++i) s += qt[i] * k[j * d + i];
                for (int32_t i = 0; i < d; ++i) dp += dot[i] * v[j * d + i];
                double P = exp(scale * s - lse[(int64_t)g * N + t]);
                double dS = P * (dp - D);
                for (int32_t i = 0; i < d; ++i) {
                    dvj[i] += P * dot[i];
                    dkj[i] += scale * dS * qt[i];
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------- */
/* Paged cache: block-table compaction and decode                            */
/* ------------------------------------------------------------------------- */

/*
 * Drop every live block of every sequence whose logical span
 * [lpos, lpos + bs) lies inside one of the given ranges; keep the order of the
 * rest (a list filter). A range that overlaps a block only in part, or touches
 * the partly filled tail block, is rejected (returns ORC_ERR_UNALIGNED and
 * changes nothing for that sequence). Freed block ids are written in original
 * table order to freed[b][..], their count to n_freed[b].
 */
int orc_compact(int32_t *bt, int32_t *blpos, int32_t *nblk, int32_t *ntok, int32_t B,
                int32_t max_blocks, int32_t bs, const int32_t *ev, int64_t n_ev, int32_t *freed,
                int32_t *n_freed) {
    int rc = ORC_OK;
    int32_t *kb = (int32_t *)malloc(sizeof(int32_t) * (size_t)max_blocks);
    int32_t *kl = (int32_t *)malloc(sizeof(int32_t) * (size_t)max_blocks);
    for (int32_t b = 0; b < B; ++b) {
        int32_t *t = bt + (int64_t)b * max_blocks, *l = blpos + (int64_t)b * max_blocks;
        int32_t n = nblk[b], nk = 0, nf = 0, bad = 0;
        int32_t tail_partial = (ntok[b] % bs) != 0;
        for (int32_t i = 0; i < n && !bad; ++i) {
            int64_t a = l[i], z = (int64_t)l[i] + bs;
            int drop = 0;
            for (int64_t e = 0; e < n_ev; ++e) {
                if (ev[4 * e] != b) continue;
                int64_t s = ev[4 * e + 2], f = ev[4 * e + 3];
                int64_t lo = a > s ? a : s, hi = z < f ? z : f;
                if (lo >= hi) continue;                          /* no overlap */
                if (s <= a && z <= f && !(tail_partial && i == n - 1)) drop = 1;
                else bad = 1;                                    /* part of a block */
            }
            if (drop) freed[(int64_t)b * max_blocks + nf++] = t[i];
            else { kb[nk] = t[i]; kl[nk] = l[i]; ++nk; }
        }
        if (bad) { rc = ORC_ERR_UNALIGNED; n_freed[b] = 0; continue; }
        for (int32_t i = 0; i < nk; ++i) { t[i] = kb[i]; l[i] = kl[i]; }
        for (int32_t i = nk; i < n; ++i) { t[i] = -1; l[i] = -1; }
        ntok[b] -= (n - nk) * bs;
        nblk[b] = nk;
        n_freed[b] = nf;
    }
    free(kb);
    free(kl);
    return rc;
}

/*
 * One decode step: o[b][h] = attention of q[b][h] over the live entries of
 * sequence b, visited in block-table order: entry i is slot (i % bs) of block
 * block_table[b][i / bs]. Caches are [pool][Hkv][bs][d].
 */
void orc_paged_decode(const double *q, const double *kc, const double *vc, const int32_t *bt,
                      const int32_t *ntok, int32_t B, int32_t Hq, int32_t Hkv, int32_t d,
                      int32_t bs, int32_t max_blocks, double scale, double *o) {
    const int32_t G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t b = 0; b < B; ++b)
        for (int32_t h = 0; h < Hq; ++h) {
            int64_t n = ntok[b];
            const double **kp = (const double **)malloc(sizeof(double *) * (size_t)(n + 1));
            const double **vp = (const double **)malloc(sizeof(double *) * (size_t)(n + 1));
            double *sb = (double *)malloc(sizeof(double) * (size_t)(n + 1));
            int32_t kvh = h / G;
            for (int64_t i = 0; i < n; ++i) {
                int64_t blk = bt[(int64_t)b * max_blocks + i / bs], off = i % bs;
                int64_t row = ((blk * Hkv + kvh) * bs + off) * d;
                kp[i] = kc + row;
                vp[i] = vc + row;
            }
            orc_attend(q + ((int64_t)b * Hq + h) * d, kp, vp, n, d, scale,
                       o + ((int64_t)b * Hq + h) * d, NULL, sb);
            free(kp);
            free(vp);
            free(sb);
        }
}

/* ------------------------------------------------------------------------- */
/* Toy multi-layer model: generation with physical eviction, replay, re-prefill */
/* ------------------------------------------------------------------------- */

/*
 * L layers; layer l maps hidden x_t (dim Dm) to q = x Wq[l] (Hq*d), k = x Wk[l],
 * v = x Wv[l] (Hkv*d); rotates q, k at the logical position; attends; and
 * adds a Wo[l] (Hq*d -> Dm) to the residual. attn_out[l] is [N][Hq*d].
 */
typedef struct {
    int32_t L, Dm, Hq, Hkv, d;
    const double *Wq, *Wk, *Wv, *Wo;
    double theta, scale;
} orc_toy;

static void toy_proj(const double *x, const double *W, int32_t Din, int32_t Dout, double *y) {
    for (int32_t c = 0; c < Dout; ++c) y[c] = 0.0;
    for (int32_t r = 0; r < Din; ++r)
        for (int32_t c = 0; c < Dout; ++c) y[c] += x[r] * W[(int64_t)r * Dout + c];
}

/* Rotate the H head rows of x in place at logical position pos: the same
 * per-row rotation as orc_rope. */
static void toy_rotate(double *x, int32_t H, int32_t d, double pos, double theta) {
    double tmp[512];
    for (int32_t h = 0; h < H; ++h) {
        double *r = x + (int64_t)h * d;
        rope_row(r, tmp, d, pos, theta);
        memcpy(r, tmp, sizeof(double) * (size_t)d);
    }
}

/* Test hooks for the toy model's two building blocks: y[n] = x[n] W for n rows
 * (toy_proj), and the in-place rotation of n tokens of H heads (toy_rotate). */
void orc_toy_project(const double *x, const double *W, int64_t n, int32_t Din, int32_t Dout,
                     double *y) {
    for (int64_t r = 0; r < n; ++r) toy_proj(x + r * Din, W, Din, Dout, y + r * Dout);
}

void orc_toy_rotate(double *x, const int32_t *lpos, int64_t n, int32_t H, int32_t d,
                    double theta) {
    for (int64_t r = 0; r < n; ++r) toy_rotate(x + r * H * d, H, d, (double)lpos[r], theta);
}

/* A per-layer paged cache: pool of blocks, free list, block table. */
typedef struct {
    int32_t bs, pool, Hkv, d;
    double *kpool, *vpool;       /* [pool][Hkv][bs][d] */
    int32_t *table, *lpos;       /* [pool] */
    int32_t nblk, ntok;
    int32_t *freelist;           /* FIFO ring */
    int32_t fhead, fcount;
} toy_cache;

static void cache_init(toy_cache *c, int32_t bs, int32_t pool, int32_t Hkv, int32_t d) {
    c->bs = bs; c->pool = pool; c->Hkv = Hkv; c->d = d;
    c->kpool = (double *)calloc((size_t)pool * Hkv * bs * d, sizeof(double));
    c->vpool = (double *)calloc((size_t)pool * Hkv * bs * d, sizeof(double));
    c->table = (int32_t *)malloc(sizeof(int32_t) * (size_t)pool);
    c->lpos = (int32_t *)malloc(sizeof(int32_t) * (size_t)pool);
    c->freelist = (int32_t *)malloc(sizeof(int32_t) * (size_t)pool);
    for (int32_t i = 0; i < pool; ++i) c->freelist[i] = i;
    c->fhead = 0; c->fcount = pool; c->nblk = 0; c->ntok = 0;
}

static void cache_reset(toy_cache *c) {
    for (int32_t i = 0; i < c->nblk; ++i) {
        c->freelist[(c->fhead + c->fcount) % c->pool] = c->table[i];
        c->fcount++;
    }
    c->nblk = 0; c->ntok = 0;
}

static void cache_free(toy_cache *c) {
    free(c->kpool); free(c->vpool); free(c->table); free(c->lpos); free(c->freelist);
}

static int cache_append(toy_cache *c, int32_t pos, const double *k, const double *v) {
    if (c->ntok % c->bs == 0) {
        if (c->fcount == 0) return ORC_ERR_CAPACITY;
        c->table[c->nblk] = c->freelist[c->fhead];
        c->lpos[c->nblk] = pos;
        c->fhead = (c->fhead + 1) % c->pool;
        c->fcount--;
        c->nblk++;
    }
    int64_t blk = c->table[c->nblk - 1], off = c->ntok % c->bs;
    for (int32_t h = 0; h < c->Hkv; ++h) {
        int64_t row = ((blk * c->Hkv + h) * c->bs + off) * c->d;
        memcpy(c->kpool + row, k + (int64_t)h * c->d, sizeof(double) * (size_t)c->d);
        memcpy(c->vpool + row, v + (int64_t)h * c->d, sizeof(double) * (size_t)c->d);
    }
    c->ntok++;
    return ORC_OK;
}

/* Remove whole blocks inside [s, e); keep the rest in order; free the removed ones. */
static int cache_evict(toy_cache *c, int32_t s, int32_t e) {
    int32_t nk = 0;
    int tail_partial = (c->ntok % c->bs) != 0;
    for (int32_t i = 0; i < c->nblk; ++i) {
        int64_t a = c->lpos[i], z = (int64_t)c->lpos[i] + c->bs;
        int64_t lo = a > s ? a : s, hi = z < e ? z : e;
        if (lo < hi && !(s <= a && z <= e && !(tail_partial && i == c->nblk - 1)))
            return ORC_ERR_UNALIGNED;
    }
    for (int32_t i = 0; i < c->nblk; ++i) {
        int64_t a = c->lpos[i], z = (int64_t)c->lpos[i] + c->bs;
        if (s <= a && z <= e) {
            c->freelist[(c->fhead + c->fcount) % c->pool] = c->table[i];
            c->fcount++;
            c->ntok -= c->bs;
        } else {
            c->table[nk] = c->table[i];
            c->lpos[nk] = c->lpos[i];
            ++nk;
        }
    }
    c->nblk = nk;
    return ORC_OK;
}

/* Attend rotated query heads over the cache, entries in block-table order. */
static void cache_attend(const toy_cache *c, const double *q, int32_t Hq, double scale,
                         double *out, const double **kp, const double **vp, double *sb) {
    const int32_t G = Hq / c->Hkv;
    for (int32_t h = 0; h < Hq; ++h) {
        int32_t kvh = h / G;
        for (int64_t i = 0; i < c->ntok; ++i) {
            int64_t blk = c->table[i / c->bs], off = i % c->bs;
            int64_t row = ((blk * c->Hkv + kvh) * c->bs + off) * c->d;
            kp[i] = c->kpool + row;
            vp[i] = c->vpool + row;
        }
        orc_attend(q + (int64_t)h * c->d, kp, vp, c->ntok, c->d, scale, out + (int64_t)h * c->d,
                   NULL, sb);
    }
}

/* One token through all layers of the toy model at logical position pos. */
static int toy_token(const orc_toy *m, toy_cache *caches, const double *x_in, int32_t pos,
                     double *x_out, double *attn_rows /* [L][Hq*d] or NULL */, double *buf,
                     const double **kp, const double **vp, double *sb) {
    const int32_t Dm = m->Dm, Dq = m->Hq * m->d, Dk = m->Hkv * m->d;
    double *x = buf, *q = x + Dm, *k = q + Dq, *v = k + Dk, *a = v + Dk, *t = a + Dq;
    memcpy(x, x_in, sizeof(double) * (size_t)Dm);
    for (int32_t l = 0; l < m->L; ++l) {
        toy_proj(x, m->Wq + (int64_t)l * Dm * Dq, Dm, Dq, q);
        toy_proj(x, m->Wk + (int64_t)l * Dm * Dk, Dm, Dk, k);
        toy_proj(x, m->Wv + (int64_t)l * Dm * Dk, Dm, Dk, v);
        toy_rotate(q, m->Hq, m->d, (double)pos, m->theta);
        toy_rotate(k, m->Hkv, m->d, (double)pos, m->theta);
        int rc = cache_append(&caches[l], pos, k, v);
        if (rc) return rc;
        cache_attend(&caches[l], q, m->Hq, m->scale, a, kp, vp, sb);
        if (attn_rows) memcpy(attn_rows + (int64_t)l * Dq, a, sizeof(double) * (size_t)Dq);
        toy_proj(a, m->Wo + (int64_t)l * Dq * Dm, Dq, Dm, t);
        for (int32_t i = 0; i < Dm; ++i) x[i] += t[i];
    }
    memcpy(x_out, x, sizeof(double) * (size_t)Dm);
    return ORC_OK;
}

/*
 * Generation with compaction, token by token (the definition):
 *   mode 0 (KV-streams): at time t first apply every event with tau == t by
 *     physically removing whole blocks from every layer's cache; the next token
 *     keeps logical position t.
 *   mode 1 (re-prefill): at an event, rebuild a shorter sequence from the
 *     retained tokens' inputs, renumber their positions 0..n-1, recompute all
 *     layers for them in a fresh cache, and continue with position n.
 * Events (tau, start, end) are this sequence's, sorted by tau.
 * x0: [N][Dm] inputs; x_out: [N][Dm]; attn: [N][L][Hq*d].
 * Final block table / lpos of layer 0 go to out_table / out_lpos (length
 * *out_nblk), and the live token count to *out_ntok.
 */
int orc_toy_generate(int32_t L, int32_t Dm, int32_t Hq, int32_t Hkv, int32_t d, const double *Wq,
                     const double *Wk, const double *Wv, const double *Wo, double theta,
                     double scale, const double *x0, int32_t N, const int32_t *ev3, int64_t n_ev,
                     int32_t bs, int32_t pool, int32_t mode, double *x_out, double *attn,
                     int32_t *out_table, int32_t *out_lpos, int32_t *out_nblk, int32_t *out_ntok) {
    orc_toy m = {L, Dm, Hq, Hkv, d, Wq, Wk, Wv, Wo, theta, scale};
    toy_cache *caches = (toy_cache *)malloc(sizeof(toy_cache) * (size_t)L);
    for (int32_t l = 0; l < L; ++l) cache_init(&caches[l], bs, pool, Hkv, d);
    const int32_t Dq = Hq * d;
    double *buf = (double *)malloc(sizeof(double) * (size_t)(2 * Dm + 3 * Dq + 2 * Hkv * d));
    const double **kp = (const double **)malloc(sizeof(double *) * (size_t)(N + 1));
    const double **vp = (const double **)malloc(sizeof(double *) * (size_t)(N + 1));
    double *sb = (double *)malloc(sizeof(double) * (size_t)(N + 1));
    double *scratch = (double *)malloc(sizeof(double) * (size_t)Dm);
    /* retained token ids (for re-prefill) */
    int32_t *alive = (int32_t *)malloc(sizeof(int32_t) * (size_t)N);
    int32_t nalive = 0, pos = 0, rc = ORC_OK;
    int64_t e = 0;
    for (int32_t t = 0; t < N && rc == ORC_OK; ++t) {
        int fired = 0;
        while (e < n_ev && ev3[3 * e] == t) {
            int32_t s = ev3[3 * e + 1], f = ev3[3 * e + 2];
            if (mode == 0)
                for (int32_t l = 0; l < L && rc == ORC_OK; ++l) rc = cache_evict(&caches[l], s, f);
            int32_t na = 0;
            for (int32_t i = 0; i < nalive; ++i)
                if (!(alive[i] >= s && alive[i] < f)) alive[na++] = alive[i];
            nalive = na;
            fired = 1;
            ++e;
        }
        if (rc) break;
        if (mode == 1 && fired) {
            for (int32_t l = 0; l < L; ++l) cache_reset(&caches[l]);
            for (int32_t i = 0; i < nalive && rc == ORC_OK; ++i)
                rc = toy_token(&m, caches, x0 + (int64_t)alive[i] * Dm, i, scratch, NULL, buf, kp,
                               vp, sb);
            pos = nalive;
        }
        if (rc) break;
        rc = toy_token(&m, caches, x0 + (int64_t)t * Dm, mode == 0 ? t : pos,
                       x_out + (int64_t)t * Dm, attn + (int64_t)t * L * Dq, buf, kp, vp, sb);
        alive[nalive++] = t;
        ++pos;
    }
    if (out_nblk) {
        *out_nblk = caches[0].nblk;
        *out_ntok = caches[0].ntok;
        for (int32_t i = 0; i < caches[0].nblk; ++i) {
            out_table[i] = caches[0].table[i];
            out_lpos[i] = caches[0].lpos[i];
        }
    }
    for (int32_t l = 0; l < L; ++l) cache_free(&caches[l]);
    free(caches); free(buf); free(kp); free(vp); free(sb); free(scratch); free(alive);
    return rc;
}

/*
 * Replay of the continuous trace (KV-streams training side): layer by layer
 * over all N tokens, queries see keys j <= t < kappa_j, ascending j.
 */
void orc_toy_replay(int32_t L, int32_t Dm, int32_t Hq, int32_t Hkv, int32_t d, const double *Wq,
                    const double *Wk, const double *Wv, const double *Wo, double theta,
                    double scale, const double *x0, int32_t N, const int32_t *kappa,
                    double *x_out, double *attn) {
    const int32_t Dq = Hq * d, Dk = Hkv * d, G = Hq / Hkv;
    double *x = (double *)malloc(sizeof(double) * (size_t)N * Dm);
    double *Q = (double *)malloc(sizeof(double) * (size_t)N * Dq);
    double *K = (double *)malloc(sizeof(double) * (size_t)N * Dk);
    double *V = (double *)malloc(sizeof(double) * (size_t)N * Dk);
    double *A = (double *)malloc(sizeof(double) * (size_t)N * Dq);
    double *t1 = (double *)malloc(sizeof(double) * (size_t)Dm);
    const double **kp = (const double **)malloc(sizeof(double *) * (size_t)N);
    const double **vp = (const double **)malloc(sizeof(double *) * (size_t)N);
    double *sb = (double *)malloc(sizeof(double) * (size_t)N);
    memcpy(x, x0, sizeof(double) * (size_t)N * Dm);
    for (int32_t l = 0; l < L; ++l) {
        for (int32_t t = 0; t < N; ++t) {
            toy_proj(x + (int64_t)t * Dm, Wq + (int64_t)l * Dm * Dq, Dm, Dq, Q + (int64_t)t * Dq);
            toy_proj(x + (int64_t)t * Dm, Wk + (int64_t)l * Dm * Dk, Dm, Dk, K + (int64_t)t * Dk);
            toy_proj(x + (int64_t)t * Dm, Wv + (int64_t)l * Dm * Dk, Dm, Dk, V + (int64_t)t * Dk);
            toy_rotate(Q + (int64_t)t * Dq, Hq, d, (double)t, theta);
            toy_rotate(K + (int64_t)t * Dk, Hkv, d, (double)t, theta);
        }
        for (int32_t t = 0; t < N; ++t) {
            for (int32_t h = 0; h < Hq; ++h) {
                int32_t kvh = h / G;
                int64_t n = 0;
                for (int64_t j = 0; j <= t; ++j)
                    if (orc_visible(kappa, N, t, j)) {
                        kp[n] = K + j * Dk + (int64_t)kvh * d;
                        vp[n] = V + j * Dk + (int64_t)kvh * d;
                        ++n;
                    }
                orc_attend(Q + (int64_t)t * Dq + (int64_t)h * d, kp, vp, n, d, scale,
                           A + (int64_t)t * Dq + (int64_t)h * d, NULL, sb);
            }
            memcpy(attn + ((int64_t)t * L + l) * Dq, A + (int64_t)t * Dq, sizeof(double) * (size_t)Dq);
        }
        for (int32_t t = 0; t < N; ++t) {
            toy_proj(A + (int64_t)t * Dq, Wo + (int64_t)l * Dq * Dm, Dq, Dm, t1);
            for (int32_t i = 0; i < Dm; ++i) x[(int64_t)t * Dm + i] += t1[i];
        }
    }
    memcpy(x_out, x, sizeof(double) * (size_t)N * Dm);
    free(x); free(Q); free(K); free(V); free(A); free(t1); free(kp); free(vp); free(sb);
}
