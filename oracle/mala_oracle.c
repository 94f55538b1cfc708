/*
 * MALA (MassAlloc Attention) CPU oracle -- TEST INFRASTRUCTURE ONLY.
 *
 * A plain, slow, fp64 restatement of what the MALA operator computes, used to
 * check the CUDA path. Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load it; the product path never does.
 * It shares no code, header, table or constant with the CUDA library.
 *
 * Source of the method: agihunt.info, "MassAlloc Attention: Let Attention
 * Allocate Its Own Compute" (arXiv 2609.32712 digest), method paragraphs:
 *   - every legal causal QK tile is scored; QK is never skipped;
 *   - after each QK tile the largest per-key contribution ratio of the tile is
 *     compared with the length-normalised threshold tau/Lq, Lq = number of
 *     causally visible keys of the query (i+1 for 0-based row i);
 *   - forward: the ratio is taken against the evolving online-softmax state;
 *     tiles run from the diagonal toward earlier keys; the first legal tile is
 *     always kept; one row that fails to skip keeps the tile for the whole
 *     query block; a skipped tile does no V load, no softmax update, no PV;
 *     the final log-normaliser (LSE) is written;
 *   - backward: scores are recomputed and every tile is tested against the
 *     final LSE (no stored mask); a skipped tile does no P, dP, dS, dQ, dK, dV;
 *   - tau -> 0 recovers full attention in both passes.
 *
 * Readings where the pages are silent (each one also listed in the design
 * notes of this repository):
 *   R1 the forward ratio uses the state over previously KEPT tiles (the state
 *      before the tile): exp(s - m)/l with (m, l) before the update;
 *   R2 skip iff ratio < tau/Lq strictly; ties keep; tau == 0 keeps every tile;
 *   R3 Lq = i + 1;
 *   R4 non-live entries (j > i, or outside the sequence) take part in neither
 *      the max nor the sums; a row with an empty state has an infinite ratio;
 *   R5 the backward uses D_i = <dO_i, O_i> with the forward O;
 *   R6 the backward has no forced tile;
 *   R7 decode with split-KV: each split runs its own evolving state over its
 *      tiles from newest to oldest and always keeps its newest tile; the
 *      partial results are merged by their LSEs;
 *   R8 GQA: decisions are per query head.
 *
 * Prefill against an existing cache (oracle_prefill): Lq new queries at the
 * positions Lk - Lq, ..., Lk - 1 of a sequence of Lk keys; row i (0-based
 * among the new queries) sees keys 0 .. P0 + i, P0 = Lk - Lq, and its
 * threshold uses Lq_i = P0 + i + 1 (the count of causally visible keys); the
 * query blocks are cut from the first new query. With Lq == Lk it is the
 * forward above.
 *
 * Layouts: q, o, dO, dq [B, L, Hq, d]; k, v, dk, dv [B, L, Hkv, d];
 * lse [B, Hq, L] (natural log); keep maps [B, Hq, nq, nk] (1 kept, 0 skipped
 * or illegal); margins [B, Hq, nq, nk] (g = max over rows of ratio/(tau/Lq),
 * NaN where the tile is illegal or forced); counts [B * Hq].
 * Tile (qb, kb) is legal iff kb*Bk <= min((qb+1)*Bq, L) - 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define IDX4(a, b, c, dd, B_, C_, D_) ((((size_t)(a) * (B_) + (b)) * (C_) + (c)) * (D_) + (dd))

static inline int imin(int a, int b) { return a < b ? a : b; }
static inline int imax(int a, int b) { return a > b ? a : b; }

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* s = scale * <q[b, i, hq, :], k[b, j, hkv, :]> */
static double score(const double* q, const double* k, int b, int i, int j, int hq, int hkv,
                    int L, int Hq, int Hkv, int d, double scale) {
    const double* qi = q + IDX4(b, i, hq, 0, L, Hq, d);
    const double* kj = k + IDX4(b, j, hkv, 0, L, Hkv, d);
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
    return scale * acc;
}

/* s = scale * <q[b, i, hq, :], k[b, j, hkv, :]> with q holding Lq rows and k
 * holding Lk rows (prefill) */
static double score2(const double* q, const double* k, int b, int i, int j, int hq, int hkv,
                     int Lq, int Lk, int Hq, int Hkv, int d, double scale) {
    const double* qi = q + IDX4(b, i, hq, 0, Lq, Hq, d);
    const double* kj = k + IDX4(b, j, hkv, 0, Lk, Hkv, d);
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += qi[c] * kj[c];
    return scale * acc;
}

/* ------------------------------------------------------------------------
 * Forward: one query block (b, hq, qb) of Lq queries at positions P0 + i
 * (P0 = Lk - Lq) against Lk keys; P0 = 0 is the training forward.
 * ---------------------------------------------------------------------- */
static void fwd_block(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                      int Lq, int Lk, int d, double scale, double tau, int Bq, int Bk, int b, int hq,
                      int qb, double* o, double* lse, uint8_t* keep_map, double* margin,
                      int64_t* n_kept) {
    (void)B;
    const int G = Hq / Hkv;
    const int hkv = hq / G;
    const int P0 = Lk - Lq;
    const int nq = (Lq + Bq - 1) / Bq;
    const int nk = (Lk + Bk - 1) / Bk;
    const int i0 = qb * Bq;
    const int i1 = imin((qb + 1) * Bq, Lq); /* rows [i0, i1) among the new queries */
    const int R = i1 - i0;
    const int kb_first = (P0 + i1 - 1) / Bk; /* largest legal key block */

    double* m = (double*)malloc(sizeof(double) * R);
    double* l = (double*)malloc(sizeof(double) * R);
    double* thr = (double*)malloc(sizeof(double) * R);
    double* acc = (double*)calloc((size_t)R * d, sizeof(double));
    double* s = (double*)malloc(sizeof(double) * (size_t)R * Bk);
    double* M = (double*)malloc(sizeof(double) * R);
    for (int r = 0; r < R; ++r) {
        m[r] = -INFINITY;
        l[r] = 0.0;
        thr[r] = tau > 0.0 ? log(tau) - log((double)(P0 + i0 + r + 1)) : -INFINITY; /* ln(tau/Lq) */
    }
    int64_t kept = 0;
    size_t map_row = ((size_t)(b * Hq + hq) * nq + qb) * nk;

    for (int kb = kb_first; kb >= 0; --kb) { /* diagonal toward earlier keys */
        const int j0 = kb * Bk;
        const int j1 = imin((kb + 1) * Bk, Lk);
        /* 1. scores of every live entry of the tile (never skipped) */
        for (int r = 0; r < R; ++r) {
            const int i = i0 + r;
            M[r] = -INFINITY;
            for (int j = j0; j < j1; ++j) {
                double sv = -INFINITY;
                if (j <= P0 + i) sv = score2(q, k, b, i, j, hq, hkv, Lq, Lk, Hq, Hkv, d, scale);
                s[(size_t)r * Bk + (j - j0)] = sv;
                if (sv > M[r]) M[r] = sv;
            }
        }
        /* 2. gate against the state over previously kept tiles */
        int keep;
        double g = NAN;
        if (kb == kb_first) {
            keep = 1;                      /* first legal tile always retained */
        } else if (tau == 0.0) {
            keep = 1;                      /* tau = 0: full attention */
        } else {
            keep = 0;
            g = 0.0;
            for (int r = 0; r < R; ++r) {
                if (M[r] == -INFINITY) continue;          /* no live key in this row */
                /* log of the row's largest ratio exp(s - m)/l, minus log(tau/Lq) */
                double lr = (l[r] > 0.0) ? (M[r] - m[r] - log(l[r])) - thr[r] : INFINITY;
                if (lr >= 0.0) keep = 1;                  /* one row keeps the block */
                double gr = exp(lr);
                if (gr > g) g = gr;
            }
        }
        if (keep_map) keep_map[map_row + kb] = (uint8_t)keep;
        if (margin) margin[map_row + kb] = g;
        if (!keep) continue;               /* skipped: no V, no softmax update, no PV */
        ++kept;
        /* 3. online-softmax update and PV for every row of the block */
        for (int r = 0; r < R; ++r) {
            if (M[r] == -INFINITY) continue;
            const double mn = M[r] > m[r] ? M[r] : m[r];
            const double alpha = (m[r] == -INFINITY) ? 0.0 : exp(m[r] - mn);
            double* ar = acc + (size_t)r * d;
            l[r] *= alpha;
            for (int c = 0; c < d; ++c) ar[c] *= alpha;
            for (int j = j0; j < j1; ++j) {
                const double sv = s[(size_t)r * Bk + (j - j0)];
                if (sv == -INFINITY) continue;
                const double p = exp(sv - mn);
                l[r] += p;
                const double* vj = v + IDX4(b, j, hkv, 0, Lk, Hkv, d);
                for (int c = 0; c < d; ++c) ar[c] += p * vj[c];
            }
            m[r] = mn;
        }
    }
    /* 4. O = acc / l, LSE = m + ln l */
    for (int r = 0; r < R; ++r) {
        const int i = i0 + r;
        double* oi = o + IDX4(b, i, hq, 0, Lq, Hq, d);
        for (int c = 0; c < d; ++c) oi[c] = acc[(size_t)r * d + c] / l[r];
        lse[((size_t)b * Hq + hq) * Lq + i] = m[r] + log(l[r]);
    }
    *n_kept = kept;
    free(m); free(l); free(thr); free(acc); free(s); free(M);
}

/*
 * oracle_prefill: MALA forward of Lq queries against Lk >= Lq keys (see the
 * header), over all query blocks (sel == NULL) or over the
 * nsel blocks listed in sel as (b, hq, qb) triples. Only the selected rows of
 * o / lse and the selected rows of keep_map / margin are written; kept_tiles
 * receives the number of kept tiles per (b, hq) over the selected blocks.
 * keep_map, margin and kept_tiles may be NULL.
 */
void oracle_prefill(const double* q, const double* k, const double* v, int B, int Hq, int Hkv,
                    int Lq, int Lk, int d, double scale, double tau, int Bq, int Bk,
                    const int32_t* sel, int nsel, double* o, double* lse, uint8_t* keep_map,
                    double* margin, int64_t* kept_tiles) {
    const int nq = (Lq + Bq - 1) / Bq;
    const long total = sel ? (long)nsel : (long)B * Hq * nq;
    int64_t* per = (int64_t*)calloc((size_t)(total > 0 ? total : 1), sizeof(int64_t));
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < total; ++t) {
        int b, hq, qb;
        if (sel) {
            b = sel[3 * t]; hq = sel[3 * t + 1]; qb = sel[3 * t + 2];
        } else {
            /* longest blocks first */
            long u = t;
            qb = nq - 1 - (int)(u / ((long)B * Hq));
            u %= (long)B * Hq;
            b = (int)(u / Hq); hq = (int)(u % Hq);
        }
        fwd_block(q, k, v, B, Hq, Hkv, Lq, Lk, d, scale, tau, Bq, Bk, b, hq, qb, o, lse, keep_map,
                  margin, &per[t]);
    }
    if (kept_tiles) {
        memset(kept_tiles, 0, sizeof(int64_t) * (size_t)B * Hq);
        for (long t = 0; t < total; ++t) {
            int b, hq;
            if (sel) { b = sel[3 * t]; hq = sel[3 * t + 1]; }
            else { long u = t % ((long)B * Hq); b = (int)(u / Hq); hq = (int)(u % Hq); }
            kept_tiles[b * Hq + hq] += per[t];
        }
    }
    free(per);
}

/* oracle_fwd: the training forward (queries and keys of one sequence). */
void oracle_fwd(const double* q, const double* k, const double* v, int B, int Hq, int Hkv, int L,
                int d, double scale, double tau, int Bq, int Bk, const int32_t* sel, int nsel,
                double* o, double* lse, uint8_t* keep_map, double* margin, int64_t* kept_tiles) {
    oracle_prefill(q, k, v, B, Hq, Hkv, L, L, d, scale, tau, Bq, Bk, sel, nsel, o, lse, keep_map,
                   margin, kept_tiles);
}

/*
 * oracle_dense_lse: logsumexp over all causally visible keys (no gate) for
 * every row, used for the omitted-mass diagnostic
 * omega_i = 1 - exp(LSE_i - LSEdense_i).
 */
void oracle_dense_lse(const double* q, const double* k, int B, int Hq, int Hkv, int L, int d,
                      double scale, double* lse_dense) {
    const int G = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int bh = 0; bh < B * Hq; ++bh) {
        for (int i = 0; i < L; ++i) {
            const int b = bh / Hq, hq = bh % Hq, hkv = hq / G;
            double mx = -INFINITY;
            for (int j = 0; j <= i; ++j) {
                double sv = score(q, k, b, i, j, hq, hkv, L, Hq, Hkv, d, scale);
                if (sv > mx) mx = sv;
            }
            double z = 0.0;
            for (int j = 0; j <= i; ++j) z += exp(score(q, k, b, i, j, hq, hkv, L, Hq, Hkv, d, scale) - mx);
            lse_dense[(size_t)bh * L + i] = mx + log(z);
        }
    }
}

/* ------------------------------------------------------------------------
 * Backward.
 * ---------------------------------------------------------------------- */

/* Backward gate of tile (b, hq, qb, kb) against the final LSE. */
static int bwd_keep(const double* q, const double* k, const double* lse, int Hq, int Hkv, int L,
                    int d, double scale, double tau, int Bq, int Bk, int b, int hq, int qb, int kb,
                    double* g_out) {
    const int hkv = hq / (Hq / Hkv);
    const int i0 = qb * Bq, i1 = imin((qb + 1) * Bq, L);
    const int j0 = kb * Bk, j1 = imin((kb + 1) * Bk, L);
    if (tau == 0.0) { *g_out = NAN; return 1; }
    int keep = 0;
    double g = 0.0;
    for (int i = i0; i < i1; ++i) {
        const double LSEi = lse[((size_t)b * Hq + hq) * L + i];
        const double thr = log(tau) - log((double)(i + 1));
        for (int j = j0; j < imin(j1, i + 1); ++j) {
            const double lr = score(q, k, b, i, j, hq, hkv, L, Hq, Hkv, d, scale) - LSEi - thr;
            if (lr >= 0.0) keep = 1;
            const double gr = exp(lr);
            if (gr > g) g = gr;
        }
    }
    *g_out = g;
    return keep;
}

/*
 * oracle_bwd: MALA backward.
 *   dq rows for the query blocks in selq ((b, hq, qb) triples; NULL = all),
 *   dk / dv rows for the key blocks in selk ((b, hkv, kb) triples; NULL = all).
 * D_i = <dO_i, O_i>; on a kept tile, for every live (i, j):
 *   P = exp(s - LSE_i), dP = <dO_i, v_j>, dS = P (dP - D_i),
 *   dv_j += P dO_i, dk_j += scale dS q_i, dq_i += scale dS k_j.
 * dk / dv sum over the query heads of the GQA group. The keep map / margins
 * / counts are produced by the dq sweep (so they cover selq's blocks).
 * nsel* are the triple counts. Outputs are zeroed on the selected rows first.
 */
void oracle_bwd(const double* q, const double* k, const double* v, const double* o,
                const double* dO, const double* lse, int B, int Hq, int Hkv, int L, int d,
                double scale, double tau, int Bq, int Bk, const int32_t* selq, int nselq,
                const int32_t* selk, int nselk, double* dq, double* dk, double* dv,
                uint8_t* keep_map, double* margin, int64_t* kept_tiles) {
    const int G = Hq / Hkv;
    const int nq = (L + Bq - 1) / Bq;
    const int nk = (L + Bk - 1) / Bk;

    /* D_i = <dO_i, O_i> for every row */
    double* D = (double*)malloc(sizeof(double) * (size_t)B * Hq * L);
#pragma omp parallel for collapse(2)
    for (int bh = 0; bh < B * Hq; ++bh)
        for (int i = 0; i < L; ++i) {
            const int b = bh / Hq, hq = bh % Hq;
            const double* oi = o + IDX4(b, i, hq, 0, L, Hq, d);
            const double* gi = dO + IDX4(b, i, hq, 0, L, Hq, d);
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += gi[c] * oi[c];
            D[(size_t)bh * L + i] = acc;
        }

    /* dq sweep: one task per query block */
    const long tq = selq ? (long)nselq : (long)B * Hq * nq;
    int64_t* per = (int64_t*)calloc((size_t)(tq > 0 ? tq : 1), sizeof(int64_t));
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < tq; ++t) {
        int b, hq, qb;
        if (selq) { b = selq[3 * t]; hq = selq[3 * t + 1]; qb = selq[3 * t + 2]; }
        else { qb = (int)(t % nq); long u = t / nq; hq = (int)(u % Hq); b = (int)(u / Hq); }
        const int hkv = hq / G;
        const int i0 = qb * Bq, i1 = imin((qb + 1) * Bq, L);
        for (int i = i0; i < i1; ++i) memset(dq + IDX4(b, i, hq, 0, L, Hq, d), 0, sizeof(double) * d);
        const int kb_last = (i1 - 1) / Bk;
        const size_t map_row = ((size_t)(b * Hq + hq) * nq + qb) * nk;
        for (int kb = 0; kb <= kb_last; ++kb) {
            double g;
            const int keep = bwd_keep(q, k, lse, Hq, Hkv, L, d, scale, tau, Bq, Bk, b, hq, qb, kb, &g);
            if (keep_map) keep_map[map_row + kb] = (uint8_t)keep;
            if (margin) margin[map_row + kb] = g;
            if (!keep) continue;
            per[t] += 1;
            const int j0 = kb * Bk, j1 = imin((kb + 1) * Bk, L);
            for (int i = i0; i < i1; ++i) {
                const double LSEi = lse[((size_t)b * Hq + hq) * L + i];
                const double Di = D[((size_t)b * Hq + hq) * L + i];
                const double* gi = dO + IDX4(b, i, hq, 0, L, Hq, d);
                double* dqi = dq + IDX4(b, i, hq, 0, L, Hq, d);
                for (int j = j0; j < imin(j1, i + 1); ++j) {
                    const double P = exp(score(q, k, b, i, j, hq, hkv, L, Hq, Hkv, d, scale) - LSEi);
                    const double* vj = v + IDX4(b, j, hkv, 0, L, Hkv, d);
                    const double* kj = k + IDX4(b, j, hkv, 0, L, Hkv, d);
                    double dP = 0.0;
                    for (int c = 0; c < d; ++c) dP += gi[c] * vj[c];
                    const double dS = P * (dP - Di);
                    for (int c = 0; c < d; ++c) dqi[c] += scale * dS * kj[c];
                }
            }
        }
    }
    if (kept_tiles) {
        memset(kept_tiles, 0, sizeof(int64_t) * (size_t)B * Hq);
        for (long t = 0; t < tq; ++t) {
            int b, hq;
            if (selq) { b = selq[3 * t]; hq = selq[3 * t + 1]; }
            else { long u = t / nq; hq = (int)(u % Hq); b = (int)(u / Hq); }
            kept_tiles[b * Hq + hq] += per[t];
        }
    }
    free(per);

    /* dk / dv sweep: one task per key block of a KV head */
    const long tk = selk ? (long)nselk : (long)B * Hkv * nk;
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < tk; ++t) {
        int b, hkv, kb;
        if (selk) { b = selk[3 * t]; hkv = selk[3 * t + 1]; kb = selk[3 * t + 2]; }
        else { kb = (int)(t % nk); long u = t / nk; hkv = (int)(u % Hkv); b = (int)(u / Hkv); }
        const int j0 = kb * Bk, j1 = imin((kb + 1) * Bk, L);
        for (int j = j0; j < j1; ++j) {
            memset(dk + IDX4(b, j, hkv, 0, L, Hkv, d), 0, sizeof(double) * d);
            memset(dv + IDX4(b, j, hkv, 0, L, Hkv, d), 0, sizeof(double) * d);
        }
        for (int hq = hkv * G; hq < (hkv + 1) * G; ++hq) {
            for (int qb = 0; qb < nq; ++qb) {
                const int i0 = qb * Bq, i1 = imin((qb + 1) * Bq, L);
                if (kb * Bk > i1 - 1) continue; /* illegal tile */
                double g;
                if (!bwd_keep(q, k, lse, Hq, Hkv, L, d, scale, tau, Bq, Bk, b, hq, qb, kb, &g)) continue;
                for (int i = i0; i < i1; ++i) {
                    const double LSEi = lse[((size_t)b * Hq + hq) * L + i];
                    const double Di = D[((size_t)b * Hq + hq) * L + i];
                    const double* gi = dO + IDX4(b, i, hq, 0, L, Hq, d);
                    const double* qi = q + IDX4(b, i, hq, 0, L, Hq, d);
                    for (int j = j0; j < imin(j1, i + 1); ++j) {
                        const double P = exp(score(q, k, b, i, j, hq, hkv, L, Hq, Hkv, d, scale) - LSEi);
                        const double* vj = v + IDX4(b, j, hkv, 0, L, Hkv, d);
                        double* dkj = dk + IDX4(b, j, hkv, 0, L, Hkv, d);
                        double* dvj = dv + IDX4(b, j, hkv, 0, L, Hkv, d);
                        double dP = 0.0;
                        for (int c = 0; c < d; ++c) dP += gi[c] * vj[c];
                        const double dS = P * (dP - Di);
                        for (int c = 0; c < d; ++c) {
                            dvj[c] += P * gi[c];
                            dkj[c] += scale * dS * qi[c];
                        }
                    }
                }
            }
        }
    }
    free(D);
}

/* ------------------------------------------------------------------------
 * Decode: one query per (b, hq) against a KV cache of Lk keys, split-KV.
 * ---------------------------------------------------------------------- */

/* Tile range of split s: [s*T, min((s+1)*T, nk)), T = ceil(nk / n_splits). */
static void split_range(int nk, int n_splits, int s, int* t0, int* t1) {
    const int T = (nk + n_splits - 1) / n_splits;
    *t0 = imin(s * T, nk);
    *t1 = imin((s + 1) * T, nk);
}

/*
 * oracle_decode: q [B, Hq, d]; kc, vc [B, Lk, Hkv, d]. The query is row
 * i = Lk - 1 (every key visible, Lq = Lk). Each split runs the forward gate
 * with its own fresh state from its newest tile to its oldest, always keeping
 * its newest tile; partials (O_s, LSE_s) are then merged:
 * LSE = log sum_s exp(LSE_s), O = sum_s exp(LSE_s - LSE) O_s.
 * Outputs: o [B, Hq, d], lse [B, Hq], keep_map [B, Hq, nk] and margin
 * [B, Hq, nk] (nullable), kept_tiles [B * Hq] (nullable); o_part
 * [B, Hq, n_splits, d] and lse_part [B, Hq, n_splits] (nullable; empty
 * splits hold LSE = -inf and O = 0). sel lists (b, hq) pairs (NULL = all).
 */
void oracle_decode(const double* q, const double* kc, const double* vc, int B, int Hq, int Hkv,
                   int Lk, int d, double scale, double tau, int Bk, int n_splits,
                   const int32_t* sel, int nsel, double* o, double* lse, uint8_t* keep_map,
                   double* margin, int64_t* kept_tiles, double* o_part, double* lse_part) {
    const int G = Hq / Hkv;
    const int nk = (Lk + Bk - 1) / Bk;
    const long total = sel ? (long)nsel : (long)B * Hq;
    if (kept_tiles) memset(kept_tiles, 0, sizeof(int64_t) * (size_t)B * Hq);
#pragma omp parallel for schedule(dynamic, 1)
    for (long t = 0; t < total; ++t) {
        int b, hq;
        if (sel) { b = sel[2 * t]; hq = sel[2 * t + 1]; }
        else { b = (int)(t / Hq); hq = (int)(t % Hq); }
        const int hkv = hq / G;
        const int i = Lk - 1;
        const double thr = tau > 0.0 ? log(tau) - log((double)Lk) : -INFINITY;
        const double* qi = q + ((size_t)b * Hq + hq) * d;
        double* pm = (double*)malloc(sizeof(double) * n_splits);
        double* pl = (double*)malloc(sizeof(double) * n_splits);
        double* pacc = (double*)calloc((size_t)n_splits * d, sizeof(double));
        double* s = (double*)malloc(sizeof(double) * Bk);
        int64_t kept = 0;
        for (int sp = 0; sp < n_splits; ++sp) {
            int t0, t1;
            split_range(nk, n_splits, sp, &t0, &t1);
            double m = -INFINITY, l = 0.0;
            double* acc = pacc + (size_t)sp * d;
            for (int kb = t1 - 1; kb >= t0; --kb) { /* newest toward oldest */
                const int j0 = kb * Bk, j1 = imin((kb + 1) * Bk, Lk);
                double M = -INFINITY;
                for (int j = j0; j < j1; ++j) {
                    const double* kj = kc + IDX4(b, j, hkv, 0, Lk, Hkv, d);
                    double a = 0.0;
                    for (int c = 0; c < d; ++c) a += qi[c] * kj[c];
                    s[j - j0] = (j <= i) ? scale * a : -INFINITY;
                    if (s[j - j0] > M) M = s[j - j0];
                }
                int keep;
                double g = NAN;
                if (kb == t1 - 1) keep = 1;
                else if (tau == 0.0) keep = 1;
                else {
                    const double lr = (l > 0.0) ? (M - m - log(l)) - thr : INFINITY;
                    keep = lr >= 0.0;
                    g = exp(lr);
                }
                const size_t mi = ((size_t)b * Hq + hq) * nk + kb;
                if (keep_map) keep_map[mi] = (uint8_t)keep;
                if (margin) margin[mi] = g;
                if (!keep) continue;
                ++kept;
                const double mn = M > m ? M : m;
                const double alpha = (m == -INFINITY) ? 0.0 : exp(m - mn);
                l *= alpha;
                for (int c = 0; c < d; ++c) acc[c] *= alpha;
                for (int j = j0; j < j1; ++j) {
                    if (s[j - j0] == -INFINITY) continue;
                    const double p = exp(s[j - j0] - mn);
                    l += p;
                    const double* vj = vc + IDX4(b, j, hkv, 0, Lk, Hkv, d);
                    for (int c = 0; c < d; ++c) acc[c] += p * vj[c];
                }
                m = mn;
            }
            pm[sp] = m;
            pl[sp] = l;
        }
        /* combine the splits by their LSEs */
        double lmax = -INFINITY;
        for (int sp = 0; sp < n_splits; ++sp) {
            const double ls = (pl[sp] > 0.0) ? pm[sp] + log(pl[sp]) : -INFINITY;
            if (lse_part) lse_part[((size_t)b * Hq + hq) * n_splits + sp] = ls;
            if (o_part)
                for (int c = 0; c < d; ++c)
                    o_part[(((size_t)b * Hq + hq) * n_splits + sp) * d + c] =
                        (pl[sp] > 0.0) ? pacc[(size_t)sp * d + c] / pl[sp] : 0.0;
            if (ls > lmax) lmax = ls;
        }
        double z = 0.0;
        for (int sp = 0; sp < n_splits; ++sp)
            if (pl[sp] > 0.0) z += exp(pm[sp] + log(pl[sp]) - lmax);
        const double LSE = lmax + log(z);
        double* oi = o + ((size_t)b * Hq + hq) * d;
        for (int c = 0; c < d; ++c) oi[c] = 0.0;
        for (int sp = 0; sp < n_splits; ++sp) {
            if (pl[sp] <= 0.0) continue;
            const double w = exp(pm[sp] + log(pl[sp]) - LSE);
            for (int c = 0; c < d; ++c) oi[c] += w * pacc[(size_t)sp * d + c] / pl[sp];
        }
        lse[(size_t)b * Hq + hq] = LSE;
        if (kept_tiles) {
#pragma omp atomic
            kept_tiles[b * Hq + hq] += kept;
        }
        free(pm); free(pl); free(pacc); free(s);
    }
}
