/*
 * moc_oracle.c - plain fp64 CPU restatement of the Mixture of Contexts (MoC)
 * sparse-attention forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the checker, not the product: only
 * the tests, the package smoke check and the benchmark's CPU-baseline leg
 * load it. It shares no code, header, table or helper with the CUDA library
 * and includes nothing from it. Every function is written for a reader who
 * checks it against the pages by eye: no blocking, fusion or reordering
 * beyond what the definition states.
 *
 * Pages restated (titles as they appear on the web pages):
 *  [S]  "Mixture of Contexts for Long Video Generation | Summary"
 *       §3.1: dense attention is Softmax(Q K^T / sqrt(d)) V; for the routed
 *       index set Omega(q_i) MoC computes Softmax(q_i K_Omega^T / sqrt(d)) V_Omega;
 *       each query scores a chunk by the dot product of the query with the
 *       chunk's mean-pooled key and keeps the top-k chunks; routing is done
 *       independently per head.
 *       §3.2: every visual query keeps all text (caption) tokens and its own
 *       shot as mandatory context; optional edges i->j are masked whenever
 *       j >= i before the top-k step.
 *  [W]  the jxzklqfsx.com write-up of MoC (arXiv 2508.21058), section
 *       "計算效率": the mandatory links are inserted before top-k so the
 *       router spends no budget on chunks that are already mandatory.
 *  [P4] "Miscela di Contesti per la Generazione di Video Lunghi" (abstract):
 *       mandatory anchors are the caption and local windows.
 *
 * Readings where the pages are silent (stated once, used below):
 *  - caption queries attend densely to every token of the sample;
 *  - the router score is the unscaled dot product q . Kbar_j;
 *  - ties in the top-k order go to the lower chunk index; fewer than k
 *    candidates selects all of them and pads the selection with -1;
 *  - "causal" compares chunk indices: candidate j must satisfy j < i where i
 *    is the query's own chunk;
 *  - anchor modes: SHOT = every video chunk of the query's shot; LOCAL = video
 *    chunks of the query's shot whose frame is within +-radius of the query's
 *    frame; CHUNK = the query's own chunk only.
 *
 * Inputs are bf16 bit patterns (uint16) of head-major [BH][L][d] tensors;
 * every product and sum below is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORC_NONE = 0, ORC_ANCHOR = 1, ORC_CAND = 2 };
enum { ORC_SHOT = 0, ORC_LOCAL = 1, ORC_CHUNK = 2 };
enum { ORC_CAPTION = 0, ORC_VIDEO = 1 };

static double bf16_value(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int moc_oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Role of key chunk j for a query in chunk i ([S] §3.2, [W] 計算效率).
 * role[i*C + j] is ORC_ANCHOR (mandatory), ORC_CAND (may be routed) or
 * ORC_NONE (never attended). Returns 0, or -1 on a bad anchor mode. */
int moc_oracle_roles(int C, const int32_t* kind, const int32_t* shot, const int32_t* frame,
                     int anchor_mode, int radius, int causal, uint8_t* role) {
    if (anchor_mode != ORC_SHOT && anchor_mode != ORC_LOCAL && anchor_mode != ORC_CHUNK) return -1;
    for (int i = 0; i < C; ++i) {
        for (int j = 0; j < C; ++j) {
            uint8_t r;
            if (kind[i] == ORC_CAPTION) {
                r = ORC_ANCHOR;                 /* caption query: dense */
            } else if (kind[j] == ORC_CAPTION) {
                r = ORC_ANCHOR;                 /* forced cross-modal link */
            } else {
                int anchored;
                if (anchor_mode == ORC_SHOT)
                    anchored = (shot[j] == shot[i]);
                else if (anchor_mode == ORC_LOCAL)
                    anchored = (shot[j] == shot[i]) && abs(frame[j] - frame[i]) <= radius;
                else
                    anchored = (j == i);
                if (anchored)
                    r = ORC_ANCHOR;
                else if (!causal || j < i)
                    r = ORC_CAND;
                else
                    r = ORC_NONE;               /* causal routing mask */
            }
            role[(size_t)i * C + j] = r;
        }
    }
    return 0;
}

/* Chunk of token t, from chunk offsets off[0..C] (off[0] = 0, off[C] = L). */
static int chunk_of(int C, const int64_t* off, int64_t t) {
    int lo = 0, hi = C - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) / 2;
        if (off[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

/* Mean-pooled key of every chunk ([S] §3.1): Kbar[bh][c][e] = (1/n_c) * sum over
 * tokens t of chunk c, in token order, of K[bh][t][e]. */
void moc_oracle_pool(int64_t BH, int64_t L, int d, const uint16_t* K, int C,
                     const int64_t* off, double* Kbar) {
    #pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int64_t bh = 0; bh < BH; ++bh) {
        for (int c = 0; c < C; ++c) {
            double* out = Kbar + ((size_t)bh * C + c) * d;
            for (int e = 0; e < d; ++e) out[e] = 0.0;
            for (int64_t t = off[c]; t < off[c + 1]; ++t) {
                const uint16_t* row = K + ((size_t)bh * L + t) * d;
                for (int e = 0; e < d; ++e) out[e] += bf16_value(row[e]);
            }
            double n = (double)(off[c + 1] - off[c]);
            for (int e = 0; e < d; ++e) out[e] /= n;
        }
    }
}

/* Router score of chunk j for query row q: sum_e q_e * Kbar_j,e, and the
 * magnitude sum_e |q_e * Kbar_j,e| used to judge near-ties. */
static void score(int d, const uint16_t* q, const double* kbar, double* s, double* a) {
    double acc = 0.0, mag = 0.0;
    for (int e = 0; e < d; ++e) {
        double p = bf16_value(q[e]) * kbar[e];
        acc += p;
        mag += fabs(p);
    }
    *s = acc;
    *a = mag;
}

typedef struct { double s; double a; int j; } cand_t;

/* (score descending, chunk id ascending) */
static int cand_cmp(const void* x, const void* y) {
    const cand_t* p = (const cand_t*)x;
    const cand_t* q = (const cand_t*)y;
    if (p->s > q->s) return -1;
    if (p->s < q->s) return 1;
    return (p->j < q->j) ? -1 : (p->j > q->j);
}

/* Top-k routing for the query tokens rows[0..nrows) of every head ([S] §3.1,
 * §3.2; [W] 計算效率). Candidates are the chunks whose role is ORC_CAND for
 * the query's chunk; all of them are scored, sorted by (score desc, id asc),
 * and the first min(k, n) are kept.
 * Outputs, per (bh, row):
 *   sel[k]        selected chunk ids in that order, -1 padded;
 *   ncand         number of candidates;
 *   top_s[k+1], top_a[k+1], top_j[k+1]: score, magnitude and id of the first
 *                 k+1 entries of the sorted list (NaN / -1 padded). */
void moc_oracle_route(int64_t BH, int64_t L, int d, const uint16_t* Q, int C, const int64_t* off,
                      const uint8_t* role, const double* Kbar, int k, int64_t nrows,
                      const int64_t* rows, int32_t* sel, int32_t* ncand, double* top_s,
                      double* top_a, int32_t* top_j) {
    #pragma omp parallel
    {
        cand_t* buf = (cand_t*)malloc(sizeof(cand_t) * (size_t)(C > 0 ? C : 1));
        #pragma omp for collapse(2) schedule(dynamic, 64)
        for (int64_t bh = 0; bh < BH; ++bh) {
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t t = rows[r];
                int i = chunk_of(C, off, t);
                const uint16_t* q = Q + ((size_t)bh * L + t) * d;
                int n = 0;
                for (int j = 0; j < C; ++j) {
                    if (role[(size_t)i * C + j] != ORC_CAND) continue;
                    score(d, q, Kbar + ((size_t)bh * C + j) * d, &buf[n].s, &buf[n].a);
                    buf[n].j = j;
                    ++n;
                }
                qsort(buf, (size_t)n, sizeof(cand_t), cand_cmp);
                size_t o = (size_t)bh * nrows + r;
                for (int x = 0; x < k; ++x) sel[o * k + x] = (x < n) ? buf[x].j : -1;
                for (int x = 0; x <= k; ++x) {
                    top_s[o * (k + 1) + x] = (x < n) ? buf[x].s : NAN;
                    top_a[o * (k + 1) + x] = (x < n) ? buf[x].a : NAN;
                    top_j[o * (k + 1) + x] = (x < n) ? buf[x].j : -1;
                }
                ncand[o] = n;
            }
        }
        free(buf);
    }
}

/* Router score for arbitrary (bh, token, chunk) triples, used to judge
 * whether a differing selection is a near-tie swap. */
void moc_oracle_scores(int64_t BH, int64_t L, int d, const uint16_t* Q, int C, const double* Kbar,
                       int64_t n, const int64_t* bh_idx, const int64_t* tok, const int32_t* chunk,
                       double* s, double* a) {
    (void)BH;
    #pragma omp parallel for schedule(static)
    for (int64_t x = 0; x < n; ++x) {
        const uint16_t* q = Q + ((size_t)bh_idx[x] * L + tok[x]) * d;
        score(d, q, Kbar + ((size_t)bh_idx[x] * C + chunk[x]) * d, &s[x], &a[x]);
    }
}

/* Exact softmax attention over Omega(t) ([S] §3.1) for the query tokens
 * rows[0..nrows) of every head. Omega(t) = tokens of every chunk whose role is
 * ORC_ANCHOR for t's chunk, plus tokens of the chunks listed in
 * sel[(bh*nrows + r)*k ..] (entries < 0 are empty slots). Scores are
 * scale * (q . K_u); the softmax subtracts the row maximum before exp.
 * Outputs O[bh][r][d], lse[bh][r] = log sum_u exp(score_u), and
 * nkeys[bh][r] = |Omega(t)|. */
void moc_oracle_attend(int64_t BH, int64_t L, int d, const uint16_t* Q, const uint16_t* K,
                       const uint16_t* V, int C, const int64_t* off, const uint8_t* role, int k,
                       const int32_t* sel, double scale, int64_t nrows, const int64_t* rows,
                       double* O, double* lse, int64_t* nkeys) {
    #pragma omp parallel
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        int64_t* u_of = (int64_t*)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
        unsigned char* in_omega = (unsigned char*)malloc((size_t)(C > 0 ? C : 1));
        #pragma omp for collapse(2) schedule(dynamic, 4)
        for (int64_t bh = 0; bh < BH; ++bh) {
            for (int64_t r = 0; r < nrows; ++r) {
                int64_t t = rows[r];
                int i = chunk_of(C, off, t);
                size_t o = (size_t)bh * nrows + r;
                for (int j = 0; j < C; ++j) in_omega[j] = (role[(size_t)i * C + j] == ORC_ANCHOR);
                for (int x = 0; x < k; ++x) {
                    int j = sel[o * k + x];
                    if (j >= 0 && j < C) in_omega[j] = 1;
                }
                const uint16_t* q = Q + ((size_t)bh * L + t) * d;
                int64_t n = 0;
                double m = -INFINITY;
                for (int j = 0; j < C; ++j) {
                    if (!in_omega[j]) continue;
                    for (int64_t u = off[j]; u < off[j + 1]; ++u) {
                        const uint16_t* kr = K + ((size_t)bh * L + u) * d;
                        double acc = 0.0;
                        for (int e = 0; e < d; ++e) acc += bf16_value(q[e]) * bf16_value(kr[e]);
                        s[n] = scale * acc;
                        u_of[n] = u;
                        if (s[n] > m) m = s[n];
                        ++n;
                    }
                }
                double z = 0.0;
                for (int64_t x = 0; x < n; ++x) {
                    s[x] = exp(s[x] - m);
                    z += s[x];
                }
                double* out = O + o * d;
                for (int e = 0; e < d; ++e) out[e] = 0.0;
                for (int64_t x = 0; x < n; ++x) {
                    const uint16_t* vr = V + ((size_t)bh * L + u_of[x]) * d;
                    double w = s[x] / z;
                    for (int e = 0; e < d; ++e) out[e] += w * bf16_value(vr[e]);
                }
                lse[o] = m + log(z);
                nkeys[o] = n;
            }
        }
        free(s);
        free(u_of);
        free(in_omega);
    }
}

/* Number of kept (query, key) pairs of one head over all L query tokens,
 * given every token's selection sel[L][k]: sum over t of |Omega(t)|. */
int64_t moc_oracle_kept_pairs(int64_t L, int C, const int64_t* off, const uint8_t* role, int k,
                              const int32_t* sel) {
    int64_t total = 0;
    for (int i = 0; i < C; ++i) {
        int64_t anchored = 0;
        for (int j = 0; j < C; ++j)
            if (role[(size_t)i * C + j] == ORC_ANCHOR) anchored += off[j + 1] - off[j];
        for (int64_t t = off[i]; t < off[i + 1]; ++t) {
            total += anchored;
            for (int x = 0; x < k; ++x) {
                int j = sel[(size_t)t * k + x];
                if (j >= 0) total += off[j + 1] - off[j];
            }
        }
    }
    (void)L;
    return total;
}
