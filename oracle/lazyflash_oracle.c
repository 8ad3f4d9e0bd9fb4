/*
 * LazyFlash CPU oracle: plain, slow, fp64 C.  TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the bench's CPU-baseline arm may load
 * this file's library.  The CUDA product path never calls it, shares no code
 * with it and must fail loudly, not fall back here, when its own library is
 * missing.
 *
 * What it computes follows the LazyFlash article ("LazyFlash allège la
 * rétropropagation de l'attention, 5,72 fois", gyom.fr, 26 Oct 2026):
 *   - the forward is exactly dense attention, which FlashAttention reaches
 *     without approximation (article, standfirst and section "Le passage
 *     arrière fait deux fois le travail du passage avant"; voce.life course
 *     "FlashAttention et la circulation des données", section "Le mécanisme");
 *   - query blocks are ranked by the norm of their output gradient and a budget
 *     delta bounds the share of gradient mass thrown away, per head and per step
 *     (article, section "Un budget sur la masse de gradient ...");
 *   - each block is kept with probability proportional to its gradient and
 *     kept blocks are reweighted so the gradient stays unbiased in expectation
 *     (same section, second paragraph).
 * The precise reading used here: p_b = min(1, m_b / tau), tau the largest value
 * whose expected discarded mass sum_b (1 - p_b) m_b is at most delta * sum_b m_b,
 * found by 64 bisection steps (each test multiplied through by the midpoint, so
 * that it takes no division); the draw is word 0 of Philox4x32-10 (Salmon,
 * Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3", SC'11)
 * keyed on the seed and countered on (block, head, segment, step); kept blocks
 * carry weight 1/p_b.
 *
 * Everything is written from those definitions, untiled, row by row.  All
 * floating point is IEEE fp64 with contraction disabled (-ffp-contract=off);
 * inputs are bf16 values upcast exactly by the caller.
 *
 * Layout: token tensors are [T][H][d] row-major ("THD"); segment s covers rows
 * cu_seqlens[s] .. cu_seqlens[s+1]-1.  lse and D are [Hq][T].  Per-block arrays
 * are [nseq][Hq][nbmax].  Query head h reads KV head h / (Hq/Hkv).
 *
 * Parity pins (see tests/test_oracle_*.py): torch fp64 SDPA and autograd for
 * the dense forward/backward, central finite differences, the closed form of
 * tau, the budget inequality, the Philox known-answer vectors, the linear
 * block decomposition of the gradient and a Monte-Carlo unbiasedness test.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define LFO_OK 0
#define LFO_EINVAL 1

/* LFO_MUTANT selects one deliberately planted mistake, so that the tests can
 * check that the pins catch it (tests/test_oracle_mutants.py).  0 = the
 * oracle as written; every other value is used only by that test. */
#ifndef LFO_MUTANT
#define LFO_MUTANT 0
#endif

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al., SC'11, section 5): a 10-round bijection of a  */
/* 128-bit counter under a 64-bit key.  Each round multiplies words 0 and 2 by */
/* fixed odd constants, crosses the high halves with words 1 and 3 and the     */
/* round key, and the key is bumped by the Weyl increments between rounds.     */
/* ------------------------------------------------------------------------ */
static const uint32_t PHILOX_M0 = 0xD2511F53u;
static const uint32_t PHILOX_M1 = 0xCD9E8D57u;
static const uint32_t PHILOX_W0 = 0x9E3779B9u;
static const uint32_t PHILOX_W1 = 0xBB67AE85u;

void lfo_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < (LFO_MUTANT == 7 ? 9 : 10); ++round) {
        if (round > 0) { k0 += PHILOX_W0; k1 += PHILOX_W1; }
        uint64_t p0 = (uint64_t)PHILOX_M0 * (uint64_t)c0;
        uint64_t p1 = (uint64_t)PHILOX_M1 * (uint64_t)c2;
        uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        uint32_t n0 = hi1 ^ c1 ^ k0;
        uint32_t n1 = lo1;
        uint32_t n2 = hi0 ^ c3 ^ k1;
        uint32_t n3 = lo0;
        c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    }
    out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 24-bit uniform of block i, head h, segment s at (seed, step). */
uint32_t lfo_block_u24(uint64_t seed, uint64_t step, int s, int h, int i)
{
    uint32_t ctr[4] = { (uint32_t)i, (uint32_t)h, (uint32_t)s, (uint32_t)(step & 0xffffffffu) };
    uint32_t key[2] = { (uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32) };
    uint32_t out[4];
    lfo_philox4x32_10(ctr, key, out);
    return out[0] >> 8;
}

/* ------------------------------------------------------------------------ */
/* Dense attention, one query row at a time (textbook definition).            */
/* ------------------------------------------------------------------------ */

/* Scores of query row t (absolute index) of head h against the keys it may  */
/* see; returns the number of keys n (keys u0 .. u0+n-1).                      */
static int row_scores(int t, int seg0, int seg1, int causal, int hq, int hkv, int d,
                      double scale, int h, const double* q, const double* k, double* srow)
{
    int G = hq / hkv, g = (LFO_MUTANT == 2) ? h % hkv : h / G;
    int u_end = causal ? ((LFO_MUTANT == 9 && t > seg0) ? t : t + 1) : seg1;
    const double* qt = q + ((size_t)t * hq + h) * d;
    int n = 0;
    for (int u = seg0; u < u_end; ++u) {
        const double* ku = k + ((size_t)u * hkv + g) * d;
        double acc = 0.0;
        for (int c = 0; c < d; ++c) acc += qt[c] * ku[c];
        srow[n++] = (LFO_MUTANT == 1) ? acc : scale * acc;
    }
    return n;
}

/* In place: srow <- softmax(srow); returns the natural-log LSE. */
static double row_softmax(double* srow, int n)
{
    double mx = -INFINITY;
    for (int i = 0; i < n; ++i) if (srow[i] > mx) mx = srow[i];
    double l = 0.0;
    for (int i = 0; i < n; ++i) l += exp(srow[i] - mx);
    double lse = mx + log(l);
    for (int i = 0; i < n; ++i) srow[i] = exp(srow[i] - lse);
    return lse;
}

static int check_desc(int nseq, const int32_t* cu, int T, int hq, int hkv, int d)
{
    if (nseq < 1 || !cu || hq < 1 || hkv < 1 || d < 1 || hq % hkv) return LFO_EINVAL;
    if (cu[0] != 0 || cu[nseq] != T) return LFO_EINVAL;
    for (int s = 0; s < nseq; ++s) if (cu[s + 1] < cu[s]) return LFO_EINVAL;
    return LFO_OK;
}

/* O[t,h,:] = sum_u softmax_u(scale <q_t, k_u>) v_u ; lse[h][t] = ln sum_u exp(.) */
int lfo_attn_fwd(int nseq, const int32_t* cu, int T, int hq, int hkv, int d, double scale,
                 int causal, const double* q, const double* k, const double* v,
                 double* o, double* lse)
{
    if (check_desc(nseq, cu, T, hq, hkv, d)) return LFO_EINVAL;
    int G = hq / hkv;
    int maxlen = 0;
    for (int s = 0; s < nseq; ++s) if (cu[s + 1] - cu[s] > maxlen) maxlen = cu[s + 1] - cu[s];
    #pragma omp parallel
    {
        double* srow = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        #pragma omp for collapse(2) schedule(dynamic, 1)
        for (int s = 0; s < nseq; ++s)
            for (int h = 0; h < hq; ++h) {
                int g = h / G;
                for (int t = cu[s]; t < cu[s + 1]; ++t) {
                    int n = row_scores(t, cu[s], cu[s + 1], causal, hq, hkv, d, scale, h, q, k, srow);
                    double L = row_softmax(srow, n);
                    double* ot = o + ((size_t)t * hq + h) * d;
                    for (int c = 0; c < d; ++c) ot[c] = 0.0;
                    for (int i = 0; i < n; ++i) {
                        const double* vu = v + ((size_t)(cu[s] + i) * hkv + g) * d;
                        for (int c = 0; c < d; ++c) ot[c] += srow[i] * vu[c];
                    }
                    lse[(size_t)h * T + t] = L;
                }
            }
        free(srow);
    }
    return LFO_OK;
}

/* ------------------------------------------------------------------------ */
/* Selection.                                                                 */
/* ------------------------------------------------------------------------ */

/* m[s][h][i] = Frobenius norm of the dO rows of block i (rows                */
/* seg0 + i*block .. min(seg0 + (i+1)*block, seg1) - 1) of head h; zero past   */
/* the segment's last block.                                                   */
int lfo_block_norms(int nseq, const int32_t* cu, int T, int hq, int d, int block, int nbmax,
                    const double* dout, double* norms)
{
    if (check_desc(nseq, cu, T, hq, hq, d) || block < 1) return LFO_EINVAL;
    for (int s = 0; s < nseq; ++s) {
        int len = cu[s + 1] - cu[s];
        if ((len + block - 1) / block > nbmax) return LFO_EINVAL;
    }
    #pragma omp parallel for collapse(2)
    for (int s = 0; s < nseq; ++s)
        for (int h = 0; h < hq; ++h) {
            int len = cu[s + 1] - cu[s];
            int nb = (len + block - 1) / block;
            for (int i = 0; i < nbmax; ++i) {
                double acc = 0.0;
                if (i < nb) {
                    int r0 = cu[s] + i * block;
                    int r1 = cu[s] + (i + 1) * block;
                    if (r1 > cu[s + 1]) r1 = cu[s + 1];
                    for (int t = r0; t < r1; ++t) {
                        const double* row = dout + ((size_t)t * hq + h) * d;
                        for (int c = 0; c < d; ++c) acc += row[c] * row[c];
                    }
                }
                norms[((size_t)s * hq + h) * nbmax + i] = (LFO_MUTANT == 10) ? acc : sqrt(acc);
            }
        }
    return LFO_OK;
}

/* D[h][t] = <dO_t, O_t> (per head, unweighted). */
int lfo_rowdot(int T, int hq, int d, const double* dout, const double* o, double* D)
{
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < hq; ++h) {
            const double* a = dout + ((size_t)t * hq + h) * d;
            const double* b = o + ((size_t)t * hq + h) * d;
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += a[c] * b[c];
            D[(size_t)h * T + t] = acc;
        }
    return LFO_OK;
}

/* The fixed summation order of the budget sums: 32 partial sums, partial l    */
/* adding x[l], x[l+32], ... in index order, then five pairwise combination    */
/* rounds v[l] <- v[l] + v[l xor r] for r = 16, 8, 4, 2, 1.  Any order would    */
/* do for the definition; this one is fixed so that both implementations make */
/* identical keep decisions.                                                  */
double lfo_pinned_sum(const double* x, int n)
{
    double lane[32], nxt[32];
    for (int l = 0; l < 32; ++l) {
        double acc = 0.0;
        for (int i = l; i < n; i += 32) acc = acc + x[i];
        lane[l] = acc;
    }
    for (int r = 16; r >= 1; r >>= 1) {
        for (int l = 0; l < 32; ++l) nxt[l] = lane[l] + lane[l ^ r];
        memcpy(lane, nxt, sizeof lane);
    }
    return lane[0];
}

/* Expected discarded mass at threshold tau: sum_b (1 - min(1, m_b/tau)) m_b. */
double lfo_discarded_mass(const double* m, int n, double tau, double* scratch)
{
    for (int b = 0; b < n; ++b)
        scratch[b] = (m[b] >= tau) ? 0.0
                   : (LFO_MUTANT == 6 ? (m[b] / tau) * m[b] : (1.0 - m[b] / tau) * m[b]);
    return lfo_pinned_sum(scratch, n);
}

/* The bisection's test at a threshold t > 0: is the expected discarded mass   */
/* within the budget B?  The inequality sum_b [m_b < t] (1 - m_b/t) m_b <= B is */
/* multiplied through by t, so that it takes no division:                       */
/*   sum_b [m_b < t] (m_b t - m_b^2) <= B t.                                    */
/* Each term is one fused multiply-add of m_b, t and -m_b^2 (the square is      */
/* exact for fp32 norms), the sum takes the pinned order and B t is one rounded */
/* product.  Any rounding would do for the definition; this one is fixed so     */
/* that both implementations make identical bisection steps.                    */
static int lfo_budget_met(const double* m, int n, double t, double B, double* scratch)
{
    for (int b = 0; b < n; ++b)
        scratch[b] = (m[b] >= t) ? 0.0
                   : (LFO_MUTANT == 6 ? m[b] * m[b] : fma(m[b], t, -(m[b] * m[b])));
    return lfo_pinned_sum(scratch, n) <= B * t;
}

/* tau of one (segment, head): the largest feasible threshold, by bisection.   */
/* Returns 0 when every block is kept outright (delta == 0 or no mass).         */
double lfo_tau(const double* m, int n, double delta)
{
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double M = lfo_pinned_sum(m, n);
    double tau = 0.0;
    if (delta > 0.0 && M > 0.0) {
        double B = delta * M;
        double mx = 0.0;
        for (int b = 0; b < n; ++b) if (m[b] > mx) mx = m[b];
        double lo = 0.0, hi = mx / (1.0 - delta);
        for (int it = 0; it < 64; ++it) {
            double mid = 0.5 * (lo + hi);
            if (lfo_budget_met(m, n, mid, B, scratch)) lo = mid; else hi = mid;
        }
        tau = lo;
    }
    free(scratch);
    return tau;
}

/* Full selection for every (segment, head):                                  */
/*   tau by bisection; p_b = min(1, m_b/tau) (p = 1 when tau == 0);           */
/*   keep iff p_b >= 1 or u24 < p_b * 2^24; w_b = (float)(1/p_b) if kept, else 0;*/
/*   kept_idx lists kept block indices in ascending order, kept_cnt counts them.*/
/* norms: [nseq][hq][nbmax]; nb[s] = blocks of segment s.                      */
int lfo_select(int nseq, const int32_t* nb, int hq, int nbmax, const double* norms,
               double delta, uint64_t seed, uint64_t step,
               double* tau, double* p, float* w, uint8_t* keep,
               int32_t* kept_idx, int32_t* kept_cnt)
{
    if (nseq < 1 || hq < 1 || nbmax < 1 || !(delta >= 0.0 && delta < 1.0)) return LFO_EINVAL;
    for (int s = 0; s < nseq; ++s) if (nb[s] < 0 || nb[s] > nbmax) return LFO_EINVAL;
    #pragma omp parallel for collapse(2)
    for (int s = 0; s < nseq; ++s)
        for (int h = 0; h < hq; ++h) {
            size_t base = ((size_t)s * hq + h) * nbmax;
            const double* m = norms + base;
            int n = nb[s];
            double t = lfo_tau(m, n, delta);
            tau[(size_t)s * hq + h] = t;
            int cnt = 0;
            for (int i = 0; i < nbmax; ++i) {
                double pi = 0.0;
                int kb = 0;
                float wi = 0.0f;
                if (i < n) {
                    if (t == 0.0) pi = 1.0;
                    else { pi = m[i] / t; if (pi > 1.0) pi = 1.0; }
                    if (pi >= 1.0) kb = 1;
                    else {
                        uint32_t u = lfo_block_u24(seed, step, s, h, i);
                        kb = ((double)u < pi * 16777216.0);
                    }
                    if (kb) wi = (float)(LFO_MUTANT == 8 ? pi : 1.0 / pi);
                }
                p[base + i] = pi;
                keep[base + i] = (uint8_t)kb;
                w[base + i] = wi;
                kept_idx[base + i] = -1;
                if (kb) kept_idx[base + cnt++] = i;
            }
            kept_cnt[(size_t)s * hq + h] = cnt;
        }
    return LFO_OK;
}

/* ------------------------------------------------------------------------ */
/* Backward of L = sum_t <w_{b(t)} dO_t, O_t> with respect to q, k, v.         */
/* With dO~_t = w dO_t, P the softmax of row t:                               */
/*   D_t = <dO~_t, O_t>, dP_tu = <dO~_t, v_u>, dS_tu = P_tu (dP_tu - D_t),     */
/*   dQ_t = scale sum_u dS_tu k_u, dK_u = scale sum_{h in group} sum_t dS_tu q_t,*/
/*   dV_u = sum_{h in group} sum_t P_tu dO~_t.                                 */
/* wblk: [nseq][hq][nbmax] block weights, or NULL for all ones (dense).         */
/* ------------------------------------------------------------------------ */
int lfo_attn_bwd(int nseq, const int32_t* cu, int T, int hq, int hkv, int d, double scale,
                 int causal, int block, int nbmax,
                 const double* q, const double* k, const double* v, const double* dout,
                 const double* wblk, double* dq, double* dk, double* dv)
{
    if (check_desc(nseq, cu, T, hq, hkv, d) || block < 1) return LFO_EINVAL;
    int G = hq / hkv;
    int maxlen = 0;
    for (int s = 0; s < nseq; ++s) if (cu[s + 1] - cu[s] > maxlen) maxlen = cu[s + 1] - cu[s];
    memset(dq, 0, sizeof(double) * (size_t)T * hq * d);
    memset(dk, 0, sizeof(double) * (size_t)T * hkv * d);
    memset(dv, 0, sizeof(double) * (size_t)T * hkv * d);
    #pragma omp parallel
    {
        double* prow = (double*)malloc(sizeof(double) * (size_t)(maxlen > 0 ? maxlen : 1));
        double* ot = (double*)malloc(sizeof(double) * (size_t)d);
        double* dot_ = (double*)malloc(sizeof(double) * (size_t)d);
        /* one task per (segment, KV head): it owns dK/dV of that head */
        #pragma omp for collapse(2) schedule(dynamic, 1)
        for (int s = 0; s < nseq; ++s)
            for (int g = 0; g < hkv; ++g) {
                int seg0 = cu[s];
                for (int h = g * G; h < (g + 1) * G; ++h) {
                    for (int t = cu[s]; t < cu[s + 1]; ++t) {
                        double wt = 1.0;
                        if (wblk) wt = wblk[((size_t)s * hq + h) * nbmax + (t - seg0) / block];
                        const double* dot_raw = dout + ((size_t)t * hq + h) * d;
                        for (int c = 0; c < d; ++c) dot_[c] = wt * dot_raw[c];
                        int n = row_scores(t, cu[s], cu[s + 1], causal, hq, hkv, d, scale, h, q, k, prow);
                        (void)row_softmax(prow, n);
                        for (int c = 0; c < d; ++c) ot[c] = 0.0;
                        for (int i = 0; i < n; ++i) {
                            const double* vu = v + ((size_t)(seg0 + i) * hkv + g) * d;
                            for (int c = 0; c < d; ++c) ot[c] += prow[i] * vu[c];
                        }
                        double Dt = 0.0;
                        for (int c = 0; c < d; ++c)
                            Dt += (LFO_MUTANT == 3 ? dot_raw[c] : dot_[c]) * ot[c];
                        const double* qt = q + ((size_t)t * hq + h) * d;
                        double* dqt = dq + ((size_t)t * hq + h) * d;
                        for (int i = 0; i < n; ++i) {
                            int u = seg0 + i;
                            const double* vu = v + ((size_t)u * hkv + g) * d;
                            const double* ku = k + ((size_t)u * hkv + g) * d;
                            double dP = 0.0;
                            for (int c = 0; c < d; ++c) dP += dot_[c] * vu[c];
                            double P = prow[i];
                            double dS = (LFO_MUTANT == 5) ? P * (Dt - dP) : P * (dP - Dt);
                            double* dku = dk + ((size_t)u * hkv + g) * d;
                            double* dvu = dv + ((size_t)u * hkv + g) * d;
                            for (int c = 0; c < d; ++c) {
                                dqt[c] += scale * dS * ku[c];
                                dku[c] += (LFO_MUTANT == 4 ? 1.0 : scale) * dS * qt[c];
                                dvu[c] += P * dot_[c];
                            }
                        }
                    }
                }
            }
        free(prow); free(ot); free(dot_);
    }
    return LFO_OK;
}

/* ------------------------------------------------------------------------ */
/* The same definitions evaluated only at chosen rows, for parity checks at    */
/* sizes where the full oracle would take hours.  Nothing is reordered: each  */
/* requested output is the same sum over the same rows as above.              */
/* ------------------------------------------------------------------------ */

static int segment_of(int nseq, const int32_t* cu, int t)
{
    int lo = 0, hi = nseq - 1;
    while (lo < hi) {               /* last s with cu[s] <= t (skips empty segments) */
        int mid = (lo + hi + 1) / 2;
        if (cu[mid] <= t) lo = mid; else hi = mid - 1;
    }
    while (lo + 1 <= nseq - 1 && cu[lo + 1] <= t) ++lo;
    return lo;
}

/* O and LSE of query rows (rows[r], heads[r]); o_out [nrows][d], lse_out [nrows]. */
int lfo_attn_fwd_rows(int nseq, const int32_t* cu, int T, int hq, int hkv, int d, double scale,
                      int causal, const double* q, const double* k, const double* v,
                      int nrows, const int32_t* rows, const int32_t* heads,
                      double* o_out, double* lse_out)
{
    if (check_desc(nseq, cu, T, hq, hkv, d)) return LFO_EINVAL;
    int G = hq / hkv;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r], h = heads[r];
        int s = segment_of(nseq, cu, t);
        int len = cu[s + 1] - cu[s];
        double* srow = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        int n = row_scores(t, cu[s], cu[s + 1], causal, hq, hkv, d, scale, h, q, k, srow);
        lse_out[r] = row_softmax(srow, n);
        for (int c = 0; c < d; ++c) o_out[(size_t)r * d + c] = 0.0;
        for (int i = 0; i < n; ++i) {
            const double* vu = v + ((size_t)(cu[s] + i) * hkv + h / G) * d;
            for (int c = 0; c < d; ++c) o_out[(size_t)r * d + c] += srow[i] * vu[c];
        }
        free(srow);
    }
    return LFO_OK;
}

/* Weighted backward at chosen rows: dq_out[r] = dQ[qrows[r], qheads[r], :];   */
/* dk_out[r], dv_out[r] = dK, dV[kvrows[r], kvheads[r], :].  wblk as in         */
/* lfo_attn_bwd (NULL = all ones).                                              */
int lfo_attn_bwd_rows(int nseq, const int32_t* cu, int T, int hq, int hkv, int d, double scale,
                      int causal, int block, int nbmax,
                      const double* q, const double* k, const double* v, const double* dout,
                      const double* wblk,
                      int nq, const int32_t* qrows, const int32_t* qheads, double* dq_out,
                      int nkv, const int32_t* kvrows, const int32_t* kvheads,
                      double* dk_out, double* dv_out)
{
    if (check_desc(nseq, cu, T, hq, hkv, d) || block < 1) return LFO_EINVAL;
    int G = hq / hkv;
    /* dQ rows: each needs only its own softmax row */
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nq; ++r) {
        int t = qrows[r], h = qheads[r], g = h / G;
        int s = segment_of(nseq, cu, t), seg0 = cu[s];
        int len = cu[s + 1] - seg0;
        double* prow = (double*)malloc(sizeof(double) * (size_t)(len > 0 ? len : 1));
        double* ot = (double*)calloc((size_t)d, sizeof(double));
        double* dot_ = (double*)malloc(sizeof(double) * (size_t)d);
        double wt = wblk ? wblk[((size_t)s * hq + h) * nbmax + (t - seg0) / block] : 1.0;
        const double* dr = dout + ((size_t)t * hq + h) * d;
        for (int c = 0; c < d; ++c) dot_[c] = wt * dr[c];
        int n = row_scores(t, seg0, cu[s + 1], causal, hq, hkv, d, scale, h, q, k, prow);
        (void)row_softmax(prow, n);
        for (int i = 0; i < n; ++i) {
            const double* vu = v + ((size_t)(seg0 + i) * hkv + g) * d;
            for (int c = 0; c < d; ++c) ot[c] += prow[i] * vu[c];
        }
        double Dt = 0.0;
        for (int c = 0; c < d; ++c) Dt += dot_[c] * ot[c];
        double* out = dq_out + (size_t)r * d;
        for (int c = 0; c < d; ++c) out[c] = 0.0;
        for (int i = 0; i < n; ++i) {
            const double* vu = v + ((size_t)(seg0 + i) * hkv + g) * d;
            const double* ku = k + ((size_t)(seg0 + i) * hkv + g) * d;
            double dP = 0.0;
            for (int c = 0; c < d; ++c) dP += dot_[c] * vu[c];
            double dS = prow[i] * (dP - Dt);
            for (int c = 0; c < d; ++c) out[c] += scale * dS * ku[c];
        }
        free(prow); free(ot); free(dot_);
    }
    /* dK/dV rows: sum over every query row t of the group that sees key u.     */
    /* Requested rows are handled per (segment, KV head): first LSE_t and D_t of */
    /* every query row that can see one of them, then the per-pair terms.        */
    char* done = (char*)calloc((size_t)(nkv > 0 ? nkv : 1), 1);
    int* members = (int*)malloc(sizeof(int) * (size_t)(nkv > 0 ? nkv : 1));
    for (int r0 = 0; r0 < nkv; ++r0) {
        if (done[r0]) continue;
        int g = kvheads[r0];
        int s = segment_of(nseq, cu, kvrows[r0]), seg0 = cu[s], seg1 = cu[s + 1];
        int nm = 0, umin = kvrows[r0];
        for (int r = r0; r < nkv; ++r)
            if (!done[r] && kvheads[r] == g && segment_of(nseq, cu, kvrows[r]) == s) {
                done[r] = 1;
                members[nm++] = r;
                if (kvrows[r] < umin) umin = kvrows[r];
            }
        int t0 = causal ? umin : seg0;
        int nt = seg1 - t0;
        double* lse_t = (double*)malloc(sizeof(double) * (size_t)G * (nt > 0 ? nt : 1));
        double* D_t = (double*)malloc(sizeof(double) * (size_t)G * (nt > 0 ? nt : 1));
        #pragma omp parallel
        {
            double* prow = (double*)malloc(sizeof(double) * (size_t)(seg1 - seg0 > 0 ? seg1 - seg0 : 1));
            double* ot = (double*)malloc(sizeof(double) * (size_t)d);
            #pragma omp for collapse(2) schedule(dynamic, 4)
            for (int hh = 0; hh < G; ++hh)
                for (int it = 0; it < nt; ++it) {
                    int h = g * G + hh, t = t0 + it;
                    double wt = wblk ? wblk[((size_t)s * hq + h) * nbmax + (t - seg0) / block] : 1.0;
                    int n = row_scores(t, seg0, seg1, causal, hq, hkv, d, scale, h, q, k, prow);
                    double L = row_softmax(prow, n);
                    for (int c = 0; c < d; ++c) ot[c] = 0.0;
                    for (int i = 0; i < n; ++i) {
                        const double* vi = v + ((size_t)(seg0 + i) * hkv + g) * d;
                        for (int c = 0; c < d; ++c) ot[c] += prow[i] * vi[c];
                    }
                    const double* dr = dout + ((size_t)t * hq + h) * d;
                    double Dt = 0.0;
                    for (int c = 0; c < d; ++c) Dt += (wt * dr[c]) * ot[c];
                    lse_t[(size_t)hh * nt + it] = L;
                    D_t[(size_t)hh * nt + it] = Dt;
                }
            free(prow); free(ot);
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (int mi = 0; mi < nm; ++mi) {
            int r = members[mi], u = kvrows[r];
            const double* vu = v + ((size_t)u * hkv + g) * d;
            const double* ku = k + ((size_t)u * hkv + g) * d;
            double* dk = dk_out + (size_t)r * d;
            double* dv = dv_out + (size_t)r * d;
            for (int c = 0; c < d; ++c) { dk[c] = 0.0; dv[c] = 0.0; }
            for (int hh = 0; hh < G; ++hh) {
                int h = g * G + hh;
                for (int t = causal ? u : seg0; t < seg1; ++t) {
                    double wt = wblk ? wblk[((size_t)s * hq + h) * nbmax + (t - seg0) / block] : 1.0;
                    if (wt == 0.0) continue;     /* dO~_t = 0: the row adds exactly nothing */
                    const double* qt = q + ((size_t)t * hq + h) * d;
                    const double* dr = dout + ((size_t)t * hq + h) * d;
                    double sc = 0.0, dP = 0.0;
                    for (int c = 0; c < d; ++c) sc += qt[c] * ku[c];
                    for (int c = 0; c < d; ++c) dP += (wt * dr[c]) * vu[c];
                    double P = exp(scale * sc - lse_t[(size_t)hh * nt + (t - t0)]);
                    double dS = P * (dP - D_t[(size_t)hh * nt + (t - t0)]);
                    for (int c = 0; c < d; ++c) {
                        dk[c] += scale * dS * qt[c];
                        dv[c] += P * (wt * dr[c]);
                    }
                }
            }
        }
        free(lse_t); free(D_t);
    }
    free(done); free(members);
    return LFO_OK;
}

/* ------------------------------------------------------------------------ */
/* Alternative selection rules compared by the article at equal backward     */
/* time (section "Le choix des blocs pèse plus que la quantité sautée"):      */
/*  rule 1, fixed fraction f: the same proportional draw and 1/p weights, but */
/*    tau is the largest threshold whose expected kept count                  */
/*    sum_b min(1, m_b/tau) is at least f*n (a fraction fixed for the whole   */
/*    run instead of the adaptive mass budget);                               */
/*  rule 2, top-k: the k = ceil(f*n) largest norms (ties: lower index), kept  */
/*    deterministically with weight 1 (the same blocks at every step).        */
/* tau reports the threshold (rule 1) or the k-th largest norm (rule 2).      */
/* ------------------------------------------------------------------------ */
double lfo_expected_kept(const double* m, int n, double tau, double* scratch)
{
    for (int b = 0; b < n; ++b) scratch[b] = (m[b] >= tau) ? 1.0 : m[b] / tau;
    return lfo_pinned_sum(scratch, n);
}

/* The fixed-fraction test at t > 0, multiplied through by t like the budget   */
/* test: sum_b min(1, m_b/t) >= target becomes sum_b min(t, m_b) >= target t    */
/* (every term exact; pinned order; target t one rounded product).              */
static int lfo_count_met(const double* m, int n, double t, double target, double* scratch)
{
    for (int b = 0; b < n; ++b) scratch[b] = (m[b] >= t) ? t : m[b];
    return lfo_pinned_sum(scratch, n) >= target * t;
}

double lfo_tau_fixed_fraction(const double* m, int n, double f)
{
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double M = lfo_pinned_sum(m, n);
    double tau = 0.0;
    if (n > 0 && M > 0.0 && f < 1.0) {
        double target = f * (double)n;
        double lo = 0.0, hi = M / target;
        for (int it = 0; it < 64; ++it) {
            double mid = 0.5 * (lo + hi);
            if (lfo_count_met(m, n, mid, target, scratch)) lo = mid; else hi = mid;
        }
        tau = lo;
    }
    free(scratch);
    return tau;
}

static int topk_count(int n, double f)
{
    double kd = ceil(f * (double)n);
    int k = (int)kd;
    if (k > n) k = n;
    if (k < 0) k = 0;
    return k;
}

int lfo_select_rule(int rule, int nseq, const int32_t* nb, int hq, int nbmax, const double* norms,
                    double param, uint64_t seed, uint64_t step,
                    double* tau, double* p, float* w, uint8_t* keep,
                    int32_t* kept_idx, int32_t* kept_cnt)
{
    if (rule == 0)
        return lfo_select(nseq, nb, hq, nbmax, norms, param, seed, step, tau, p, w, keep,
                          kept_idx, kept_cnt);
    if (rule != 1 && rule != 2) return LFO_EINVAL;
    if (nseq < 1 || hq < 1 || nbmax < 1 || !(param > 0.0 && param <= 1.0)) return LFO_EINVAL;
    for (int s = 0; s < nseq; ++s) if (nb[s] < 0 || nb[s] > nbmax) return LFO_EINVAL;
    #pragma omp parallel for collapse(2)
    for (int s = 0; s < nseq; ++s)
        for (int h = 0; h < hq; ++h) {
            size_t base = ((size_t)s * hq + h) * nbmax;
            const double* m = norms + base;
            int n = nb[s];
            int cnt = 0;
            if (rule == 1) {
                double t = lfo_tau_fixed_fraction(m, n, param);
                tau[(size_t)s * hq + h] = t;
                for (int i = 0; i < nbmax; ++i) {
                    double pi = 0.0;
                    int kb = 0;
                    float wi = 0.0f;
                    if (i < n) {
                        if (t == 0.0) pi = 1.0;
                        else { pi = m[i] / t; if (pi > 1.0) pi = 1.0; }
                        if (pi >= 1.0) kb = 1;
                        else kb = ((double)lfo_block_u24(seed, step, s, h, i) < pi * 16777216.0);
                        if (kb) wi = (float)(1.0 / pi);
                    }
                    p[base + i] = pi;
                    keep[base + i] = (uint8_t)kb;
                    w[base + i] = wi;
                    kept_idx[base + i] = -1;
                    if (kb) kept_idx[base + cnt++] = i;
                }
            } else {
                int k = topk_count(n, param);
                double kth = 0.0;
                for (int i = 0; i < nbmax; ++i) {
                    int kb = 0;
                    if (i < n) {
                        /* rank: blocks with a larger norm, or an equal norm and lower index */
                        int rank = 0;
                        for (int j = 0; j < n; ++j)
                            if (m[j] > m[i] || (m[j] == m[i] && j < i)) ++rank;
                        kb = rank < k;
                        if (rank == k - 1) kth = m[i];
                    }
                    p[base + i] = kb ? 1.0 : 0.0;
                    keep[base + i] = (uint8_t)kb;
                    w[base + i] = kb ? 1.0f : 0.0f;
                    kept_idx[base + i] = -1;
                    if (kb) kept_idx[base + cnt++] = i;
                }
                tau[(size_t)s * hq + h] = kth;
            }
            kept_cnt[(size_t)s * hq + h] = cnt;
        }
    return LFO_OK;
}
