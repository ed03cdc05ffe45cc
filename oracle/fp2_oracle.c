/*
 * fp2_oracle.c -- plain fp64 CPU oracle of FlashPrefill V2 block-sparse causal
 * prefill attention with the block-mean correction.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file: only the tests, the smoke check and the bench's CPU-baseline leg
 * do.  It shares no code, header, table or helper with the CUDA library.
 *
 * Sources (the method as the pages state it; readings where they are silent
 * are marked READING):
 *   [ABS]  "FlashPrefill V2: block-sparse prefill attention for long-context
 *          LLM serving", abstract card (chatpaper.ai), English abstract:
 *          instantaneous pattern discovery, max-based dynamic thresholding,
 *          a mean correction term for the approximation error.
 *   [POP]  popular explainer (papers.ananclaw.com, popular__2608-19758),
 *          section 2.1 "algorithm layer": V1 keeps only the key blocks the
 *          threshold selects; V2 adds a term built from the mean of the
 *          dropped tokens' values ("V_avg_dropped").
 *   [NEWS] NetEase article on FlashPrefill V2 (163.com): the mean correction
 *          suppresses the error of skipping blocks.
 *
 * Readings taken where the pages leave a step open:
 *   - pooling = arithmetic mean over the valid rows of a block, for queries
 *     and keys; the same key means serve the score and the correction;
 *   - score s_ij = qbar_i . kbar_j / sqrt(d), one mask per query head;
 *   - keep j iff s_ij >= max_j' s_ij' - tau (inclusive), and always keep
 *     block 0 and the diagonal block;
 *   - correction: each dropped block j enters the SAME softmax as one
 *     pseudo-token with logit q.kbar_j/sqrt(d) + ln(n_j) and value vbar_j,
 *     i.e. weight n_j * exp(q.kbar_j/sqrt(d)) in the denominator and that
 *     weight times vbar_j in the numerator.  The explainer's printed formula
 *     (a bare subtraction of mu_q * V_avg_dropped) is garbled: it has no
 *     normaliser and mu_q is never defined; the pseudo-token form is the one
 *     that turns into exact dense attention when the dropped blocks have
 *     constant rows, which is what "removes the first-order bias" requires.
 *
 * Layouts (all fp64, row-major, one sequence per call):
 *   Q [Lq][Hq][d], K and V [Lk][Hkv][d]; query t sits at absolute position
 *   P + t with P = Lk - Lq (a resident prefix, any length >= 0).  Blocks are
 *   cut at absolute positions, for queries as for keys: query block i of the
 *   call is absolute block P/B + i (integer division) and holds the call's
 *   rows that fall in [(P/B + i)B, (P/B + i + 1)B).  When P is not a multiple
 *   of B the first query block is partial (READING: the pages' "mixed
 *   prefill + decode chunk" puts rows at arbitrary positions; a decode row is
 *   a call with Lq = 1), and its pooled query is the mean of the rows it
 *   holds.  nqb = ceil((P mod B + Lq) / B).
 *   kbar, vbar [Hkv][nkb][d]; cnt [nkb]; qbar [Hq][nqb][d];
 *   S [Hq][nqb][nkb] (entries with j > i_abs are left untouched);
 *   keep [Hq][nqb][nkb] bytes, 1 = kept, 0 = dropped or non-causal.
 *
 * Parity pins live in tests/test_oracle_pins.py.
 *
 * Compile-time mutants (used only by the mutation tests, which compile this
 * file a second time with -DFP2_ORACLE_MUTANT=k to check that the pins catch
 * a plausible slip): 1 drops the ln(n_j) term, 2 flips the inequality of the
 * threshold to strict and forgets the forced diagonal, 3 adds the correction
 * term's weight to the numerator only, 4 uses the mean of the first row of a
 * block's keys instead of the mean of the block, 5 picks a row's mask by its
 * offset in the call (t / B) instead of its absolute block, 6 pools the
 * query blocks as if the prefix were a multiple of B.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifndef FP2_ORACLE_MUTANT
#define FP2_ORACLE_MUTANT 0
#endif

static int ceil_div(int a, int b) { return (a + b - 1) / b; }

/* ---- step: block means of K and V ([POP] 2.1 "V_avg_dropped") ----------- */
void oracle_blockmean(const double* K, const double* V, int Lk, int Hkv, int d, int B,
                      double* kbar, double* vbar, int* cnt)
{
    int nkb = ceil_div(Lk, B);
    for (int j = 0; j < nkb; ++j) {
        int t0 = j * B, t1 = (j + 1) * B < Lk ? (j + 1) * B : Lk;
        cnt[j] = t1 - t0;
        for (int h = 0; h < Hkv; ++h) {
            double* kb = kbar + ((size_t)h * nkb + j) * d;
            double* vb = vbar + ((size_t)h * nkb + j) * d;
            for (int c = 0; c < d; ++c) {
                double sk = 0.0, sv = 0.0;
                for (int t = t0; t < t1; ++t) {
#if FP2_ORACLE_MUTANT == 4
                    sk += K[((size_t)t0 * Hkv + h) * d + c];
#else
                    sk += K[((size_t)t * Hkv + h) * d + c];
#endif
                    sv += V[((size_t)t * Hkv + h) * d + c];
                }
                kb[c] = sk / (double)(t1 - t0);
                vb[c] = sv / (double)(t1 - t0);
            }
        }
    }
}

/* ---- step: pooled query blocks ([ABS] instantaneous pattern discovery) ---
 * off = P mod B, the offset of the call's first row inside its block. */
void oracle_pool_q(const double* Q, int Lq, int Hq, int d, int B, int off, double* qbar)
{
    int nqb = ceil_div(off + Lq, B);
#if FP2_ORACLE_MUTANT == 6
    off = 0;
#endif
    for (int i = 0; i < nqb; ++i) {
        int t0 = i * B - off, t1 = (i + 1) * B - off;
        if (t0 < 0) t0 = 0;
        if (t1 > Lq) t1 = Lq;
        for (int h = 0; h < Hq; ++h)
            for (int c = 0; c < d; ++c) {
                double s = 0.0;
                for (int t = t0; t < t1; ++t) s += Q[((size_t)t * Hq + h) * d + c];
                qbar[((size_t)h * nqb + i) * d + c] = s / (double)(t1 - t0);
            }
    }
}

/* ---- step: block scores s_ij = qbar_i . kbar_j / sqrt(d), j <= i_abs ----- */
void oracle_score(const double* qbar, const double* kbar, int Hq, int Hkv, int nqb, int nkb,
                  int d, int prefix_blocks, double* S)
{
    int G = Hq / Hkv;
    double scale = 1.0 / sqrt((double)d);
    for (int h = 0; h < Hq; ++h) {
        int hk = h / G;
        for (int i = 0; i < nqb; ++i) {
            int iabs = prefix_blocks + i;
            for (int j = 0; j <= iabs && j < nkb; ++j) {
                double s = 0.0;
                for (int c = 0; c < d; ++c)
                    s += qbar[((size_t)h * nqb + i) * d + c] * kbar[((size_t)hk * nkb + j) * d + c];
                S[((size_t)h * nqb + i) * nkb + j] = s * scale;
            }
        }
    }
}

/* ---- step: max-based dynamic threshold ([ABS]) -------------------------- */
void oracle_mask(const double* S, int Hq, int nqb, int nkb, int prefix_blocks, double tau,
                 unsigned char* keep)
{
    for (int h = 0; h < Hq; ++h)
        for (int i = 0; i < nqb; ++i) {
            int iabs = prefix_blocks + i;
            const double* row = S + ((size_t)h * nqb + i) * nkb;
            unsigned char* kr = keep + ((size_t)h * nqb + i) * nkb;
            memset(kr, 0, (size_t)nkb);
            double m = -INFINITY;
            for (int j = 0; j <= iabs; ++j) if (row[j] > m) m = row[j];
            for (int j = 0; j <= iabs; ++j) {
#if FP2_ORACLE_MUTANT == 2
                kr[j] = (row[j] > m - tau) || j == 0;
#else
                kr[j] = (row[j] >= m - tau) || j == 0 || j == iabs;
#endif
            }
        }
}

/*
 * ---- step: attention over kept tokens + one pseudo-token per dropped block
 * For query row t (absolute position p = P + t), head h:
 *   kept token u (block kept, u <= p):   logit z_u = q.k_u / sqrt(d), value v_u
 *   dropped block j (j < p/B, not kept): logit q.kbar_j / sqrt(d) + ln n_j, value vbar_j
 *   out = sum_x exp(z_x - M) val_x / sum_x exp(z_x - M),  M = max_x z_x.
 * If wsum is given, it receives sum_x w_x with w_x = exp(z_x-M)/den computed
 * term by term (the weight-sum invariant).
 * rows[r] are local query indices, heads[r] their heads; out is [nrows][d].
 */
void oracle_attn_rows(const double* Q, const double* K, const double* V,
                      const double* kbar, const double* vbar, const int* cnt,
                      const unsigned char* keep, int Lq, int Lk, int Hq, int Hkv, int d, int B,
                      const int* rows, const int* heads, int nrows, double* out, double* wsum)
{
    int G = Hq / Hkv;
    int P = Lk - Lq;
    int nqb = ceil_div(P % B + Lq, B), nkb = ceil_div(Lk, B);
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r], h = heads[r], hk = h / G;
        int p = P + t;
        int iabs = p / B;           /* absolute query block */
#if FP2_ORACLE_MUTANT == 5
        int i = t / B;
#else
        int i = iabs - P / B;       /* query block of the call */
#endif
        const double* q = Q + ((size_t)t * Hq + h) * d;
        const unsigned char* kr = keep + ((size_t)h * nqb + i) * nkb;
        /* logits and values: at most Lk tokens + nkb pseudo-tokens */
        int cap = Lk + nkb;
        double* z = (double*)malloc(sizeof(double) * (size_t)cap);
        const double** val = (const double**)malloc(sizeof(double*) * (size_t)cap);
        int nx = 0;
        for (int j = 0; j <= iabs; ++j) {
            if (kr[j]) {
                int u1 = (j + 1) * B - 1 < p ? (j + 1) * B - 1 : p;
                for (int u = j * B; u <= u1; ++u) {
                    const double* k = K + ((size_t)u * Hkv + hk) * d;
                    double s = 0.0;
                    for (int c = 0; c < d; ++c) s += q[c] * k[c];
                    z[nx] = s * scale;
                    val[nx] = V + ((size_t)u * Hkv + hk) * d;
                    ++nx;
                }
            } else {
                const double* kb = kbar + ((size_t)hk * nkb + j) * d;
                double s = 0.0;
                for (int c = 0; c < d; ++c) s += q[c] * kb[c];
#if FP2_ORACLE_MUTANT == 1
                z[nx] = s * scale;
#else
                z[nx] = s * scale + log((double)cnt[j]);
#endif
                val[nx] = vbar + ((size_t)hk * nkb + j) * d;
                ++nx;
            }
        }
        double M = -INFINITY;
        for (int x = 0; x < nx; ++x) if (z[x] > M) M = z[x];
        double den = 0.0;
        double* o = out + (size_t)r * d;
        for (int c = 0; c < d; ++c) o[c] = 0.0;
        for (int x = 0; x < nx; ++x) {
            double w = exp(z[x] - M);
#if FP2_ORACLE_MUTANT == 3
            if (val[x] < V || val[x] >= V + (size_t)Lk * Hkv * d) { /* pseudo-token */
                for (int c = 0; c < d; ++c) o[c] += w * val[x][c];
                continue;
            }
#endif
            den += w;
            for (int c = 0; c < d; ++c) o[c] += w * val[x][c];
        }
        for (int c = 0; c < d; ++c) o[c] /= den;
        if (wsum) {
            double sw = 0.0;
            for (int x = 0; x < nx; ++x) sw += exp(z[x] - M) / den;
            wsum[r] = sw;
        }
        free(z);
        free((void*)val);
    }
}

/*
 * Brute-force dense causal softmax(Q K^T / sqrt(d)) V (textbook), written
 * independently of the sparse routine above: the full causal logit row is
 * formed, the softmax taken, then V weighted.  GQA: head h reads KV head h/G.
 */
void oracle_dense_rows(const double* Q, const double* K, const double* V, int Lq, int Lk,
                       int Hq, int Hkv, int d, const int* rows, const int* heads, int nrows,
                       double* out)
{
    int G = Hq / Hkv;
    int P = Lk - Lq;
    double scale = 1.0 / sqrt((double)d);
#pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < nrows; ++r) {
        int t = rows[r], h = heads[r], hk = h / G, p = P + t;
        double* a = (double*)malloc(sizeof(double) * (size_t)(p + 1));
        double mx = -INFINITY;
        for (int u = 0; u <= p; ++u) {
            double s = 0.0;
            for (int c = 0; c < d; ++c)
                s += Q[((size_t)t * Hq + h) * d + c] * K[((size_t)u * Hkv + hk) * d + c];
            a[u] = s * scale;
            if (a[u] > mx) mx = a[u];
        }
        double den = 0.0;
        for (int u = 0; u <= p; ++u) { a[u] = exp(a[u] - mx); den += a[u]; }
        for (int c = 0; c < d; ++c) {
            double s = 0.0;
            for (int u = 0; u <= p; ++u) s += a[u] * V[((size_t)u * Hkv + hk) * d + c];
            out[(size_t)r * d + c] = s / den;
        }
        free(a);
    }
}

/* Thread count OpenMP will use (reported beside the CPU baseline). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
