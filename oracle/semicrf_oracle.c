/*
 * semicrf_oracle.c -- plain float64 CPU oracle for the semi-Markov CRF that the
 * Flash-SemiCRF pages describe.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or load
 * this file: only the tests, the package smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, table or helper with the
 * CUDA library; both sides are fed the same seeded inputs from the synthetic
 * generator, which holds none of the method's arithmetic.
 *
 * What it computes (one sequence per call, everything in float64):
 *
 *   Model ("Streaming Structured Inference with Flash-SemiCRF", explainer
 *   section 1 "Problem Statement"; abstract): a segmentation of positions
 *   0..L-1 into segments [s, t) of duration k = t - s in 1..K, each with a
 *   label c in 0..C-1.  Its score is the sum over segments of
 *       content(s, t, c) + dur[k-1, c]
 *   plus trans[c', c] between consecutive segments (labels c' then c).  There
 *   is no start or end transition (the first segment carries no trans term).
 *   content(s, t, c) is the sum of the (centred) emissions of label c over the
 *   positions s..t-1 (explainer section 2, "On-the-Fly Edge Computation via
 *   Prefix Sums": the segment content score).  Optional boundary projections
 *   (explainer section 2, "Boundary Projections") add P_start[s, c] +
 *   P_end[t-1, c] to the segment: a score for starting at position s and one
 *   for ending at position t-1.
 *
 *   Centering (explainer section 2, "Emission Baseline Centering"): a
 *   per-sequence, per-label baseline nu[c] = mean over the L valid positions
 *   of e[u, c] is subtracted before anything else.
 *
 *   log Z is the log-sum-exp of the scores of all segmentations.  The oracle
 *   materialises every edge explicitly, one end-position block W[k, c', c] at a
 *   time: segment content is an explicit running sum over the k positions (no
 *   prefix differences), alpha and beta are full-length arrays with no ring,
 *   no checkpoint and no normalisation, and every log-sum-exp is the two-pass
 *   max / sum-of-exp form.  Marginals are accumulated from the explicit edge
 *   posteriors:
 *     start_marg[s, c]  = P(a segment with label c starts at boundary s)
 *     end_marg[t, c]    = P(a segment with label c ends at boundary t)
 *     pos_marg[u, c]    = P(position u lies in a segment with label c),
 *                         summed explicitly over every segment covering u
 *     grad_dur[k-1, c]  = g * expected number of label-c segments of duration k
 *     grad_trans[c', c] = g * expected number of c' -> c transitions
 *     grad_e[u, c]      = g * d logZ / d e[u, c]; with centering this is
 *                         pos_marg[u, c] - mean_v pos_marg[v, c]
 *   (explainer section 4, "Correctness": marginals, boundary probabilities and
 *   gradients of log Z).
 *
 *   Viterbi: the same recursion in the max semiring, with ties broken towards
 *   the smallest duration k, then the smallest previous label c', and at the
 *   end towards the smallest final label.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* log(sum(exp(x[i]))) by the two-pass max / sum form.  NaN in, NaN out. */
static double lse(const double *x, int n)
{
    double m = -INFINITY;
    for (int i = 0; i < n; ++i) {
        if (isnan(x[i])) return NAN;
        if (x[i] > m) m = x[i];
    }
    if (m == -INFINITY) return -INFINITY;
    if (m == INFINITY) return INFINITY;
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += exp(x[i] - m);
    return m + log(s);
}

/* nu[c] = mean of e[u, c] over u < L (0 when centering is off or L == 0), and
 * the centred emissions et[u, c] = e[u, c] - nu[c]. */
void oracle_center(const double *e, int L, int C, int center, double *et, double *nu)
{
    for (int c = 0; c < C; ++c) {
        double acc = 0.0;
        if (center && L > 0) {
            for (int u = 0; u < L; ++u) acc += e[(size_t)u * C + c];
            acc /= (double)L;
        }
        nu[c] = acc;
    }
    for (int u = 0; u < L; ++u)
        for (int c = 0; c < C; ++c)
            et[(size_t)u * C + c] = e[(size_t)u * C + c] - nu[c];
}

/* S[t, c] = sum_{u < t} et[u, c] for t = 0..L (the prefix-sum array of the
 * centred emissions). */
void oracle_prefix(const double *et, int L, int C, double *S)
{
    for (int c = 0; c < C; ++c) S[c] = 0.0;
    for (int t = 1; t <= L; ++t)
        for (int c = 0; c < C; ++c)
            S[(size_t)t * C + c] = S[(size_t)(t - 1) * C + c] + et[(size_t)(t - 1) * C + c];
}

/* content[k-1, c] = sum_{u = t-k}^{t-1} et[u, c] for k = 1..kmax, as an
 * explicit running sum walking back from position t-1. */
static void contents_ending_at(const double *et, int C, int t, int kmax, double *content)
{
    for (int c = 0; c < C; ++c) content[c] = et[(size_t)(t - 1) * C + c];
    for (int k = 2; k <= kmax; ++k)
        for (int c = 0; c < C; ++c)
            content[(size_t)(k - 1) * C + c] =
                content[(size_t)(k - 2) * C + c] + et[(size_t)(t - k) * C + c];
}

/* content[k-1, c] = sum_{u = s}^{s+k-1} et[u, c] for k = 1..kmax, walking
 * forward from position s. */
static void contents_starting_at(const double *et, int C, int s, int kmax, double *content)
{
    for (int c = 0; c < C; ++c) content[c] = et[(size_t)s * C + c];
    for (int k = 2; k <= kmax; ++k)
        for (int c = 0; c < C; ++c)
            content[(size_t)(k - 1) * C + c] =
                content[(size_t)(k - 2) * C + c] + et[(size_t)(s + k - 1) * C + c];
}

/* Boundary projection terms of segment [s, t) with label c
 * ("Streaming Structured Inference with Flash-SemiCRF", explainer section 2,
 * "Boundary Projections": start and end features added to the edge
 * potential): ps[s, c] + pe[t-1, c], either array may be NULL (no term). */
static double proj(const double *ps, const double *pe, int C, int s, int t, int c)
{
    double v = 0.0;
    if (ps) v += ps[(size_t)s * C + c];
    if (pe) v += pe[(size_t)(t - 1) * C + c];
    return v;
}

/* The explicit edge block for segments ending at boundary t:
 *   W[k-1, c', c] = content(t-k, t, c) + dur[k-1, c] + proj + trans[c', c]   (t-k >= 1)
 *   W[k-1, 0,  c] = content(0,   t, c) + dur[k-1, c] + proj                  (t-k == 0)
 */
static void edge_block(const double *content, const double *trans, const double *dur,
                       const double *ps, const double *pe, int C, int t, int kmax, double *W)
{
    for (int k = 1; k <= kmax; ++k) {
        double *Wk = W + (size_t)(k - 1) * C * C;
        for (int cp = 0; cp < C; ++cp)
            for (int c = 0; c < C; ++c) {
                double v = content[(size_t)(k - 1) * C + c] + dur[(size_t)(k - 1) * C + c] +
                           proj(ps, pe, C, t - k, t, c);
                if (t - k >= 1) v += trans[(size_t)cp * C + c];
                Wk[(size_t)cp * C + c] = v;
            }
    }
}

/*
 * Forward-backward for one sequence of length L (positions 0..L-1).
 * e [L, C] raw emissions; trans [C, C] (trans[c', c]); dur [K, C].
 * g is d loss / d logZ for this sequence (scales the three gradients only).
 *
 * ps, pe [L, C] boundary projection scores (NULL: none), see proj().
 * Outputs (each may be NULL except logZ):
 *   alpha, beta        [(L+1), C]  full float64 forward / backward arrays
 *                                  (beta row 0 is left at 0: no segment
 *                                  precedes the first one)
 *   start_marg, end_marg [(L+1), C]
 *   pos_marg, grad_e   [L, C]
 *   grad_trans [C, C], grad_dur [K, C]: ADDED to (so a batch can share them)
 *   seg_marg  [L, K, C]  P(segment [s, s+k) with label c) at [s, k-1, c], the
 *                        explicit edge posteriors summed over the previous
 *                        label (explainer section 4, "Correctness": the
 *                        boundary and segment probabilities); entries with
 *                        s + k > L are left as passed (zero)
 * logZ_beta receives log Z recomputed from the backward side.
 * Returns 0, or -1 if the scratch allocation failed.
 */
int oracle_fb(const double *e, int L, int C, int K, const double *trans, const double *dur,
              const double *ps, const double *pe, int center, double g, double *logZ, double *logZ_beta,
              double *alpha_out, double *beta_out, double *start_marg, double *end_marg,
              double *pos_marg, double *grad_e, double *grad_trans, double *grad_dur,
              double *seg_marg)
{
    if (L <= 0) {
        *logZ = 0.0;
        if (logZ_beta) *logZ_beta = 0.0;
        if (alpha_out) memset(alpha_out, 0, sizeof(double) * (size_t)C);
        if (beta_out) memset(beta_out, 0, sizeof(double) * (size_t)C);
        if (start_marg) memset(start_marg, 0, sizeof(double) * (size_t)C);
        if (end_marg) memset(end_marg, 0, sizeof(double) * (size_t)C);
        return 0;
    }
    const size_t LC = (size_t)L * C, L1C = (size_t)(L + 1) * C;
    double *et = malloc(sizeof(double) * LC);
    double *nu = malloc(sizeof(double) * (size_t)C);
    double *alpha = malloc(sizeof(double) * L1C);
    double *beta = malloc(sizeof(double) * L1C);
    double *content = malloc(sizeof(double) * (size_t)K * C);
    double *W = malloc(sizeof(double) * (size_t)K * C * C);
    double *terms = malloc(sizeof(double) * ((size_t)K * C + 1));
    double *St = calloc(L1C, sizeof(double));
    double *En = calloc(L1C, sizeof(double));
    double *mu = calloc(LC, sizeof(double));
    if (!et || !nu || !alpha || !beta || !content || !W || !terms || !St || !En || !mu) {
        free(et); free(nu); free(alpha); free(beta); free(content); free(W); free(terms);
        free(St); free(En); free(mu);
        return -1;
    }
    oracle_center(e, L, C, center, et, nu);

    /* ---- forward: alpha[t, c] = LSE over (k, c') of alpha[t-k, c'] + W ---- */
    for (int c = 0; c < C; ++c) alpha[c] = 0.0; /* row 0 is never read */
    for (int t = 1; t <= L; ++t) {
        int kmax = t < K ? t : K;
        contents_ending_at(et, C, t, kmax, content);
        edge_block(content, trans, dur, ps, pe, C, t, kmax, W);
        for (int c = 0; c < C; ++c) {
            int n = 0;
            for (int k = 1; k <= kmax; ++k) {
                const double *Wk = W + (size_t)(k - 1) * C * C;
                if (t - k >= 1) {
                    for (int cp = 0; cp < C; ++cp)
                        terms[n++] = alpha[(size_t)(t - k) * C + cp] + Wk[(size_t)cp * C + c];
                } else {
                    terms[n++] = Wk[c]; /* first segment: no previous label */
                }
            }
            alpha[(size_t)t * C + c] = lse(terms, n);
        }
    }
    *logZ = lse(alpha + (size_t)L * C, C);

    /* ---- backward: beta[s, c'] = LSE over (k, c) of W + beta[s+k, c] ---- */
    for (int c = 0; c < C; ++c) beta[(size_t)L * C + c] = 0.0;
    for (int s = L - 1; s >= 0; --s) {
        int kmax = (L - s) < K ? (L - s) : K;
        contents_starting_at(et, C, s, kmax, content);
        if (s >= 1) {
            for (int cp = 0; cp < C; ++cp) {
                int n = 0;
                for (int k = 1; k <= kmax; ++k)
                    for (int c = 0; c < C; ++c)
                        terms[n++] = trans[(size_t)cp * C + c] + content[(size_t)(k - 1) * C + c] +
                                     dur[(size_t)(k - 1) * C + c] + proj(ps, pe, C, s, s + k, c) +
                                     beta[(size_t)(s + k) * C + c];
                beta[(size_t)s * C + cp] = lse(terms, n);
            }
        } else {
            int n = 0;
            for (int k = 1; k <= kmax; ++k)
                for (int c = 0; c < C; ++c)
                    terms[n++] = content[(size_t)(k - 1) * C + c] + dur[(size_t)(k - 1) * C + c] +
                                 proj(ps, pe, C, 0, k, c) + beta[(size_t)k * C + c];
            if (logZ_beta) *logZ_beta = lse(terms, n);
            for (int c = 0; c < C; ++c) beta[c] = 0.0;
        }
    }

    /* ---- explicit edge posteriors ---- */
    const double lz = *logZ;
    for (int t = 1; t <= L; ++t) {
        int kmax = t < K ? t : K;
        contents_ending_at(et, C, t, kmax, content);
        edge_block(content, trans, dur, ps, pe, C, t, kmax, W);
        for (int k = 1; k <= kmax; ++k) {
            const int s = t - k;
            const double *Wk = W + (size_t)(k - 1) * C * C;
            for (int c = 0; c < C; ++c) {
                double P = 0.0; /* P(segment [s, t) with label c) */
                if (s >= 1) {
                    for (int cp = 0; cp < C; ++cp) {
                        double p = exp(alpha[(size_t)s * C + cp] + Wk[(size_t)cp * C + c] +
                                       beta[(size_t)t * C + c] - lz);
                        if (grad_trans) grad_trans[(size_t)cp * C + c] += g * p;
                        P += p;
                    }
                } else {
                    P = exp(Wk[c] + beta[(size_t)t * C + c] - lz);
                }
                if (grad_dur) grad_dur[(size_t)(k - 1) * C + c] += g * P;
                if (seg_marg) seg_marg[((size_t)s * K + (k - 1)) * C + c] = P;
                St[(size_t)s * C + c] += P;
                En[(size_t)t * C + c] += P;
                for (int u = s; u < t; ++u) mu[(size_t)u * C + c] += P;
            }
        }
    }
    if (alpha_out) memcpy(alpha_out, alpha, sizeof(double) * L1C);
    if (beta_out) memcpy(beta_out, beta, sizeof(double) * L1C);
    if (start_marg) memcpy(start_marg, St, sizeof(double) * L1C);
    if (end_marg) memcpy(end_marg, En, sizeof(double) * L1C);
    if (pos_marg) memcpy(pos_marg, mu, sizeof(double) * LC);
    if (grad_e) {
        for (int c = 0; c < C; ++c) {
            double mean = 0.0;
            if (center) {
                for (int u = 0; u < L; ++u) mean += mu[(size_t)u * C + c];
                mean /= (double)L;
            }
            for (int u = 0; u < L; ++u) grad_e[(size_t)u * C + c] = g * (mu[(size_t)u * C + c] - mean);
        }
    }
    free(et); free(nu); free(alpha); free(beta); free(content); free(W); free(terms);
    free(St); free(En); free(mu);
    return 0;
}

/*
 * Max-semiring (Viterbi) decoding of one sequence.  Writes the best score, the
 * label of every position (labels[u]) and seg_start[u] = 1 where a segment of
 * the best segmentation starts.  Ties: smallest k, then smallest c', then the
 * smallest final label.  Returns 0, or -1 on allocation failure.
 */
int oracle_viterbi(const double *e, int L, int C, int K, const double *trans, const double *dur,
                   const double *ps, const double *pe, int center, double *score, int32_t *labels, uint8_t *seg_start)
{
    if (L <= 0) {
        *score = 0.0;
        return 0;
    }
    const size_t LC = (size_t)L * C, L1C = (size_t)(L + 1) * C;
    double *et = malloc(sizeof(double) * LC);
    double *nu = malloc(sizeof(double) * (size_t)C);
    double *V = malloc(sizeof(double) * L1C);
    int32_t *bk = malloc(sizeof(int32_t) * L1C);
    int32_t *bc = malloc(sizeof(int32_t) * L1C);
    double *content = malloc(sizeof(double) * (size_t)K * C);
    double *W = malloc(sizeof(double) * (size_t)K * C * C);
    if (!et || !nu || !V || !bk || !bc || !content || !W) {
        free(et); free(nu); free(V); free(bk); free(bc); free(content); free(W);
        return -1;
    }
    oracle_center(e, L, C, center, et, nu);
    for (int t = 1; t <= L; ++t) {
        int kmax = t < K ? t : K;
        contents_ending_at(et, C, t, kmax, content);
        edge_block(content, trans, dur, ps, pe, C, t, kmax, W);
        for (int c = 0; c < C; ++c) {
            double best = -INFINITY;
            int best_k = 0, best_c = -1, have = 0;
            for (int k = 1; k <= kmax; ++k) {
                const double *Wk = W + (size_t)(k - 1) * C * C;
                if (t - k >= 1) {
                    for (int cp = 0; cp < C; ++cp) {
                        double v = V[(size_t)(t - k) * C + cp] + Wk[(size_t)cp * C + c];
                        if (!have || v > best) { best = v; best_k = k; best_c = cp; have = 1; }
                    }
                } else {
                    double v = Wk[c];
                    if (!have || v > best) { best = v; best_k = k; best_c = -1; have = 1; }
                }
            }
            V[(size_t)t * C + c] = best;
            bk[(size_t)t * C + c] = best_k;
            bc[(size_t)t * C + c] = best_c;
        }
    }
    int cbest = 0;
    for (int c = 1; c < C; ++c)
        if (V[(size_t)L * C + c] > V[(size_t)L * C + cbest]) cbest = c;
    *score = V[(size_t)L * C + cbest];
    int t = L, c = cbest;
    while (t > 0) {
        int k = bk[(size_t)t * C + c];
        int cp = bc[(size_t)t * C + c];
        int s = t - k;
        for (int u = s; u < t; ++u) {
            labels[u] = c;
            seg_start[u] = (uint8_t)(u == s);
        }
        t = s;
        c = cp;
    }
    free(et); free(nu); free(V); free(bk); free(bc); free(content); free(W);
    return 0;
}

/*
 * Score of a given segmentation of one sequence (labels[u], seg_start[u] as
 * Viterbi writes them), summing content, duration and transition terms
 * explicitly.  Returns NaN if the segmentation is malformed: no start at
 * position 0, a label that changes inside a segment, a label out of range,
 * or a segment longer than K.
 */
double oracle_path_score(const double *e, int L, int C, int K, const double *trans,
                         const double *dur, const double *ps, const double *pe, int center, const int32_t *labels,
                         const uint8_t *seg_start)
{
    if (L <= 0) return 0.0;
    if (!seg_start[0]) return NAN;
    double *et = malloc(sizeof(double) * (size_t)L * C);
    double *nu = malloc(sizeof(double) * (size_t)C);
    if (!et || !nu) { free(et); free(nu); return NAN; }
    oracle_center(e, L, C, center, et, nu);
    double total = 0.0;
    int prev = -1;
    int s = 0;
    while (s < L) {
        int c = labels[s];
        if (c < 0 || c >= C) { total = NAN; break; }
        int t = s + 1;
        while (t < L && !seg_start[t]) {
            if (labels[t] != c) { total = NAN; break; }
            ++t;
        }
        if (isnan(total)) break;
        int k = t - s;
        if (k > K) { total = NAN; break; }
        double seg = 0.0;
        for (int u = s; u < t; ++u) seg += et[(size_t)u * C + c];
        seg += dur[(size_t)(k - 1) * C + c] + proj(ps, pe, C, s, t, c);
        if (prev >= 0) seg += trans[(size_t)prev * C + c];
        total += seg;
        prev = c;
        s = t;
    }
    free(et); free(nu);
    return total;
}

/*
 * Derivatives of the path score above with respect to the parameters, for
 * the training loss log Z - score(gold) ("Streaming Structured Inference with
 * Flash-SemiCRF", explainer section 4, Correctness: training to the CRF loss).
 * The score is linear in every parameter, so each derivative is a count read
 * off the segmentation:
 *   de[u, c]     = [labels[u] = c] - (centred ? n_c / L : 0), u < L,
 *                  where n_c counts the positions labelled c (the second term
 *                  is the derivative through the centring mean nu[c]);
 *   dtrans[c',c] = number of consecutive segment pairs labelled c' then c;
 *   ddur[k-1, c] = number of label-c segments of length k.
 * The outputs are overwritten.  Returns 0, or -1 (outputs zero) if the
 * segmentation is malformed in the sense of oracle_path_score.
 */
int oracle_path_counts(int L, int C, int K, int center, const int32_t *labels,
                       const uint8_t *seg_start, double *de, double *dtrans, double *ddur)
{
    memset(dtrans, 0, sizeof(double) * (size_t)C * C);
    memset(ddur, 0, sizeof(double) * (size_t)K * C);
    if (L <= 0) return 0;
    memset(de, 0, sizeof(double) * (size_t)L * C);
    if (!seg_start[0]) return -1;
    double *n = calloc((size_t)C, sizeof(double));
    if (!n) return -1;
    int prev = -1, s = 0, bad = 0;
    while (s < L && !bad) {
        const int c = labels[s];
        if (c < 0 || c >= C) { bad = 1; break; }
        int t = s + 1;
        while (t < L && !seg_start[t]) {
            if (labels[t] != c) { bad = 1; break; }
            ++t;
        }
        if (bad || t - s > K) { bad = 1; break; }
        for (int u = s; u < t; ++u) de[(size_t)u * C + c] += 1.0;
        n[c] += (double)(t - s);
        ddur[(size_t)(t - s - 1) * C + c] += 1.0;
        if (prev >= 0) dtrans[(size_t)prev * C + c] += 1.0;
        prev = c;
        s = t;
    }
    if (bad) {
        memset(de, 0, sizeof(double) * (size_t)L * C);
        memset(dtrans, 0, sizeof(double) * (size_t)C * C);
        memset(ddur, 0, sizeof(double) * (size_t)K * C);
        free(n);
        return -1;
    }
    if (center)
        for (int u = 0; u < L; ++u)
            for (int c = 0; c < C; ++c) de[(size_t)u * C + c] -= n[c] / (double)L;
    free(n);
    return 0;
}
