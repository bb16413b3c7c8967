/*
 * CPU oracle for Reformer LSH self-attention with shared query-key.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * CPU-baseline leg of the benchmark load this library.  It shares no code,
 * header, table or constant with the CUDA library: it is the plain,
 * slow, double-precision statement of what the CUDA path must compute.
 *
 * Sources.  The method is the one described in the paper note
 * "Reformer" (eightmm.github.io, notes on Kitaev, Kaiser, Levskaya,
 * "Reformer: The Efficient Transformer", ICLR 2020):
 *   [HASH]   section "LSH Attention", hash equation h(x) in {1..B}
 *   [CAND]   section "LSH Attention", candidate-set equation N_LSH(i)
 *   [OUT]    section "LSH Attention", output equation y_i = sum softmax(q.k/sqrt(d_k)) v_j
 *   [SHARED] section "Shared Query-Key Space", Q = K
 *   [SORT]   section "Sorting and Chunking", hash -> sort -> chunked attention
 *   [ROUNDS] section "Multiple Hash Rounds", N(i) = union over rounds
 *   [MASK]   section "Implementation Reading", causal mask kept after sorting,
 *            and the question of attending to the same-token position
 *
 * The note leaves several steps open; this oracle takes these readings:
 *   hash family   angular LSH: bucket = argmax over the n_buckets-vector
 *                 [x R_r ; -x R_r], R_r a d x (n_buckets/2) Gaussian matrix
 *                 per round, 0-based ids, lowest index wins an exact tie;
 *   sort          stable by original position inside a bucket;
 *   chunks        sorted slots cut into chunks of m; chunk c attends to its
 *                 own chunk and chunk c-1 (chunk 0 only to itself, no wrap);
 *                 no bucket-equality mask inside that window;
 *   keys          unit-normalised, k_j = x_j / |x_j| (0 when |x_j| = 0);
 *                 queries are x_i as stored; scale 1/sqrt(d);
 *   self          the query's own position is removed from its candidates
 *                 unless nothing else is left, in which case it attends to
 *                 itself alone;
 *   causal        key position must not exceed the query position, compared
 *                 on ORIGINAL positions;
 *   rounds        per-round outputs merged with weights softmax_r(lse_r),
 *                 no correction for keys found in several rounds;
 *   backward      gradients w.r.t. x (query role, key role through the
 *                 normalisation) and v; buckets and permutation held fixed.
 *
 * Two optional readings, each switched on by an argument:
 *   bucket mask   the strict candidate set N_LSH(i) = {j : h(q_i) = h(k_j)}
 *                 of [CAND]: inside the window only keys in the query's
 *                 bucket (of that round) are candidates;
 *   local window  the local self-attention of the HF blog summary (page
 *                 "The Reformer - Pushing the limits of language modeling",
 *                 "Approach / What changed"): no hashing, positions in their
 *                 own order, chunk c attends to chunks c - before .. c + after
 *                 (the LSH window is before = 1, after = 0 on sorted slots);
 *   self penalty  the other answer to the same-token question of [MASK]:
 *                 the query's own position is always a candidate, with the
 *                 fixed score ORACLE_SELF_PENALTY instead of q.k/sqrt(d), so
 *                 it matters only when nothing else is left (its score does
 *                 not depend on x, so it passes no gradient to x).
 *
 * Parity pins: see the oracle tests (dense special case, softmax sums,
 * stable order, identical rounds, finite differences, brute-force
 * candidate enumeration, two-bucket sign hash).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_EXPORT __attribute__((visibility("default")))

/* Score of the query's own position in the self-penalty reading (natural-log
 * units, the same scale as q.k/sqrt(d)). */
#define ORACLE_SELF_PENALTY (-1.0e5)

/* ------------------------------------------------------------------ */
/* [HASH] one hash round for n rows: bucket = argmax [x.R ; -x.R].      */
/* margin = (top1 - top2) / max(|top1|, tiny), top2 the runner-up entry  */
/* of the same n_buckets-vector; used to report near ties.               */
/* ------------------------------------------------------------------ */
ORACLE_EXPORT int oracle_hash(const double *x, long n, int d, const double *Rr,
                              int n_buckets, int32_t *bucket, double *margin)
{
    const int half = n_buckets / 2;
    double *u = (double *)malloc(sizeof(double) * (size_t)n_buckets);
    if (!u) return -1;
    for (long i = 0; i < n; ++i) {
        const double *xi = x + (size_t)i * d;
        for (int k = 0; k < half; ++k) {
            double p = 0.0;
            for (int t = 0; t < d; ++t) p += xi[t] * Rr[(size_t)t * half + k];
            u[k] = p;
            u[half + k] = -p;
        }
        int best = 0;
        for (int k = 1; k < n_buckets; ++k)
            if (u[k] > u[best]) best = k;          /* strict: first maximum kept */
        double top2 = -INFINITY;
        for (int k = 0; k < n_buckets; ++k)
            if (k != best && u[k] > top2) top2 = u[k];
        bucket[i] = best;
        if (margin) {
            double den = fabs(u[best]);
            if (den < 1e-300) den = 1e-300;
            margin[i] = (u[best] - top2) / den;
        }
    }
    free(u);
    return 0;
}

/* ------------------------------------------------------------------ */
/* [SORT] stable sort of positions by bucket: sort the unique keys      */
/* bucket * L + pos ascending.  perm[s] = original position at slot s.  */
/* ------------------------------------------------------------------ */
static int cmp_i64(const void *a, const void *b)
{
    int64_t x = *(const int64_t *)a, y = *(const int64_t *)b;
    return (x > y) - (x < y);
}

ORACLE_EXPORT int oracle_sort(const int32_t *bucket, long L, int32_t *perm)
{
    int64_t *key = (int64_t *)malloc(sizeof(int64_t) * (size_t)(L > 0 ? L : 1));
    if (!key) return -1;
    for (long p = 0; p < L; ++p) key[p] = (int64_t)bucket[p] * (int64_t)L + p;
    qsort(key, (size_t)L, sizeof(int64_t), cmp_i64);
    for (long s = 0; s < L; ++s) perm[s] = (int32_t)(key[s] % L);
    free(key);
    return 0;
}

/* Unit-normalised key k_j = x_j / |x_j| ([SHARED] with normalised keys). */
static void normalise_keys(const double *x, long L, int d, double *khat, double *norm)
{
    for (long j = 0; j < L; ++j) {
        double s = 0.0;
        for (int t = 0; t < d; ++t) s += x[(size_t)j * d + t] * x[(size_t)j * d + t];
        double nj = sqrt(s);
        norm[j] = nj;
        for (int t = 0; t < d; ++t)
            khat[(size_t)j * d + t] = nj > 0.0 ? x[(size_t)j * d + t] / nj : 0.0;
    }
}

/* [CAND] + [SORT] + [MASK]: the candidate positions of sorted slot s.
 * Window: slots of chunks c - before .. c + after, c = s / m, clipped to
 * [0, L) (before = 1, after = 0 for LSH attention).
 * bucket (nullable): bucket id of every position in this round; when given,
 * only keys in the query's bucket are candidates.  Returns the number of
 * candidates written to cand; *self_in = 1 when the query's own position is
 * among them (then it is the last entry): always in the self-penalty reading,
 * else only when nothing else is left. */
static long candidates(const int32_t *perm, long L, int m, int before, int after, int causal,
                       const int32_t *bucket, int self_penalty, long s, int32_t *cand, int *self_in)
{
    long c = s / m;
    long w0 = (c - before) * m;
    if (w0 < 0) w0 = 0;
    long w1 = (c + after + 1) * m;
    if (w1 > L) w1 = L;
    int32_t i = perm[s];
    long nc = 0;
    for (long t = w0; t < w1; ++t) {
        if (t == s) continue;                    /* self removed ... */
        int32_t j = perm[t];
        if (causal && j > i) continue;           /* causal on original positions */
        if (bucket && bucket[j] != bucket[i]) continue;   /* strict N_LSH */
        cand[nc++] = j;
    }
    *self_in = 0;
    if (self_penalty || nc == 0) {               /* ... unless it is the only candidate */
        cand[nc++] = i;
        *self_in = 1;
    }
    return nc;
}

/* [OUT] one round of chunked LSH attention for the slots in `slots`
 * (all slots when slots == NULL).  Writes o and lse at the ORIGINAL
 * position of each query when scatter != 0, else at the list index. */
static int attn_round_impl(const double *x, const double *v, long L, int d,
                           const int32_t *perm, int m, int before, int after, int causal, const int32_t *bucket,
                           int self_penalty, const int64_t *slots, long nslots, int scatter,
                           double *o, double *lse)
{
    const size_t wmax = (size_t)(before + after + 1) * m + 1;
    double *khat = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *norm = (double *)malloc(sizeof(double) * (size_t)L);
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * wmax);
    double *z = (double *)malloc(sizeof(double) * wmax);
    if (!khat || !norm || !cand || !z) { free(khat); free(norm); free(cand); free(z); return -1; }
    normalise_keys(x, L, d, khat, norm);
    const double tau = 1.0 / sqrt((double)d);
    long count = slots ? nslots : L;
    for (long q = 0; q < count; ++q) {
        long s = slots ? (long)slots[q] : q;
        int32_t i = perm[s];
        int self_in;
        long nc = candidates(perm, L, m, before, after, causal, bucket, self_penalty, s, cand, &self_in);
        double zmax = -INFINITY;
        for (long a = 0; a < nc; ++a) {
            double dot = 0.0;
            for (int t = 0; t < d; ++t) dot += x[(size_t)i * d + t] * khat[(size_t)cand[a] * d + t];
            z[a] = (self_penalty && self_in && a == nc - 1) ? ORACLE_SELF_PENALTY : tau * dot;
            if (z[a] > zmax) zmax = z[a];
        }
        double l = 0.0;
        for (long a = 0; a < nc; ++a) l += exp(z[a] - zmax);
        double lse_i = zmax + log(l);
        long dst = scatter ? (long)i : q;
        double *oi = o + (size_t)dst * d;
        for (int t = 0; t < d; ++t) oi[t] = 0.0;
        for (long a = 0; a < nc; ++a) {
            double p = exp(z[a] - lse_i);
            for (int t = 0; t < d; ++t) oi[t] += p * v[(size_t)cand[a] * d + t];
        }
        lse[dst] = lse_i;
    }
    free(khat); free(norm); free(cand); free(z);
    return 0;
}

ORACLE_EXPORT int oracle_attn_round(const double *x, const double *v, long L, int d,
                                    const int32_t *perm, int m, int causal, const int32_t *bucket,
                                    int self_penalty, double *o, double *lse)
{
    return attn_round_impl(x, v, L, d, perm, m, 1, 0, causal, bucket, self_penalty, NULL, L, 1, o, lse);
}

/* Same as oracle_attn_round for a list of sorted slots; outputs follow the list. */
ORACLE_EXPORT int oracle_attn_slots(const double *x, const double *v, long L, int d,
                                    const int32_t *perm, int m, int causal, const int32_t *bucket,
                                    int self_penalty, const int64_t *slots, long nslots,
                                    double *o, double *lse)
{
    return attn_round_impl(x, v, L, d, perm, m, 1, 0, causal, bucket, self_penalty, slots, nslots, 0, o, lse);
}

/* [ROUNDS] y_i = sum_r softmax_r(lse_r,i) o_r,i; also returns LSE_i = logsumexp_r lse_r,i. */
ORACLE_EXPORT int oracle_combine(const double *o, const double *lse, int R, long L, int d,
                                 double *y, double *lse_all)
{
    for (long i = 0; i < L; ++i) {
        double mx = -INFINITY;
        for (int r = 0; r < R; ++r) if (lse[(size_t)r * L + i] > mx) mx = lse[(size_t)r * L + i];
        double s = 0.0;
        for (int r = 0; r < R; ++r) s += exp(lse[(size_t)r * L + i] - mx);
        double big = mx + log(s);
        if (lse_all) lse_all[i] = big;
        for (int t = 0; t < d; ++t) y[(size_t)i * d + t] = 0.0;
        for (int r = 0; r < R; ++r) {
            double w = exp(lse[(size_t)r * L + i] - big);
            for (int t = 0; t < d; ++t) y[(size_t)i * d + t] += w * o[((size_t)r * L + i) * d + t];
        }
    }
    return 0;
}

/* Whole forward for one (batch, head): hash every round, sort, attend, combine.
 * x, v [L, d]; R [n_hashes, d, n_buckets/2]; outputs y [L, d], lse [n_hashes, L],
 * perm [n_hashes, L], bucket [n_hashes, L], margin [n_hashes, L] (nullable).
 * bucket_mask / self_penalty: the optional readings (see the top of the file). */
ORACLE_EXPORT int oracle_fwd_head(const double *x, const double *v, long L, int d,
                                  const double *R, int n_buckets, int n_hashes, int m, int causal,
                                  int bucket_mask, int self_penalty,
                                  double *y, double *lse, int32_t *perm, int32_t *bucket, double *margin)
{
    const int half = n_buckets / 2;
    double *o = (double *)malloc(sizeof(double) * (size_t)n_hashes * L * d);
    if (!o) return -1;
    int rc = 0;
    for (int r = 0; r < n_hashes && rc == 0; ++r) {
        rc |= oracle_hash(x, L, d, R + (size_t)r * d * half, n_buckets, bucket + (size_t)r * L,
                          margin ? margin + (size_t)r * L : NULL);
        rc |= oracle_sort(bucket + (size_t)r * L, L, perm + (size_t)r * L);
        rc |= oracle_attn_round(x, v, L, d, perm + (size_t)r * L, m, causal,
                                bucket_mask ? bucket + (size_t)r * L : NULL, self_penalty,
                                o + (size_t)r * L * d, lse + (size_t)r * L);
    }
    if (rc == 0) rc = oracle_combine(o, lse, n_hashes, L, d, y, NULL);
    free(o);
    return rc;
}

/* Forward with given permutations (one per round); same outputs minus hashing.
 * bucket (nullable, [n_hashes, L] by position): given -> the bucket mask. */
ORACLE_EXPORT int oracle_fwd_head_perm(const double *x, const double *v, long L, int d,
                                       const int32_t *perm, int n_hashes, int m, int causal,
                                       const int32_t *bucket, int self_penalty, double *y, double *lse)
{
    double *o = (double *)malloc(sizeof(double) * (size_t)n_hashes * L * d);
    if (!o) return -1;
    int rc = 0;
    for (int r = 0; r < n_hashes && rc == 0; ++r)
        rc |= oracle_attn_round(x, v, L, d, perm + (size_t)r * L, m, causal,
                                bucket ? bucket + (size_t)r * L : NULL, self_penalty,
                                o + (size_t)r * L * d, lse + (size_t)r * L);
    if (rc == 0) rc = oracle_combine(o, lse, n_hashes, L, d, y, NULL);
    free(o);
    return rc;
}

/* Backward for one (batch, head) with the permutations held fixed.
 *
 * With LSE_i = logsumexp over all rounds and candidates of z_ij, the merged
 * output is y_i = sum_r sum_j exp(z_rij - LSE_i) v_j.  Writing
 * P_rij = exp(z_rij - LSE_i) and G = dL/dy:
 *   dv_j      += P_rij G_i
 *   dz_rij     = P_rij (G_i . v_j - G_i . y_i)
 *   dx_i      += dz_rij / sqrt(d) * k_j                 (query role)
 *   dk_j      += dz_rij / sqrt(d) * x_i                 (key role)
 *   dx_j      += (dk_j - k_j (k_j . dk_j)) / |x_j|      (through k_j = x_j/|x_j|)
 * Accumulated in a fixed order (round, slot, candidate).  In the self-penalty
 * reading the query's own entry has a constant score: it adds P G_i to dv_i
 * and nothing to dx.  bucket (nullable, [n_hashes, L]): given -> bucket mask. */
static int bwd_impl(const double *x, const double *v, const double *dy, long L, int d, const int32_t *perm,
                    int n_hashes, int m, int before, int after, int causal, const int32_t *bucket,
                    int self_penalty, double *dx, double *dv)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *lse = (double *)malloc(sizeof(double) * (size_t)n_hashes * L);
    double *o = (double *)malloc(sizeof(double) * (size_t)n_hashes * L * d);
    double *big = (double *)malloc(sizeof(double) * (size_t)L);
    double *khat = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *norm = (double *)malloc(sizeof(double) * (size_t)L);
    double *dk = (double *)calloc((size_t)L * d, sizeof(double));
    int32_t *cand = (int32_t *)malloc(sizeof(int32_t) * ((size_t)(before + after + 1) * m + 1));
    int rc = -1;
    if (!y || !lse || !o || !big || !khat || !norm || !dk || !cand) goto done;
    rc = 0;
    for (int r = 0; r < n_hashes && rc == 0; ++r)
        rc |= attn_round_impl(x, v, L, d, perm + (size_t)r * L, m, before, after, causal,
                              bucket ? bucket + (size_t)r * L : NULL, self_penalty, NULL, L, 1,
                              o + (size_t)r * L * d, lse + (size_t)r * L);
    if (rc) goto done;
    oracle_combine(o, lse, n_hashes, L, d, y, big);
    normalise_keys(x, L, d, khat, norm);
    memset(dx, 0, sizeof(double) * (size_t)L * d);
    memset(dv, 0, sizeof(double) * (size_t)L * d);
    const double tau = 1.0 / sqrt((double)d);
    for (int r = 0; r < n_hashes; ++r) {
        const int32_t *pr = perm + (size_t)r * L;
        for (long s = 0; s < L; ++s) {
            int32_t i = pr[s];
            const double *xi = x + (size_t)i * d, *gi = dy + (size_t)i * d;
            double delta = 0.0;
            for (int t = 0; t < d; ++t) delta += gi[t] * y[(size_t)i * d + t];
            int self_in;
            long nc = candidates(pr, L, m, before, after, causal, bucket ? bucket + (size_t)r * L : NULL,
                                 self_penalty, s, cand, &self_in);
            for (long a = 0; a < nc; ++a) {
                int32_t j = cand[a];
                const double *kj = khat + (size_t)j * d, *vj = v + (size_t)j * d;
                double dot = 0.0, gv = 0.0;
                for (int t = 0; t < d; ++t) { dot += xi[t] * kj[t]; gv += gi[t] * vj[t]; }
                if (self_penalty && self_in && a == nc - 1) {
                    /* constant score: value path only */
                    double p = exp(ORACLE_SELF_PENALTY - big[i]);
                    for (int t = 0; t < d; ++t) dv[(size_t)j * d + t] += p * gi[t];
                    continue;
                }
                double p = exp(tau * dot - big[i]);
                double dz = p * (gv - delta);
                for (int t = 0; t < d; ++t) {
                    dv[(size_t)j * d + t] += p * gi[t];
                    dx[(size_t)i * d + t] += dz * tau * kj[t];
                    dk[(size_t)j * d + t] += dz * tau * xi[t];
                }
            }
        }
    }
    for (long j = 0; j < L; ++j) {
        if (!(norm[j] > 0.0)) continue;
        const double *kj = khat + (size_t)j * d, *gj = dk + (size_t)j * d;
        double kg = 0.0;
        for (int t = 0; t < d; ++t) kg += kj[t] * gj[t];
        for (int t = 0; t < d; ++t) dx[(size_t)j * d + t] += (gj[t] - kj[t] * kg) / norm[j];
    }
done:
    free(y); free(lse); free(o); free(big); free(khat); free(norm); free(dk); free(cand);
    return rc;
}

ORACLE_EXPORT int oracle_bwd_head(const double *x, const double *v, const double *dy, long L, int d,
                                  const int32_t *perm, int n_hashes, int m, int causal,
                                  const int32_t *bucket, int self_penalty, double *dx, double *dv)
{
    return bwd_impl(x, v, dy, L, d, perm, n_hashes, m, 1, 0, causal, bucket, self_penalty, dx, dv);
}

/* Local (non-hashed) chunk attention for one (batch, head): positions in their
 * own order, chunk c attends to chunks c - before .. c + after, the same keys,
 * self rule and causal mask as above.  y [L, d], lse [L]. */
ORACLE_EXPORT int oracle_local_fwd_head(const double *x, const double *v, long L, int d, int m, int before,
                                        int after, int causal, int self_penalty, double *y, double *lse)
{
    int32_t *ident = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
    if (!ident) return -1;
    for (long i = 0; i < L; ++i) ident[i] = (int32_t)i;
    int rc = attn_round_impl(x, v, L, d, ident, m, before, after, causal, NULL, self_penalty, NULL, L, 1, y, lse);
    free(ident);
    return rc;
}

ORACLE_EXPORT int oracle_local_bwd_head(const double *x, const double *v, const double *dy, long L, int d, int m,
                                        int before, int after, int causal, int self_penalty, double *dx,
                                        double *dv)
{
    int32_t *ident = (int32_t *)malloc(sizeof(int32_t) * (size_t)(L > 0 ? L : 1));
    if (!ident) return -1;
    for (long i = 0; i < L; ++i) ident[i] = (int32_t)i;
    int rc = bwd_impl(x, v, dy, L, d, ident, 1, m, before, after, causal, NULL, self_penalty, dx, dv);
    free(ident);
    return rc;
}

/* ------------------------------------------------------------------ */
/* Batched drivers: independent (batch, head) slices run in parallel   */
/* with OpenMP when the library is built with it.                       */
/* x, v, dy, y, dx, dv [BH, L, d]; lse, perm, bucket, margin [BH, R, L]. */
/* ------------------------------------------------------------------ */
ORACLE_EXPORT int oracle_fwd_batch(const double *x, const double *v, long BH, long L, int d,
                                   const double *R, int n_buckets, int n_hashes, int m, int causal,
                                   int bucket_mask, int self_penalty,
                                   double *y, double *lse, int32_t *perm, int32_t *bucket, double *margin)
{
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
    for (long h = 0; h < BH; ++h) {
        size_t rows = (size_t)h * L, segs = (size_t)h * n_hashes * L;
        rc |= oracle_fwd_head(x + rows * d, v + rows * d, L, d, R, n_buckets, n_hashes, m, causal, bucket_mask,
                              self_penalty, y + rows * d, lse + segs, perm + segs, bucket + segs,
                              margin ? margin + segs : NULL);
    }
    return rc;
}

/* bucket (nullable) [BH, n_hashes, L] by position: given -> the bucket mask. */
ORACLE_EXPORT int oracle_fwd_perm_batch(const double *x, const double *v, long BH, long L, int d,
                                        const int32_t *perm, int n_hashes, int m, int causal,
                                        const int32_t *bucket, int self_penalty, double *y, double *lse)
{
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
    for (long h = 0; h < BH; ++h) {
        size_t rows = (size_t)h * L, segs = (size_t)h * n_hashes * L;
        rc |= oracle_fwd_head_perm(x + rows * d, v + rows * d, L, d, perm + segs, n_hashes, m, causal,
                                   bucket ? bucket + segs : NULL, self_penalty, y + rows * d, lse + segs);
    }
    return rc;
}

ORACLE_EXPORT int oracle_bwd_batch(const double *x, const double *v, const double *dy, long BH, long L,
                                   int d, const int32_t *perm, int n_hashes, int m, int causal,
                                   const int32_t *bucket, int self_penalty, double *dx, double *dv)
{
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
    for (long h = 0; h < BH; ++h) {
        size_t rows = (size_t)h * L, segs = (size_t)h * n_hashes * L;
        rc |= oracle_bwd_head(x + rows * d, v + rows * d, dy + rows * d, L, d, perm + segs, n_hashes,
                              m, causal, bucket ? bucket + segs : NULL, self_penalty, dx + rows * d,
                              dv + rows * d);
    }
    return rc;
}

ORACLE_EXPORT int oracle_local_fwd_batch(const double *x, const double *v, long BH, long L, int d, int m,
                                         int before, int after, int causal, int self_penalty, double *y,
                                         double *lse)
{
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
    for (long h = 0; h < BH; ++h)
        rc |= oracle_local_fwd_head(x + (size_t)h * L * d, v + (size_t)h * L * d, L, d, m, before, after, causal,
                                    self_penalty, y + (size_t)h * L * d, lse + (size_t)h * L);
    return rc;
}

ORACLE_EXPORT int oracle_local_bwd_batch(const double *x, const double *v, const double *dy, long BH, long L, int d,
                                         int m, int before, int after, int causal, int self_penalty, double *dx,
                                         double *dv)
{
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : rc)
    for (long h = 0; h < BH; ++h) {
        size_t rows = (size_t)h * L * d;
        rc |= oracle_local_bwd_head(x + rows, v + rows, dy + rows, L, d, m, before, after, causal, self_penalty,
                                    dx + rows, dv + rows);
    }
    return rc;
}

ORACLE_EXPORT int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
