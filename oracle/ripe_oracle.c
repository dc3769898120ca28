/*
 * RIPE verification attention, CPU oracle in fp64.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the package's smoke check and the CPU-baseline leg
 * of the benchmark do.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes follows "Prefix Keys and Values Matter Late: RIPE Caching
 * for Self-Speculative Decoding in Looped Language Models" (arXiv 2610.34436),
 * abstract:
 *   - a looped model keeps R planes of keys/values per recurrent layer; the
 *     verify pass at loop r reads the cache (abstract, first sentence);
 *   - RIPE keeps the deepest plane (r = R-1) for every position and all R
 *     planes only for a window of recent positions (abstract, fourth sentence);
 *   - a window at least as long as the draft block makes batched verification
 *     independent of the block split (abstract, fifth sentence).  That property
 *     only holds when the window is measured back from each query position, so
 *     that is the default rule here (mode 0); the literal "window of the cache"
 *     reading is kept as mode 1 so tests can show that it breaks the property.
 *
 * Plane rule for a query at position p = T + j (T committed positions, j the
 * index inside the draft block) and key t <= p at loop r:
 *     t >= T                  -> plane r   (draft block: deeper planes do not exist yet)
 *     mode 0: t >= p - W      -> plane r   (inside the query's window)
 *     mode 1: t >= T - W      -> plane r   (inside the cache's window)
 *     otherwise               -> plane R-1 (the shared deepest plane)
 * Attention is the textbook causal softmax over keys t = 0..p, with the
 * caller's scale applied to the dot products, everything in fp64.
 *
 * Absent planes are marked by NaN in the inputs; reading one is an error
 * (return code 2), so the oracle also proves that the rule never reads a plane
 * that RIPE does not store.
 */
#include <math.h>
#include <stddef.h>
#include <stdint.h>

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_EABSENT 2

/* Plane that query position p reads for key t (t <= p). */
int oracle_plane(long p, long t, int r, int R, long T, long W, int mode)
{
    if (t >= T)
        return r;
    if (mode == 0)
        return (t >= p - W) ? r : R - 1;
    return (t >= T - W) ? r : R - 1;
}

/*
 * Verification attention for a batch of sequences at loop r.
 *   T[n]            committed prefix length of sequence n
 *   Kr, Vr          plane r,   [N][kvH][ld][d], positions [0, T[n] + B)
 *   Kl, Vl          plane R-1, [N][kvH][ld][d], positions [0, T[n])
 *   q               [N][B][kvH*g][d]; query head h uses key/value head h / g
 *   out             [N][B][kvH*g][d]
 *   lse             [N][B][kvH*g]   natural log of the softmax normaliser
 * Returns 0, or ORACLE_EABSENT if a selected key or value is NaN.
 */
int oracle_verify(int N, int kvH, int g, int d, int R, long W, int r, int mode, int B,
                  const long *T, long ld,
                  const double *Kr, const double *Vr,
                  const double *Kl, const double *Vl,
                  const double *q, double scale, double *out, double *lse)
{
    if (N < 0 || kvH <= 0 || g <= 0 || d <= 0 || R <= 0 || W < 0 || r < 0 || r >= R ||
        B <= 0 || (mode != 0 && mode != 1))
        return ORACLE_EINVAL;
    for (int n = 0; n < N; ++n)
        if (T[n] < 0 || T[n] + B > ld)
            return ORACLE_EINVAL;

    const int Hq = kvH * g;
    const long total = (long)N * B * Hq;
    int status = ORACLE_OK;

#pragma omp parallel for schedule(dynamic, 1) reduction(max : status)
    for (long idx = 0; idx < total; ++idx) {
        const int h = (int)(idx % Hq);
        const int j = (int)((idx / Hq) % B);
        const int n = (int)(idx / ((long)Hq * B));
        const int kh = h / g;
        const long Tn = T[n];
        const long p = Tn + j;
        const double *qv = q + idx * d;
        const size_t base = ((size_t)n * kvH + kh) * (size_t)ld * d;

        /* logits s_t = scale * <q, K_plane(t)[t]> for t = 0..p */
        /* two passes over the keys: first the maximum logit, then the sums */
        double m = -INFINITY;
        int bad = 0;
        for (long t = 0; t <= p; ++t) {
            const int pl = oracle_plane(p, t, r, R, Tn, W, mode);
            const double *kv = (pl == r ? Kr : Kl) + base + (size_t)t * d;
            double s = 0.0;
            for (int e = 0; e < d; ++e)
                s += qv[e] * kv[e];
            s *= scale;
            if (isnan(s)) {
                bad = 1;
                break;
            }
            if (s > m)
                m = s;
        }
        double *o = out + idx * d;
        for (int e = 0; e < d; ++e)
            o[e] = 0.0;
        double Z = 0.0;
        for (long t = 0; t <= p && !bad; ++t) {
            const int pl = oracle_plane(p, t, r, R, Tn, W, mode);
            const double *kv = (pl == r ? Kr : Kl) + base + (size_t)t * d;
            const double *vv = (pl == r ? Vr : Vl) + base + (size_t)t * d;
            double s = 0.0;
            for (int e = 0; e < d; ++e)
                s += qv[e] * kv[e];
            const double w = exp(s * scale - m);
            Z += w;
            for (int e = 0; e < d; ++e) {
                if (isnan(vv[e]))
                    bad = 1;
                o[e] += w * vv[e];
            }
        }
        if (bad) {
            status = ORACLE_EABSENT;
            continue;
        }
        for (int e = 0; e < d; ++e)
            o[e] /= Z;
        lse[idx] = m + log(Z);
    }
    return status;
}

/*
 * Softmax weights of one query (for the weights-sum-to-one check).
 * Writes w[0..p] and returns 0; same plane rule and inputs as oracle_verify,
 * for the single sequence and key/value head given by the pointers.
 */
int oracle_weights(int d, int R, long W, int r, int mode, long T, int j,
                   const double *Kr, const double *Kl, const double *qv, double scale,
                   double *w)
{
    const long p = T + j;
    double m = -INFINITY;
    for (long t = 0; t <= p; ++t) {
        const int pl = oracle_plane(p, t, r, R, T, W, mode);
        const double *kv = (pl == r ? Kr : Kl) + (size_t)t * d;
        double s = 0.0;
        for (int e = 0; e < d; ++e)
            s += qv[e] * kv[e];
        w[t] = s * scale;
        if (isnan(w[t]))
            return ORACLE_EABSENT;
        if (w[t] > m)
            m = w[t];
    }
    double Z = 0.0;
    for (long t = 0; t <= p; ++t) {
        w[t] = exp(w[t] - m);
        Z += w[t];
    }
    for (long t = 0; t <= p; ++t)
        w[t] /= Z;
    return ORACLE_OK;
}
