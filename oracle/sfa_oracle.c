/*
 * sfa_oracle.c -- fp64 CPU oracle for the Hidden Decoding hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, obviously-correct
 * definition that the CUDA library is checked against.  Only the tests, the
 * package smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header or constant with the CUDA library and includes
 * nothing from it.
 *
 * What it computes ("Hidden Decoding at Scale" review, section "Method";
 * Tencent/Sequential-Hidden-Decoding README, section "Key Idea"; arXiv
 * 2607.08186 abstract):
 *
 *   - token expansion: every token x_t of a length-L sequence becomes n
 *     vectors, one from each of n independent embedding tables E_0..E_{n-1}.
 *     The n vectors are laid out token-major, so expanded position p = t*n + s
 *     holds E_s[x_t] (the length-nL sequence).
 *
 *   - Stream-Factorized Attention on that sequence, per (batch b, query head h):
 *       within-stream: query (t,s) attends keys (t',s') with s' == s, t' <= t
 *       cross-stream:  query p attends every expanded position p' <= p
 *       cross-stream sliding window of W tokens (the mixing layers follow the
 *       base model's own pattern, full or sliding-window; review "Method"):
 *                      query p attends p' <= p whose token t' > t - W
 *       transient intermediate streams (the PHD-style control: intermediate
 *       streams help only their own token; review "Prior limitations"):
 *                      query (t,s) attends (t',n-1) for t' < t, and (t,s'), s' <= s
 *     O[p] = sum_{p' in A(p)} softmax_p'(scale * <Q[p], K[p']>) V[p'],
 *     LSE[p] = log sum_{p' in A(p)} exp(scale * <Q[p], K[p']>).
 *     Query head h reads key/value head h / (Hq/Hkv) (consecutive groups).
 *
 *   - decode: the n new positions of token T (p = n(T-1)+s) attend the
 *     retained expanded cache of n*T positions under the same masks; the K/V
 *     rows of the new positions are already in the cache.
 *
 * Everything is computed in fp64 from the exact fp64 value of each bf16
 * input.  Rows are independent, so OpenMP spreads whole rows over threads;
 * nothing inside a row is blocked or reordered.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC sfa_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* The exact value of a bf16 number: its 16 bits are the high half of an
 * IEEE-754 binary32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Token expansion into n streams (review "Method": "expands each token into n
 * streams with independent embedding tables"; README "Key Idea" item 1).
 *
 * ids    : [B][L] token ids
 * tables : n pointers, table s is [V][d] bf16 bits, row-major
 * out    : [B][L*n][d] bf16 bits; row t*n+s of batch b is tables[s][ids[b][t]]
 *
 * An id outside [0, V) yields a zero row.  Returns how many ids were out of
 * range (each counted once per token, not per stream).
 */
int64_t oracle_expand_embed(const int64_t *ids, int64_t B, int64_t L,
                            const uint16_t *const *tables, int n, int64_t V,
                            int64_t d, uint16_t *out)
{
    int64_t bad = 0;
    for (int64_t b = 0; b < B; ++b) {
        for (int64_t t = 0; t < L; ++t) {
            int64_t x = ids[b * L + t];
            int in_range = (x >= 0 && x < V);
            if (!in_range)
                ++bad;
            for (int s = 0; s < n; ++s) {
                uint16_t *dst = out + ((b * L + t) * (int64_t)n + s) * d;
                if (in_range)
                    memcpy(dst, tables[s] + x * d, (size_t)d * sizeof(uint16_t));
                else
                    memset(dst, 0, (size_t)d * sizeof(uint16_t));
            }
        }
    }
    return bad;
}

/*
 * Final-stream rows (review "Method": next-token cross-entropy is applied only
 * at the final-stream positions; README "Key Idea" item 3: only the final
 * stream predicts the next token).
 *
 * x   : [B][L*n][d] bf16 bits (the expanded sequence's hidden states)
 * out : [B][L][d] bf16 bits; row t of batch b := x[b][t*n + n-1]
 */
void oracle_final_stream_rows(const uint16_t *x, int64_t B, int64_t L, int n,
                              int64_t d, uint16_t *out)
{
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < L; ++t)
            memcpy(out + (b * L + t) * d, x + ((b * L + t) * (int64_t)n + n - 1) * d,
                   (size_t)d * sizeof(uint16_t));
}

/*
 * Gradient of the token expansion with respect to the n embedding tables:
 * out row t*n+s of batch b is tables[s][ids[b][t]], so
 *   grad_tables[s][v] = sum over (b, t) with ids[b][t] == v of grad_out[b][t*n+s].
 *
 * grad_out    : [B][L*n][d] bf16 bits
 * grad_tables : n pointers, each [V][d] fp64, ACCUMULATED into (callers zero them)
 * Ids outside [0, V) contribute nothing.
 */
void oracle_expand_embed_backward(const int64_t *ids, int64_t B, int64_t L,
                                  const uint16_t *grad_out, int n, int64_t V,
                                  int64_t d, double *const *grad_tables)
{
    for (int64_t b = 0; b < B; ++b)
        for (int64_t t = 0; t < L; ++t) {
            const int64_t x = ids[b * L + t];
            if (x < 0 || x >= V)
                continue;
            for (int s = 0; s < n; ++s) {
                const uint16_t *g = grad_out + ((b * L + t) * (int64_t)n + s) * d;
                double *dst = grad_tables[s] + x * d;
                for (int64_t c = 0; c < d; ++c)
                    dst[c] += bf16_value(g[c]);
            }
        }
}

/*
 * The SFA mask, stated in the (token, stream) coordinates of the pages:
 * expanded position p is token t = p / n, stream s = p % n.
 *   mode 0 (within-stream): same stream, earlier-or-same token.
 *   mode 1 (cross-stream):  any earlier-or-same expanded position.
 *   mode 2 (cross-stream, sliding window of `window` tokens): any
 *          earlier-or-same expanded position of the last `window` tokens
 *          (token t' with t - window < t' <= t).
 *   mode 3 (transient intermediate streams, the PHD-style control of the
 *          shared-KV ablation; review "Prior limitations"): earlier tokens
 *          are seen only through their final stream n-1; the current token's
 *          streams s' <= s stay visible.
 */
static int sfa_allowed(int64_t p, int64_t pk, int n, int mode, int64_t window)
{
    int64_t t = p / n, s = p % n;
    int64_t tk = pk / n, sk = pk % n;
    if (mode == 0)
        return sk == s && tk <= t;
    if (mode == 2)
        return pk <= p && tk > t - window;
    if (mode == 3)
        return (tk < t && sk == n - 1) || (tk == t && sk <= s);
    return pk <= p;
}

/*
 * One query row of masked softmax attention, the textbook two-pass form:
 * logits of the allowed keys, their maximum, then exp(l - max) weights.
 *
 * q      : D bf16 bits (the query vector)
 * k, v   : [B][Nk][Hkv][D] bf16 bits
 * p      : expanded position of the query
 * nkeys  : key rows 0 .. nkeys-1 of batch b are valid
 * logit  : scratch of nkeys doubles
 * o      : D doubles out; *lse out
 */
static void attend_row(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                       int64_t b, int64_t p, int g, int64_t Nk, int Hkv, int D,
                       int64_t nkeys, int n, int mode, int64_t window,
                       double scale, double *logit, double *o, double *lse)
{
    double qd[256];
    for (int c = 0; c < D; ++c)
        qd[c] = bf16_value(q[c]);

    double m = -INFINITY;
    for (int64_t pk = 0; pk < nkeys; ++pk) {
        if (!sfa_allowed(p, pk, n, mode, window))
            continue;
        const uint16_t *kr = k + ((b * Nk + pk) * Hkv + g) * (int64_t)D;
        double dot = 0.0;
        for (int c = 0; c < D; ++c)
            dot += qd[c] * bf16_value(kr[c]);
        logit[pk] = scale * dot;
        if (logit[pk] > m)
            m = logit[pk];
    }

    for (int c = 0; c < D; ++c)
        o[c] = 0.0;
    double sum = 0.0;
    for (int64_t pk = 0; pk < nkeys; ++pk) {
        if (!sfa_allowed(p, pk, n, mode, window))
            continue;
        double w = exp(logit[pk] - m);
        sum += w;
        const uint16_t *vr = v + ((b * Nk + pk) * Hkv + g) * (int64_t)D;
        for (int c = 0; c < D; ++c)
            o[c] += w * bf16_value(vr[c]);
    }
    if (sum > 0.0) {
        for (int c = 0; c < D; ++c)
            o[c] /= sum;
        *lse = m + log(sum);
    } else {
        /* no allowed key: cannot happen for p < nkeys (the diagonal is always
         * allowed); reported as NaN so a caller mistake is visible */
        for (int c = 0; c < D; ++c)
            o[c] = NAN;
        *lse = NAN;
    }
}

/*
 * Attention for an explicit list of R query rows.
 *
 * q_rows : [R][D] bf16 bits, the query vector of each row
 * rb, rp, rh : [R] batch index, expanded position, query head of each row
 * k, v   : [B][Nk][Hkv][D] bf16 bits
 * nkeys  : [B] number of valid key rows per batch (keys 0..nkeys[b]-1)
 * mode   : 0 within-stream, 1 cross-stream, 2 cross-stream sliding window,
 *          3 transient intermediate streams
 * window : tokens in the sliding window (mode 2; ignored otherwise, >= 1)
 * o      : [R][D] fp64 out, lse : [R] fp64 out
 *
 * Returns 0, or -1 on a bad argument (D > 256, Hq % Hkv != 0, index out of
 * range) without writing anything.
 */
int oracle_attend_rows(const uint16_t *q_rows, const int64_t *rb,
                       const int64_t *rp, const int64_t *rh, int64_t R,
                       const uint16_t *k, const uint16_t *v, int64_t B,
                       int64_t Nk, int Hq, int Hkv, int D,
                       const int64_t *nkeys, int n, int mode, int64_t window,
                       double scale, double *o, double *lse)
{
    if (D < 1 || D > 256 || Hkv < 1 || Hq % Hkv != 0 || n < 1 ||
        mode < 0 || mode > 3 || (mode == 2 && window < 1))
        return -1;
    for (int64_t r = 0; r < R; ++r) {
        if (rb[r] < 0 || rb[r] >= B || rh[r] < 0 || rh[r] >= Hq ||
            rp[r] < 0 || rp[r] >= nkeys[rb[r]] || nkeys[rb[r]] > Nk)
            return -1;
    }
    const int group = Hq / Hkv;
    int failed = 0;
#pragma omp parallel
    {
        double *logit = (double *)malloc((size_t)Nk * sizeof(double));
        if (!logit) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < R; ++r) {
            if (!logit)
                continue;
            attend_row(q_rows + r * (int64_t)D, k, v, rb[r], rp[r],
                       (int)(rh[r] / group), Nk, Hkv, D, nkeys[rb[r]], n, mode,
                       window, scale, logit, o + r * (int64_t)D, lse + r);
        }
        free(logit);
    }
    return failed ? -2 : 0;
}

/*
 * Backward of the masked softmax attention above, for training through the
 * SFA layers (review "Method": the model is trained end to end with the loss
 * at the final-stream positions, so the gradient flows back through every
 * within- and cross-stream layer).  Written from the derivation of
 * O = softmax(scale * Q K^T) V restricted to the allowed set A(p):
 *
 *   P[p, p']  = exp(scale <Q[p], K[p']> - LSE[p])          (p' in A(p))
 *   dV[p']   += P[p, p'] dO[p]
 *   dP[p, p'] = <dO[p], V[p']>
 *   Delta[p]  = sum_{p'} P[p, p'] dP[p, p'] = <dO[p], O[p]>
 *   dS[p, p'] = P[p, p'] (dP[p, p'] - Delta[p])
 *   dQ[p]     = scale sum_{p'} dS[p, p'] K[p']
 *   dK[p']   += scale dS[p, p'] Q[p]
 *
 * K/V head g collects the gradients of every query head that reads it.
 * O, LSE and Delta are recomputed here in fp64 from the inputs; nothing from
 * a forward pass is taken in.
 *
 * q, dout : [B][N][Hq][D] bf16 bits;  k, v : [B][N][Hkv][D] bf16 bits
 * dq      : [B][N][Hq][D] fp64 out;   dk, dv : [B][N][Hkv][D] fp64 out
 * Returns 0, -1 on a bad argument, -2 if scratch could not be allocated.
 */
int oracle_attend_backward(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                           const uint16_t *dout, int64_t B, int64_t N, int Hq,
                           int Hkv, int D, int n, int mode, int64_t window,
                           double scale, double *dq, double *dk, double *dv)
{
    if (D < 1 || D > 256 || Hkv < 1 || Hq % Hkv != 0 || n < 1 || N % n != 0 ||
        mode < 0 || mode > 3 || (mode == 2 && window < 1))
        return -1;
    const int group = Hq / Hkv;
    memset(dq, 0, (size_t)(B * N * Hq * D) * sizeof(double));
    memset(dk, 0, (size_t)(B * N * Hkv * D) * sizeof(double));
    memset(dv, 0, (size_t)(B * N * Hkv * D) * sizeof(double));
    int failed = 0;
    /* one (batch, KV head) per iteration: it owns its rows of dk and dv */
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bg = 0; bg < B * Hkv; ++bg) {
        const int64_t b = bg / Hkv;
        const int g = (int)(bg % Hkv);
        double *p_row = (double *)malloc((size_t)N * sizeof(double));
        double *o_row = (double *)malloc((size_t)D * sizeof(double));
        double *q_row = (double *)malloc((size_t)D * sizeof(double));
        double *do_row = (double *)malloc((size_t)D * sizeof(double));
        if (!p_row || !o_row || !q_row || !do_row) {
#pragma omp atomic write
            failed = 1;
            free(p_row); free(o_row); free(q_row); free(do_row);
            continue;
        }
        for (int h = g * group; h < (g + 1) * group; ++h) {
            for (int64_t p = 0; p < N; ++p) {
                const int64_t qi = ((b * N + p) * Hq + h) * (int64_t)D;
                for (int c = 0; c < D; ++c) {
                    q_row[c] = bf16_value(q[qi + c]);
                    do_row[c] = bf16_value(dout[qi + c]);
                }
                /* probabilities of the allowed keys (two-pass softmax) */
                double m = -INFINITY;
                for (int64_t pk = 0; pk < N; ++pk) {
                    if (!sfa_allowed(p, pk, n, mode, window))
                        continue;
                    const uint16_t *kr = k + ((b * N + pk) * Hkv + g) * (int64_t)D;
                    double dot = 0.0;
                    for (int c = 0; c < D; ++c)
                        dot += q_row[c] * bf16_value(kr[c]);
                    p_row[pk] = scale * dot;
                    if (p_row[pk] > m)
                        m = p_row[pk];
                }
                double sum = 0.0;
                for (int64_t pk = 0; pk < N; ++pk)
                    if (sfa_allowed(p, pk, n, mode, window)) {
                        p_row[pk] = exp(p_row[pk] - m);
                        sum += p_row[pk];
                    }
                for (int c = 0; c < D; ++c)
                    o_row[c] = 0.0;
                for (int64_t pk = 0; pk < N; ++pk) {
                    if (!sfa_allowed(p, pk, n, mode, window))
                        continue;
                    p_row[pk] /= sum;
                    const uint16_t *vr = v + ((b * N + pk) * Hkv + g) * (int64_t)D;
                    for (int c = 0; c < D; ++c)
                        o_row[c] += p_row[pk] * bf16_value(vr[c]);
                }
                double delta = 0.0;
                for (int c = 0; c < D; ++c)
                    delta += do_row[c] * o_row[c];
                /* gradients through each allowed key */
                for (int64_t pk = 0; pk < N; ++pk) {
                    if (!sfa_allowed(p, pk, n, mode, window))
                        continue;
                    const int64_t kvi = ((b * N + pk) * Hkv + g) * (int64_t)D;
                    double dp = 0.0;
                    for (int c = 0; c < D; ++c)
                        dp += do_row[c] * bf16_value(v[kvi + c]);
                    const double ds = p_row[pk] * (dp - delta);
                    for (int c = 0; c < D; ++c) {
                        dv[kvi + c] += p_row[pk] * do_row[c];
                        dk[kvi + c] += scale * ds * q_row[c];
                        dq[qi + c] += scale * ds * bf16_value(k[kvi + c]);
                    }
                }
            }
        }
        free(p_row); free(o_row); free(q_row); free(do_row);
    }
    return failed ? -2 : 0;
}
