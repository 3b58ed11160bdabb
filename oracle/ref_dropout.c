/*
 * ref_dropout.c -- fp64 CPU oracle for exact attention with dropout on the
 * attention probabilities, and the counter-based generator that draws the
 * dropout mask.
 *
 * TEST INFRASTRUCTURE ONLY (see ref_attn.c): nothing in the product path may
 * link, load or call this file.  It shares no code with the CUDA path; the two
 * sides each implement the generator below from its published definition.
 *
 * Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random
 * numbers: as easy as 1, 2, 3", SC 2011).  A 128-bit counter (c0..c3) and a
 * 64-bit key (k0, k1) go through ten rounds; each round multiplies c0 and c2 by
 * the two round multipliers (keeping the high and low 32-bit halves of the
 * 64-bit products), mixes the high halves with the other two counter words and
 * the key, and then bumps the key by the two Weyl constants.
 *
 * Mask: for head bh = b*H + h, query row i and key j, the counter is
 * (i, j >> 4, bh, offset) and the key (seed & 0xffffffff, seed >> 32); the 8-bit
 * draw for key j is byte (j & 3) of output word ((j & 15) >> 2), so one call
 * serves 16 keys.  Key j is kept for row i iff that draw is >= T, with
 * T = floor(rate * 256); kept entries are scaled by 256 / (256 - T), the
 * inverse of the exact keep probability (the rate takes steps of 1/256).
 *
 * Attention with dropout (the mask applied to the normalised probabilities,
 * after the causal mask and the softmax; the log-sum-exp is the one without
 * dropout):
 *   P_ij  = softmax_j(scale * Q_i . K_j)       (as in ref_attn.c)
 *   Z_ij  = keep_ij * 256 / (256 - T)
 *   O_i   = sum_j P_ij Z_ij V_j,   LSE_i = m_i + ln l_i
 * Backward (chain rule; the softmax Jacobian acts on dP = Z o (dO V^T)):
 *   dP_ij = Z_ij (dO_i . V_j),   D_i = sum_j P_ij dP_ij,   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale sum_j dS_ij K_j,  dK_j = scale sum_i dS_ij Q_i,  dV_j = sum_i P_ij Z_ij dO_i
 *
 * Layout: [BH, N, d] row-major fp64 per tensor, lse [BH, N]; single-threaded
 * (test sizes only).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>

/* ------------------------------------------------------------ Philox4x32-10 */

/* Round multipliers and Weyl key increments of Philox4x32 (Salmon et al. 2011). */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void ref_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4])
{
    uint32_t c0 = ctr[0], c1 = ctr[1], c2 = ctr[2], c3 = ctr[3];
    uint32_t k0 = key[0], k1 = key[1];
    for (int round = 0; round < 10; ++round) {
        const uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
        const uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
        const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
        const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
        c0 = hi1 ^ c1 ^ k0;
        c1 = lo1;
        c2 = hi0 ^ c3 ^ k1;
        c3 = lo0;
        k0 += PHILOX_W0;
        k1 += PHILOX_W1;
    }
    out[0] = c0;
    out[1] = c1;
    out[2] = c2;
    out[3] = c3;
}

/* The 8-bit draw of (bh, i, j). */
static uint32_t draw8(uint64_t seed, uint32_t offset, long bh, long i, long j)
{
    const uint32_t ctr[4] = {(uint32_t)i, (uint32_t)(j >> 4), (uint32_t)bh, offset};
    const uint32_t key[2] = {(uint32_t)(seed & 0xffffffffu), (uint32_t)(seed >> 32)};
    uint32_t w[4];
    ref_philox4x32_10(ctr, key, w);
    return (w[(j & 15) >> 2] >> (8 * (j & 3))) & 0xffu;
}

/* keep[bh, i, j] in {0, 1} for every head, row and key. */
void ref_dropout_mask(long BH, long N, uint64_t seed, uint32_t offset, uint32_t T, uint8_t *keep)
{
    for (long bh = 0; bh < BH; ++bh)
        for (long i = 0; i < N; ++i)
            for (long j = 0; j < N; ++j)
                keep[(bh * N + i) * N + j] = draw8(seed, offset, bh, i, j) >= T ? 1 : 0;
}

/* ------------------------------------------------------ attention + dropout */

/* Softmax row i of one head (safe softmax, causal mask): p[0..N), returns m, l. */
static void prob_row(const double *q, const double *k, long N, long d, double scale, int causal, long i,
                     double *p, double *m_out, double *l_out)
{
    double m = -INFINITY;
    for (long j = 0; j < N; ++j) {
        if (causal && j > i) {
            p[j] = -INFINITY;
            continue;
        }
        double s = 0.0;
        for (long c = 0; c < d; ++c)
            s += q[i * d + c] * k[j * d + c];
        p[j] = scale * s;
        if (p[j] > m)
            m = p[j];
    }
    double l = 0.0;
    for (long j = 0; j < N; ++j) {
        p[j] = exp(p[j] - m);
        l += p[j];
    }
    for (long j = 0; j < N; ++j)
        p[j] /= l;
    *m_out = m;
    *l_out = l;
}

static double zval(uint64_t seed, uint32_t offset, uint32_t T, long bh, long i, long j)
{
    return draw8(seed, offset, bh, i, j) >= T ? 256.0 / (256.0 - (double)T) : 0.0;
}

/* bh0: global head index of the first head passed (the mask's counter uses b*H + h), so
   that single heads of a large workload can be checked on their own. */
int ref_attn_fwd_dropout(const double *Q, const double *K, const double *V, double *O, double *LSE, long BH,
                         long N, long d, double scale, int causal, uint64_t seed, uint32_t offset, uint32_t T,
                         long bh0)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p)
        return -1;
    for (long bh = 0; bh < BH; ++bh) {
        const double *q = Q + bh * N * d, *k = K + bh * N * d, *v = V + bh * N * d;
        for (long i = 0; i < N; ++i) {
            double m, l;
            prob_row(q, k, N, d, scale, causal, i, p, &m, &l);
            double *o = O + (bh * N + i) * d;
            for (long c = 0; c < d; ++c)
                o[c] = 0.0;
            for (long j = 0; j < N; ++j) {
                const double w = p[j] * zval(seed, offset, T, bh0 + bh, i, j);
                if (w == 0.0)
                    continue;
                for (long c = 0; c < d; ++c)
                    o[c] += w * v[j * d + c];
            }
            LSE[bh * N + i] = m + log(l);
        }
    }
    free(p);
    return 0;
}

int ref_attn_bwd_dropout(const double *Q, const double *K, const double *V, const double *dO, double *dQ,
                         double *dK, double *dV, long BH, long N, long d, double scale, int causal, uint64_t seed,
                         uint32_t offset, uint32_t T, long bh0)
{
    double *p = (double *)malloc(sizeof(double) * (size_t)N);
    double *dp = (double *)malloc(sizeof(double) * (size_t)N);
    if (!p || !dp) {
        free(p);
        free(dp);
        return -1;
    }
    for (long x = 0; x < BH * N * d; ++x) {
        dQ[x] = 0.0;
        dK[x] = 0.0;
        dV[x] = 0.0;
    }
    for (long bh = 0; bh < BH; ++bh) {
        const double *q = Q + bh * N * d, *k = K + bh * N * d, *v = V + bh * N * d, *go = dO + bh * N * d;
        double *gq = dQ + bh * N * d, *gk = dK + bh * N * d, *gv = dV + bh * N * d;
        for (long i = 0; i < N; ++i) {
            double m, l;
            prob_row(q, k, N, d, scale, causal, i, p, &m, &l);
            double D = 0.0;
            for (long j = 0; j < N; ++j) {
                const double z = zval(seed, offset, T, bh0 + bh, i, j);
                double s = 0.0;
                for (long c = 0; c < d; ++c)
                    s += go[i * d + c] * v[j * d + c];
                dp[j] = z * s;
                D += p[j] * dp[j];
                const double pz = p[j] * z;
                if (pz != 0.0)
                    for (long c = 0; c < d; ++c)
                        gv[j * d + c] += pz * go[i * d + c];
            }
            for (long j = 0; j < N; ++j) {
                const double ds = p[j] * (dp[j] - D);
                if (ds == 0.0)
                    continue;
                for (long c = 0; c < d; ++c) {
                    gq[i * d + c] += scale * ds * k[j * d + c];
                    gk[j * d + c] += scale * ds * q[i * d + c];
                }
            }
        }
    }
    free(p);
    free(dp);
    return 0;
}
