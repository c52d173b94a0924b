/*
 * Oracle for the causal linear-attention forward: a plain per-token
 * recurrence in fp64 on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into a separate shared
 * object that only the tests, the package's smoke check and the bench's CPU
 * baseline load.  It shares no code with the CUDA library and must never be
 * used as a fallback for it.
 *
 * Every function walks the tokens of one (batch, head) sequence in order and
 * applies the update rule exactly as the pages write it, then reads the output
 * from the state AFTER the update of the same token.  Sequences are
 * independent; OpenMP runs them in parallel (the order of floating-point
 * operations inside one sequence is fixed, so results do not depend on the
 * thread count).
 *
 * Layouts (row-major, contiguous):
 *   q, k  [B,T,H,dk]   v, o  [B,T,H,dv]
 *   GLA gate g [B,T,H,dk];  gated-delta alpha, beta [B,T,H]
 *   S0, S_out [B,H,dk,dv]  (S is dk x dv: row = key dim, column = value dim)
 *   z0, z_out [B,H,dk]     (ELU normaliser)
 * S0 / z0 may be NULL (zero initial state).  S_out / z_out may be NULL.
 *
 * Sources (page title, section):
 *   ELU+1: "Linear / RNN 路线：砍 softmax，固定 state 替代 KV", §2.1
 *     (recurrence S_t = S_{t-1} + phi(k_t) v_t^T, z_t = z_{t-1} + phi(k_t),
 *     phi = ELU + 1); epsilon added to the denominator after the dot product
 *     as in "状态空间与线性注意力", section 线性注意力.
 *   GLA: "Linear / RNN 路线", §2.2 (S_t = diag(g_t) S_{t-1} + k_t v_t^T,
 *     o_t = q_t^T S_t; g_t scales row i of the state).
 *   Gated delta rule: "线性注意力与 SSM：把整张关系表变成一条状态流", GDN box
 *     (S_t = alpha_t S_{t-1}(I - beta_t k_t k_t^T) + beta_t v_t k_t^T, written
 *     there with S as dv x dk).  Here S is dk x dv, i.e. the transpose:
 *     S_t = alpha_t (I - beta_t k_t k_t^T) S_{t-1} + beta_t k_t v_t^T, the
 *     orientation of "状态空间与线性注意力", section Retention、衰减与 Delta
 *     Rule; output o_t = S_t^T q_t read after the write, as in that page's
 *     KDA recurrent reference.
 *   KDA (per-key-channel retention with the delta rule): "状态空间与线性注意力",
 *     section KDA：逐通道遗忘与误差写入.  The old state is first decayed row by
 *     row, Sbar = Diag(alpha_t) S_{t-1}; the residual of the decayed state's
 *     prediction is then written, S_t = Sbar + beta_t k_t (v_t - Sbar^T k_t)^T;
 *     o_t = S_t^T q_t.  alpha [B,T,H,dk], beta [B,T,H].
 *   Output normalisation: Lightning attention reads o_t = Norm(q_t^T S_t)
 *     with an RMSNorm at the output ("Linear / RNN 路线", §2.4); K3 applies a
 *     head-wise RMSNorm to the recurrent output ("状态空间与线性注意力", KDA
 *     section).  The pages name the norm without writing it out; the oracle
 *     takes the root-mean-square normalisation of each (token, head) row over
 *     its dv values, times an optional per-channel weight (oracle_head_rmsnorm).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define IDX4(b, t, h, d, T, H, D) ((((int64_t)(b) * (T) + (t)) * (H) + (h)) * (D) + (d))
#define IDX3(b, t, h, T, H) (((int64_t)(b) * (T) + (t)) * (H) + (h))

/* phi(x) = ELU(x) + 1 with ELU's alpha = 1: x + 1 for x > 0, exp(x) otherwise. */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

static void load_state(double *S, const double *S0, int64_t b, int64_t h, int64_t H,
                       int64_t n) {
    if (S0)
        memcpy(S, S0 + ((int64_t)b * H + h) * n, (size_t)n * sizeof(double));
    else
        memset(S, 0, (size_t)n * sizeof(double));
}

static void store_state(double *dst, const double *S, int64_t b, int64_t h, int64_t H,
                        int64_t n) {
    if (dst) memcpy(dst + ((int64_t)b * H + h) * n, S, (size_t)n * sizeof(double));
}

/* Normalized ELU+1 linear attention. */
void oracle_elu(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                const double *q, const double *k, const double *v,
                const double *S0, const double *z0, double eps,
                double *o, double *S_out, double *z_out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv + 3 * dk + dv));
        double *z = S + dk * dv, *pk = z + dk, *pq = pk + dk, *num = pq + dk;
        load_state(S, S0, b, h, H, dk * dv);
        load_state(z, z0, b, h, H, dk);
        for (int64_t t = 0; t < T; ++t) {
            const double *qt = q + IDX4(b, t, h, 0, T, H, dk);
            const double *kt = k + IDX4(b, t, h, 0, T, H, dk);
            const double *vt = v + IDX4(b, t, h, 0, T, H, dv);
            for (int64_t d = 0; d < dk; ++d) { pq[d] = phi(qt[d]); pk[d] = phi(kt[d]); }
            /* S_t = S_{t-1} + phi(k_t) v_t^T ;  z_t = z_{t-1} + phi(k_t) */
            for (int64_t d = 0; d < dk; ++d) {
                for (int64_t j = 0; j < dv; ++j) S[d * dv + j] += pk[d] * vt[j];
                z[d] += pk[d];
            }
            /* o_t = phi(q_t)^T S_t / (phi(q_t)^T z_t + eps) */
            double den = 0.0;
            for (int64_t d = 0; d < dk; ++d) den += pq[d] * z[d];
            den += eps;
            for (int64_t j = 0; j < dv; ++j) num[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) num[j] += pq[d] * S[d * dv + j];
            double *ot = o + IDX4(b, t, h, 0, T, H, dv);
            for (int64_t j = 0; j < dv; ++j) ot[j] = num[j] / den;
        }
        store_state(S_out, S, b, h, H, dk * dv);
        store_state(z_out, z, b, h, H, dk);
        free(S);
    }
}

/* Gated linear attention with a per-key-dimension gate. */
void oracle_gla(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                const double *q, const double *k, const double *v, const double *g,
                const double *S0, double *o, double *S_out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv + dv));
        double *acc = S + dk * dv;
        load_state(S, S0, b, h, H, dk * dv);
        for (int64_t t = 0; t < T; ++t) {
            const double *qt = q + IDX4(b, t, h, 0, T, H, dk);
            const double *kt = k + IDX4(b, t, h, 0, T, H, dk);
            const double *gt = g + IDX4(b, t, h, 0, T, H, dk);
            const double *vt = v + IDX4(b, t, h, 0, T, H, dv);
            /* S_t = diag(g_t) S_{t-1} + k_t v_t^T */
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j)
                    S[d * dv + j] = gt[d] * S[d * dv + j] + kt[d] * vt[j];
            /* o_t = S_t^T q_t */
            for (int64_t j = 0; j < dv; ++j) acc[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) acc[j] += qt[d] * S[d * dv + j];
            memcpy(o + IDX4(b, t, h, 0, T, H, dv), acc, sizeof(double) * (size_t)dv);
        }
        store_state(S_out, S, b, h, H, dk * dv);
        free(S);
    }
}

/* Gated delta rule with scalar alpha_t, beta_t per token and head. */
void oracle_gdn(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                const double *q, const double *k, const double *v,
                const double *alpha, const double *beta,
                const double *S0, double *o, double *S_out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv + 2 * dv));
        double *kS = S + dk * dv, *acc = kS + dv;
        load_state(S, S0, b, h, H, dk * dv);
        for (int64_t t = 0; t < T; ++t) {
            const double *qt = q + IDX4(b, t, h, 0, T, H, dk);
            const double *kt = k + IDX4(b, t, h, 0, T, H, dk);
            const double *vt = v + IDX4(b, t, h, 0, T, H, dv);
            const double a = alpha[IDX3(b, t, h, T, H)];
            const double be = beta[IDX3(b, t, h, T, H)];
            /* (I - beta k k^T) S = S - beta k (k^T S):  kS = k^T S_{t-1} */
            for (int64_t j = 0; j < dv; ++j) kS[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) kS[j] += kt[d] * S[d * dv + j];
            /* S_t = alpha (S - beta k (k^T S)) + beta k v^T */
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j)
                    S[d * dv + j] = a * (S[d * dv + j] - be * kt[d] * kS[j]) + be * kt[d] * vt[j];
            /* o_t = S_t^T q_t */
            for (int64_t j = 0; j < dv; ++j) acc[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) acc[j] += qt[d] * S[d * dv + j];
            memcpy(o + IDX4(b, t, h, 0, T, H, dv), acc, sizeof(double) * (size_t)dv);
        }
        store_state(S_out, S, b, h, H, dk * dv);
        free(S);
    }
}

/* KDA: decay each key row of the state, then the delta-rule write. */
void oracle_kda(int64_t B, int64_t T, int64_t H, int64_t dk, int64_t dv,
                const double *q, const double *k, const double *v,
                const double *alpha, const double *beta,
                const double *S0, double *o, double *S_out) {
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t bh = 0; bh < B * H; ++bh) {
        const int64_t b = bh / H, h = bh % H;
        double *S = (double *)malloc(sizeof(double) * (size_t)(dk * dv + 2 * dv));
        double *pred = S + dk * dv, *acc = pred + dv;
        load_state(S, S0, b, h, H, dk * dv);
        for (int64_t t = 0; t < T; ++t) {
            const double *qt = q + IDX4(b, t, h, 0, T, H, dk);
            const double *kt = k + IDX4(b, t, h, 0, T, H, dk);
            const double *vt = v + IDX4(b, t, h, 0, T, H, dv);
            const double *at = alpha + IDX4(b, t, h, 0, T, H, dk);
            const double be = beta[IDX3(b, t, h, T, H)];
            /* Sbar = Diag(alpha_t) S_{t-1} */
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) S[d * dv + j] *= at[d];
            /* pred = Sbar^T k_t, then S_t = Sbar + beta k (v - pred)^T */
            for (int64_t j = 0; j < dv; ++j) pred[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) pred[j] += kt[d] * S[d * dv + j];
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) S[d * dv + j] += be * kt[d] * (vt[j] - pred[j]);
            /* o_t = S_t^T q_t */
            for (int64_t j = 0; j < dv; ++j) acc[j] = 0.0;
            for (int64_t d = 0; d < dk; ++d)
                for (int64_t j = 0; j < dv; ++j) acc[j] += qt[d] * S[d * dv + j];
            memcpy(o + IDX4(b, t, h, 0, T, H, dv), acc, sizeof(double) * (size_t)dv);
        }
        store_state(S_out, S, b, h, H, dk * dv);
        free(S);
    }
}

/* Head-wise RMS normalisation: for each of `rows` rows x of dv values,
 * y_j = w_j x_j / sqrt((1/dv) sum_i x_i^2 + eps), w NULL = all ones. */
void oracle_head_rmsnorm(int64_t rows, int64_t dv, const double *x, const double *w, double eps,
                         double *y) {
    for (int64_t r = 0; r < rows; ++r) {
        const double *xr = x + r * dv;
        double ss = 0.0;
        for (int64_t j = 0; j < dv; ++j) ss += xr[j] * xr[j];
        const double scale = 1.0 / sqrt(ss / (double)dv + eps);
        for (int64_t j = 0; j < dv; ++j) y[r * dv + j] = xr[j] * scale * (w ? w[j] : 1.0);
    }
}

int oracle_abi_version(void) { return 2; }
