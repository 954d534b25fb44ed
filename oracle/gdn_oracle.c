/*
 * gdn_oracle.c -- plain CPU oracle for the fused sigmoid-gating Gated
 * DeltaNet decode update.  TEST INFRASTRUCTURE ONLY (see gdn_oracle.h for
 * what it computes, the layouts and the passages it follows).
 *
 * The loop nest is the definition written out: sequence -> value head ->
 * token -> (gating, q/k normalisation, decay, S^T k, delta, rank-1 update,
 * output, optional intermediate copy).  No step is fused, reordered or
 * blocked.  The file is compiled three times: as-is for the fp64 oracle,
 * from gdn_oracle_f32.c with GDN_ORACLE_REAL=float for the fp32 drift study,
 * and from gdn_oracle_fin.c with fp32 (instead of bf16-pattern) inputs.
 * <tgmath.h> makes exp/log1p/sqrt follow the working type.
 */
#include <stddef.h>
#include <stdlib.h>
#include <string.h>
#include <tgmath.h>

#include "gdn_oracle.h"

/* Three builds of this file: fp64 with bf16-pattern inputs (the oracle),
 * fp32 with bf16-pattern inputs (drift study), fp64 with fp32 inputs. */
#ifndef GDN_ORACLE_REAL
#define GDN_ORACLE_REAL double
#define GDN_ORACLE_FN gdn_oracle_update
#define GDN_ORACLE_GATING_FN gdn_oracle_gating
#endif
#ifndef GDN_ORACLE_IN_T
#define GDN_ORACLE_IN_T uint16_t
#define GDN_ORACLE_IN_BF16 1
#endif

typedef GDN_ORACLE_REAL real;
typedef GDN_ORACLE_IN_T in_t;

#ifdef GDN_ORACLE_IN_BF16
/* A bf16 value is the upper half of an IEEE binary32 pattern. */
static real bf16_bits_to_real(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (real)f;
}
#else
/* fp32 inputs: the value itself. */
static real bf16_bits_to_real(float x)
{
    return (real)x;
}
#endif

/* softplus(x) = ln(1 + e^x); above 20 the correction e^-x is below 2e-9
 * relative and the function returns x (reading: threshold 20). */
static real softplus(real x)
{
    if (x > (real)20)
        return x;
    return log1p(exp(x));
}

/* sigmoid(x) = 1 / (1 + e^-x); exact 0 at -inf and 1 at +inf. */
static real sigmoid(real x)
{
    return (real)1 / ((real)1 + exp(-x));
}

/* g, beta = -exp(A_log) softplus(a + dt_bias), sigmoid(b), per (token, value
 * head): the gating step on its own (the pages' fused_gdn_gating). */
int GDN_ORACLE_GATING_FN(const in_t *a, const in_t *b, const float *A_log, const float *dt_bias,
                         int32_t T_tot, int32_t HV, real *g_out, real *beta_out)
{
    if (!a || !b || !A_log || !dt_bias || !g_out || !beta_out || T_tot < 0 || HV <= 0)
        return GDN_ORACLE_BAD_ARGUMENT;
    for (int64_t tok = 0; tok < T_tot; ++tok)
        for (int32_t hv = 0; hv < HV; ++hv) {
            const real x = bf16_bits_to_real(a[(size_t)tok * HV + hv]) + (real)dt_bias[hv];
            g_out[(size_t)tok * HV + hv] = -exp((real)A_log[hv]) * softplus(x);
            beta_out[(size_t)tok * HV + hv] = sigmoid(bf16_bits_to_real(b[(size_t)tok * HV + hv]));
        }
    return 0;
}

int GDN_ORACLE_FN(const in_t *q, const in_t *k, const in_t *v,
                  const in_t *a, const in_t *b,
                  const float *A_log, const float *dt_bias,
                  const float *g_in, const float *beta_in,
                  const float *state_in, const int32_t *state_indices,
                  const int32_t *cu_seqlens,
                  int32_t N, int32_t T_fixed, int32_t T_tot,
                  int32_t H, int32_t HV, int32_t K, int32_t V,
                  int32_t num_slots, double scale, uint32_t flags,
                  real *out, real *state_out, real *inter)
{
    const real eps = (real)1e-6;
    const int l2norm = (flags & GDN_ORACLE_L2NORM_QK) != 0;
    const int keep_inter = (flags & GDN_ORACLE_WRITE_INTERMEDIATE) != 0;
    const int final_write = (flags & GDN_ORACLE_NO_FINAL_WRITEBACK) == 0;
    int status = 0;

    /* Gates: from (a, b, A_log, dt_bias), or given as (g, beta) arrays. */
    const int given_gates = g_in != NULL || beta_in != NULL;
    if (given_gates ? (!g_in || !beta_in) : (!a || !b || !A_log || !dt_bias))
        return GDN_ORACLE_BAD_ARGUMENT;
    if (!q || !k || !v || !state_in || !state_indices || !out || !state_out)
        return GDN_ORACLE_BAD_ARGUMENT;
    if (N < 0 || T_tot < 0 || H <= 0 || HV <= 0 || K <= 0 || V <= 0 ||
        num_slots < 0 || HV % H != 0)
        return GDN_ORACLE_BAD_ARGUMENT;
    if (!cu_seqlens && (T_fixed < 0 || (int64_t)T_fixed * N != T_tot))
        return GDN_ORACLE_BAD_ARGUMENT;
    if (keep_inter && !inter)
        return GDN_ORACLE_BAD_ARGUMENT;

    const int32_t G = HV / H; /* value heads per key head */
    const size_t head_elems = (size_t)K * V;

    /* The pool after the call starts as the pool before it. */
    const size_t pool_elems = (size_t)num_slots * HV * head_elems;
    for (size_t e = 0; e < pool_elems; ++e)
        state_out[e] = (real)state_in[e];

    real *S = malloc(head_elems * sizeof(real));
    real *k_hat = malloc((size_t)K * sizeof(real));
    real *q_hat = malloc((size_t)K * sizeof(real));
    real *kv = malloc((size_t)V * sizeof(real));
    real *delta = malloc((size_t)V * sizeof(real));
    if (!S || !k_hat || !q_hat || !kv || !delta) {
        free(S); free(k_hat); free(q_hat); free(kv); free(delta);
        return GDN_ORACLE_BAD_ARGUMENT;
    }

    for (int32_t i = 0; i < N; ++i) {
        /* Token range of sequence i. */
        int64_t bos, eos;
        if (cu_seqlens) {
            bos = cu_seqlens[i];
            eos = cu_seqlens[i + 1];
            if (bos < 0 || eos < bos || eos > T_tot) {
                status |= GDN_ORACLE_BAD_SEQLENS;
                continue;
            }
        } else {
            bos = (int64_t)i * T_fixed;
            eos = bos + T_fixed;
        }

        const int32_t slot = state_indices[i];
        if (slot < -1 || slot >= num_slots) {
            status |= GDN_ORACLE_BAD_SLOT;
            continue;
        }
        if (slot == -1) {
            /* Padded sequence: zero output rows, state untouched. */
            for (int64_t tok = bos; tok < eos; ++tok)
                for (int32_t hv = 0; hv < HV; ++hv)
                    for (int32_t c = 0; c < V; ++c)
                        out[((size_t)tok * HV + hv) * V + c] = 0;
            continue;
        }

        for (int32_t hv = 0; hv < HV; ++hv) {
            const int32_t h = hv / G; /* key head of this value head */
            const float *S_in = state_in + ((size_t)slot * HV + hv) * head_elems;
            for (size_t e = 0; e < head_elems; ++e)
                S[e] = (real)S_in[e];

            for (int64_t tok = bos; tok < eos; ++tok) {
                real g, beta;
                if (given_gates) {
                    g = (real)g_in[(size_t)tok * HV + hv];
                    beta = (real)beta_in[(size_t)tok * HV + hv];
                } else {
                    /* Gating: g = -exp(A_log) softplus(a + dt_bias), beta = sigmoid(b). */
                    const real x = bf16_bits_to_real(a[(size_t)tok * HV + hv]) + (real)dt_bias[hv];
                    g = -exp((real)A_log[hv]) * softplus(x);
                    beta = sigmoid(bf16_bits_to_real(b[(size_t)tok * HV + hv]));
                }

                /* q and k of key head h, L2-normalised; q scaled. */
                const in_t *k_row = k + ((size_t)tok * H + h) * K;
                const in_t *q_row = q + ((size_t)tok * H + h) * K;
                real sum_kk = 0, sum_qq = 0;
                for (int32_t r = 0; r < K; ++r) {
                    const real kr = bf16_bits_to_real(k_row[r]);
                    const real qr = bf16_bits_to_real(q_row[r]);
                    sum_kk += kr * kr;
                    sum_qq += qr * qr;
                }
                const real k_norm = l2norm ? (real)1 / sqrt(sum_kk + eps) : (real)1;
                const real q_norm = l2norm ? (real)1 / sqrt(sum_qq + eps) : (real)1;
                for (int32_t r = 0; r < K; ++r) {
                    k_hat[r] = bf16_bits_to_real(k_row[r]) * k_norm;
                    q_hat[r] = bf16_bits_to_real(q_row[r]) * q_norm * (real)scale;
                }

                /* Decay: S <- exp(g) S. */
                const real decay = exp(g);
                for (size_t e = 0; e < head_elems; ++e)
                    S[e] *= decay;

                /* kv = S^T k^ (a length-V vector; sum over the K rows). */
                for (int32_t c = 0; c < V; ++c) {
                    real acc = 0;
                    for (int32_t r = 0; r < K; ++r)
                        acc += S[(size_t)r * V + c] * k_hat[r];
                    kv[c] = acc;
                }

                /* delta = beta (v - kv). */
                const in_t *v_row = v + ((size_t)tok * HV + hv) * V;
                for (int32_t c = 0; c < V; ++c)
                    delta[c] = beta * (bf16_bits_to_real(v_row[c]) - kv[c]);

                /* Rank-1 update: S <- S + k^ delta^T. */
                for (int32_t r = 0; r < K; ++r)
                    for (int32_t c = 0; c < V; ++c)
                        S[(size_t)r * V + c] += k_hat[r] * delta[c];

                /* Output o = S^T q^ on the updated state. */
                real *o = out + ((size_t)tok * HV + hv) * V;
                for (int32_t c = 0; c < V; ++c) {
                    real acc = 0;
                    for (int32_t r = 0; r < K; ++r)
                        acc += S[(size_t)r * V + c] * q_hat[r];
                    o[c] = acc;
                }

                if (keep_inter) {
                    real *dst = inter + ((size_t)tok * HV + hv) * head_elems;
                    for (size_t e = 0; e < head_elems; ++e)
                        dst[e] = S[e];
                }
            }

            if (final_write) {
                real *dst = state_out + ((size_t)slot * HV + hv) * head_elems;
                for (size_t e = 0; e < head_elems; ++e)
                    dst[e] = S[e];
            }
        }
    }

    free(S); free(k_hat); free(q_hat); free(kv); free(delta);
    return status;
}
