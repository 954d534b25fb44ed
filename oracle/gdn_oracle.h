/*
 * gdn_oracle.h -- CPU oracle for the fused sigmoid-gating Gated DeltaNet
 * decode / speculative-decode state update.
 *
 * TEST INFRASTRUCTURE ONLY.  This oracle exists to check the CUDA path; only
 * the test suite, the smoke check and the CPU-baseline leg of the benchmark
 * may call it.  It is a plain, slow, single-threaded loop nest that follows
 * the update in the order the method states it, and it shares no code,
 * header, constant or helper with the CUDA library.
 *
 * What it computes (sources, by page title and section):
 *   - "[Qwen3Next] Optimize fused_sigmoid_gating_delta_rule_update_kernel"
 *     (sglang PR 18271), Motivation / Highlights: the one kernel that does
 *     the sigmoid gating and the recurrent delta-rule step together.
 *   - vLLM PR 35777 summary, sections "执行摘要" and "实现拆解": the fused
 *     op replaces fused_gdn_gating + fused_recurrent_gated_delta_rule, takes
 *     A_log, a, b, dt_bias, serves the spec and non-spec decode paths, and
 *     normalises q/k with rsqrt.
 *   - The update rule itself (the pages name the kernels but print no
 *     formula; the plainest reading that fits every name they use):
 *         g    = -exp(A_log[hv]) * softplus(a[t,hv] + dt_bias[hv])
 *         beta = sigmoid(b[t,hv])
 *         k^ = k / sqrt(sum k^2 + eps),  q^ = scale * q / sqrt(sum q^2 + eps)
 *         S  <- exp(g) * S                      (S is the [K,V] state)
 *         S  <- S + k^ (beta * (v - S^T k^))^T
 *         o  =  S^T q^
 *   - vLLM PR 37975 report, "实现拆解" (the `ba` reshape to
 *     (num_k_heads, 2*num_v_heads/num_k_heads)): value heads are grouped
 *     contiguously under key heads, h = hv / (HV/H).
 *
 * Readings taken where the pages are silent (each one is listed in the
 * design notes): softplus(x) = x for x > 20; eps = 1e-6 inside the square
 * root; `scale` multiplies q^ only; o is taken after the update; a slot
 * index of -1 marks a padded sequence whose output rows are written as 0
 * and whose state is not touched; a sequence of length 0 touches nothing.
 *
 * Layouts (all contiguous, row-major; bf16 values are passed as their
 * 16-bit patterns):
 *   q, k           [T_tot, H, K]        bf16 bits
 *   v              [T_tot, HV, V]       bf16 bits
 *   a, b           [T_tot, HV]          bf16 bits
 *   A_log, dt_bias [HV]                 fp32
 *   state_in       [num_slots, HV, K, V] fp32, V fastest
 *   state_indices  [N]                  int32, -1 = padded
 *   cu_seqlens     [N+1]                int32, or NULL for fixed length T
 *   out            [T_tot, HV, V]       REAL (written for every token of a
 *                                       valid or padded sequence)
 *   state_out      [num_slots, HV, K, V] REAL (a copy of state_in with the
 *                                       touched slots replaced)
 *   inter          [T_tot, HV, K, V]    REAL or NULL (state after each token)
 *
 * Return value: a bit mask, 0 when every sequence was valid.  Bit 0 is set
 * when a slot index is < -1 or >= num_slots, bit 1 when cu_seqlens is not
 * monotone or runs past T_tot; the offending sequence is skipped (nothing of
 * it is written).  A negative value means a bad argument (NULL pointer or a
 * non-positive size); nothing is written then.
 */
#ifndef GDN_ORACLE_H
#define GDN_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ORACLE_L2NORM_QK          1u
#define GDN_ORACLE_WRITE_INTERMEDIATE 2u
#define GDN_ORACLE_NO_FINAL_WRITEBACK 4u

#define GDN_ORACLE_BAD_SLOT     1
#define GDN_ORACLE_BAD_SEQLENS  2
#define GDN_ORACLE_BAD_ARGUMENT (-1)

/* fp64 oracle: every step in double precision.  Gates come from (a, b,
 * A_log, dt_bias), or -- when g and beta are given (both non-NULL; a, b,
 * A_log and dt_bias are then ignored and may be NULL) -- from the per
 * (token, value head) arrays g [T_tot, HV] (S <- exp(g) S) and beta
 * [T_tot, HV]: the recurrence of the unfused pair (the pages'
 * fused_recurrent_gated_delta_rule with precomputed gates). */
int gdn_oracle_update(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                      const uint16_t *a, const uint16_t *b,
                      const float *A_log, const float *dt_bias,
                      const float *g, const float *beta,
                      const float *state_in, const int32_t *state_indices,
                      const int32_t *cu_seqlens,
                      int32_t N, int32_t T_fixed, int32_t T_tot,
                      int32_t H, int32_t HV, int32_t K, int32_t V,
                      int32_t num_slots, double scale, uint32_t flags,
                      double *out, double *state_out, double *inter);

/* The same loop nest evaluated in fp32 (float math functions).  Used only
 * to size how far a correct fp32 evaluation drifts from the fp64 one. */
int gdn_oracle_update_f32(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                          const uint16_t *a, const uint16_t *b,
                          const float *A_log, const float *dt_bias,
                          const float *g, const float *beta,
                          const float *state_in, const int32_t *state_indices,
                          const int32_t *cu_seqlens,
                          int32_t N, int32_t T_fixed, int32_t T_tot,
                          int32_t H, int32_t HV, int32_t K, int32_t V,
                          int32_t num_slots, double scale, uint32_t flags,
                          float *out, float *state_out, float *inter);

/* The fp64 oracle with q, k, v, a, b given as fp32 values. */
int gdn_oracle_update_fin(const float *q, const float *k, const float *v,
                          const float *a, const float *b,
                          const float *A_log, const float *dt_bias,
                          const float *g, const float *beta,
                          const float *state_in, const int32_t *state_indices,
                          const int32_t *cu_seqlens,
                          int32_t N, int32_t T_fixed, int32_t T_tot,
                          int32_t H, int32_t HV, int32_t K, int32_t V,
                          int32_t num_slots, double scale, uint32_t flags,
                          double *out, double *state_out, double *inter);

/* The gating step alone: g = -exp(A_log) softplus(a + dt_bias) and
 * beta = sigmoid(b) for every (token, value head), [T_tot, HV] each. */
int gdn_oracle_gating(const uint16_t *a, const uint16_t *b, const float *A_log, const float *dt_bias,
                      int32_t T_tot, int32_t HV, double *g, double *beta);
int gdn_oracle_gating_f32(const uint16_t *a, const uint16_t *b, const float *A_log, const float *dt_bias,
                          int32_t T_tot, int32_t HV, float *g, float *beta);
int gdn_oracle_gating_fin(const float *a, const float *b, const float *A_log, const float *dt_bias,
                          int32_t T_tot, int32_t HV, double *g, double *beta);

#ifdef __cplusplus
}
#endif

#endif /* GDN_ORACLE_H */
