/*
 * gdn_oracle_fin.c -- the fp64 oracle with fp32 inputs (q, k, v, a, b given
 * as fp32 values instead of bf16 patterns).  TEST INFRASTRUCTURE ONLY.
 */
#define GDN_ORACLE_REAL double
#define GDN_ORACLE_FN gdn_oracle_update_fin
#define GDN_ORACLE_GATING_FN gdn_oracle_gating_fin
#define GDN_ORACLE_IN_T float
#include "gdn_oracle.c"
