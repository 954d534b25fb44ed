/*
 * gdn_oracle_f32.c -- the oracle's loop nest evaluated in fp32.
 * TEST INFRASTRUCTURE ONLY: it sizes how far a correct single-precision
 * evaluation drifts from the fp64 oracle; it is never a parity reference.
 */
#define GDN_ORACLE_REAL float
#define GDN_ORACLE_FN gdn_oracle_update_f32
#define GDN_ORACLE_GATING_FN gdn_oracle_gating_f32
#include "gdn_oracle.c"
