/*
 * gdn_oracle_ld.c -- the same CPU oracle as gdn_oracle.c, compiled with
 * long double arithmetic.  TEST INFRASTRUCTURE ONLY.  Used to bound the
 * rounding error of the double oracle itself on extreme gate regimes.
 * Exported names carry an `_ld` suffix and take long double state/outputs.
 */
#define ORACLE_REAL long double
#define ORACLE_SUFFIX(name) name##_ld
#include "gdn_oracle.c"
