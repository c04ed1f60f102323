/*
 * Element-wise check of rotated K rows against the oracle, for the
 * full-size parity tests (test infrastructure; the same rule as
 * tests/test_gpu_parity.py k_out_of_tolerance, checked against it on the
 * CPU): with got the library's bf16 output and ref the oracle's fp64 value,
 *   ref NaN       -> got must be a NaN (any sign or payload);
 *   ref +-inf     -> got must be that infinity;
 *   ref finite    -> |got - ref| <= rel |ref| + abs, where an infinite got
 *                    stands for every magnitude from the bf16 overflow
 *                    threshold 2^128 - 2^119 up (same sign as ref).
 * Also counts got equal bit for bit to the oracle's own bf16 rounding
 * (refs that are NaN excluded).  OpenMP over elements.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

static double bf16_value(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* Returns the number of elements outside the bar; *first_bad the index of
 * the first of them (or -1), *n_exact the bit-identical count, *n_compared
 * the elements whose ref is not NaN. */
int64_t kcheck(const uint16_t* got, const double* ref, const uint16_t* oracle_bits, int64_t n,
               double rel, double abs_tol, int64_t* first_bad, int64_t* n_exact,
               int64_t* n_compared) {
  const double over = ldexp(1.0, 128) - ldexp(1.0, 119);
  int64_t bad = 0, exact = 0, cmp = 0, first = -1;
#pragma omp parallel for reduction(+ : bad, exact, cmp) schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    const double g = bf16_value(got[i]);
    const double r = ref[i];
    int ok;
    if (isnan(r)) {
      ok = isnan(g);
    } else {
      ++cmp;
      if (got[i] == oracle_bits[i]) ++exact;
      if (isinf(r)) {
        ok = g == r;
      } else if (isnan(g)) {
        ok = 0;
      } else if (isinf(g)) {
        const double d = over - fabs(r);
        ok = ((signbit(g) != 0) == (signbit(r) != 0)) && (d <= 0.0 || d <= rel * fabs(r) + abs_tol);
      } else {
        ok = fabs(g - r) <= rel * fabs(r) + abs_tol;
      }
    }
    if (!ok) {
      ++bad;
#pragma omp critical
      if (first < 0 || i < first) first = i;
    }
  }
  *first_bad = first;
  *n_exact = exact;
  *n_compared = cmp;
  return bad;
}
