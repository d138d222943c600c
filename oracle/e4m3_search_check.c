/*
 * e4m3_search_check.c -- TEST INFRASTRUCTURE ONLY.
 *
 * A second, independent E4M3 encoder (nearest-value search over the sorted
 * table of finite E4M3 magnitudes, ties to the even code) and an exhaustive
 * driver that compares it with the bit-manipulation encoder of the oracle over
 * every binary32 bit pattern.  The table comes from the oracle's decoder,
 * which the tests pin separately against hand-computed values and against
 * PyTorch's float8_e4m3fn decoding.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

double orc_e4m3_decode(uint8_t code);
uint8_t orc_e4m3_encode(float v);

/* magnitudes of codes 0x00..0x7E, strictly increasing (0 .. 448) */
static void positive_table(double* t127) {
  for (int c = 0; c < 127; ++c) t127[c] = orc_e4m3_decode((uint8_t)c);
}

/* Nearest E4M3 code by search.  The comparison is against the exact midpoint
 * of two neighbouring grid values (a short binary fraction, exact in double),
 * so no subtraction can round. */
static uint8_t encode_by_search(float v, const double* t) {
  if (isnan(v)) return 0x7F;
  uint8_t sign = signbit(v) ? 0x80 : 0x00;
  double a = fabs((double)v);
  if (a >= t[126]) return sign | 0x7E; /* saturate at 448 */
  int lo = 0, hi = 126;                /* invariant: t[lo] <= a < t[hi] */
  while (hi - lo > 1) {
    int mid = (lo + hi) / 2;
    if (t[mid] <= a)
      lo = mid;
    else
      hi = mid;
  }
  double midpoint = 0.5 * (t[lo] + t[hi]);
  int code;
  if (a < midpoint)
    code = lo;
  else if (a > midpoint)
    code = hi;
  else
    code = (lo % 2 == 0) ? lo : hi; /* tie: even mantissa LSB */
  return sign | (uint8_t)code;
}

uint8_t orc_e4m3_encode_by_search(float v) {
  double t[127];
  positive_table(t);
  return encode_by_search(v, t);
}

/* Compare both encoders on bit patterns first, first+stride, ... < end
 * (64-bit bounds so the full 2^32 range fits).  Returns the number of
 * mismatches and stores the first mismatching pattern in *first_bad. */
int64_t orc_e4m3_exhaustive_check(uint64_t first, uint64_t end, uint64_t stride, uint32_t* first_bad) {
  double t[127];
  positive_table(t);
  int64_t bad = 0;
  uint64_t worst = UINT64_MAX;
  if (stride == 0) return -1;
  const int64_t n = (int64_t)((end - first + stride - 1) / stride);
#pragma omp parallel for schedule(static) reduction(+ : bad) reduction(min : worst)
  for (int64_t i = 0; i < n; ++i) {
    uint32_t bits = (uint32_t)(first + (uint64_t)i * stride);
    float v;
    memcpy(&v, &bits, sizeof v);
    if (orc_e4m3_encode(v) != encode_by_search(v, t)) {
      bad += 1;
      if (bits < worst) worst = bits;
    }
  }
  if (first_bad) *first_bad = bad ? (uint32_t)worst : 0u;
  return bad;
}
