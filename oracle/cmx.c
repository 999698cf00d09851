/*
 * MX block quantisation in plain C, fp64 arithmetic.  TEST INFRASTRUCTURE ONLY.
 *
 * The same rule as oracle/mx.py (quantize_mx), restated in C so that the parity tests at
 * the Kimi-K3 shapes can quantise hundreds of experts' weights (66M values each) in
 * seconds.  It follows the OCP Microscaling Formats (MX) v1.0 block rule with the readings
 * of oracle/mx.py:
 *   - a block is 32 consecutive values of a row; amax = its largest magnitude;
 *   - scale exponent e = floor(log2 amax) - emax, clamped to [-127, 127]; an all-zero block
 *     takes e = -127 (R3, R4); the scale byte is e + 127;
 *   - element = the value v / 2^e rounded to the nearest entry of the format's positive
 *     value list (ties to the even code), saturating at the largest entry (R1), with the
 *     sign bit of v kept, also for a value that rounds to zero (R2).
 * The positive value lists come from the caller (oracle/mx.py builds them from the formats'
 * sign/exponent/mantissa definitions), so the two restatements share one table.  The
 * decoder (mx_dequantize_f64) restates oracle/mx.py's dequantize_mx the same way.
 */
#include <math.h>
#include <stdint.h>

/* Index of the entry of pos[0..n) nearest to a (0 <= a <= pos[n-1]), ties to the even
 * index: the largest lo with pos[lo] <= a, then lo or lo + 1 by distance. */
static int nearest_even(const double* pos, int n, double a) {
  int lo = 0;
  if (n <= 16) { /* short list (E2M1): count the entries above pos[0] that are <= a */
    for (int i = 1; i < n; ++i) lo += pos[i] <= a;
  } else {
    int hi = n - 1;
    while (lo < hi) { /* largest lo with pos[lo] <= a */
      const int mid = (lo + hi + 1) / 2;
      if (pos[mid] <= a) lo = mid; else hi = mid - 1;
    }
  }
  const int up = lo + 1 < n ? lo + 1 : lo;
  const double d_lo = a - pos[lo], d_up = pos[up] - a;
  if (d_up < d_lo || (d_up == d_lo && (up & 1) == 0)) return up;
  return lo;
}

/* v: fp32 [rows][K] (K % 32 == 0), read as exact fp64.  codes: uint8 [rows][K] (sign bit =
 * sign_bit | index), scales: uint8 [rows][K / 32].  pos: the n positive values in
 * increasing order (code = index); max_mag = pos[n - 1]; emax: the format's emax. */
void mx_quantize_f32(const float* v, long rows, long K, const double* pos, int n, int emax,
                     int sign_bit, uint8_t* codes, uint8_t* scales) {
  const double max_mag = pos[n - 1];
  for (long r = 0; r < rows; ++r) {
    for (long b = 0; b < K / 32; ++b) {
      const float* x = v + r * K + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) {
        const double m = fabs((double)x[i]);
        if (m > amax) amax = m;
      }
      int e = -127;
      if (amax > 0.0) {
        int ex;
        frexp(amax, &ex); /* amax = f * 2^ex, f in [0.5, 1): floor(log2 amax) = ex - 1 */
        e = ex - 1 - emax;
      }
      if (e < -127) e = -127;
      if (e > 127) e = 127;
      scales[r * (K / 32) + b] = (uint8_t)(e + 127);
      const double inv = ldexp(1.0, -e); /* 2^-e, exact in fp64 for e in [-127, 127] */
      for (int i = 0; i < 32; ++i) {
        const double q = (double)x[i] * inv; /* exact: a power-of-two scaling */
        double a = fabs(q);
        if (a > max_mag) a = max_mag;
        const int idx = nearest_even(pos, n, a);
        codes[r * K + b * 32 + i] = (uint8_t)(idx | (signbit(q) ? sign_bit : 0));
      }
    }
  }
}

/* Exact fp64 values of MX data: table[code & code_mask] * 2^(scale - 127) per block of 32
 * (a scale byte of 0xFF is NaN).  codes: uint8 [rows][K]; scales: uint8 [rows][K / 32];
 * table: the format's value of every code (16 or 256 entries, from oracle/mx.py). */
void mx_dequantize_f64(const uint8_t* codes, const uint8_t* scales, long rows, long K, const double* table,
                       int code_mask, double* out) {
  for (long r = 0; r < rows; ++r) {
    for (long b = 0; b < K / 32; ++b) {
      const int sb = scales[r * (K / 32) + b];
      const double sc = sb == 255 ? NAN : ldexp(1.0, sb - 127);
      const uint8_t* c = codes + r * K + b * 32;
      double* o = out + r * K + b * 32;
      for (int i = 0; i < 32; ++i) o[i] = table[c[i] & code_mask] * sc;
    }
  }
}
