/*
 * Plain C restatement of one PhaseQuant stage, for full-size oracle runs.
 * TEST INFRASTRUCTURE ONLY: used by tests/ and bench.py's CPU-baseline leg,
 * never by the library.  Same definitions as oracle/phasequant.py, element by
 * element, in IEEE double with no contraction (-ffp-contract=off):
 *
 *   residual ("Fairy2i write-up" §4.1): r = w - sum_{u<t} (s_re,u Br_u + i s_im,u Bi_u),
 *     subtracted one earlier stage at a time, in stage order; an entry with a
 *     non-finite part is taken as 0;
 *   phase rule (§3.1): sector k = floor(2 arg(r)/pi + 0.5) mod 4, written as
 *     comparisons; ties on a diagonal go counter-clockwise; r = 0 -> 0;
 *   axis scales (§3.2): S_re = sum |Re r| over k even, S_im = sum |Im r| over k odd.
 */
#include <math.h>
#include <stdint.h>

static int sector(double a, double b) {
  double aa = fabs(a), ab = fabs(b);
  if (b > aa || (a == b && b > 0)) return 1;
  if (-a > ab || (b == -a && a < 0)) return 2;
  if (-b > aa || (a == b && b < 0)) return 3;
  return 0;
}

/*
 * Codes of stage t (0-based) for n weights (n % 4 == 0), given the packed codes
 * prev[u][n/4] and float32 scales prev_scales[u][2] of stages u < t.
 *   out_codes  [n/4] packed, code i in bits 2(i%4) of byte i/4
 *   sums       {S_re, C_re, S_im, C_im}
 *   near       optional [n]: 1 where |(|a|-|b|)| <= 1e-6 (|a|+|b|) or
 *              |a|+|b| <= 1e-6 * sum_{u<t} (s_re,u + s_im,u)
 */
void ref_stage(const float* w_re, const float* w_im, int64_t n, int t, const uint8_t* prev,
               const float* prev_scales, uint8_t* out_codes, double* sums, uint8_t* near) {
  const int64_t nq = n / 4;
  double S_re = 0.0, S_im = 0.0, C_re = 0.0, C_im = 0.0, sprev = 0.0;
  for (int u = 0; u < t; ++u) sprev += (double)prev_scales[2 * u] + (double)prev_scales[2 * u + 1];
  for (int64_t q = 0; q < nq; ++q) out_codes[q] = 0;
  for (int64_t i = 0; i < n; ++i) {
    double a = w_re[i], b = w_im[i];
    if (!isfinite(w_re[i]) || !isfinite(w_im[i])) {
      a = 0.0;
      b = 0.0;
    }
    for (int u = 0; u < t; ++u) {
      int ku = (prev[(int64_t)u * nq + i / 4] >> (2 * (i % 4))) & 3;
      double br = ku == 0 ? 1.0 : (ku == 2 ? -1.0 : 0.0);
      double bi = ku == 1 ? 1.0 : (ku == 3 ? -1.0 : 0.0);
      double pr = (double)prev_scales[2 * u] * br;
      double pi = (double)prev_scales[2 * u + 1] * bi;
      a = a - pr;
      b = b - pi;
    }
    int k = sector(a, b);
    out_codes[i / 4] |= (uint8_t)(k << (2 * (i % 4)));
    if ((k & 1) == 0) {
      S_re += fabs(a);
      C_re += 1.0;
    } else {
      S_im += fabs(b);
      C_im += 1.0;
    }
    if (near) {
      double aa = fabs(a), ab = fabs(b);
      near[i] = (fabs(aa - ab) <= 1e-6 * (aa + ab)) || (aa + ab <= 1e-6 * sprev);
    }
  }
  sums[0] = S_re;
  sums[1] = C_re;
  sums[2] = S_im;
  sums[3] = C_im;
}
