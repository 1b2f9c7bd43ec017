// Host-side construction of the 4-bit code tables and their decision
// thresholds.
//
// NF4 -- page "QLoRA Explained", sections "Put the rows where the weights
// are" and "That is NF4": the 16 rows sit at quantiles of a standard normal,
// are computed once (not from the model) and include an exact zero; the table
// is normalised onto [-1, 1] so that a block's absmax stretches it onto the
// weights.  The page gives no construction for the exact zero; this library
// uses 8 positive levels, the zero and 7 negative levels:
//   delta = (1/30 + 1/32) / 2, top = 1 - delta
//   positive: Phi^-1 at 8 probabilities spaced evenly from top towards 1/2
//             (9 points including 1/2, which is dropped)
//   negative: -Phi^-1 at 7 such probabilities (8 points, 1/2 dropped)
//   divide by Phi^-1(top) so the ends are exactly -1 and +1; round to fp32.
// Phi^-1 is found by bisection on Phi(z) = erfc(-z / sqrt 2) / 2 in double
// precision, which converges to the double nearest the root (well inside the
// fp32 rounding of the final values).  Codes are the ranks 0..15.
//
// FP4 -- the same page's config walk-through names the library's other 4-bit
// option, "a small floating-point layout" at the same memory cost, and
// section "That is NF4" contrasts NF4 with a number made of exponent and
// mantissa fields.  This library reads it as the 4-bit float with a sign
// bit, 2 exponent bits and 1 mantissa bit (no infinities or NaNs): code c
// holds sign = bit 3 and magnitude {0, 0.5, 1, 1.5, 2, 3, 4, 6}[c & 7],
// divided by 6 so that the largest magnitude meets the block absmax.  Code 8
// (-0) decodes to -0 but is never produced: the quantiser searches the 15
// distinct values.
//
// Thresholds: a value x goes to the nearest row, a tie to the higher row
// (page "QLoRA Explained", section "The two failures that motivate the next
// section": 0, exactly between two rows, comes back as the upper one).  For
// distinct values v_k < v_{k+1} the decision point is their exact midpoint
// (exact in double); for an fp32 x, "x >= midpoint" equals "x >= T_k" with
// T_k the smallest float not below the midpoint.

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <algorithm>
#include <vector>

#include "common.cuh"

namespace qnf4 {

static double normal_cdf(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

static double normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int i = 0; i < 2000 && lo < hi; ++i) {
    double mid = 0.5 * (lo + hi);
    if (mid == lo || mid == hi) break;
    if (normal_cdf(mid) < p) lo = mid; else hi = mid;
  }
  return 0.5 * (lo + hi);
}

static void nf4_values(float* q) {
  const double delta = 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  const double top = 1.0 - delta;
  std::vector<double> lv;
  for (int i = 0; i < 8; ++i) lv.push_back(normal_quantile(top + (0.5 - top) * i / 8.0));
  for (int i = 0; i < 7; ++i) lv.push_back(-normal_quantile(top + (0.5 - top) * i / 7.0));
  lv.push_back(0.0);
  std::sort(lv.begin(), lv.end());
  double mx = 0.0;
  for (double v : lv) mx = std::max(mx, std::fabs(v));
  for (int i = 0; i < 16; ++i) q[i] = (float)(lv[i] / mx);
}

static void fp4_values(float* q) {
  static const double mag[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};
  for (int c = 0; c < 16; ++c) {
    const float v = (float)(mag[c & 7] / 6.0);
    q[c] = (c & 8) ? -v : v;
  }
}

static CodeTables build_tables(int quant_type) {
  CodeTables tb{};
  if (quant_type == QLORA_QUANT_FP4) fp4_values(tb.q);
  else nf4_values(tb.q);

  // distinct values, ascending, each with the code that stores it (the
  // first code holding the value: +0 rather than -0)
  std::vector<std::pair<float, int>> vals;
  for (int c = 0; c < 16; ++c) {
    bool seen = false;
    for (auto& v : vals) seen |= (v.first == tb.q[c]);
    if (!seen) vals.push_back({tb.q[c], c});
  }
  std::sort(vals.begin(), vals.end(),
            [](const std::pair<float, int>& a, const std::pair<float, int>& b) { return a.first < b.first; });
  const int nv = (int)vals.size();
  tb.nt = nv - 1;
  tb.monotone = 1;
  for (int k = 0; k < nv; ++k) {
    tb.rank_code[k] = (uint8_t)vals[k].second;
    tb.monotone &= vals[k].second == k;
  }
  for (int j = 0; j < tb.nt; ++j) {
    double m = ((double)vals[j].first + (double)vals[j + 1].first) * 0.5;   // exact
    float t = (float)m;
    if ((double)t < m) t = std::nextafter(t, INFINITY);
    tb.t[j] = t;
  }

  // Bucket table for the quantise kernel's code search.  Every threshold
  // must sit well away from a bucket edge so that the rounding in the
  // bucket index (x + 1) * 16 can never put x on the wrong side of an edge
  // that a threshold shares.
  for (int b = 0; b < 64; ++b) {
    double lo = -1.0 + (b - 0.5) / 16.0, hi = lo + 1.0 / 16.0;
    int below = 0;
    float thr = 2.0f;                         // "no threshold here": above every |x| <= 1
    for (int j = 0; j < tb.nt; ++j) {
      if ((double)tb.t[j] < lo) ++below;
      else if ((double)tb.t[j] < hi) {
        if (thr != 2.0f) { std::fprintf(stderr, "qlora_nf4: two thresholds in a bucket\n"); std::abort(); }
        thr = tb.t[j];
      }
      double edge_gap = std::min(std::fabs((double)tb.t[j] - lo), std::fabs((double)tb.t[j] - hi));
      if (edge_gap < 1e-4) { std::fprintf(stderr, "qlora_nf4: threshold too near a bucket edge\n"); std::abort(); }
    }
    tb.bucket_thr[b] = thr;
    tb.bucket_lo[b] = tb.rank_code[std::min(below, nv - 1)];
    tb.bucket_hi[b] = tb.rank_code[std::min(below + 1, nv - 1)];
  }
  return tb;
}

const CodeTables& host_tables(int quant_type) {
  static const CodeTables nf4 = build_tables(QLORA_QUANT_NF4);
  static const CodeTables fp4 = build_tables(QLORA_QUANT_FP4);
  return quant_type == QLORA_QUANT_FP4 ? fp4 : nf4;
}

}  // namespace qnf4
