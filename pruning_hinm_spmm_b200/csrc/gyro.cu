// Gyro-style refinement of a tile's 2:4 grouping (FlexHiNM-GP notes, 关键设计 2: channel
// permutation reorders channels without changing the product, so that important weights
// land where they are kept; per tile, sampled vectors are re-assigned by the Hungarian
// algorithm on the pruning-cost matrix, iterated to refine).  Host code: an offline,
// once-per-layer step whose output -- the 2:4 band's working order -- is the permutation
// the hot path takes.
//
// Iteration i takes the caller's S (group, slot) samples (distinct groups): the sampled
// vectors leave their slots and return by the assignment that maximises the sum over the
// sampled groups of their retained 2:4 importance (each row's two largest of the group's
// four values, summed over the tile's rows in fp64).  Keeping every vector in place is one
// assignment, so the retained importance never decreases.
#include <algorithm>
#include <cstdint>
#include <limits>
#include <vector>

#include "hinm_internal.h"

namespace hinm {
namespace {

// Retained 2:4 importance of four channels over the tile's rows: per row the two largest
// values, each as fp64, added to the row-ascending fp64 sum.
double group_retained(const float* I, int T, int K, const int32_t (&m)[4]) {
  double acc = 0.0;
  for (int r = 0; r < T; ++r) {
    const float* row = I + (size_t)r * K;
    const float a = row[m[0]], b = row[m[1]], c = row[m[2]], d = row[m[3]];
    const float hi1 = std::max(a, b), lo1 = std::min(a, b);
    const float hi2 = std::max(c, d), lo2 = std::min(c, d);
    const float t1 = std::max(hi1, hi2);
    const float t2 = std::max(std::min(hi1, hi2), std::max(lo1, lo2));
    acc += (double)t1 + (double)t2;
  }
  return acc;
}

// Minimum-cost perfect assignment of a dense n x n matrix c (row-major); returns the
// column of every row.  Rows join one at a time, each by the cheapest augmenting path in
// the reduced costs c[i][j] - pr[i] - pc[j], found by a Dijkstra over the columns
// (O(n^2) per row).  With delta the path's length and d[j] the settled columns' distances,
// pr[r] += delta and, for every settled column j, pc[j] -= delta - d[j] and the row
// matched to it gains delta - d[j]: the reduced costs stay >= 0 and every matched edge,
// old and new, stays at 0.  Ties go to the lowest column index.
std::vector<int> min_cost_assignment(const std::vector<double>& c, int n) {
  const double kInf = std::numeric_limits<double>::infinity();
  std::vector<double> pr(n, 0.0), pc(n, 0.0), d(n);
  std::vector<int> row_of(n, -1), col_of(n, -1), from(n);
  std::vector<char> settled(n);
  for (int r = 0; r < n; ++r) {
    for (int j = 0; j < n; ++j) {
      d[j] = c[(size_t)r * n + j] - pr[r] - pc[j];
      from[j] = -1;
      settled[j] = 0;
    }
    int jfree = -1;
    double delta = 0.0;
    for (;;) {
      int jm = -1;
      double dm = kInf;
      for (int j = 0; j < n; ++j)
        if (!settled[j] && d[j] < dm) {
          dm = d[j];
          jm = j;
        }
      if (jm < 0) return {};  // no finite reduced cost left (the callers pass finite costs)
      settled[jm] = 1;
      if (row_of[jm] < 0) {
        jfree = jm;
        delta = dm;
        break;
      }
      const int i = row_of[jm];
      for (int j = 0; j < n; ++j) {
        if (settled[j]) continue;
        const double nd = dm + c[(size_t)i * n + j] - pr[i] - pc[j];
        if (nd < d[j]) {
          d[j] = nd;
          from[j] = jm;
        }
      }
    }
    pr[r] += delta;
    for (int j = 0; j < n; ++j) {
      if (!settled[j]) continue;
      pc[j] -= delta - d[j];
      if (row_of[j] >= 0) pr[row_of[j]] += delta - d[j];
    }
    // augment: each column on the path takes the row of the column it was reached from
    for (int j = jfree;;) {
      const int jp = from[j];
      const int i = jp < 0 ? r : row_of[jp];
      row_of[j] = i;
      col_of[i] = j;
      if (jp < 0) break;
      j = jp;
    }
  }
  return col_of;
}

}  // namespace

double gyro_band_retained(const float* I, int T, int K, const int32_t* band, int n) {
  double acc = 0.0;
  for (int g = 0; g < n / 4; ++g) {
    const int32_t m[4] = {band[4 * g], band[4 * g + 1], band[4 * g + 2], band[4 * g + 3]};
    acc += group_retained(I, T, K, m);
  }
  return acc;
}

void gyro_refine(const float* I, int T, int K, int32_t* band, int n, const int32_t* schedule,
                 int iters, int S, double* retained) {
  if (retained) retained[0] = gyro_band_retained(I, T, K, band, n);
  std::vector<double> cost((size_t)S * S);
  std::vector<int32_t> vec(S);
  std::vector<float> top2((size_t)S * T * 2);  // per sampled group and row: the two largest
  std::vector<float> xv((size_t)S * T);        // of its three remaining values; the vectors
  for (int it = 0; it < iters; ++it) {
    const int32_t* sc = schedule + (size_t)it * S * 2;
    for (int a = 0; a < S; ++a) {
      vec[a] = band[4 * sc[2 * a] + sc[2 * a + 1]];
      for (int r = 0; r < T; ++r) xv[(size_t)a * T + r] = I[(size_t)r * K + vec[a]];
    }
    for (int b = 0; b < S; ++b) {
      const int g = sc[2 * b], k = sc[2 * b + 1];
      int32_t m[3];
      int q = 0;
      for (int j = 0; j < 4; ++j)
        if (j != k) m[q++] = band[4 * g + j];
      for (int r = 0; r < T; ++r) {
        const float* row = I + (size_t)r * K;
        float v0 = row[m[0]], v1 = row[m[1]], v2 = row[m[2]];
        if (v1 > v0) std::swap(v0, v1);
        if (v2 > v1) std::swap(v1, v2);
        if (v1 > v0) std::swap(v0, v1);
        top2[((size_t)b * T + r) * 2] = v0;
        top2[((size_t)b * T + r) * 2 + 1] = v1;
      }
    }
    // cost[a][b] = -(retained importance of group b with vector a in its freed slot): per row
    // the two largest of {x, s1, s2, s3} are {x, s1} (x >= s1), {s1, x} (s2 <= x < s1) or
    // {s1, s2}, added as fp64 and summed over the rows in ascending order (the values and
    // the order of group_retained, so the sums are the same)
    for (int a = 0; a < S; ++a) {
      const float* x = xv.data() + (size_t)a * T;
      for (int b = 0; b < S; ++b) {
        const float* t2 = top2.data() + (size_t)b * T * 2;
        double acc = 0.0;
        for (int r = 0; r < T; ++r) {
          const float s1 = t2[2 * r], s2 = t2[2 * r + 1], xr = x[r];
          acc += xr >= s1 ? (double)xr + (double)s1
                          : (xr >= s2 ? (double)s1 + (double)xr : (double)s1 + (double)s2);
        }
        cost[(size_t)a * S + b] = -acc;  // maximise the retained importance
      }
    }
    const std::vector<int> to = min_cost_assignment(cost, S);
    if ((int)to.size() != S) return;
    for (int a = 0; a < S; ++a) band[4 * sc[2 * to[a]] + sc[2 * to[a] + 1]] = vec[a];
    if (retained) retained[it + 1] = gyro_band_retained(I, T, K, band, n);
  }
}

}  // namespace hinm
