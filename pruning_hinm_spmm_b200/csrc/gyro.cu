// Gyro-permutation (FlexHiNM-GP notes, 关键设计 2: channel permutation reorders input and
// output channels without changing the product, so that important weights land where they
// are kept; the pipeline runs output-channel permutation, column-vector pruning and the
// in-tile input-channel permutation, and each round samples vectors per tile, clusters them
// with a balanced K-means and assigns the clusters by the Hungarian algorithm on the
// pruning-cost matrix, smaller cost better; iterated to refine).  Offline, once per layer:
// its outputs -- a tile's 2:4 band in a better working order, a layer's output-row order --
// are the permutations the hot path takes.
//
// Host code for the rounds (the sampled sizes are small: the K-means and the assignment are
// O(S^3)), and gyro_cost_kernel, which builds the input rounds' pruning-cost matrices of
// every tile of a layer on the GPU (the O(G^2 T) part).  Both compute every cost as the
// row-ascending fp64 sum of the two smallest of the group's four fp32 values per row, so
// host, device and the fp64 oracle agree bit for bit.
#include <algorithm>
#include <cstdint>
#include <limits>
#include <numeric>
#include <vector>

#include "hinm_internal.h"

namespace hinm {
namespace {

// Minimum-cost perfect assignment of a dense n x n matrix c (row-major); returns the
// column of every row.  Rows join one at a time, each by the cheapest augmenting path in
// the reduced costs c[i][j] - pr[i] - pc[j], found by a Dijkstra over the columns
// (O(n^2) per row).  With delta the path's length and d[j] the settled columns' distances,
// pr[r] += delta and, for every settled column j, pc[j] -= delta - d[j] and the row
// matched to it gains delta - d[j]: the reduced costs stay >= 0 and every matched edge,
// old and new, stays at 0.  Ties go to the lowest column index.  Empty if a cost is not
// finite (the callers check their inputs).
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
      if (jm < 0) return {};  // no finite reduced cost left
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

// The two smallest of four values: (third largest, smallest).
inline void two_smallest(float a, float b, float c, float e, float& s1, float& s2) {
  const float lo1 = std::min(a, b), hi1 = std::max(a, b);
  const float lo2 = std::min(c, e), hi2 = std::max(c, e);
  s2 = std::min(lo1, lo2);
  s1 = std::min(std::max(lo1, lo2), std::min(hi1, hi2));
}

// Pruning cost of four channels over the tile's rows: per row the two smallest values (the
// larger first, each as fp64) added to the row-ascending fp64 sum.
double group_cost(const float* I, int T, int K, const int32_t (&m)[4]) {
  double acc = 0.0;
  for (int r = 0; r < T; ++r) {
    const float* row = I + (size_t)r * K;
    float s1, s2;
    two_smallest(row[m[0]], row[m[1]], row[m[2]], row[m[3]], s1, s2);
    acc += (double)s1 + (double)s2;
  }
  return acc;
}

// Balanced K-means of S = G k points (rows of F, S x d, fp64) into G clusters of k members,
// seeded with cluster i = points i k .. i k + k - 1: per iteration the centroids (members
// summed in ascending order, divided by k) and the min-cost assignment of the points to the
// G k seats under the squared distance (coordinates ascending), until the partition repeats.
// Returns the clusters as ascending point lists.
std::vector<std::vector<int>> balanced_kmeans(const std::vector<double>& F, int S, int d, int k,
                                              int iters) {
  const int G = S / k;
  std::vector<std::vector<int>> cl(G);
  for (int i = 0; i < G; ++i)
    for (int j = 0; j < k; ++j) cl[i].push_back(i * k + j);
  std::vector<double> C((size_t)G * d), cost((size_t)S * S), acc(d);
  for (int it = 0; it < iters; ++it) {
    for (int c = 0; c < G; ++c) {
      std::fill(acc.begin(), acc.end(), 0.0);
      for (int p : cl[c])
        for (int x = 0; x < d; ++x) acc[x] = acc[x] + F[(size_t)p * d + x];
      for (int x = 0; x < d; ++x) C[(size_t)c * d + x] = acc[x] / (double)k;
    }
    for (int p = 0; p < S; ++p)
      for (int c = 0; c < G; ++c) {
        double dist = 0.0;
        for (int x = 0; x < d; ++x) {
          const double diff = F[(size_t)p * d + x] - C[(size_t)c * d + x];
          dist += diff * diff;
        }
        for (int j = 0; j < k; ++j) cost[(size_t)p * S + c * k + j] = dist;
      }
    const std::vector<int> seat = min_cost_assignment(cost, S);
    if ((int)seat.size() != S) break;
    std::vector<std::vector<int>> nw(G);
    for (int p = 0; p < S; ++p) nw[seat[p] / k].push_back(p);  // p ascending: lists sorted
    if (nw == cl) break;
    cl.swap(nw);
  }
  return cl;
}

// The n0 smallest column sums of the rows `rows` (in the given order) of I, summed in
// ascending order of (sum, channel): the cost of column-vector pruning of that tile.
double column_cost(const float* I, int K, const std::vector<int>& rows, int n0,
                   std::vector<double>& V, std::vector<int>& order) {
  std::fill(V.begin(), V.end(), 0.0);
  for (int r : rows) {
    const float* row = I + (size_t)r * K;
    for (int j = 0; j < K; ++j) V[j] = V[j] + (double)row[j];
  }
  std::iota(order.begin(), order.end(), 0);
  std::partial_sort(order.begin(), order.begin() + n0, order.end(), [&](int a, int b) {
    return V[a] < V[b] || (V[a] == V[b] && a < b);
  });
  double acc = 0.0;
  for (int i = 0; i < n0; ++i) acc += V[order[i]];
  return acc;
}

}  // namespace

double gyro_band_cost(const float* I, int T, int K, const int32_t* band, int n) {
  double acc = 0.0;
  for (int g = 0; g < n / 4; ++g) {
    const int32_t m[4] = {band[4 * g], band[4 * g + 1], band[4 * g + 2], band[4 * g + 3]};
    acc += group_cost(I, T, K, m);
  }
  return acc;
}

// One in-tile input-channel round (arguments checked by the caller): returns false if the
// assignment could not be formed (non-finite costs).
bool gyro_input_round(const float* I, int T, int K, int32_t* band, const int32_t* groups,
                      const int32_t* slots, int G, int k, int kmeans_iters, double* cost_out) {
  const int S = G * k;
  std::vector<int32_t> vec(S);
  std::vector<double> F((size_t)S * T);
  for (int i = 0; i < G; ++i)
    for (int j = 0; j < k; ++j) {
      const int p = i * k + j;
      vec[p] = band[4 * groups[i] + slots[p]];
      for (int r = 0; r < T; ++r) F[(size_t)p * T + r] = (double)I[(size_t)r * K + vec[p]];
    }
  const std::vector<std::vector<int>> cl = balanced_kmeans(F, S, T, k, kmeans_iters);
  // group i's members with its sampled slots (ascending) holding cluster c (ascending)
  auto members = [&](int i, const std::vector<int>& c, int32_t (&m)[4]) {
    for (int q = 0; q < 4; ++q) m[q] = band[4 * groups[i] + q];
    std::vector<int> ss(slots + (size_t)i * k, slots + (size_t)(i + 1) * k);
    std::sort(ss.begin(), ss.end());
    for (int j = 0; j < k; ++j) m[ss[j]] = vec[c[j]];
  };
  std::vector<double> cost((size_t)G * G);
  int32_t m[4];
  for (int c = 0; c < G; ++c)
    for (int i = 0; i < G; ++i) {
      members(i, cl[c], m);
      cost[(size_t)c * G + i] = group_cost(I, T, K, m);
    }
  const std::vector<int> to = min_cost_assignment(cost, G);  // cluster c -> group to[c]
  if ((int)to.size() != G) return false;
  std::vector<int> cl_of(G);
  for (int c = 0; c < G; ++c) cl_of[to[c]] = c;
  double before = 0.0, after = 0.0;
  for (int i = 0; i < G; ++i) {
    const int32_t o[4] = {band[4 * groups[i]], band[4 * groups[i] + 1], band[4 * groups[i] + 2],
                          band[4 * groups[i] + 3]};
    before += group_cost(I, T, K, o);
  }
  for (int i = 0; i < G; ++i) after += cost[(size_t)cl_of[i] * G + i];
  if (after <= before) {
    std::vector<int32_t> nb((size_t)G * 4);
    for (int i = 0; i < G; ++i) {
      members(i, cl[cl_of[i]], m);
      for (int q = 0; q < 4; ++q) nb[(size_t)i * 4 + q] = m[q];
    }
    for (int i = 0; i < G; ++i)
      for (int q = 0; q < 4; ++q) band[4 * groups[i] + q] = nb[(size_t)i * 4 + q];
  } else {
    after = before;
  }
  if (cost_out) {
    cost_out[0] = before;
    cost_out[1] = after;
  }
  return true;
}

// One output-channel round over a layer's tiles (arguments checked by the caller).
bool gyro_output_round(const float* I, int M, int K, int T, const int32_t* n0, int32_t* order,
                       const int32_t* tiles, const int32_t* rows, int G, int k, int kmeans_iters,
                       double* cost_out) {
  (void)M;
  const int S = G * k;
  std::vector<int32_t> ch(S);
  std::vector<double> F((size_t)S * K);
  for (int i = 0; i < G; ++i)
    for (int j = 0; j < k; ++j) {
      const int p = i * k + j;
      ch[p] = order[(size_t)tiles[i] * T + rows[p]];
      for (int x = 0; x < K; ++x) F[(size_t)p * K + x] = (double)I[(size_t)ch[p] * K + x];
    }
  const std::vector<std::vector<int>> cl = balanced_kmeans(F, S, K, k, kmeans_iters);
  auto tile_rows = [&](int i, const std::vector<int>* c, std::vector<int>& out) {
    out.assign(order + (size_t)tiles[i] * T, order + (size_t)(tiles[i] + 1) * T);
    if (!c) return;
    std::vector<int> rr(rows + (size_t)i * k, rows + (size_t)(i + 1) * k);
    std::sort(rr.begin(), rr.end());
    for (int j = 0; j < k; ++j) out[rr[j]] = ch[(*c)[j]];
  };
  std::vector<double> V(K), cost((size_t)G * G);
  std::vector<int> ord(K), tr;
  for (int c = 0; c < G; ++c)
    for (int i = 0; i < G; ++i) {
      tile_rows(i, &cl[c], tr);
      cost[(size_t)c * G + i] = column_cost(I, K, tr, n0[tiles[i]], V, ord);
    }
  const std::vector<int> to = min_cost_assignment(cost, G);
  if ((int)to.size() != G) return false;
  std::vector<int> cl_of(G);
  for (int c = 0; c < G; ++c) cl_of[to[c]] = c;
  double before = 0.0, after = 0.0;
  for (int i = 0; i < G; ++i) {
    tile_rows(i, nullptr, tr);
    before += column_cost(I, K, tr, n0[tiles[i]], V, ord);
  }
  for (int i = 0; i < G; ++i) after += cost[(size_t)cl_of[i] * G + i];
  if (after <= before) {
    std::vector<std::vector<int>> nt(G);
    for (int i = 0; i < G; ++i) tile_rows(i, &cl[cl_of[i]], nt[i]);
    for (int i = 0; i < G; ++i)
      for (int r = 0; r < T; ++r) order[(size_t)tiles[i] * T + r] = nt[i][r];
  } else {
    after = before;
  }
  if (cost_out) {
    cost_out[0] = before;
    cost_out[1] = after;
  }
  return true;
}

// ------------------------------------------------------------------ device: cost matrices
namespace {

__device__ __forceinline__ void two_smallest_d(float a, float b, float c, float e, float& s1,
                                               float& s2) {
  const float lo1 = fminf(a, b), hi1 = fmaxf(a, b);
  const float lo2 = fminf(c, e), hi2 = fmaxf(c, e);
  s2 = fminf(lo1, lo2);
  s1 = fminf(fmaxf(lo1, lo2), fminf(hi1, hi2));
}

// cost[t][c][i] for every tile t, cluster c and sampled group i: thread per (t, c, i), the
// tile's rows ascending.  Inputs as hinm_gyro_cost_matrix documents; every index was
// checked on the host except the band's channels, which are clamped (a bad one is reported).
__global__ void gyro_cost_kernel(const float* __restrict__ I, int K, int T, int nt,
                                 const int32_t* __restrict__ bands, int nb,
                                 const int32_t* __restrict__ groups,
                                 const int32_t* __restrict__ slots,
                                 const int32_t* __restrict__ clusters, int G, int k,
                                 double* __restrict__ cost, int* status) {
  const long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  const long long per = (long long)G * G;
  if (e >= per * nt) return;
  const int t = (int)(e / per);
  const int c = (int)((e - (long long)t * per) / G);
  const int i = (int)(e - (long long)t * per - (long long)c * G);
  const int32_t* band = bands + (size_t)t * nb;
  const int g = groups[(size_t)t * G + i];
  int m[4];
  for (int q = 0; q < 4; ++q) m[q] = band[4 * g + q];
  // the group's sampled slots in ascending order take cluster c's samples in order; sample
  // p = i' k + j is the vector in slot slots[t][i'][j] of group groups[t][i']
  int ss[4], sv[4];
  for (int j = 0; j < k; ++j) ss[j] = slots[((size_t)t * G + i) * k + j];
  for (int a = 1; a < k; ++a)  // insertion sort of at most 4 slots
    for (int b = a; b > 0 && ss[b - 1] > ss[b]; --b) {
      const int x = ss[b];
      ss[b] = ss[b - 1];
      ss[b - 1] = x;
    }
  for (int j = 0; j < k; ++j) {
    const int p = clusters[((size_t)t * G + c) * k + j];
    const int gi = p / k, sj = p - gi * k;
    sv[j] = band[4 * groups[(size_t)t * G + gi] + slots[((size_t)t * G + gi) * k + sj]];
  }
  for (int j = 0; j < k; ++j) m[ss[j]] = sv[j];
  for (int q = 0; q < 4; ++q)
    if ((unsigned)m[q] >= (unsigned)K) {
      if (status) atomicCAS(status, 0, (int)HINM_ERR_INVALID_ARG);
      m[q] = 0;
    }
  const float* rows = I + (size_t)t * T * K;
  double acc = 0.0;
  for (int r = 0; r < T; ++r) {
    const float* row = rows + (size_t)r * K;
    float s1, s2;
    two_smallest_d(__ldg(row + m[0]), __ldg(row + m[1]), __ldg(row + m[2]), __ldg(row + m[3]),
                   s1, s2);
    acc = __dadd_rn(acc, __dadd_rn((double)s1, (double)s2));
  }
  cost[e] = acc;
}

}  // namespace

cudaError_t launch_gyro_cost(const float* I, int K, int T, int nt, const int32_t* bands, int nb,
                             const int32_t* groups, const int32_t* slots,
                             const int32_t* clusters, int G, int k, double* cost, int* status,
                             cudaStream_t s) {
  const long long n = (long long)nt * G * G;
  if (n == 0) return cudaSuccess;
  const long long blocks = (n + 255) / 256;
  gyro_cost_kernel<<<(unsigned)blocks, 256, 0, s>>>(I, K, T, nt, bands, nb, groups, slots,
                                                     clusters, G, k, cost, status);
  return cudaGetLastError();
}

}  // namespace hinm
