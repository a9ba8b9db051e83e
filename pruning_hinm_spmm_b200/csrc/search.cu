// a2 + a3. Vector scores, vector ranking and the boundary search
// (FlexHiNM-GP notes, 整体框架: every tile runs the search; 关键设计 1: the scan of v_s
// from t_s downward by alpha, stopping at the first drop of the retained importance
// R_total = R_dense + R_24; 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned).
//
// Kernels:
//   vector_score_kernel   V[t, c] = sum of I over the tile's rows, ascending, fp64
//   rank_sort_kernel      one CTA per tile: bitonic sort of (V desc, j asc) in shared
//                         memory; writes rank[t][j]
//   candidate_kernel      one CTA per (candidate m, tile): regions, 2:4 groups, top-2,
//                         and the EXACT sum of the kept importance (integer exponent
//                         buckets), rounded once to fp64 -> R[t][m]
//   select_kernel         first m with R(m+1) < R(m), else the last candidate
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "ptx.cuh"

namespace hinm {

// ------------------------------------------------------------------ vector scores
// Exact sums.  Every non-negative finite fp32 value is m * 2^(p - 149) with an integer
// mantissa m < 2^24 and p = max(biased exponent, 1) - 1 in [0, 253].  Within a tile the
// sums are kept as 128-bit integers in units of 2^(lsb - 149), lsb = max(P - 83, 0),
// P = the tile's largest p: a value then needs at most 107 bits and 2^21 of them (128
// rows x 16384 columns) still fit.  A value more than 2^83 below the tile's largest
// (p < lsb) would lose bits there, so it goes to 64-bit exponent buckets instead.
constexpr int kHeadroomShift = 83;

__device__ __forceinline__ void split_f32(float v, uint32_t& m, int& p) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t e = (u >> 23) & 0xFF;
  m = (u & 0x7FFFFF) | (e ? 0x800000u : 0u);
  p = (e ? (int)e : 1) - 1;
}

struct U128 {
  unsigned long long lo, hi;
};

// a += m * 2^sh, 0 <= sh <= 104
__device__ __forceinline__ void add_shifted(U128& a, uint32_t m, int sh) {
  unsigned long long lo, hi;
  if (sh < 64) {
    lo = (unsigned long long)m << sh;
    hi = sh > 40 ? ((unsigned long long)m >> (64 - sh)) : 0ull;
  } else {
    lo = 0ull;
    hi = (unsigned long long)m << (sh - 64);
  }
  a.lo += lo;
  a.hi += hi + (a.lo < lo ? 1ull : 0ull);
}

__device__ __forceinline__ void add128(U128& a, const U128& b) {
  a.lo += b.lo;
  a.hi += b.hi + (a.lo < b.lo ? 1ull : 0ull);
}

// acc += v (a non-negative finite fp32) exactly: at the tile's scale when v >= 2^lsb-ish,
// else into the exponent buckets.
__device__ __forceinline__ void acc_value(U128& acc, float v, int lsb, unsigned long long* bucket) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t e = u >> 23;
  const uint32_t m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  const int sh = (int)(e ? e : 1u) - 1 - lsb;
  if (sh >= 0) {
    const unsigned long long x = m;
    const unsigned long long lo = sh < 64 ? (x << sh) : 0ull;
    const unsigned long long hi =
        sh >= 64 ? (x << (sh - 64)) : (sh > 40 ? (x >> (64 - sh)) : 0ull);
    acc.lo += lo;
    acc.hi += hi + (acc.lo < lo ? 1ull : 0ull);
  } else if (m) {
    atomicAdd(bucket + (sh + lsb), (unsigned long long)m);
  }
}

__device__ __forceinline__ int tile_lsb(int pmax) {
  return pmax > kHeadroomShift ? pmax - kHeadroomShift : 0;
}

// Pass 1, thread per (tile, channel): V[t, c] = sum over the tile's rows, ascending, of
// I (fp64), and the tile's largest exponent P.
__global__ void vector_score_kernel(const float* __restrict__ I, int K, int T,
                                    double* __restrict__ Vc, int* __restrict__ tile_pmax) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  int pm = 0;
  if (c < K) {
    const float* p = I + (size_t)t * T * K + c;
    double acc = 0.0;
    for (int i = 0; i < T; ++i) {
      const float v = __ldg(p + (size_t)i * K);
      acc = __dadd_rn(acc, (double)v);
      uint32_t m;
      int e;
      split_f32(v, m, e);
      if (m) pm = max(pm, e);
    }
    Vc[(size_t)t * K + c] = acc;
  }
  for (int o = 16; o > 0; o >>= 1) pm = max(pm, __shfl_xor_sync(0xffffffffu, pm, o));
  if ((threadIdx.x & 31) == 0) atomicMax(tile_pmax + t, pm);
}

// Pass 2, thread per (tile, channel): the column's exact sum at the tile's scale, and a
// flag when some of its values fell below that scale (summed exactly elsewhere).
__global__ void column_sum_kernel(const float* __restrict__ I, int K, int T,
                                  const int* __restrict__ tile_pmax, U128* __restrict__ colsum,
                                  unsigned char* __restrict__ coltiny) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (c >= K) return;
  const int lsb = tile_lsb(tile_pmax[t]);
  const float* p = I + (size_t)t * T * K + c;
  U128 acc{0ull, 0ull};
  unsigned char tiny = 0;
  for (int i = 0; i < T; ++i) {
    uint32_t m;
    int e;
    split_f32(__ldg(p + (size_t)i * K), m, e);
    if (!m) continue;
    if (e >= lsb) add_shifted(acc, m, e - lsb);
    else tiny = 1;
  }
  colsum[(size_t)t * K + c] = acc;
  coltiny[(size_t)t * K + c] = tiny;
}

// ------------------------------------------------------------------ rank sort
// Sort key: (~bits(V), j) ascending == (V descending, j ascending); V >= 0 so its bit
// pattern orders like its value.  Padding entries (j = 0xFFFF) sort last.
__global__ void __launch_bounds__(1024) rank_sort_kernel(const double* __restrict__ Vc,
                                                         const int32_t* __restrict__ perm, int K,
                                                         int Kp, int32_t* __restrict__ rank) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* key = reinterpret_cast<unsigned long long*>(smem);
  unsigned short* idx = reinterpret_cast<unsigned short*>(key + Kp);
  const int t = blockIdx.x;
  const double* V = Vc + (size_t)t * K;
  for (int j = threadIdx.x; j < Kp; j += blockDim.x) {
    if (j < K) {
      const int c = ptx::perm_at(perm, j, K);
      key[j] = ~static_cast<unsigned long long>(__double_as_longlong(__ldg(V + c)));
      idx[j] = (unsigned short)j;
    } else {
      key[j] = ~0ull;
      idx[j] = 0xFFFF;
    }
  }
  __syncthreads();
  for (int k = 2; k <= Kp; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < Kp; i += blockDim.x) {
        const int l = i ^ jj;
        if (l > i) {
          const unsigned long long ki = key[i], kl = key[l];
          const unsigned short ii = idx[i], il = idx[l];
          const bool i_gt = (ki > kl) || (ki == kl && ii > il);
          const bool ascending = (i & k) == 0;
          if (i_gt == ascending) {
            key[i] = kl;
            key[l] = ki;
            idx[i] = il;
            idx[l] = ii;
          }
        }
      }
      __syncthreads();
    }
  }
  int32_t* r = rank + (size_t)t * K;
  for (int p = threadIdx.x; p < K; p += blockDim.x) r[idx[p]] = p;
}

cudaError_t launch_vector_rank(const float* I, const int32_t* perm, int M, int K, int T,
                               double* V, int32_t* rank, int* tile_pmax, cudaStream_t s) {
  const int nt = M / T;
  cudaError_t e = cudaMemsetAsync(tile_pmax, 0, (size_t)nt * sizeof(int), s);
  if (e != cudaSuccess) return e;
  dim3 g1((K + 255) / 256, nt);
  vector_score_kernel<<<g1, 256, 0, s>>>(I, K, T, V, tile_pmax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int Kp = 1;
  while (Kp < K) Kp <<= 1;
  const size_t smem = (size_t)Kp * (sizeof(unsigned long long) + sizeof(unsigned short));
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(rank_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)((size_t)kMaxK * 10));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  rank_sort_kernel<<<nt, 1024, smem, s>>>(V, perm, K, Kp, rank);
  return cudaGetLastError();
}

// Adds v * 2^sh (v < 2^64) into the little-endian multi-limb integer z[0..5].
__device__ __forceinline__ void big_add_shifted(unsigned long long* z, unsigned long long v, int sh) {
  const int limb = sh >> 6, off = sh & 63;
  const unsigned long long lo = v << off;
  const unsigned long long hi = off ? (v >> (64 - off)) : 0ull;
  unsigned long long s0 = z[limb] + lo;
  unsigned long long carry = s0 < lo;
  z[limb] = s0;
  unsigned long long s1 = z[limb + 1] + hi;
  unsigned long long c1 = s1 < hi;
  s1 += carry;
  c1 |= (s1 < carry);
  z[limb + 1] = s1;
  carry = c1;
  for (int l = limb + 2; l < 6 && carry; ++l) {
    z[l] += carry;
    carry = (z[l] == 0);
  }
}

// value = Z * 2^-149 with Z = main * 2^lsb + sum_p bucket[p] * 2^p (a 384-bit integer),
// rounded to the nearest fp64, ties to even.
__device__ double exact_to_double(U128 main, int lsb, const unsigned long long* bucket) {
  unsigned long long z[6] = {0, 0, 0, 0, 0, 0};
  if (main.lo) big_add_shifted(z, main.lo, lsb);
  if (main.hi) big_add_shifted(z, main.hi, lsb + 64);
  for (int p = 0; p < 254; ++p)
    if (bucket[p]) big_add_shifted(z, bucket[p], p);
  int top = -1;
  for (int l = 5; l >= 0 && top < 0; --l)
    if (z[l]) top = l * 64 + 63 - __clzll((long long)z[l]);
  if (top < 0) return 0.0;
  if (top < 53) return ldexp((double)z[0], -149);  // exact
  const int lo = top - 52;  // keep bits [lo, lo + 53)
  const int limb = lo >> 6, off = lo & 63;
  unsigned long long mant = z[limb] >> off;
  if (off && limb + 1 < 6) mant |= z[limb + 1] << (64 - off);
  mant &= (1ull << 53) - 1;
  const int hb = lo - 1;  // rounding bit
  const bool half = (z[hb >> 6] >> (hb & 63)) & 1ull;
  bool sticky = false;  // any bit in [0, hb)
  for (int l = 0; l < (hb >> 6); ++l) sticky |= (z[l] != 0);
  if (hb & 63) sticky |= (z[hb >> 6] & ((1ull << (hb & 63)) - 1)) != 0;
  int ex = lo - 149;
  if (half && (sticky || (mant & 1ull))) {
    mant += 1;
    if (mant == (1ull << 53)) {
      mant >>= 1;
      ex += 1;
    }
  }
  return ldexp((double)mant, ex);
}

// ------------------------------------------------------------------ candidates
struct CandidateList {
  Candidate c[kMaxCandidates];
};

// blockIdx.x = candidate m, blockIdx.y = tile.  512 threads.
// R(m) = sum of the column sums of the dense vectors + sum over the 2:4 groups of the
// top-2 of every row, all exact (128-bit per thread at the tile's scale, exponent buckets
// for values below it), rounded once to fp64.
__global__ void __launch_bounds__(512) candidate_kernel(
    const float* __restrict__ I, const int32_t* __restrict__ perm, const int32_t* __restrict__ rank,
    const int* __restrict__ tile_pmax, const U128* __restrict__ colsum,
    const unsigned char* __restrict__ coltiny, int K, int T, CandidateList cl,
    double* __restrict__ R, int ncand) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* bucket = reinterpret_cast<unsigned long long*>(smem);  // [256]
  unsigned short* member = reinterpret_cast<unsigned short*>(bucket + 256);   // [K]
  __shared__ int warp_tot[16];
  __shared__ U128 warp_acc[16];

  const int m = blockIdx.x, t = blockIdx.y;
  const Candidate cand = cl.c[m];
  const int n4 = cand.n4, n24 = cand.n24;
  const int32_t* rk = rank + (size_t)t * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lsb = tile_lsb(tile_pmax[t]);
  const float* It = I + (size_t)t * T * K;

  for (int i = threadIdx.x; i < 256; i += blockDim.x) bucket[i] = 0;
  U128 acc{0ull, 0ull};

  // pass over the working positions: dense column sums, and the 2:4 members in
  // ascending working position (block-wide prefix count)
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per, j1 = min(K, j0 + per);
  int cnt = 0;
  for (int j = j0; j < j1; ++j) {
    const int r = __ldg(rk + j);
    cnt += (r >= n4 && r < n4 + n24);
  }
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();  // also publishes the cleared buckets
  int pos = incl - cnt;
  for (int w = 0; w < warp; ++w) pos += warp_tot[w];
  for (int j = j0; j < j1; ++j) {
    const int r = __ldg(rk + j);
    if (r < n4) {
      const int c = ptx::perm_at(perm, j, K);
      add128(acc, colsum[(size_t)t * K + c]);
      if (coltiny[(size_t)t * K + c]) {  // values below the tile's scale: exact buckets
        for (int i = 0; i < T; ++i) {
          uint32_t mm;
          int e;
          split_f32(__ldg(It + (size_t)i * K + c), mm, e);
          if (mm && e < lsb) atomicAdd(bucket + e, (unsigned long long)mm);
        }
      }
    } else if (r < n4 + n24) {
      member[pos++] = (unsigned short)j;
    }
  }
  __syncthreads();

  // 2:4 groups: the two largest of the four importances of every row are kept (which of
  // two equal values is kept does not change the sum).  One thread per group walks all
  // rows, so the group's channels are looked up once.
  const int ng = n24 / 4;
  for (int g = threadIdx.x; g < ng; g += blockDim.x) {
    int c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int j = member[4 * g + k];
      j = j < K ? j : 0;
      c[k] = ptx::perm_at(perm, j, K);
    }
    const float* row = It;
    for (int i = 0; i < T; ++i, row += K) {
      const float v0 = __ldg(row + c[0]), v1 = __ldg(row + c[1]);
      const float v2 = __ldg(row + c[2]), v3 = __ldg(row + c[3]);
      const float a = fmaxf(v0, v1), b = fminf(v0, v1);
      const float cc = fmaxf(v2, v3), d = fminf(v2, v3);
      acc_value(acc, fmaxf(a, cc), lsb, bucket);
      acc_value(acc, fmaxf(fminf(a, cc), fmaxf(b, d)), lsb, bucket);
    }
  }

  // block reduction of the 128-bit partial sums (integer adds: order-independent)
  for (int o = 16; o > 0; o >>= 1) {
    U128 other;
    other.lo = __shfl_xor_sync(0xffffffffu, acc.lo, o);
    other.hi = __shfl_xor_sync(0xffffffffu, acc.hi, o);
    add128(acc, other);
  }
  if (lane == 0) warp_acc[warp] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    U128 tot{0ull, 0ull};
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) add128(tot, warp_acc[w]);
    R[(size_t)t * ncand + m] = exact_to_double(tot, lsb, bucket);
  }
}

__global__ void select_kernel(const double* __restrict__ R, int nt, int ncand, CandidateList cl,
                              double t_s, double alpha, int32_t* __restrict__ counts,
                              double* __restrict__ vs) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= nt) return;
  const double* r = R + (size_t)t * ncand;
  int ms = ncand - 1;
  for (int m = 0; m + 1 < ncand; ++m) {
    if (r[m + 1] < r[m]) {
      ms = m;
      break;
    }
  }
  counts[3 * t + 0] = cl.c[ms].n0;
  counts[3 * t + 1] = cl.c[ms].n24;
  counts[3 * t + 2] = cl.c[ms].n4;
  vs[t] = __dsub_rn(t_s, __dmul_rn((double)ms, alpha));
}

size_t search_workspace_bytes(int M, int K, int T, int ncand) {
  const int nt = M / T;
  Carve c{nullptr, 0};
  c.take<double>((size_t)nt * K);         // V
  c.take<int32_t>((size_t)nt * K);        // rank (when the caller passes none)
  c.take<double>((size_t)nt * ncand);     // R
  c.take<int>((size_t)nt);                // tile max exponent
  c.take<U128>((size_t)nt * K);           // exact column sums
  c.take<unsigned char>((size_t)nt * K);  // column has values below the tile scale
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_boundary_search(const float* I, const int32_t* perm, int M, int K, int T,
                                   double t_s, double alpha, const Candidate* cands, int ncand,
                                   int32_t* counts_out, double* vs_out, int32_t* rank_out,
                                   double* retained_out, void* ws, int* status, cudaStream_t s) {
  (void)status;
  const int nt = M / T;
  Carve c{static_cast<char*>(ws), 0};
  double* V = c.take<double>((size_t)nt * K);
  int32_t* rank_ws = c.take<int32_t>((size_t)nt * K);
  double* R_ws = c.take<double>((size_t)nt * ncand);
  double* R = retained_out ? retained_out : R_ws;
  int* pmax = c.take<int>((size_t)nt);
  U128* colsum = c.take<U128>((size_t)nt * K);
  unsigned char* coltiny = c.take<unsigned char>((size_t)nt * K);
  int32_t* rank = rank_out ? rank_out : rank_ws;
  cudaError_t e = launch_vector_rank(I, perm, M, K, T, V, rank, pmax, s);
  if (e != cudaSuccess) return e;
  dim3 gc((K + 255) / 256, nt);
  column_sum_kernel<<<gc, 256, 0, s>>>(I, K, T, pmax, colsum, coltiny);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CandidateList cl;
  for (int i = 0; i < kMaxCandidates; ++i) cl.c[i] = i < ncand ? cands[i] : Candidate{0, 0, 0};
  const size_t smem = 256 * sizeof(unsigned long long) + (size_t)K * sizeof(unsigned short);
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(candidate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(256 * sizeof(unsigned long long) + kMaxK * 2));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 g(ncand, nt);
  candidate_kernel<<<g, 512, smem, s>>>(I, perm, rank, pmax, colsum, coltiny, K, T, cl, R, ncand);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_kernel<<<(nt + 127) / 128, 128, 0, s>>>(R, nt, ncand, cl, t_s, alpha, counts_out, vs_out);
  return cudaGetLastError();
}

}  // namespace hinm
