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
__global__ void vector_score_kernel(const float* __restrict__ I, int K, int T,
                                    double* __restrict__ Vc) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (c >= K) return;
  const float* p = I + (size_t)t * T * K + c;
  double acc = 0.0;
  for (int i = 0; i < T; ++i) acc = __dadd_rn(acc, (double)__ldg(p + (size_t)i * K));
  Vc[(size_t)t * K + c] = acc;
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
                               double* V, int32_t* rank, cudaStream_t s) {
  const int nt = M / T;
  dim3 g1((K + 255) / 256, nt);
  vector_score_kernel<<<g1, 256, 0, s>>>(I, K, T, V);
  cudaError_t e = cudaGetLastError();
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

// ------------------------------------------------------------------ exact sums
// Exact sum of non-negative finite fp32 values: every value is m * 2^(b - 150) with an
// integer mantissa m < 2^24 and b = max(biased exponent, 1); bucket[b] accumulates m in
// 64-bit integers (at most 2^24 values per sum keeps every bucket below 2^48).
// Called by all 32 lanes of a warp together (v = 0 contributes nothing).
__device__ __forceinline__ void bucket_add(unsigned long long* buckets, float v) {
  const uint32_t u = __float_as_uint(v);
  const uint32_t e = (u >> 23) & 0xFF;
  const uint32_t m = (u & 0x7FFFFF) | (e ? 0x800000u : 0u);
  const uint32_t b = e ? e : 1u;
  // lanes with the same bucket are summed first (mantissas < 2^24, 32 lanes < 2^29)
  const unsigned peers = __match_any_sync(0xffffffffu, b);
  const unsigned sum = __reduce_add_sync(peers, m);
  if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31) && sum != 0u)
    atomicAdd(buckets + b, (unsigned long long)sum);
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

// Z = sum_b bucket[b] * 2^(b-1) (bucket[b] < 2^48, so Z < 2^303), value = Z * 2^-149,
// rounded to the nearest fp64, ties to even.
__device__ double buckets_to_double(const unsigned long long* bucket) {
  unsigned long long z[6] = {0, 0, 0, 0, 0, 0};
  for (int b = 1; b < 256; ++b)
    if (bucket[b]) big_add_shifted(z, bucket[b], b - 1);
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
// Shared memory: 16 warps x 256 buckets (32 KB) + group members (K int16).
__global__ void __launch_bounds__(512) candidate_kernel(const float* __restrict__ I,
                                                        const int32_t* __restrict__ perm,
                                                        const int32_t* __restrict__ rank, int K,
                                                        int T, CandidateList cl,
                                                        double* __restrict__ R, int ncand) {
  extern __shared__ __align__(16) unsigned char smem[];
  unsigned long long* buckets = reinterpret_cast<unsigned long long*>(smem);  // [16][256]
  unsigned short* member = reinterpret_cast<unsigned short*>(buckets + 16 * 256);  // [K]
  __shared__ int warp_tot[16];

  const int m = blockIdx.x, t = blockIdx.y;
  const Candidate cand = cl.c[m];
  const int n4 = cand.n4, n24 = cand.n24;
  const int32_t* rk = rank + (size_t)t * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int i = threadIdx.x; i < 16 * 256; i += blockDim.x) buckets[i] = 0;

  // 2:4 members in ascending working position: block-wide prefix count over j.
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per;
  int cnt = 0;
  for (int j = j0; j < min(K, j0 + per); ++j) {
    const int r = __ldg(rk + j);
    cnt += (r >= n4 && r < n4 + n24);
  }
  // exclusive scan of cnt over the block
  int incl = cnt;
  for (int o = 1; o < 32; o <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += warp_tot[w];
  int pos = wbase + incl - cnt;
  for (int j = j0; j < min(K, j0 + per); ++j) {
    const int r = __ldg(rk + j);
    if (r >= n4 && r < n4 + n24) member[pos++] = (unsigned short)j;
  }
  __syncthreads();

  unsigned long long* my = buckets + warp * 256;
  const float* It = I + (size_t)t * T * K;
  // dense vectors: every element kept.  Loops advance whole warps together so every
  // lane takes part in the warp-aggregated bucket adds.
  const int total_d = T * K;
  for (int base = threadIdx.x - lane; base < total_d; base += blockDim.x) {
    const int q = base + lane;
    float v = 0.0f;
    if (q < total_d) {
      const int i = q / K, j = q - (q / K) * K;
      if (__ldg(rk + j) < n4) {
        const int c = ptx::perm_at(perm, j, K);
        v = __ldg(It + (size_t)i * K + c);
      }
    }
    bucket_add(my, v);
  }
  // 2:4 groups: top-2 of 4 per row (lower position wins ties)
  const int ng = n24 / 4;
  const int total_s = T * ng;
  for (int base = threadIdx.x - lane; base < total_s; base += blockDim.x) {
    const int q = base + lane;
    float v[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    bool keep[4] = {false, false, false, false};
    if (q < total_s) {
      const int i = q / ng, g = q - (q / ng) * ng;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int j = member[4 * g + k];
        j = j < K ? j : 0;
        const int c = ptx::perm_at(perm, j, K);
        v[k] = __ldg(It + (size_t)i * K + c);
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        int beats = 0;
#pragma unroll
        for (int l = 0; l < 4; ++l) beats += (v[l] > v[k]) || (v[l] == v[k] && l < k);
        keep[k] = beats < 2;
      }
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) bucket_add(my, keep[k] ? v[k] : 0.0f);
  }
  __syncthreads();
  // fold the 16 warp copies into copy 0
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    unsigned long long s = 0;
    for (int w = 0; w < 16; ++w) s += buckets[w * 256 + b];
    buckets[b] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) R[(size_t)t * ncand + m] = buckets_to_double(buckets);
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
  c.take<double>((size_t)nt * K);      // V
  c.take<int32_t>((size_t)nt * K);     // rank (when the caller passes none)
  c.take<double>((size_t)nt * ncand);  // R
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_boundary_search(const float* I, const int32_t* perm, int M, int K, int T,
                                   double t_s, double alpha, const Candidate* cands, int ncand,
                                   int32_t* counts_out, double* vs_out, int32_t* rank_out,
                                   void* ws, int* status, cudaStream_t s) {
  (void)status;
  const int nt = M / T;
  Carve c{static_cast<char*>(ws), 0};
  double* V = c.take<double>((size_t)nt * K);
  int32_t* rank_ws = c.take<int32_t>((size_t)nt * K);
  double* R = c.take<double>((size_t)nt * ncand);
  int32_t* rank = rank_out ? rank_out : rank_ws;
  cudaError_t e = launch_vector_rank(I, perm, M, K, T, V, rank, s);
  if (e != cudaSuccess) return e;
  CandidateList cl;
  for (int i = 0; i < kMaxCandidates; ++i) cl.c[i] = i < ncand ? cands[i] : Candidate{0, 0, 0};
  const size_t smem = 16 * 256 * sizeof(unsigned long long) + (size_t)K * sizeof(unsigned short);
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(candidate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(16 * 256 * sizeof(unsigned long long) + kMaxK * 2));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 g(ncand, nt);
  candidate_kernel<<<g, 512, smem, s>>>(I, perm, rank, K, T, cl, R, ncand);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  select_kernel<<<(nt + 127) / 128, 128, 0, s>>>(R, nt, ncand, cl, t_s, alpha, counts_out, vs_out);
  return cudaGetLastError();
}

}  // namespace hinm
