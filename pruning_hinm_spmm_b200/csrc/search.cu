// a2 + a3. Vector scores, vector ranking and the boundary search
// (FlexHiNM-GP notes, 整体框架: every tile runs the search; 关键设计 1: the scan of v_s
// from t_s downward by alpha, stopping at the first drop of the retained importance
// R_total = R_dense + R_24; 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned).
//
// Kernels:
//   vector_score_kernel   V[t, c] = sum of I over the tile's rows, ascending, fp64, and
//                         each tile's largest exponent
//   chunk_sort_kernel,    rank[t][j] of (V desc, j asc): bitonic sort of 1024-position
//   merge_rank_kernel     chunks, then a binary-search count over the sorted chunks
//   column_sum_kernel     exact column sums (128-bit integers at the tile's scale)
//   candidate_lists_kernel  one CTA per (candidate m, tile): the 2:4 band's channels in
//                         ascending working position and the exact sum of the dense
//                         vectors' column sums
//   band_sum_kernel       one CTA per (tile, chunk of rows): the rows are staged in shared
//                         memory once and every candidate's groups are evaluated from there
//                         (top-2 of 4 per row, exact 128-bit partial sums)
//   finalize_kernel       per tile: R(m) = exact total rounded once to fp64; the first m
//                         with R(m+1) < R(m), else the last candidate
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

// acc += t1 + t2 (t1 >= t2 >= 0, fp32) exactly.  When their fp64 sum is exact (Fast2Sum
// error 0) and at or above the tile's scale it is added once (a 53-bit mantissa shifted by
// at most 56 bits); otherwise each value goes through acc_value.
__device__ __forceinline__ void acc_pair(U128& acc, float t1, float t2, int lsb,
                                         unsigned long long* bucket) {
  const double a = t1, b = t2;
  const double s = __dadd_rn(a, b);
  const double err = __dsub_rn(b, __dsub_rn(s, a));
  if (err == 0.0 && s != 0.0) {
    const unsigned long long bits = (unsigned long long)__double_as_longlong(s);
    const int sh = (int)(bits >> 52) - 926 - lsb;  // s = m53 * 2^sh in units of 2^(lsb-149)
    if (sh >= 0) {
      const unsigned long long m = (bits & 0xFFFFFFFFFFFFFull) | (1ull << 52);
      const unsigned long long lo = m << sh;
      const unsigned long long hi = sh ? (m >> (64 - sh)) : 0ull;
      acc.lo += lo;
      acc.hi += hi + (acc.lo < lo ? 1ull : 0ull);
      return;
    }
  }
  acc_value(acc, t1, lsb, bucket);
  acc_value(acc, t2, lsb, bucket);
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
    constexpr int kBatch = 16;  // loads in flight per thread (T is a multiple of 16)
    for (int i0 = 0; i0 < T; i0 += kBatch) {
      float v[kBatch];
#pragma unroll
      for (int k = 0; k < kBatch; ++k) v[k] = __ldg(p + (size_t)(i0 + k) * K);
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {  // rows ascending
        acc = __dadd_rn(acc, (double)v[k]);
        uint32_t m;
        int e;
        split_f32(v[k], m, e);
        if (m) pm = max(pm, e);
      }
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
  constexpr int kBatch = 16;
  for (int i0 = 0; i0 < T; i0 += kBatch) {
    float v[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) v[k] = __ldg(p + (size_t)(i0 + k) * K);
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      uint32_t m;
      int e;
      split_f32(v[k], m, e);
      if (!m) continue;
      if (e >= lsb) add_shifted(acc, m, e - lsb);
      else tiny = 1;
    }
  }
  colsum[(size_t)t * K + c] = acc;
  coltiny[(size_t)t * K + c] = tiny;
}

// ------------------------------------------------------------------ rank sort
// Order key of working position j: (~bits(V), j) ascending == (V descending, j ascending);
// V >= 0, so its bit pattern orders like its value.  Every (key, j) pair is distinct.
// Phase 1 sorts chunks of 1024 positions in shared memory (bitonic); phase 2 gives every
// position its rank = sum over chunks of the number of smaller pairs (binary search).
constexpr int kRankChunk = 1024;

__device__ __forceinline__ bool pair_less(unsigned long long ka, unsigned ia,
                                          unsigned long long kb, unsigned ib) {
  return ka < kb || (ka == kb && ia < ib);
}

__global__ void __launch_bounds__(512) chunk_sort_kernel(const double* __restrict__ Vc,
                                                         const int32_t* __restrict__ perm, int K,
                                                         int Kp, unsigned long long* __restrict__ skey,
                                                         unsigned short* __restrict__ sidx) {
  __shared__ unsigned long long key[kRankChunk];
  __shared__ unsigned short idx[kRankChunk];
  const int t = blockIdx.y, base = blockIdx.x * kRankChunk;
  const double* V = Vc + (size_t)t * K;
  for (int i = threadIdx.x; i < kRankChunk; i += blockDim.x) {
    const int j = base + i;
    if (j < K) {
      key[i] = ~static_cast<unsigned long long>(__double_as_longlong(__ldg(V + ptx::perm_at(perm, j, K))));
      idx[i] = (unsigned short)j;
    } else {
      key[i] = ~0ull;
      idx[i] = 0xFFFF;
    }
  }
  __syncthreads();
  for (int k = 2; k <= kRankChunk; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      for (int i = threadIdx.x; i < kRankChunk; i += blockDim.x) {
        const int l = i ^ jj;
        if (l > i) {
          const unsigned long long ki = key[i], kl = key[l];
          const unsigned short ii = idx[i], il = idx[l];
          const bool i_gt = pair_less(kl, il, ki, ii);
          if (i_gt == ((i & k) == 0)) {
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
  for (int i = threadIdx.x; i < kRankChunk; i += blockDim.x) {
    skey[(size_t)t * Kp + base + i] = key[i];
    sidx[(size_t)t * Kp + base + i] = idx[i];
  }
}

__global__ void merge_rank_kernel(const double* __restrict__ Vc, const int32_t* __restrict__ perm,
                                  const unsigned long long* __restrict__ skey,
                                  const unsigned short* __restrict__ sidx, int K, int Kp,
                                  int32_t* __restrict__ rank) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  if (j >= K) return;
  const unsigned long long kj =
      ~static_cast<unsigned long long>(__double_as_longlong(__ldg(Vc + (size_t)t * K + ptx::perm_at(perm, j, K))));
  const unsigned ij = (unsigned)j;
  int r = 0;
  for (int base = 0; base < Kp; base += kRankChunk) {
    const unsigned long long* ck = skey + (size_t)t * Kp + base;
    const unsigned short* ci = sidx + (size_t)t * Kp + base;
    int lo = 0, hi = kRankChunk;  // count of pairs < (kj, ij) in this sorted chunk
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pair_less(__ldg(ck + mid), __ldg(ci + mid), kj, ij)) lo = mid + 1;
      else hi = mid;
    }
    r += lo;
  }
  rank[(size_t)t * K + j] = r;
}

size_t rank_scratch_bytes(int M, int K, int T) {
  const int nt = M / T;
  const size_t Kp = (size_t)((K + kRankChunk - 1) / kRankChunk) * kRankChunk;
  Carve c{nullptr, 0};
  c.take<unsigned long long>((size_t)nt * Kp);
  c.take<unsigned short>((size_t)nt * Kp);
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_vector_rank(const float* I, const int32_t* perm, int M, int K, int T,
                               double* V, int32_t* rank, int* tile_pmax, void* scratch,
                               cudaStream_t s) {
  const int nt = M / T;
  cudaError_t e = cudaMemsetAsync(tile_pmax, 0, (size_t)nt * sizeof(int), s);
  if (e != cudaSuccess) return e;
  dim3 g1((K + 255) / 256, nt);
  vector_score_kernel<<<g1, 256, 0, s>>>(I, K, T, V, tile_pmax);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int nchunk = (K + kRankChunk - 1) / kRankChunk;
  const int Kp = nchunk * kRankChunk;
  Carve c{static_cast<char*>(scratch), 0};
  unsigned long long* skey = c.take<unsigned long long>((size_t)nt * Kp);
  unsigned short* sidx = c.take<unsigned short>((size_t)nt * Kp);
  chunk_sort_kernel<<<dim3(nchunk, nt), 512, 0, s>>>(V, perm, K, Kp, skey, sidx);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  merge_rank_kernel<<<dim3((K + 255) / 256, nt), 256, 0, s>>>(V, perm, skey, sidx, K, Kp, rank);
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

// Per (candidate m, tile), 512 threads: the channels of the 2:4 band in ascending working
// position (block-wide prefix count) -> band[t][m][q], and the exact sum of the dense
// vectors' column sums -> rdense[t][m] (values below the tile's scale go to the buckets).
__global__ void __launch_bounds__(512) candidate_lists_kernel(
    const float* __restrict__ I, const int32_t* __restrict__ perm, const int32_t* __restrict__ rank,
    const int* __restrict__ tile_pmax, const U128* __restrict__ colsum,
    const unsigned char* __restrict__ coltiny, int K, int T, CandidateList cl, int ncand,
    unsigned short* __restrict__ band, U128* __restrict__ rdense,
    unsigned long long* __restrict__ bucket, int* __restrict__ bucket_used) {
  __shared__ int warp_tot[16];
  __shared__ U128 warp_acc[16];
  const int m = blockIdx.x, t = blockIdx.y;
  const Candidate cand = cl.c[m];
  const int n4 = cand.n4, n24 = cand.n24;
  const int32_t* rk = rank + (size_t)t * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lsb = tile_lsb(tile_pmax[t]);
  const float* It = I + (size_t)t * T * K;
  unsigned long long* bkt = bucket + ((size_t)t * ncand + m) * 256;
  unsigned short* out = band + ((size_t)t * ncand + m) * K;
  U128 acc{0ull, 0ull};

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
  __syncthreads();
  int pos = incl - cnt;
  for (int w = 0; w < warp; ++w) pos += warp_tot[w];
  bool used = false;
  for (int j = j0; j < j1; ++j) {
    const int r = __ldg(rk + j);
    const int c = ptx::perm_at(perm, j, K);
    if (r < n4) {
      add128(acc, colsum[(size_t)t * K + c]);
      if (coltiny[(size_t)t * K + c]) {  // values below the tile's scale: exact buckets
        for (int i = 0; i < T; ++i) {
          uint32_t mm;
          int e;
          split_f32(__ldg(It + (size_t)i * K + c), mm, e);
          if (mm && e < lsb) {
            atomicAdd(bkt + e, (unsigned long long)mm);
            used = true;
          }
        }
      }
    } else if (r < n4 + n24) {
      out[pos++] = (unsigned short)c;
    }
  }
  if (used) atomicOr(bucket_used + (size_t)t * ncand + m, 1);
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
    rdense[(size_t)t * ncand + m] = tot;
  }
}

// An fp64 value as a 128-bit integer in units of 2^(lsb-149); false when it is not a whole
// number of units (it then holds values below the tile's scale).
__device__ __forceinline__ bool f64_to_fixed(double s, int lsb, U128& r) {
  r = U128{0ull, 0ull};
  if (s == 0.0) return true;
  const unsigned long long bits = (unsigned long long)__double_as_longlong(s);
  const unsigned long long m = (bits & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  const int sh = (int)(bits >> 52) - 926 - lsb;
  if (sh >= 64) {
    r.hi = m << (sh - 64);
  } else if (sh >= 0) {
    r.lo = m << sh;
    r.hi = sh ? (m >> (64 - sh)) : 0ull;
  } else {
    if (sh <= -53 || (m & ((1ull << (-sh)) - 1ull))) return false;
    r.lo = m >> (-sh);
  }
  return true;
}

// acc (fp64) += x (fp64 >= 0); err |= the addition rounded (Fast2Sum on max/min).
__device__ __forceinline__ void add_checked(double& acc, double x, bool& err) {
  const double a = fmax(acc, x), b = fmin(acc, x);
  const double s = __dadd_rn(a, b);
  err |= __dsub_rn(b, __dsub_rn(s, a)) != 0.0;
  acc = s;
}

// Per (tile, chunk of RB rows), 512 threads.  The chunk's rows of I are staged in shared
// memory once; then, candidate by candidate, each thread takes 2:4 groups g = tid,
// tid + 512, ... and evaluates the top-2 of every row of the chunk.  A thread sums its
// values in fp64 with every addition checked for rounding: when nothing rounded (and the
// sum is a whole number of the tile's fixed-point units) the sum is exact; otherwise the
// same groups are summed again through the exact integer path.  Warps combine their
// 128-bit partials with shuffles into per-warp slots; one barrier at the end, then
// part[t][m][chunk] = the CTA's exact total of candidate m.
__global__ void __launch_bounds__(512) band_sum_kernel(
    const float* __restrict__ I, const unsigned short* __restrict__ band,
    const int* __restrict__ tile_pmax, int K, int T, int RB, CandidateList cl, int ncand,
    U128* __restrict__ part, unsigned long long* __restrict__ bucket,
    int* __restrict__ bucket_used) {
  extern __shared__ __align__(16) float rows_s[];  // [RB][K]
  // per candidate, the CTA's total as four 32-bit digits held in 64-bit words
  __shared__ unsigned long long digits[kMaxCandidates][4];
  const int chunk = blockIdx.x, t = blockIdx.y;
  const int nchunks = gridDim.x;
  const int lane = threadIdx.x & 31;
  for (int x = threadIdx.x; x < kMaxCandidates * 4; x += blockDim.x) (&digits[0][0])[x] = 0ull;
  const int lsb = tile_lsb(tile_pmax[t]);
  const float4* src = reinterpret_cast<const float4*>(I + ((size_t)t * T + (size_t)chunk * RB) * K);
  for (int x = threadIdx.x; x < RB * K / 4; x += blockDim.x)
    reinterpret_cast<float4*>(rows_s)[x] = __ldg(src + x);
  __syncthreads();

  for (int m = 0; m < ncand; ++m) {
    const int ng = cl.c[m].n24 / 4;
    const unsigned short* bl = band + ((size_t)t * ncand + m) * K;
    unsigned long long* bkt = bucket + ((size_t)t * ncand + m) * 256;
    U128 ex{0ull, 0ull};
    if ((int)threadIdx.x < ng) {
      // pass 1: checked fp64
      double acc = 0.0;
      bool err = false;
      for (int g = threadIdx.x; g < ng; g += blockDim.x) {
        const ushort4 cq = __ldg(reinterpret_cast<const ushort4*>(bl) + g);
        const int c0 = min((int)cq.x, K - 1), c1 = min((int)cq.y, K - 1);
        const int c2 = min((int)cq.z, K - 1), c3 = min((int)cq.w, K - 1);
        for (int r = 0; r < RB; ++r) {
          const float* row = rows_s + r * K;
          const float v0 = row[c0], v1 = row[c1], v2 = row[c2], v3 = row[c3];
          const float a = fmaxf(v0, v1), b = fminf(v0, v1);
          const float cc = fmaxf(v2, v3), d = fminf(v2, v3);
          const float t1 = fmaxf(a, cc), t2 = fmaxf(fminf(a, cc), fmaxf(b, d));
          const double p = __dadd_rn((double)t1, (double)t2);  // Fast2Sum, t1 >= t2
          err |= __dsub_rn((double)t2, __dsub_rn(p, (double)t1)) != 0.0;
          add_checked(acc, p, err);
        }
      }
      if (!err && !f64_to_fixed(acc, lsb, ex)) err = true;
      if (err) {
        // pass 2: exact integers (values below the tile's scale into the buckets)
        ex = U128{0ull, 0ull};
        bool used = false;
        for (int g = threadIdx.x; g < ng; g += blockDim.x) {
          const ushort4 cq = __ldg(reinterpret_cast<const ushort4*>(bl) + g);
          const int c0 = min((int)cq.x, K - 1), c1 = min((int)cq.y, K - 1);
          const int c2 = min((int)cq.z, K - 1), c3 = min((int)cq.w, K - 1);
          for (int r = 0; r < RB; ++r) {
            const float* row = rows_s + r * K;
            const float v0 = row[c0], v1 = row[c1], v2 = row[c2], v3 = row[c3];
            const float a = fmaxf(v0, v1), b = fminf(v0, v1);
            const float cc = fmaxf(v2, v3), d = fminf(v2, v3);
            const float tv[2] = {fmaxf(a, cc), fmaxf(fminf(a, cc), fmaxf(b, d))};
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              uint32_t mm;
              int e;
              split_f32(tv[q], mm, e);
              if (!mm) continue;
              if (e >= lsb) {
                add_shifted(ex, mm, e - lsb);
              } else {
                atomicAdd(bkt + e, (unsigned long long)mm);
                used = true;
              }
            }
          }
        }
        if (used) atomicOr(bucket_used + (size_t)t * ncand + m, 1);
      }
    }
    __syncwarp();
    for (int o = 16; o > 0; o >>= 1) {
      U128 other;
      other.lo = __shfl_xor_sync(0xffffffffu, ex.lo, o);
      other.hi = __shfl_xor_sync(0xffffffffu, ex.hi, o);
      add128(ex, other);
    }
    if (lane == 0 && (ex.lo | ex.hi)) {
      atomicAdd(&digits[m][0], ex.lo & 0xFFFFFFFFull);
      atomicAdd(&digits[m][1], ex.lo >> 32);
      atomicAdd(&digits[m][2], ex.hi & 0xFFFFFFFFull);
      atomicAdd(&digits[m][3], ex.hi >> 32);
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < ncand) {
    // fold the digits' carries (each digit word is below 2^37: at most 16 warps add)
    const unsigned long long* d = digits[threadIdx.x];
    const unsigned long long d0 = d[0];
    const unsigned long long d1 = d[1] + (d0 >> 32);
    const unsigned long long d2 = d[2] + (d1 >> 32);
    const unsigned long long d3 = d[3] + (d2 >> 32);
    U128 tot;
    tot.lo = (d0 & 0xFFFFFFFFull) | (d1 << 32);
    tot.hi = (d2 & 0xFFFFFFFFull) | (d3 << 32);
    part[((size_t)t * ncand + threadIdx.x) * nchunks + chunk] = tot;
  }
}

// Per tile, one thread per candidate: R(m) = exact total rounded once to fp64; then the
// first m with R(m+1) < R(m) (else the last candidate) gives the counts and v_s.
__global__ void finalize_kernel(const U128* __restrict__ rdense, const U128* __restrict__ part,
                                int nchunks, const unsigned long long* __restrict__ bucket,
                                const int* __restrict__ bucket_used,
                                const int* __restrict__ tile_pmax, int ncand, CandidateList cl,
                                double t_s, double alpha, double* __restrict__ R,
                                int32_t* __restrict__ counts, double* __restrict__ vs) {
  __shared__ double Rs[kMaxCandidates];
  __shared__ unsigned long long zero_bkt[256];
  const int t = blockIdx.x, m = threadIdx.x;
  for (int i = threadIdx.x; i < 256; i += blockDim.x) zero_bkt[i] = 0ull;
  __syncthreads();
  if (m < ncand) {
    const size_t tm = (size_t)t * ncand + m;
    U128 tot = rdense[tm];
    for (int c = 0; c < nchunks; ++c) add128(tot, part[tm * nchunks + c]);
    const unsigned long long* bk = bucket_used[tm] ? bucket + tm * 256 : zero_bkt;
    const double r = exact_to_double(tot, tile_lsb(tile_pmax[t]), bk);
    Rs[m] = r;
    R[tm] = r;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int ms = ncand - 1;
    for (int k = 0; k + 1 < ncand; ++k) {
      if (Rs[k + 1] < Rs[k]) {
        ms = k;
        break;
      }
    }
    counts[3 * t + 0] = cl.c[ms].n0;
    counts[3 * t + 1] = cl.c[ms].n24;
    counts[3 * t + 2] = cl.c[ms].n4;
    vs[t] = __dsub_rn(t_s, __dmul_rn((double)ms, alpha));
  }
}

// Rows per band_sum CTA: the largest power of two <= 8 whose rows fit in ~96 KB of shared
// memory, so that two CTAs share an SM (T is a multiple of it).  Wider rows (K > 24576)
// would need one row of more than 96 KB; K is at most 16384.
static int band_rows(int K) {
  int rb = 8;
  while (rb > 1 && (size_t)rb * K * sizeof(float) > 96u * 1024u) rb >>= 1;
  return rb;
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
  c.take<char>(rank_scratch_bytes(M, K, T));  // chunk-sorted keys for the ranking
  const int nchunks = T / band_rows(K);
  c.take<unsigned short>((size_t)nt * ncand * K);      // band channel lists
  c.take<U128>((size_t)nt * ncand);                    // dense exact sums
  c.take<U128>((size_t)nt * ncand * nchunks);          // 2:4 partial sums per row chunk
  c.take<unsigned long long>((size_t)nt * ncand * 256);  // exponent buckets
  c.take<int>((size_t)nt * ncand);                     // buckets used
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
  char* rank_scratch = c.take<char>(rank_scratch_bytes(M, K, T));
  int32_t* rank = rank_out ? rank_out : rank_ws;
  cudaError_t e = launch_vector_rank(I, perm, M, K, T, V, rank, pmax, rank_scratch, s);
  if (e != cudaSuccess) return e;
  dim3 gc((K + 255) / 256, nt);
  column_sum_kernel<<<gc, 256, 0, s>>>(I, K, T, pmax, colsum, coltiny);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CandidateList cl;
  for (int i = 0; i < kMaxCandidates; ++i) cl.c[i] = i < ncand ? cands[i] : Candidate{0, 0, 0};
  const int RB = band_rows(K);
  const int nchunks = T / RB;
  unsigned short* band = c.take<unsigned short>((size_t)nt * ncand * K);
  U128* rdense = c.take<U128>((size_t)nt * ncand);
  U128* part = c.take<U128>((size_t)nt * ncand * nchunks);
  unsigned long long* bucket = c.take<unsigned long long>((size_t)nt * ncand * 256);
  int* bucket_used = c.take<int>((size_t)nt * ncand);
  e = cudaMemsetAsync(bucket, 0, (size_t)nt * ncand * 256 * sizeof(unsigned long long), s);
  if (e != cudaSuccess) return e;
  e = cudaMemsetAsync(bucket_used, 0, (size_t)nt * ncand * sizeof(int), s);
  if (e != cudaSuccess) return e;
  candidate_lists_kernel<<<dim3(ncand, nt), 512, 0, s>>>(I, perm, rank, pmax, colsum, coltiny, K, T,
                                                         cl, ncand, band, rdense, bucket,
                                                         bucket_used);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)RB * K * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(band_sum_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             96 * 1024);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  band_sum_kernel<<<dim3(nchunks, nt), 512, smem, s>>>(I, band, pmax, K, T, RB, cl, ncand, part,
                                                       bucket, bucket_used);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  finalize_kernel<<<nt, 64, 0, s>>>(rdense, part, nchunks, bucket, bucket_used, pmax, ncand, cl,
                                    t_s, alpha, R, counts_out, vs_out);
  return cudaGetLastError();
}

}  // namespace hinm
